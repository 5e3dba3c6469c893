"""Pins of the oracle's FP8 SWA window ("Le cache KV en FP4": the SWA KV stays in
FP8; one E4M3 code per channel, no scale): exact round trip of every finite
E4M3 value, agreement with a library float8 cast in range, ties, saturation,
and the model-level effect on attention."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from fp4_sparse_attention_pack_b200 import workloads as W


def _bf16(x):
    return (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_every_finite_e4m3_value_round_trips(ref):
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)   # 0x7F / 0xFF are NaN
    vals = np.array([ref.e4m3_value(int(c)) for c in codes], np.float32)
    vals[codes == 0x80] = -0.0
    bits = _bf16(vals)
    assert np.array_equal(ref.bf16_to_f32(bits), vals)        # E4M3 values are bf16 values
    assert np.array_equal(ref.window_fp8(bits), codes)
    assert np.array_equal(ref.e4m3_values(codes), vals)


def test_matches_library_float8_cast_in_range(ref):
    rng = np.random.default_rng(4)
    x = np.concatenate([rng.normal(size=20000) * 10 ** rng.uniform(-3, 2, 20000),
                        rng.uniform(-448, 448, 5000)]).astype(np.float32)
    x = ref.bf16_to_f32(_bf16(x))                              # window inputs are bf16
    x = x[np.abs(x) <= 448]
    lib = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ref.window_fp8(_bf16(x)), lib)


def test_ties_go_to_the_even_code_and_large_values_saturate(ref):
    # 1.0625 lies halfway between 1 (0x38) and 1.125 (0x39); 1.1875 between 0x39 and 0x3A
    assert list(ref.window_fp8(_bf16([1.0625, 1.1875, -1.0625]))) == [0x38, 0x3A, 0xB8]
    # 2^-10 lies halfway between 0 and the smallest subnormal 2^-9: even code 0, sign kept
    assert list(ref.window_fp8(_bf16([2.0 ** -10, -(2.0 ** -10), 3 * 2.0 ** -10]))) == [0x00, 0x80, 0x02]
    assert list(ref.window_fp8(_bf16([448.0, 464.0, 1e6, -3e38]))) == [0x7E, 0x7E, 0x7E, 0xFE]


def _model(ref, win_fp8, wtok_fn):
    t = W.ModeTable((W.SWA_ONLY, W.FULL, W.REUSE), (-1, 0, 0), (-1, 1, 1), (2,))
    rng = np.random.default_rng(2)
    B, H, Hi, K, T = 2, 4, 4, 6, 40
    Ws = [(rng.normal(size=(512, 128)) / np.sqrt(512)).astype(np.float32)]
    m = ref.RefModel(t, B, [64], Ws, H, Hi, K, 1 / np.sqrt(512), win_fp8=win_fp8)
    for b in range(B):
        m.caches[0].append(b, _bf16(rng.normal(size=(T, 512))), rng.normal(size=T).astype(np.float32))
    for l in range(3):
        for b in range(B):
            for _ in range(5):
                m.window_append(l, b, wtok_fn(rng))
    inp = dict(x_new=[[_bf16(rng.normal(size=512)) for _ in range(B)]],
               g_new=[rng.normal(size=B).astype(np.float32)],
               q=[[_bf16(rng.normal(size=(H, 512))) for _ in range(B)] for _ in range(3)],
               qidx=[[_bf16(rng.normal(size=(Hi, 128))) for _ in range(B)] for _ in range(3)],
               wh=[[rng.uniform(0, 1, Hi).astype(np.float32) for _ in range(B)] for _ in range(3)],
               wtok=[[wtok_fn(rng) for _ in range(B)] for _ in range(3)])
    return m, inp


def test_fp8_window_holds_half_the_bytes_and_its_codes(ref):
    m, inp = _model(ref, True, lambda r: _bf16(r.normal(size=512)))
    m.step(**inp)
    assert m.win8.nbytes * 2 == m.win.nbytes and m.win8.shape == m.win.shape
    for l in range(3):
        for b in range(2):
            assert np.array_equal(m.win8[l, b, :6], ref.window_fp8(m.win[l, b, :6]))


def test_fp8_window_equals_bf16_window_on_representable_tokens(ref):
    # tokens that are E4M3 values already: the FP8 model attends exactly as the bf16 one
    def tok(r):
        return _bf16(ref.e4m3_values(r.integers(0, 0x7F, 512) | (r.integers(0, 2, 512) << 7)))
    m8, inp = _model(ref, True, tok)
    m16, _ = _model(ref, False, tok)
    out8, idx8 = m8.step(**inp)
    out16, idx16 = m16.step(**inp)
    for l in range(3):
        for b in range(2):
            assert np.array_equal(out8[l][b], out16[l][b])


def test_fp8_window_changes_attention_only_through_the_window(ref):
    m8, inp = _model(ref, True, lambda r: _bf16(r.normal(size=512) * 3))
    m16, _ = _model(ref, False, lambda r: _bf16(r.normal(size=512) * 3))
    out8, idx8 = m8.step(**inp)
    out16, _ = m16.step(**inp)
    b, l = 1, 1
    wl = m8.win_len(l, b)
    c = m8.caches[0]
    items = ref.attention_items(c.mc[b], c.ms[b], int(c.n[b]), idx8[l][b], np.zeros((1, 512), np.uint16), 0)
    win = ref.e4m3_values(ref.window_fp8(m16.win[l, b, :wl]))
    want = ref.attention(inp["q"][l][b], np.concatenate([items, win]), m8.scale)
    assert np.array_equal(out8[l][b], want)
    assert not np.array_equal(out8[l][b], out16[l][b])
