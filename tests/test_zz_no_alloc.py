"""csa2_index_topk_noalloc gives what csa2_index_topk gives.

The non-allocating entry point exists for callers that cannot allocate device
memory (a fixed memory pool reserved before decoding, or an interface without a
workspace argument); its scratch is a fixed array inside the library.  Here it
is called twice in a row through the C ABI -- the second call finds the first
call's leftovers in that array -- and both results are compared with the
workspace entry point on the same inputs.  This file is collected last.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from fp4_sparse_attention_pack_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from fp4_sparse_attention_pack_b200 import _build
    _build.build()
    import fp4_sparse_attention_pack_b200 as m
    from fp4_sparse_attention_pack_b200 import engine
    m.engine = engine
    return m


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


@pytest.mark.parametrize("H_idx", [64, 4])
def test_noalloc_matches_workspace_entry_point(csa, H_idx):
    B, T, K = 3, 3001, 512
    wl = W.small(W.WORKLOADS[1], B=B, T=T, H_idx=H_idx, K=K)
    dc = csa.engine.DeviceCache(B, (T // 2 + 63) // 64 + 1, 2, "cuda", page_seed=2)
    x = np.stack([W.tokens(wl, 0, b, 0, T) for b in range(B)])
    g = np.stack([W.gates(wl, 0, b, 0, T) for b in range(B)])
    csa.pack_cache(dc.desc, _bf16(x), _f32(g), _f32(W.w_idx(wl, 0)))
    q, w = _bf16(W.query_idx(wl, 0, 0)), _f32(W.head_weights(wl, 0, 0))

    ws = torch.empty(csa.index_topk_workspace(B, dc.max_pages * 64, H_idx, K), dtype=torch.uint8,
                     device="cuda")
    idx_ref = torch.empty(B, K, dtype=torch.int32, device="cuda")
    sc_ref = torch.empty(B, K, dtype=torch.float32, device="cuda")
    csa.index_topk(dc.desc, q, w, K, idx_ref, ws, score_out=sc_ref)
    torch.cuda.synchronize()
    for _ in range(2):
        idx = torch.full((B, K), -7, dtype=torch.int32, device="cuda")
        sc = torch.full((B, K), -7.0, dtype=torch.float32, device="cuda")
        csa.index_topk_noalloc(dc.desc, q, w, K, idx, score_out=sc)
        torch.cuda.synchronize()
        assert torch.equal(idx, idx_ref)
        np.testing.assert_allclose(sc.cpu().numpy(), sc_ref.cpu().numpy(), rtol=1e-5, atol=0)
    assert dc.status_bits() == 0

    # a request beyond the fixed scratch is refused before anything is launched
    big = csa.csa2_cache.from_buffer_copy(dc.desc)
    big.max_pages = 50000
    with pytest.raises(csa.Csa2Error) as e:
        csa.index_topk_noalloc(big, q, w, K, idx_ref)
    assert e.value.status == -3
