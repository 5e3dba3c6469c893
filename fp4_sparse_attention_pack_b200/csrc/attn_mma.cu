// Sparse + window attention on the 5th-generation tensor cores (tcgen05.mma
// kind::f16, fp16 operands, fp32 accumulation in TMEM).
//
// Per (problem, sequence) the items are the K selected entries (dequantised
// from E2M1 x E4M3: exact in fp16) and the valid window tokens (bf16 -> fp16,
// exact for |x| in fp16's normal range); the latent item is key and value.
// Items go through 128-item tiles with an online softmax:
//
//   S^T[128 items x 64 heads] = Items . Q^T            (M = 128, N = 64, K = 512)
//   P^T = exp(scale * S^T - m_head)                    (fp16, per item lane)
//   O^T[4 x 128 latent x 64 heads] += Items^T . P^T    (M = 128, N = 64, K = 128)
//
// A tile is consumed as eight slabs of 64 latent channels (128 rows x 128 B,
// 128-byte swizzle), each read as the K-major A operand of S^T and, two at a
// time, as the MN-major A operand of O^T.  The running per-head maximum is only
// moved when a tile's maximum exceeds it by more than 8 (so p <= e^8 fits
// fp16), which makes the O rescale (TMEM load, scale, store) rare.  Heads are
// padded to 64.
//
// Warp-specialised CTA (416 threads, one unit = (problem, sequence, split)):
//   warps 8-11  slab producers, one item row per thread: dequantise the row's
//               cache entry (16-byte loads issued three slabs ahead) or convert
//               its window token (slab boxes by TMA, 3-D tensor map per window,
//               started four slabs ahead) into a ring of eight 16 KB slab slots;
//   warp 12     MMA issuer (one elected lane of the converged warp) in the
//               order S(0), S(1), O(0), S(2), O(1), ..., O(last), so that the
//               softmax of tile t overlaps the S MMAs of tile t + 1; the slabs of
//               a tile are produced twice (once for S, once for O);
//   warps 0-7   softmax (two per TMEM lane quadrant, 32 heads each) into a
//               double-buffered S^T, P^T to shared memory, rescale of O^T, and
//               the final normalised write of O.
// Every wait is bounded; a timeout sets CSA2_DEVERR_TIMEOUT and the CTA drains.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>

#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace csa2 {

namespace {

using namespace sm100;

constexpr int kT = 128;            // items per tile (MMA M of S^T)
constexpr int kHp = 64;            // heads, padded (MMA N)
constexpr int kSlots = 8;          // slab ring
constexpr int kSlabBytes = kT * 128;
constexpr int kSoftWarps = 8;      // warps 0-7
constexpr int kProdWarp0 = 8;      // warps 8-11
constexpr int kMmaWarp = 12;
constexpr int kThreads = 32 * 13;
constexpr int kMaxUnitTiles = (CSA2_MAX_K + WIN + kT - 1) / kT;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;      // S^T: 2 x 64 columns
constexpr uint32_t kColO = 128;    // O^T: 4 x 64 columns
constexpr float kRescaleGap = 8.0f;
constexpr int kRowEmpty = -1, kRowWindow = -2;  // lookup codes (else: entry row in the pools)

struct AttnMaps {
    CUtensorMap win[kMaxProblems];  // window [batch][128][512] bf16, box 64 x 128 x 1, SW128
};

struct __align__(1024) Smem {
    uint8_t slab[kSlots][kSlabBytes];  // 128 rows x 128 B (SW128) each
    uint8_t q[8][kHp * 128];           // 8 slabs x 64 rows x 128 B (SW128)
    uint8_t p[kT * 128];               // P^T: 128 item rows x 64 heads fp16 (SW128)
    int32_t lk[kMaxUnitTiles][kT];     // per unit tile and row: entry row, kRowWindow or kRowEmpty
    float red_max[4][kHp];             // per-quadrant partial max
    float red_sum[4][kHp];             // per-quadrant partial sum
    float m_used[kHp];
    float l[kHp];
    float alpha[kHp];
    int rescale[2];                    // per head warp: some head's maximum moved
    uint64_t slot_full[kSlots], slot_empty[kSlots], tma_bar[kSlots];
    uint64_t s_full[2], s_empty[2], p_full, o_done, drained;
    uint32_t tmem_base;
};
static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory beyond the 227 KB per-block limit");

// Byte offset of 16-byte chunk c of row r inside a 128B-swizzled slab.
__device__ __forceinline__ uint32_t sw128(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

// Convert the 8 bf16 chunks (64 channels) of row r of a slab to fp16 in place
// (exact for values in fp16's normal range).
__device__ __forceinline__ void bf16_row_to_f16(uint8_t* slab, int r) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint4* ptr = reinterpret_cast<uint4*>(slab + sw128(r, c));
        const uint4 w = *ptr;
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
        uint4 o;
        uint32_t* os = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const __half2 hv = __floats2half2_rn(__uint_as_float(ws[k] << 16), __uint_as_float(ws[k] & 0xFFFF0000u));
            os[k] = *reinterpret_cast<const uint32_t*>(&hv);
        }
        *ptr = o;
    }
}

// Two E2M1 codes (one byte, channel 2i in the low nibble) -> f16x2 (low half first).
__device__ __forceinline__ uint32_t e2m1x2_to_h2(uint32_t byte) {
    uint32_t out;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(out) : "r"(byte));
    return out;
}

__device__ __forceinline__ void zero_row(uint8_t* slab, int r) {
#pragma unroll
    for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(slab + sw128(r, c)) = make_uint4(0, 0, 0, 0);
}

// Reduce-scatter over the warp: v[N] per lane (N = 32 or 64) -> lane l holds the
// reduction over the 32 lanes of element N/32 * l + i in v[i], i < N/32.
template <bool kMax, int N>
__device__ __forceinline__ void warp_reduce_scatter(float (&v)[N]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int step = 0; step < 5; ++step) {
        const int o = 16 >> step;
        const int half = (N / 2) >> step;
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float keep = upper ? v[half + i] : v[i];
            const float send = upper ? v[i] : v[half + i];
            const float got = __shfl_xor_sync(0xffffffffu, send, o);
            v[i] = kMax ? fmaxf(keep, got) : keep + got;
        }
    }
}

// All 256 softmax threads meet (named barrier 1); returns the OR of pred over them.
__device__ __forceinline__ bool soft_sync_or(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.or.pred q, 1, 256, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void soft_sync() { asm volatile("barrier.cta.sync 1, 256;" ::: "memory"); }

// Dequantise one entry row of slab j: 32 code bytes (64 E2M1 values, channel 2i
// in the low nibble) and 4 E4M3 scale bytes (one per 16 channels) -> fp16.
__device__ __forceinline__ void dequant_row(uint8_t* slab, int r, uint4 c0, uint4 c1, uint32_t sc) {
    const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int c2 = 0; c2 < 4; ++c2) {  // chunks 2*c2, 2*c2+1 share scale byte c2
        const __half2 s2 = __float2half2_rn(e4m3_decode_pos((sc >> (8 * c2)) & 0xFFu));
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const int c = 2 * c2 + cc;
            uint4 o;
            uint32_t* os = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t h = e2m1x2_to_h2((cw[c] >> (8 * k)) & 0xFFu);
                const __half2 v = __hmul2(*reinterpret_cast<const __half2*>(&h), s2);
                os[k] = *reinterpret_cast<const uint32_t*>(&v);
            }
            *reinterpret_cast<uint4*>(slab + sw128(r, c)) = o;
        }
    }
}

// Step s of a unit with n tiles: S(0), S(1), O(0), S(2), O(1), ..., S(n-1), O(n-2), O(n-1).
__device__ __forceinline__ void unit_step(int s, int n, int& tile, bool& is_s) {
    if (s == 0) {
        tile = 0, is_s = true;
    } else if (s == 2 * n - 1) {
        tile = n - 1, is_s = false;
    } else if (s & 1) {
        tile = (s + 1) >> 1, is_s = true;
    } else {
        tile = (s >> 1) - 1, is_s = false;
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    k_attn_mma(const __grid_constant__ AttnBatch ab, const __grid_constant__ AttnMaps maps, int splits,
               int tiles_per_split) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int unit = blockIdx.x;
    const int split = unit % splits;
    const int pb = unit / splits;
    const int b = pb % ab.batch;
    const int prob = pb / ab.batch;
    const AttnProblem& P = ab.p[prob];
    const int K = P.K;
    const int H = ab.H;
    const int n_tiles = (K + WIN + kT - 1) / kT;
    const int t_begin = split * tiles_per_split;
    const int nt = max(0, min(n_tiles, t_begin + tiles_per_split) - t_begin);  // tiles of this unit

    if (tid == 0) {
        for (int i = 0; i < kSlots; ++i) {
            mbar_init(&sm.slot_full[i], 4);  // the four producer warps
            mbar_init(&sm.slot_empty[i], 1);
            mbar_init(&sm.tma_bar[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.s_full[i], 1);
            mbar_init(&sm.s_empty[i], kSoftWarps);
        }
        mbar_init(&sm.p_full, kSoftWarps);
        mbar_init(&sm.o_done, 1);
        mbar_init(&sm.drained, 1);
        fence_mbar_init();
        prefetch_tmap(&maps.win[prob]);
    }
    if (warp == kMmaWarp) tmem_alloc(&sm.tmem_base, kTmemCols);
    if (tid < kHp) {
        sm.m_used[tid] = -INFINITY;
        sm.l[tid] = 0.0f;
    }
    // Q -> fp16 slabs (rows >= H are zero): cp.async in place, then convert.
    if (warp < 8) {
        const int j = warp;
        for (int h = lane; h < kHp; h += 32) {
            if (h < H) {
                const uint16_t* src = P.q + ((int64_t)b * H + h) * D + 64 * j;
#pragma unroll
                for (int c = 0; c < 8; ++c) cp_async16(sm.q[j] + sw128(h, c), src + 8 * c);
            } else {
                zero_row(sm.q[j], h);
            }
        }
        cp_async_commit();
        cp_async_wait_all();
        for (int h = lane; h < H && h < kHp; h += 32) bf16_row_to_f16(sm.q[j], h);
    }
    const int wcount = P.win_count[b];
    const int wlen = wcount < WIN ? (wcount < 0 ? 0 : wcount) : WIN;
    const int n = (K > 0) ? entries_of(P.cache, b) : 0;
    // Where every item of the unit comes from, and its entries into L2 now.
    for (int i = tid; i < nt * kT; i += kThreads) {
        const int u = i / kT, r = i - u * kT;
        const int pos = (t_begin + u) * kT + r;
        int32_t code = kRowEmpty;
        if (pos < K) {
            const int e = P.idx[(int64_t)b * K + pos];
            if (e >= 0 && e < n) {
                const int pg = page_of(P.cache, b, e);
                if (pg >= 0) {
                    code = pg * PAGE + (e % PAGE);
                    bulk_prefetch_l2(P.cache.main_codes + (int64_t)code * MCB, MCB);
                    bulk_prefetch_l2(P.cache.main_scales + (int64_t)code * MSB, MSB);
                }
            }
        } else if (pos - K < wlen) {
            code = kRowWindow;
        }
        sm.lk[u][r] = code;
    }
    if (tid == 0 && nt > 0 && (t_begin + nt) * kT > K && wlen > 0)
        bulk_prefetch_l2(P.win + (int64_t)b * WIN * D, (uint32_t)wlen * D * 2);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = sm.tmem_base;
    bool timed_out = false;

    if (warp >= kProdWarp0 && warp < kMmaWarp) {
        // ------------------------------------------------------------ producers
        const int r = tid - kProdWarp0 * 32;  // item row of this thread
        const bool issuer = warp == kProdWarp0;
        uint32_t tma_par = 0, tma_pending = 0;
        const int n_prod = 16 * nt;
        auto prod_at = [&](int q, int& u, int& j) {
            bool is_s;
            unit_step(q >> 3, nt, u, is_s);
            j = q & 7;
        };
        auto load_raw = [&](int q, uint4& c0, uint4& c1, uint32_t& sc) {
            int u, j;
            prod_at(q, u, j);
            const int32_t code = sm.lk[u][r];
            if (code >= 0) {
                const uint4* cs = reinterpret_cast<const uint4*>(P.cache.main_codes + (int64_t)code * MCB + 32 * j);
                c0 = __ldg(cs);
                c1 = __ldg(cs + 1);
                sc = __ldg(reinterpret_cast<const uint32_t*>(P.cache.main_scales + (int64_t)code * MSB + 4 * j));
            } else {
                c0 = c1 = make_uint4(0, 0, 0, 0);
                sc = 0;
            }
        };
        auto window_tile = [&](int u) {
            const int t = t_begin + u;
            return (t * kT + kT > K) && (t * kT < K + wlen);
        };
        // Window boxes: the issuing warp acquires slots and starts their TMA loads
        // kTmaAhead productions ahead of the one being built.
        constexpr int kTmaAhead = 4;
        auto acquire = [&](int qa) -> bool {
            int u, j;
            prod_at(qa, u, j);
            const int slot = qa & (kSlots - 1);
            if (!mbar_wait_warp(&sm.slot_empty[slot], ((qa >> 3) & 1) ^ 1)) return false;
            if (window_tile(u)) {
                mbar_expect_tx_w(&sm.tma_bar[slot], kSlabBytes);
                tma_load_3d_w(sm.slab[slot], &maps.win[prob], 64 * j, (t_begin + u) * kT - K, b, &sm.tma_bar[slot]);
                tma_pending |= 1u << slot;
            }
            return true;
        };
        if (issuer)
            for (int qa = 0; qa < kTmaAhead && qa < n_prod && !timed_out; ++qa) timed_out = !acquire(qa);
        // Entry bytes: three productions ahead in registers.
        uint4 ra0[3], ra1[3];
        uint32_t rsc[3];
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            if (i < n_prod) {
                load_raw(i, ra0[i], ra1[i], rsc[i]);
            } else {
                ra0[i] = ra1[i] = make_uint4(0, 0, 0, 0);
                rsc[i] = 0;
            }
        }
        for (int q = 0; q < n_prod && !timed_out; ++q) {
            const uint4 c0 = ra0[0], c1 = ra1[0];
            const uint32_t sc = rsc[0];
            ra0[0] = ra0[1], ra1[0] = ra1[1], rsc[0] = rsc[1];
            ra0[1] = ra0[2], ra1[1] = ra1[2], rsc[1] = rsc[2];
            if (q + 3 < n_prod) load_raw(q + 3, ra0[2], ra1[2], rsc[2]);
            if (issuer && q + kTmaAhead < n_prod && !acquire(q + kTmaAhead)) { timed_out = true; break; }
            int u, j;
            prod_at(q, u, j);
            const int slot = q & (kSlots - 1);
            if (!mbar_wait_warp(&sm.slot_empty[slot], ((q >> 3) & 1) ^ 1)) { timed_out = true; break; }
            uint8_t* slab = sm.slab[slot];
            if (window_tile(u)) {
                if (!mbar_wait_warp(&sm.tma_bar[slot], (tma_par >> slot) & 1u)) { timed_out = true; break; }
                tma_par ^= 1u << slot;
                tma_pending &= ~(1u << slot);
            }
            const int32_t code = sm.lk[u][r];
            if (code >= 0)
                dequant_row(slab, r, c0, c1, sc);
            else if (code == kRowWindow)
                bf16_row_to_f16(slab, r);
            else
                zero_row(slab, r);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.slot_full[slot]);
        }
        // a window box still in flight lands before the CTA moves on
        if (issuer && lane == 0)
            for (int i = 0; i < kSlots; ++i)
                if ((tma_pending >> i) & 1u) (void)mbar_wait(&sm.tma_bar[i], (tma_par >> i) & 1u);
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t idesc_s = idesc_f16(128, kHp, 0, 0, 0);
        const uint32_t idesc_o = idesc_f16(128, kHp, 0, 1, 1);
        const uint64_t desc_slab0 = smem_desc(sm.slab[0], 16, 1024, kLayoutSw128);
        const uint64_t desc_vt0 = smem_desc(sm.slab[0], kSlabBytes, 1024, kLayoutSw128);
        const uint64_t desc_q = smem_desc(sm.q[0], 16, 1024, kLayoutSw128);
        const uint64_t desc_p = smem_desc(sm.p, kSlabBytes, 1024, kLayoutSw128);
        int q = 0;
        for (int st = 0; st < 2 * nt && !timed_out; ++st) {
            int u;
            bool is_s;
            unit_step(st, nt, u, is_s);
            if (is_s) {
                if (u >= 2 && !mbar_wait_warp(&sm.s_empty[u & 1], ((u - 2) >> 1) & 1)) { timed_out = true; break; }
                const uint32_t d = tbase + kColS + 64 * (u & 1);
                for (int j = 0; j < 8; ++j, ++q) {
                    const int slot = q & (kSlots - 1);
                    if (!mbar_wait_warp(&sm.slot_full[slot], (q >> 3) & 1)) { timed_out = true; break; }
                    tc_fence_after();
                    const uint64_t da = desc_slab0 + (uint64_t)((slot * kSlabBytes) >> 4);
#pragma unroll
                    for (int k = 0; k < 4; ++k)  // 16 latent channels per MMA
                        tc_mma_f16_w(d, da + 2 * k, desc_q + (uint64_t)((j * kHp * 128 + 32 * k) >> 4), idesc_s,
                                     (j | k) ? 1u : 0u);
                    tc_commit_w(&sm.slot_empty[slot]);
                }
                if (timed_out) break;
                tc_commit_w(&sm.s_full[u & 1]);
            } else {
                if (!mbar_wait_warp(&sm.p_full, u & 1)) { timed_out = true; break; }
                for (int c = 0; c < 4; ++c, q += 2) {
                    const int slot = q & (kSlots - 1);  // slabs 2c, 2c+1 sit in adjacent slots
                    if (!mbar_wait_warp(&sm.slot_full[slot], (q >> 3) & 1) ||
                        !mbar_wait_warp(&sm.slot_full[slot + 1], ((q + 1) >> 3) & 1)) {
                        timed_out = true;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t da = desc_vt0 + (uint64_t)((slot * kSlabBytes) >> 4);
#pragma unroll
                    for (int i = 0; i < 8; ++i)  // 16 items per MMA
                        tc_mma_f16_w(tbase + kColO + 64 * c, da + (uint64_t)((2048 * i) >> 4),
                                     desc_p + (uint64_t)((2048 * i) >> 4), idesc_o, (u > 0 || i > 0) ? 1u : 0u);
                    tc_commit_w(&sm.slot_empty[slot]);
                    tc_commit_w(&sm.slot_empty[slot + 1]);
                }
                if (timed_out) break;
                tc_commit_w(&sm.o_done);
            }
        }
        // every tcgen05 operation of this warp has completed before TMEM is freed
        tc_commit_w(&sm.drained);
        (void)mbar_wait_warp(&sm.drained, 0);
    } else {
        // ------------------------------------------------------------ softmax + output
        const int quad = warp & 3, hh = warp >> 2;
        const int row = quad * 32 + lane;
        for (int u = 0; u < nt; ++u) {
            bool ok_wait = mbar_wait(&sm.s_full[u & 1], (u >> 1) & 1);
            if (soft_sync_or(!ok_wait)) { timed_out = true; break; }
            tc_fence_after();
            const uint32_t s_addr = tbase + ((uint32_t)(quad * 32) << 16) + kColS + 64 * (u & 1) + 32 * hh;
            const bool ok = sm.lk[u][row] != kRowEmpty;
            {
                float v[32];
                tmem_ld_32x32b_x32(s_addr, v);
#pragma unroll
                for (int h = 0; h < 32; ++h) v[h] = ok ? v[h] * ab.scale : -INFINITY;
                warp_reduce_scatter<true, 32>(v);
                sm.red_max[quad][32 * hh + lane] = v[0];
            }
            soft_sync();
            if (tid < kHp) {
                const float mt = fmaxf(fmaxf(sm.red_max[0][tid], sm.red_max[1][tid]),
                                       fmaxf(sm.red_max[2][tid], sm.red_max[3][tid]));
                const float mo = sm.m_used[tid];
                float a = 1.0f;
                bool rs = false;
                if (mt > mo + kRescaleGap || (mo == -INFINITY && mt != -INFINITY)) {
                    a = (mo == -INFINITY) ? 0.0f : expf(mo - mt);
                    sm.m_used[tid] = mt;
                    rs = u > 0 && mo != -INFINITY;
                }
                sm.alpha[tid] = a;
                const unsigned any = __ballot_sync(0xffffffffu, rs);
                if (lane == 0) sm.rescale[warp] = any ? 1 : 0;
            }
            // P^T and O^T of the previous tile are in use until its O MMAs complete
            ok_wait = (u == 0) || mbar_wait(&sm.o_done, (u - 1) & 1);
            if (soft_sync_or(!ok_wait)) { timed_out = true; break; }
            tc_fence_after();
            const bool rescale = (sm.rescale[0] | sm.rescale[1]) != 0;
            // ---- P^T = exp(s - m) in fp16 (S reloaded from TMEM), sums of the rounded p
            {
                float v[32];
                tmem_ld_32x32b_x32(s_addr, v);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.s_empty[u & 1]);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint4 o;
                    uint32_t* os = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int h = 8 * c + 2 * k;
                        const float p0 = ok ? __expf(v[h] * ab.scale - sm.m_used[32 * hh + h]) : 0.0f;
                        const float p1 = ok ? __expf(v[h + 1] * ab.scale - sm.m_used[32 * hh + h + 1]) : 0.0f;
                        const __half2 hv = __floats2half2_rn(p0, p1);
                        const float2 back = __half22float2(hv);
                        v[h] = back.x;
                        v[h + 1] = back.y;
                        os[k] = *reinterpret_cast<const uint32_t*>(&hv);
                    }
                    *reinterpret_cast<uint4*>(sm.p + sw128(row, 4 * hh + c)) = o;
                }
                warp_reduce_scatter<false, 32>(v);
                sm.red_sum[quad][32 * hh + lane] = v[0];
            }
            // ---- rescale O^T where a head's reference maximum moved
            if (rescale) {
                for (int c = hh * 2; c < hh * 2 + 2; ++c) {
                    const uint32_t ta = tbase + ((uint32_t)(quad * 32) << 16) + kColO + 64 * c;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        float o[32];
                        tmem_ld_32x32b_x32(ta + 32 * half, o);
#pragma unroll
                        for (int h = 0; h < 32; ++h) o[h] *= sm.alpha[32 * half + h];
                        tmem_st_32x32b_x32(ta + 32 * half, o);
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            soft_sync();
            if (tid < kHp)
                sm.l[tid] = sm.l[tid] * sm.alpha[tid] + (sm.red_sum[0][tid] + sm.red_sum[1][tid]) +
                            (sm.red_sum[2][tid] + sm.red_sum[3][tid]);
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.p_full);
        }
        if (!timed_out && nt > 0) {
            const bool ok_wait = mbar_wait(&sm.o_done, (nt - 1) & 1);
            timed_out = soft_sync_or(!ok_wait);
        } else {
            soft_sync();
        }
        if (!timed_out) {
            tc_fence_after();
            // ---- write O (normalised) or the split's partial (O, m, l)
            const bool partial = splits > 1;
            float* dst = partial ? ab.part_o + (int64_t)unit * H * D : P.out + (int64_t)b * H * D;
            for (int c = hh * 2; c < hh * 2 + 2; ++c) {
                const int lat = 128 * c + quad * 32 + lane;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float o[32];
                    if (nt > 0) {
                        tmem_ld_32x32b_x32(tbase + ((uint32_t)(quad * 32) << 16) + kColO + 64 * c + 32 * half, o);
                    } else {
#pragma unroll
                        for (int h = 0; h < 32; ++h) o[h] = 0.0f;
                    }
#pragma unroll
                    for (int h = 0; h < 32; ++h) {
                        const int hd = 32 * half + h;
                        if (hd < H) {
                            const float l = sm.l[hd];
                            dst[(int64_t)hd * D + lat] = partial ? o[h] : (l > 0.0f ? o[h] / l : 0.0f);
                        }
                    }
                }
            }
            if (partial && tid < H) {
                ab.part_ml[((int64_t)unit * H + tid) * 2 + 0] = sm.m_used[tid];
                ab.part_ml[((int64_t)unit * H + tid) * 2 + 1] = sm.l[tid];
            }
        }
    }
    if (timed_out && K > 0 && lane == 0) atomicOr(P.cache.status, CSA2_DEVERR_TIMEOUT);

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tbase, kTmemCols);
    }
}

// out = sum_s O_s e^(m_s - M) / sum_s l_s e^(m_s - M) over the splits of (problem, sequence)
__global__ void k_attn_mma_combine(const __grid_constant__ AttnBatch ab, int splits) {
    const int h = blockIdx.x, b = blockIdx.y, prob = blockIdx.z;
    const AttnProblem& P = ab.p[prob];
    const int H = ab.H;
    const int64_t u0 = ((int64_t)prob * ab.batch + b) * splits;
    float M = -INFINITY;
    for (int s = 0; s < splits; ++s) M = fmaxf(M, ab.part_ml[((u0 + s) * H + h) * 2]);
    float L = 0.0f;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (M != -INFINITY) {
        for (int s = 0; s < splits; ++s) {
            const float m = ab.part_ml[((u0 + s) * H + h) * 2];
            const float l = ab.part_ml[((u0 + s) * H + h) * 2 + 1];
            if (m == -INFINITY || l == 0.0f) continue;
            const float f = expf(m - M);
            L += l * f;
            const float* po = ab.part_o + ((u0 + s) * H + h) * D;
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[i] = fmaf(f, po[threadIdx.x + 128 * i], acc[i]);
        }
    }
    float* o = P.out + ((int64_t)b * H + h) * D;
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) o[threadIdx.x + 128 * i] = acc[i] * inv;
}

int sm_count_attn() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

}  // namespace

// Splits of the item tiles per (problem, sequence): enough units to fill the
// SMs when the batch is small, none when there are already plenty.
int attn_mma_splits(int n_problems, int batch, int Kmax) {
    const int tiles = (Kmax + WIN + kT - 1) / kT;
    const int pairs = n_problems * batch;
    const int want = (sm_count_attn() + pairs - 1) / pairs;
    return std::max(1, std::min(tiles, want));
}

bool attn_mma_supported(const AttnBatch& ab) {
    if (ab.H < 1 || ab.H > kHp || ab.Kmax > CSA2_MAX_K) return false;
    for (int i = 0; i < ab.n; ++i)  // entry rows are kept as 32-bit ints
        if (ab.p[i].K > 0 && (int64_t)ab.p[i].cache.num_pages * PAGE > INT32_MAX) return false;
    return true;
}

size_t attn_mma_workspace_bytes(int n_problems, int batch, int H, int Kmax) {
    const int splits = attn_mma_splits(n_problems, batch, Kmax);
    if (splits == 1) return 0;
    const size_t units = (size_t)n_problems * batch * splits;
    return units * H * D * sizeof(float) + units * H * 2 * sizeof(float);
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 attn_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void* p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// Window ring [batch][128][512] bf16 as a 3-D tensor, boxes of 64 channels x 128 rows.
bool make_window_map(CUtensorMap* m, const void* base, int batch) {
    auto fn = attn_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)WIN, (cuuint64_t)batch};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)WIN * D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)WIN, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_attn_mma(const AttnBatch& ab_in, cudaStream_t st, cudaEvent_t* ev) {
    AttnBatch ab = ab_in;
    AttnMaps maps;  // kernel parameter (copied at launch)
    std::memset(&maps, 0, sizeof(maps));
    for (int i = 0; i < ab.n; ++i)
        if (!make_window_map(&maps.win[i], ab.p[i].win, ab.batch)) return cudaErrorInvalidValue;
    const int splits = attn_mma_splits(ab.n, ab.batch, ab.Kmax);
    const int tiles = (ab.Kmax + WIN + kT - 1) / kT;
    const int tps = (tiles + splits - 1) / splits;
    if (splits > 1) {
        const size_t units = (size_t)ab.n * ab.batch * splits;
        ab.part_ml = ab.part_o + units * ab.H * D;
    }
    const size_t smem = sizeof(Smem) + 1024;
    static const bool attr = [smem] {
        cudaFuncSetAttribute(k_attn_mma, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        return true;
    }();
    (void)attr;
    k_attn_mma<<<ab.n * ab.batch * splits, kThreads, smem, st>>>(ab, maps, splits, tps);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (ev) cudaEventRecord(ev[0], st);
    if (splits > 1) {
        dim3 g(ab.H, ab.batch, ab.n);
        k_attn_mma_combine<<<g, 128, 0, st>>>(ab, splits);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess && ev) cudaEventRecord(ev[1], st);
    return e;
}

}  // namespace csa2
