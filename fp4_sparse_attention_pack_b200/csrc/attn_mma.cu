// Sparse + window attention on the 5th-generation tensor cores (tcgen05.mma
// kind::f16, fp16 operands, fp32 accumulation in TMEM).
//
// Per (problem, sequence) the items are the K selected entries (dequantised
// from E2M1 x E4M3: exact in fp16) and the valid window tokens (bf16 -> fp16,
// exact for |x| in fp16's normal range; E4M3 -> fp16, always exact, for an FP8
// window); the latent item is key and value.
// Items go through 128-item tiles with an online softmax:
//
//   S^T[128 items x 64 heads] = Items . Q^T            (M = 128, N = 64, K = 512)
//   P^T = exp(scale * S^T - m_head)                    (fp16, per item lane)
//   O^T[4 x 128 latent x 64 heads] += Items^T . P^T    (M = 128, N = 64, K = 128)
//
// One shared-memory image of the tile serves both MMAs: 128-byte-swizzled
// slabs of 64 latent channels, read as the K-major A operand of S^T and as the
// MN-major A operand of O^T.  The running per-head maximum is only moved when
// a tile's maximum exceeds it by more than 8 (so p <= e^8 fits fp16), which
// makes the O rescale (TMEM load, scale, store) rare.  Heads are padded to 64.
//
// CTA = 512 threads, one unit (problem, sequence, split of tiles) per CTA.
// Gather: the unit's selected entries and window are prefetched into L2 first;
// window rows arrive by TMA (a 3-D tensor map per window, 128-byte swizzle, one
// box per slab, so they land directly in the slab layout and are converted
// bf16 -> fp16 in place); FP8 window rows (64 bytes a slab) are loaded with
// 16-byte loads when their tile is built; cache entries are loaded with 16-byte loads into
// registers one tile ahead (warp w: slab w % 8, rows 64 (w / 8) .. + 63, two rows
// per lane) and dequantised into the swizzled slab; a slab is rewritten as soon
// as the previous tile's O block that reads it has completed (the O MMAs commit
// per 128-channel block), so the gather overlaps O.  Warp 0 issues the MMAs (one
// elected lane, the warp converged); all sixteen warps run the softmax (four per
// TMEM lane quadrant, 16 heads each) and rescale / write O (one O^T block each).
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
constexpr int kThreads = 512;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;      // S^T: 64 columns
constexpr uint32_t kColO = 64;     // O^T: 4 x 64 columns
constexpr float kRescaleGap = 8.0f;

struct AttnMaps {
    CUtensorMap win[kMaxProblems];  // window [batch][128][512] bf16, box 64 x 128 x 1, SW128
};

struct __align__(1024) Smem {
    uint8_t items[8][kT * 128];    // 8 slabs x 128 rows x 128 B (SW128)
    uint8_t q[8][kHp * 128];       // 8 slabs x 64 rows x 128 B (SW128)
    uint8_t p[kT * 128];           // P^T: 128 item rows x 64 heads fp16 (SW128)
    float red[4][kHp];             // per-quadrant partial max / sum
    float m_used[kHp];
    float l[kHp];
    float alpha[kHp];
    int kind[2][kT];               // per tile buffer: 0 empty, 1 cache entry, 2 window token
    int64_t src_row[2][kT];        // entry row in the pools
    int n_entries[2];
    int has_window[2];
    uint64_t bar;                  // S MMA completion
    uint64_t ob[4];                // O MMA completion per 128-channel block (slabs 2c, 2c + 1)
    uint64_t wbar;                 // window TMA
    uint64_t drained;              // every MMA of the unit completed
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

// Reduce-scatter over the warp: v[N] per lane (N = 16, 32 or 64).  For N >= 32
// lane l ends with the reduction over the 32 lanes of element N/32 * l + i in
// v[i], i < N/32; for N = 16 lanes 2e and 2e + 1 both hold element e in v[0].
template <bool kMax, int N>
__device__ __forceinline__ void warp_reduce_scatter(float (&v)[N]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int step = 0; step < 5; ++step) {
        const int o = 16 >> step;
        const int half = (N / 2) >> step;
        if (half >= 1) {
            const bool upper = (lane & o) != 0;
#pragma unroll
            for (int i = 0; i < half; ++i) {
                const float keep = upper ? v[half + i] : v[i];
                const float send = upper ? v[i] : v[half + i];
                const float got = __shfl_xor_sync(0xffffffffu, send, o);
                v[i] = kMax ? fmaxf(keep, got) : keep + got;
            }
        } else {
            const float got = __shfl_xor_sync(0xffffffffu, v[0], o);
            v[0] = kMax ? fmaxf(v[0], got) : v[0] + got;
        }
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
    const int t_end = min(n_tiles, t_begin + tiles_per_split);

    if (tid == 0) {
        mbar_init(&sm.bar, 1);
        for (int c = 0; c < 4; ++c) mbar_init(&sm.ob[c], 1);
        mbar_init(&sm.wbar, 1);
        mbar_init(&sm.drained, 1);
        sm.n_entries[0] = sm.n_entries[1] = 0;
        sm.has_window[0] = sm.has_window[1] = 0;
        fence_mbar_init();
        prefetch_tmap(&maps.win[prob]);
    }
    if (warp == 0) tmem_alloc(&sm.tmem_base, kTmemCols);
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
    // Bring this unit's selected entries and window ring into L2 now, so that
    // every tile's gather below is served from L2 rather than waiting on DRAM.
    {
        const int p_end = min(K, t_end * kT);
        for (int pos = t_begin * kT + tid; pos < p_end; pos += kThreads) {
            const int e = P.idx[(int64_t)b * K + pos];
            if (e >= 0 && e < n) {
                const int pg = page_of(P.cache, b, e);
                if (pg >= 0) {
                    const int64_t ent = (int64_t)pg * PAGE + (e % PAGE);
                    bulk_prefetch_l2(P.cache.main_codes + ent * MCB, MCB);
                    bulk_prefetch_l2(P.cache.main_scales + ent * MSB, MSB);
                }
            }
        }
        if (tid == 0 && t_end * kT > K && wlen > 0) {
            const int tb = P.win_fp8 ? 1 : 2;  // bytes a channel
            bulk_prefetch_l2(static_cast<const uint8_t*>(P.win) + (int64_t)b * WIN * D * tb, (uint32_t)wlen * D * tb);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // lane 0's copy: a value the compiler knows is warp-uniform, so the MMA
    // operands derived from it need no per-lane handling at issue
    const uint32_t tbase = __shfl_sync(0xffffffffu, sm.tmem_base, 0);
    uint32_t phase = 0, wphase = 0;
    bool o_init = false;
    bool timed_out = false;

    const uint32_t idesc_s = idesc_f16(128, kHp, 0, 0, 0);
    const uint32_t idesc_o = idesc_f16(128, kHp, 0, 1, 1);
    const uint64_t desc_items = smem_desc(sm.items[0], 16, 1024, kLayoutSw128);
    const uint64_t desc_q = smem_desc(sm.q[0], 16, 1024, kLayoutSw128);
    const uint64_t desc_vt = smem_desc(sm.items[0], 16384, 1024, kLayoutSw128);
    const uint64_t desc_p = smem_desc(sm.p, 16384, 1024, kLayoutSw128);

    // Where each item of tile t comes from (one thread per item), into buffer buf.
    auto lookup = [&](int t, int buf) {
        if (tid < kT) {
            const int pos = t * kT + tid;
            int kind = 0;
            int64_t row = -1;
            if (pos < K) {
                const int e = P.idx[(int64_t)b * K + pos];
                if (e >= 0 && e < n) {
                    const int pg = page_of(P.cache, b, e);
                    if (pg >= 0) {
                        kind = 1;
                        row = (int64_t)pg * PAGE + (e % PAGE);
                    }
                }
            } else if (pos - K < wlen) {
                kind = P.win_fp8 ? 3 : 2;
                row = (int64_t)b * WIN + (pos - K);
            }
            sm.kind[buf][tid] = kind;
            sm.src_row[buf][tid] = row;
            const unsigned ent = __ballot_sync(0xffffffffu, kind == 1);
            const unsigned win = __ballot_sync(0xffffffffu, kind == 2);
            if (lane == 0) {
                if (ent) atomicAdd(&sm.n_entries[buf], __popc(ent));
                if (win) sm.has_window[buf] = 1;
            }
        }
    };
    // Packed bytes of the tile's cache entries: warp w takes slab w & 7 of rows
    // 64 (w >> 3) .. 64 (w >> 3) + 63, lane = rows lane + 32 i of that half.
    const int g_slab = warp & 7, g_row0 = 64 * (warp >> 3);
    uint4 raw0[2], raw1[2];
    uint32_t raws[2];
    auto load_entries = [&](int buf) {
        const int j = g_slab;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int r = g_row0 + lane + 32 * i;
            if (sm.kind[buf][r] == 1) {
                const int64_t ent = sm.src_row[buf][r];
                const uint4* cs = reinterpret_cast<const uint4*>(P.cache.main_codes + ent * MCB + 32 * j);
                raw0[i] = __ldg(cs);
                raw1[i] = __ldg(cs + 1);
                raws[i] = __ldg(reinterpret_cast<const uint32_t*>(P.cache.main_scales + ent * MSB + 4 * j));
            } else {
                raw0[i] = raw1[i] = make_uint4(0, 0, 0, 0);
                raws[i] = 0;
            }
        }
    };

    int buf = 0;
    if (t_begin < t_end) {
        lookup(t_begin, 0);
        __syncthreads();
        load_entries(0);
    }
    for (int t = t_begin; t < t_end && !timed_out; ++t, buf ^= 1) {
        const bool has_window = sm.has_window[buf] != 0;
        // The O MMAs of the previous tile read slabs 2c, 2c + 1 in block c; a slab is
        // rewritten once its block has completed (phase of the previous tile's O).
        const uint32_t opar = (uint32_t)(t - t_begin - 1) & 1u;
        // ---- window rows by TMA, one 64-channel box per slab, once every block of
        // the previous tile's O has completed (the last block's commit covers all)
        if (warp == 0 && has_window) {
            if (o_init && !mbar_wait_warp(&sm.ob[3], opar)) timed_out = true;
            mbar_expect_tx_w(&sm.wbar, 8 * kT * 128);
#pragma unroll
            for (int j = 0; j < 8; ++j) tma_load_3d_w(sm.items[j], &maps.win[prob], 64 * j, t * kT - K, b, &sm.wbar);
        }
        // ---- cache entries (bytes already in registers): warp = (slab, row half), lane = row.
        // The window boxes cover all 128 rows, so they must land first.
        if (has_window) {
            if (!mbar_wait(&sm.wbar, wphase)) timed_out = true;
            wphase ^= 1;
        } else if (o_init) {
            if (!mbar_wait(&sm.ob[g_slab >> 1], opar)) timed_out = true;
        }
        {
            const int j = g_slab;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int r = g_row0 + lane + 32 * i;
                const int kind = sm.kind[buf][r];
                if (kind == 2) {
                    bf16_row_to_f16(sm.items[j], r);
                } else if (kind == 3) {
                    // FP8 window token: the slab's 64 E4M3 codes -> fp16 (exact)
                    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(P.win) +
                                                                      sm.src_row[buf][r] * D + 64 * j);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const uint4 u = __ldg(src + q4);
                        const uint32_t cw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc) {  // 16-byte chunk 2 q4 + cc: channels 8 (2 q4 + cc) ..
                            uint4 o;
                            o.x = e4m3x2_to_h2(cw[2 * cc] & 0xFFFFu);
                            o.y = e4m3x2_to_h2(cw[2 * cc] >> 16);
                            o.z = e4m3x2_to_h2(cw[2 * cc + 1] & 0xFFFFu);
                            o.w = e4m3x2_to_h2(cw[2 * cc + 1] >> 16);
                            *reinterpret_cast<uint4*>(sm.items[j] + sw128(r, 2 * q4 + cc)) = o;
                        }
                    }
                } else if (kind == 0) {
                    zero_row(sm.items[j], r);
                } else {
                    const uint32_t cw[8] = {raw0[i].x, raw0[i].y, raw0[i].z, raw0[i].w,
                                            raw1[i].x, raw1[i].y, raw1[i].z, raw1[i].w};
#pragma unroll
                    for (int c2 = 0; c2 < 4; ++c2) {  // chunks 2*c2, 2*c2+1 share scale byte c2
                        const __half2 s2 = __float2half2_rn(e4m3_decode_pos((raws[i] >> (8 * c2)) & 0xFFu));
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
                            *reinterpret_cast<uint4*>(sm.items[j] + sw128(r, c)) = o;
                        }
                    }
                }
            }
        }
        if (tid == 0) {
            sm.n_entries[buf ^ 1] = 0;
            sm.has_window[buf ^ 1] = 0;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        if (__syncthreads_or(timed_out)) {
            timed_out = true;
            break;
        }

        // ---- S^T = Items . Q^T, and meanwhile the next tile's lookups
        if (warp == 0) {
            tc_fence_after();
#pragma unroll 4
            for (int ks = 0; ks < 32; ++ks) {  // 16 latent channels per MMA
                const uint32_t off = (uint32_t)((ks >> 2) * (kT * 128) + (ks & 3) * 32) >> 4;
                const uint32_t offq = (uint32_t)((ks >> 2) * (kHp * 128) + (ks & 3) * 32) >> 4;
                tc_mma_f16_w(tbase + kColS, desc_items + off, desc_q + offq, idesc_s, ks > 0 ? 1u : 0u);
            }
            tc_commit_w(&sm.bar);
        }
        if (t + 1 < t_end) lookup(t + 1, buf ^ 1);
        if (!mbar_wait(&sm.bar, phase)) timed_out = true;
        phase ^= 1;
        if (__syncthreads_or(timed_out)) {
            timed_out = true;
            break;
        }
        tc_fence_after();

        // ---- softmax statistics: warp = (quadrant, 16 heads); thread = item row
        const int quad = warp & 3, hq = warp >> 2;
        const int row = quad * 32 + lane;
        const uint32_t s_addr = tbase + ((uint32_t)(quad * 32) << 16) + kColS + 16 * hq;
        const bool ok = sm.kind[buf][row] != 0;
        {
            float v[16];
            tmem_ld_32x32b_x16(s_addr, v);
#pragma unroll
            for (int h = 0; h < 16; ++h) v[h] = ok ? v[h] * ab.scale : -INFINITY;
            warp_reduce_scatter<true, 16>(v);
            if ((lane & 1) == 0) sm.red[quad][16 * hq + (lane >> 1)] = v[0];
        }
        __syncthreads();
        bool rescale = false;
        if (tid < kHp) {
            const float mt = fmaxf(fmaxf(sm.red[0][tid], sm.red[1][tid]), fmaxf(sm.red[2][tid], sm.red[3][tid]));
            const float mo = sm.m_used[tid];
            float a = 1.0f;
            if (mt > mo + kRescaleGap || (mo == -INFINITY && mt != -INFINITY)) {
                a = (mo == -INFINITY) ? 0.0f : expf(mo - mt);
                sm.m_used[tid] = mt;
                rescale = o_init && mo != -INFINITY;
            }
            sm.alpha[tid] = a;
        }
        rescale = __syncthreads_or(rescale);

        // ---- P^T = exp(s - m) in fp16 (S reloaded from TMEM), row sums of the rounded p
        {
            float v[16];
            tmem_ld_32x32b_x16(s_addr, v);
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint4 o;
                uint32_t* os = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int h = 8 * c + 2 * k;
                    const float p0 = ok ? __expf(v[h] * ab.scale - sm.m_used[16 * hq + h]) : 0.0f;
                    const float p1 = ok ? __expf(v[h + 1] * ab.scale - sm.m_used[16 * hq + h + 1]) : 0.0f;
                    const __half2 hv = __floats2half2_rn(p0, p1);
                    const float2 back = __half22float2(hv);
                    v[h] = back.x;
                    v[h + 1] = back.y;
                    os[k] = *reinterpret_cast<const uint32_t*>(&hv);
                }
                *reinterpret_cast<uint4*>(sm.p + sw128(row, 2 * hq + c)) = o;
            }
            warp_reduce_scatter<false, 16>(v);
            // the max pass read red[] before the barrier above; reuse it for sums
            if ((lane & 1) == 0) sm.red[quad][16 * hq + (lane >> 1)] = v[0];
        }
        // ---- rescale O^T where a head's reference maximum moved (warp = quadrant, block hq)
        if (rescale) {
            const uint32_t ta = tbase + ((uint32_t)(quad * 32) << 16) + kColO + 64 * hq;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float o[32];
                tmem_ld_32x32b_x32(ta + 32 * half, o);
#pragma unroll
                for (int h = 0; h < 32; ++h) o[h] *= sm.alpha[32 * half + h];
                tmem_st_32x32b_x32(ta + 32 * half, o);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid < kHp)
            sm.l[tid] = sm.l[tid] * sm.alpha[tid] + (sm.red[0][tid] + sm.red[1][tid]) + (sm.red[2][tid] + sm.red[3][tid]);

        // ---- O^T += Items^T . P^T
        if (warp == 0) {
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
#pragma unroll 4
                for (int i = 0; i < 8; ++i) {  // 16 items per MMA
                    const uint32_t offa = (uint32_t)(2 * c * (kT * 128) + 2048 * i) >> 4;
                    const uint32_t offp = (uint32_t)(2048 * i) >> 4;
                    tc_mma_f16_w(tbase + kColO + 64 * c, desc_vt + offa, desc_p + offp, idesc_o,
                                 (o_init || i > 0) ? 1u : 0u);
                }
                tc_commit_w(&sm.ob[c]);
            }
        }
        o_init = true;
        // the next tile's gather overlaps these MMAs, slab pair by slab pair
        if (t + 1 < t_end) load_entries(buf ^ 1);
        if (__syncthreads_or(timed_out)) {
            timed_out = true;
            break;
        }
        tc_fence_after();
    }

    // the last tile's O has completed before it is read (its last block covers all)
    if (!timed_out && o_init) {
        const bool ok = mbar_wait(&sm.ob[3], (uint32_t)(t_end - t_begin - 1) & 1u);
        timed_out = __syncthreads_or(!ok);
        tc_fence_after();
    }
    if (timed_out) {
        if (tid == 0 && K > 0) atomicOr(P.cache.status, CSA2_DEVERR_TIMEOUT);
    } else {
        // ---- write O (normalised) or the split's partial (O, m, l)
        const int quad = warp & 3;
        const bool partial = splits > 1;
        float* dst = partial ? ab.part_o + (int64_t)unit * H * D : P.out + (int64_t)b * H * D;
        {
            const int c = warp >> 2;  // O^T block of this warp: latent 128 c + quad * 32 + lane
            const int lat = 128 * c + quad * 32 + lane;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float o[32];
                if (o_init) {
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
    // a timed-out wait may leave copies in flight: let them land before the CTA exits
    if (tid == 0) {
        (void)mbar_wait(&sm.wbar, wphase ^ 1);
    }
    // every MMA of warp 0 has completed before TMEM is freed
    if (warp == 0) {
        tc_commit_w(&sm.drained);
        (void)mbar_wait_warp(&sm.drained, 0);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
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


}  // namespace

// Splits of the item tiles per (problem, sequence): enough units to fill the
// SMs when the batch is small, none when there are already plenty.
int attn_mma_splits(int n_problems, int batch, int Kmax) {
    const int tiles = (Kmax + WIN + kT - 1) / kT;
    const int pairs = n_problems * batch;
    const int want = (device_sm_count() + pairs - 1) / pairs;
    return std::max(1, std::min(tiles, want));
}

bool attn_mma_supported(const AttnBatch& ab) { return ab.H >= 1 && ab.H <= kHp; }

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
    for (int i = 0; i < ab.n; ++i)  // FP8 windows are gathered, not loaded by TMA
        if (!ab.p[i].win_fp8 && !make_window_map(&maps.win[i], ab.p[i].win, ab.batch)) return cudaErrorInvalidValue;
    const int splits = attn_mma_splits(ab.n, ab.batch, ab.Kmax);
    const int tiles = (ab.Kmax + WIN + kT - 1) / kT;
    const int tps = (tiles + splits - 1) / splits;
    if (splits > 1) {
        const size_t units = (size_t)ab.n * ab.batch * splits;
        ab.part_ml = ab.part_o + units * ab.H * D;
    }
    const size_t smem = sizeof(Smem) + 1024;
    static std::atomic<uint64_t> attr_done{0};
    const cudaError_t ea = smem_opt_in(reinterpret_cast<const void*>(k_attn_mma), (int)smem, attr_done);
    if (ea != cudaSuccess) return ea;
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
