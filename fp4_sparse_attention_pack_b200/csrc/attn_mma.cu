// Sparse + window attention on the 5th-generation tensor cores (tcgen05.mma
// kind::f16, fp16 operands, fp32 accumulation in TMEM).
//
// Per (problem, sequence) the items are the K selected entries (dequantised
// from E2M1 x E4M3: exact in fp16) and the valid window tokens (bf16 -> fp16,
// exact for |x| in fp16's normal range, saturated at +-65504; E4M3 -> fp16,
// always exact, for an FP8 window); the latent item is key and value.  Each
// head's bf16 query row is multiplied by a power of two 2^k_h that brings its
// largest magnitude into [2^14, 2^15) before it is rounded to fp16 (exact for
// every bf16 value within 2^24 of the row's maximum), and 2^-k_h is folded
// into that head's softmax scale, so no query magnitude overflows.
// Items go through 128-item tiles with an online softmax:
//
//   S^T[128 items x 64 heads] = Items . Q^T            (M = 128, N = 64, K = 512)
//   P^T = exp(scale_h * S^T - m_h)                     (fp16, per item lane)
//   O^T[4 x 128 latent x 64 heads] += Items^T . P^T    (M = 128, N = 64, K = 128)
//
// One shared-memory image of the tile serves both MMAs: 128-byte-swizzled
// slabs of 64 latent channels, read as the K-major A operand of S^T and as the
// MN-major A operand of O^T.  The reference maximum m_h only moves when a
// tile's maximum exceeds it by more than 8 (so p <= e^8 fits fp16); the O
// rescale that a move needs is rare, and a tile that moves no maximum needs no
// cross-item reduction at all: every thread tests its own item against m_h and
// one barrier ORs the tests.
//
// Persistent CTAs (one per SM, 448 threads) walk their units (problem,
// sequence, split of tiles) tile by tile; warps specialise and hand work over
// through mbarriers, never through a block-wide barrier:
//   warp 0      issues the MMAs (one elected lane): S^T of a tile slab pair by
//               slab pair as the pairs are written, then O^T block by block;
//   warp 1      resolves each tile's 128 items (selected index -> page -> entry
//               row, or window slot) two tiles ahead, and prefetches the window
//               rows and the next unit's query into L2;
//   warps 2-5   softmax: thread = item row (TMEM lane), all 64 heads; P^T into
//               shared memory, the per-lane partial row sums in TMEM; at the end
//               of a unit the O^T readout, normalised (or the split's partial);
//   warps 6-13  gather: warp g owns slab g (latent channels 64g .. 64g + 63);
//               each tile's entry bytes are loaded into registers a tile ahead
//               and dequantised into the slab once the previous tile's O block
//               that reads it has completed; bf16 window rows arrive by TMA
//               (issued by warp 13, which waits for the last O block) and are
//               converted in place; the unit's query is converted in the slab
//               layout.
// A waiter only ever waits for the phase right after the last one it saw
// complete: a wait further ahead would alias an older phase of the same parity.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
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
constexpr int kWarpMma = 0, kWarpProd = 1, kWarpSoft = 2, kWarpGath = 6;
constexpr int kSoftWarps = 4, kGathWarps = 8;
constexpr int kThreads = 32 * (kWarpGath + kGathWarps);  // 448
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;      // O^T: 4 blocks x 64 heads
constexpr uint32_t kColS = 256;    // S^T: 64 heads
constexpr uint32_t kColL = 320;    // per-lane partial row sums of P: 64 heads
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kGap2 = 8.0f * kLog2e;  // the reference maximum moves beyond e^8 (log2 units)
constexpr int kBarSoft = 1, kBarGath = 2;  // named barriers of the softmax and gather warps

struct AttnMaps {
    CUtensorMap win[kMaxProblems];  // window [batch][128][512] bf16, box 64 x 128 x 1, SW128
};

struct __align__(1024) Smem {
    uint8_t items[8][kT * 128];    // 8 slabs x 128 rows x 128 B (SW128)
    uint8_t q[8][kHp * 128];       // 8 slabs x 64 rows x 128 B (SW128)
    uint8_t p[kT * 128];           // P^T: 128 item rows x 64 heads fp16 (SW128)
    int64_t src_row[2][kT];        // per tile buffer: entry row in the pools, or window row
    int kind[2][kT];               // 0 empty, 1 cache entry, 2 bf16 window token, 3 E4M3 window token
    int tile_win[2];               // the tile holds bf16 window rows (loaded by TMA)
    float a2[2][kHp];              // per unit parity: scale * 2^-k_h * log2(e)
    uint32_t qmax[kGathWarps][kHp];  // per slab: largest |q| bf16 magnitude bits of a head
    float mu2[kHp];                // reference maximum per head (log2 units)
    float alpha[kHp];              // O / row-sum rescale factor of a move
    float red[4][kHp];             // per-quadrant partial max / sum
    float lfin[kHp];               // row sum of the unit
    uint64_t lk_full[2], lk_empty[2];  // item lookups: producer -> gather + softmax warps
    uint64_t q_ready[2];           // the unit's query converted (per unit parity)
    uint64_t q_empty;              // every S^T MMA of the unit completed
    uint64_t w_full;               // window TMA landed
    uint64_t it_full[4];           // slab pair c of the tile written
    uint64_t s_full;               // S^T complete
    uint64_t p_full;               // P^T written, S^T read
    uint64_t o_blk[4];             // O^T block c complete (block 3: the whole tile)
    uint64_t drained;              // every MMA of the CTA completed
    uint32_t tmem_base;
    int abort;                     // a bounded wait gave up: every role winds down
};
static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory beyond the 227 KB per-block limit");

// Byte offset of 16-byte chunk c of row r inside a 128B-swizzled slab.
__device__ __forceinline__ uint32_t sw128(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

// Two E2M1 codes (one byte, channel 2i in the low nibble) -> f16x2 (low half first).
__device__ __forceinline__ uint32_t e2m1x2_to_h2(uint32_t byte) {
    uint32_t out;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(out) : "r"(byte));
    return out;
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void named_bar(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// OR of v over the n threads of named barrier id (a barrier as well).
__device__ __forceinline__ bool named_bar_or(int id, int n, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

// Bounded wait that also gives up at once when another role has given up, so
// that every role winds down within one bound of the first failure.
__device__ __forceinline__ bool wait_bar(Smem& sm, uint64_t* bar, uint32_t parity) {
    if (mbar_try(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        if (*reinterpret_cast<volatile int*>(&sm.abort)) return false;
        if (mbar_try_sleep(bar, parity, 20000u)) return true;
        if (global_ns() - t0 > kWaitNs) {
            atomicExch(&sm.abort, 1);
            return false;
        }
    }
}

__device__ __forceinline__ bool wait_bar_warp(Smem& sm, uint64_t* bar, uint32_t parity) {
    const bool ok = wait_bar(sm, bar, parity);
    return __all_sync(0xffffffffu, ok);
}

// Reduce-scatter over the warp of 32 values per lane: lane l ends with the
// reduction over the 32 lanes of element l in v[0].
template <bool kMax>
__device__ __forceinline__ float warp_reduce_scatter32(float (&v)[32]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int step = 0; step < 5; ++step) {
        const int o = 16 >> step;
        const int half = 16 >> step;
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float keep = upper ? v[half + i] : v[i];
            const float send = upper ? v[i] : v[half + i];
            const float got = __shfl_xor_sync(0xffffffffu, send, o);
            v[i] = kMax ? fmaxf(keep, got) : keep + got;
        }
    }
    return v[0];
}

// The unit a CTA takes k-th (units are strided over the CTAs).
struct Unit {
    int unit, prob, b, t0, t1;
};

__device__ __forceinline__ bool unit_at(const AttnBatch& ab, int splits, int tps, int k, Unit& u) {
    const int unit = blockIdx.x + k * gridDim.x;
    if (unit >= ab.n * ab.batch * splits) return false;
    const int split = unit % splits, pb = unit / splits;
    u.unit = unit;
    u.b = pb % ab.batch;
    u.prob = pb / ab.batch;
    const int n_tiles = (ab.p[u.prob].K + WIN + kT - 1) / kT;
    u.t0 = split * tps;
    u.t1 = min(n_tiles, u.t0 + tps);
    return true;
}

// Valid window tokens of sequence b.
__device__ __forceinline__ int window_len(const AttnProblem& P, int b) {
    const int c = P.win_count[b];
    return c < 0 ? 0 : (c < WIN ? c : WIN);
}

// ---------------------------------------------------------------- warp 1: items and window

__device__ void role_producer(Smem& sm, const AttnBatch& ab, int splits, int tps) {
    const int lane = threadIdx.x & 31;
    bool alive = true;
    uint32_t it = 0;
    Unit u;
    for (int k = 0; unit_at(ab, splits, tps, k, u); ++k) {
        // the next unit's query into L2 while this unit runs
        Unit nu;
        if (lane == 0 && unit_at(ab, splits, tps, k + 1, nu) && nu.t0 < nu.t1)
            bulk_prefetch_l2(ab.p[nu.prob].q + (int64_t)nu.b * ab.H * D, (uint32_t)(ab.H * D * 2));
        if (u.t0 >= u.t1) continue;
        const AttnProblem& P = ab.p[u.prob];
        const int K = P.K, b = u.b;
        const int wlen = window_len(P, b);
        const int n = K > 0 ? entries_of(P.cache, b) : 0;
        for (int t = u.t0; t < u.t1; ++t, ++it) {
            const int buf = it & 1;
            if (it >= 2) alive = wait_bar_warp(sm, &sm.lk_empty[buf], ((it >> 1) - 1) & 1u) && alive;
            bool win = false;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = lane + 32 * i;
                const int pos = t * kT + r;
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
                sm.kind[buf][r] = kind;
                sm.src_row[buf][r] = row;
                win |= kind == 2;
            }
            win = __any_sync(0xffffffffu, win);
            if (lane == 0) sm.tile_win[buf] = win;
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.lk_full[buf]);
            // the window rows this tile's TMA will read, into L2 two tiles ahead
            if (win && lane == 0) {
                const int r0 = max(0, t * kT - K), r1 = min(wlen, t * kT + kT - K);
                bulk_prefetch_l2(static_cast<const uint8_t*>(P.win) + ((int64_t)b * WIN + r0) * D * 2,
                                 (uint32_t)(r1 - r0) * D * 2);
            }
        }
    }
}

// ---------------------------------------------------------------- warp 0: MMA issue

__device__ void role_mma(Smem& sm, const AttnBatch& ab, int splits, int tps, uint32_t tbase) {
    const uint32_t idesc_s = idesc_f16(128, kHp, 0, 0, 0);
    const uint32_t idesc_o = idesc_f16(128, kHp, 0, 1, 1);
    const uint64_t desc_items = smem_desc(sm.items[0], 16, 1024, kLayoutSw128);
    const uint64_t desc_q = smem_desc(sm.q[0], 16, 1024, kLayoutSw128);
    const uint64_t desc_vt = smem_desc(sm.items[0], 16384, 1024, kLayoutSw128);
    const uint64_t desc_p = smem_desc(sm.p, 16384, 1024, kLayoutSw128);
    bool alive = true;
    uint32_t it = 0, ku = 0;
    Unit u;
    for (int k = 0; unit_at(ab, splits, tps, k, u); ++k) {
        if (u.t0 >= u.t1) continue;
        alive = wait_bar_warp(sm, &sm.q_ready[ku & 1], (ku >> 1) & 1u) && alive;
        for (int t = u.t0; t < u.t1; ++t, ++it) {
            // S^T = Items . Q^T, slab pair by slab pair as the gather warps finish them
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                alive = wait_bar_warp(sm, &sm.it_full[c], it & 1u) && alive;
                tc_fence_after();
                if (alive) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {  // 16 latent channels per MMA
                        const int ks = 8 * c + kk;
                        const uint32_t off = (uint32_t)((ks >> 2) * (kT * 128) + (ks & 3) * 32) >> 4;
                        const uint32_t offq = (uint32_t)((ks >> 2) * (kHp * 128) + (ks & 3) * 32) >> 4;
                        tc_mma_f16_w(tbase + kColS, desc_items + off, desc_q + offq, idesc_s, ks > 0 ? 1u : 0u);
                    }
                }
            }
            if (alive) {
                tc_commit_w(&sm.s_full);
                if (t + 1 == u.t1) tc_commit_w(&sm.q_empty);
            }
            // O^T += Items^T . P^T, one commit per 128-channel block (slabs 2c, 2c + 1)
            alive = wait_bar_warp(sm, &sm.p_full, it & 1u) && alive;
            tc_fence_after();
            if (alive) {
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {  // 16 items per MMA
                        const uint32_t offa = (uint32_t)(2 * c * (kT * 128) + 2048 * i) >> 4;
                        const uint32_t offp = (uint32_t)(2048 * i) >> 4;
                        tc_mma_f16_w(tbase + kColO + 64 * c, desc_vt + offa, desc_p + offp, idesc_o,
                                     (t > u.t0 || i > 0) ? 1u : 0u);
                    }
                    tc_commit_w(&sm.o_blk[c]);
                }
            }
        }
        ++ku;
    }
}

// ---------------------------------------------------------------- warps 6-13: gather

// The unit's query, slab g (channels 64g .. 64g + 63) of all 64 head rows,
// scaled per head by 2^k_h and rounded to fp16; lane l owns heads l and l + 32.
// k_h brings the head's largest bf16 magnitude into [2^14, 2^15).
__device__ void convert_query(Smem& sm, const AttnBatch& ab, const Unit& u, int g, uint32_t ku, bool alive) {
    const int lane = threadIdx.x & 31;
    const int H = ab.H;
    const uint16_t* qb = ab.p[u.prob].q + (int64_t)u.b * H * D + 64 * g;
#pragma unroll 1
    for (int half = 0; half < 2; ++half) {
        const int h = lane + 32 * half;
        uint4 w[8];
#pragma unroll
        for (int c = 0; c < 8; ++c)
            w[c] = h < H ? __ldg(reinterpret_cast<const uint4*>(qb + (int64_t)h * D) + c) : make_uint4(0, 0, 0, 0);
        uint32_t m = 0;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            m = __vmaxu2(m, w[c].x & 0x7FFF7FFFu);
            m = __vmaxu2(m, w[c].y & 0x7FFF7FFFu);
            m = __vmaxu2(m, w[c].z & 0x7FFF7FFFu);
            m = __vmaxu2(m, w[c].w & 0x7FFF7FFFu);
        }
        sm.qmax[g][h] = max(m & 0xFFFFu, m >> 16);
        named_bar(kBarGath, 32 * kGathWarps);
        uint32_t mh = 0;
#pragma unroll
        for (int j = 0; j < kGathWarps; ++j) mh = max(mh, sm.qmax[j][h]);
        // bf16 magnitude bits: exponent field E = mh >> 7; the maximum lies in
        // [2^(E-127), 2^(E-126)), so k = 141 - E puts it in [2^14, 2^15)
        const int E = (int)(mh >> 7);
        const int kx = mh == 0 ? 0 : min(126, 141 - E);
        const float mul = __uint_as_float((uint32_t)(127 + kx) << 23);
        if (g == 0) sm.a2[ku & 1][h] = ab.scale * __uint_as_float((uint32_t)(127 - kx) << 23) * kLog2e;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const uint32_t ws[4] = {w[c].x, w[c].y, w[c].z, w[c].w};
            uint4 o;
            uint32_t* os = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const __half2 hv = __floats2half2_rn(__uint_as_float(ws[e] << 16) * mul,
                                                     __uint_as_float(ws[e] & 0xFFFF0000u) * mul);
                os[e] = *reinterpret_cast<const uint32_t*>(&hv);
            }
            if (alive) *reinterpret_cast<uint4*>(sm.q[g] + sw128(h, c)) = o;
        }
        // no barrier after the reads: the two halves use disjoint heads, and a
        // warp writes this half's heads again (next unit) only after every warp
        // has passed the other half's barrier
    }
}

// bf16 pair -> f16x2, saturated to fp16's finite range
__device__ __forceinline__ uint32_t bf16x2_to_h2_sat(uint32_t w) {
    const float lo = fminf(fmaxf(__uint_as_float(w << 16), -65504.0f), 65504.0f);
    const float hi = fminf(fmaxf(__uint_as_float(w & 0xFFFF0000u), -65504.0f), 65504.0f);
    const __half2 hv = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&hv);
}

__device__ void role_gather(Smem& sm, const AttnBatch& ab, const AttnMaps& maps, int splits, int tps) {
    const int lane = threadIdx.x & 31;
    const int g = (threadIdx.x >> 5) - kWarpGath;  // slab
    uint8_t* slab = sm.items[g];
    bool alive = true;
    uint32_t it = 0, ku = 0, wn = 0, w_issued = 0;
    Unit u;
    for (int k = 0; unit_at(ab, splits, tps, k, u); ++k) {
        if (u.t0 >= u.t1) continue;
        const AttnProblem& P = ab.p[u.prob];
        for (int t = u.t0; t < u.t1; ++t, ++it) {
            const int buf = it & 1;
            alive = wait_bar_warp(sm, &sm.lk_full[buf], (it >> 1) & 1u) && alive;
            // this tile's rows lane + 32 i: their kind, and the entry bytes of slab g
            int kd[4];
            uint4 c0[4], c1[4];
            uint32_t sc[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = lane + 32 * i;
                kd[i] = sm.kind[buf][r];
                if (kd[i] == 1) {
                    const int64_t rw = sm.src_row[buf][r];
                    const uint4* cs = reinterpret_cast<const uint4*>(P.cache.main_codes + rw * MCB + 32 * g);
                    c0[i] = __ldg(cs);
                    c1[i] = __ldg(cs + 1);
                    sc[i] = __ldg(reinterpret_cast<const uint32_t*>(P.cache.main_scales + rw * MSB + 4 * g));
                } else {
                    c0[i] = c1[i] = make_uint4(0, 0, 0, 0);
                    sc[i] = 0;
                }
            }
            const bool win = sm.tile_win[buf] != 0;
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.lk_empty[buf]);

            if (t == u.t0) {
                // the unit's query: once the previous unit's S^T MMAs have completed
                if (ku > 0) alive = wait_bar_warp(sm, &sm.q_empty, (ku - 1) & 1u) && alive;
                convert_query(sm, ab, u, g, ku, alive);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.q_ready[ku & 1]);
            }
            // slab g is free once the previous tile's O block g / 2 has completed
            // (every gather warp waits for every tile in order, so the parity
            // never aliases an older phase)
            if (it > 0) alive = wait_bar_warp(sm, &sm.o_blk[g >> 1], (it - 1) & 1u) && alive;
            if (win) {
                // bf16 window rows by TMA, one 64-channel box per slab, covering all
                // 128 rows of every slab: issued by the warp that waited for block 3
                // (the previous tile's last O block, so all of its O)
                if (g == kGathWarps - 1 && alive) {
                    if (lane == 0) {
                        mbar_expect_tx(&sm.w_full, 8 * kT * 128);
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            tma_load_3d(sm.items[j], &maps.win[u.prob], 64 * j, t * kT - P.K, u.b, &sm.w_full);
                    }
                    ++w_issued;
                }
                alive = wait_bar_warp(sm, &sm.w_full, wn & 1u) && alive;
                ++wn;
            }
            if (alive) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int r = lane + 32 * i;
                    if (kd[i] == 1) {
                        const uint32_t cw[8] = {c0[i].x, c0[i].y, c0[i].z, c0[i].w, c1[i].x, c1[i].y, c1[i].z, c1[i].w};
#pragma unroll
                        for (int c2 = 0; c2 < 4; ++c2) {  // chunks 2 c2, 2 c2 + 1 share scale byte c2
                            const __half2 s2 = __float2half2_rn(e4m3_decode_pos((sc[i] >> (8 * c2)) & 0xFFu));
#pragma unroll
                            for (int cc = 0; cc < 2; ++cc) {
                                const int c = 2 * c2 + cc;
                                uint4 o;
                                uint32_t* os = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const uint32_t hh = e2m1x2_to_h2((cw[c] >> (8 * e)) & 0xFFu);
                                    const __half2 v = __hmul2(*reinterpret_cast<const __half2*>(&hh), s2);
                                    os[e] = *reinterpret_cast<const uint32_t*>(&v);
                                }
                                *reinterpret_cast<uint4*>(slab + sw128(r, c)) = o;
                            }
                        }
                    } else if (kd[i] == 2) {
                        // bf16 window row, landed by TMA in the slab layout: to fp16 in place
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            uint4* ptr = reinterpret_cast<uint4*>(slab + sw128(r, c));
                            const uint4 x = *ptr;
                            *ptr = make_uint4(bf16x2_to_h2_sat(x.x), bf16x2_to_h2_sat(x.y), bf16x2_to_h2_sat(x.z),
                                              bf16x2_to_h2_sat(x.w));
                        }
                    } else if (kd[i] == 3) {
                        // E4M3 window row (slot t * 128 + r - K of the ring): the slab's 64 codes -> fp16 (exact)
                        const int64_t rw = (int64_t)u.b * WIN + (t * kT + r - P.K);
                        const uint4* src =
                            reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(P.win) + rw * D + 64 * g);
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const uint4 x = __ldg(src + q4);
                            const uint32_t cw[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                            for (int cc = 0; cc < 2; ++cc) {
                                uint4 o;
                                o.x = e4m3x2_to_h2(cw[2 * cc] & 0xFFFFu);
                                o.y = e4m3x2_to_h2(cw[2 * cc] >> 16);
                                o.z = e4m3x2_to_h2(cw[2 * cc + 1] & 0xFFFFu);
                                o.w = e4m3x2_to_h2(cw[2 * cc + 1] >> 16);
                                *reinterpret_cast<uint4*>(slab + sw128(r, 2 * q4 + cc)) = o;
                            }
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(slab + sw128(r, c)) = make_uint4(0, 0, 0, 0);
                    }
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.it_full[g >> 1]);
        }
        ++ku;
    }
    // a window copy that was issued but not waited for lands before the CTA exits
    if (!alive && w_issued > 0 && lane == 0) (void)mbar_wait(&sm.w_full, (w_issued - 1) & 1u);
}

// ---------------------------------------------------------------- warps 2-5: softmax

// P^T for 32 heads of this thread's item: p = exp2(y) (0 for an empty item) to
// fp16 into chunks c0 .. c0 + 3 of the item's row; y is replaced by the
// rounded p (what the O MMA multiplies), so the row sums match it exactly.
__device__ __forceinline__ void store_p(uint8_t* prow_base, int row, int c0, bool ok, float (&y)[32]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint4 o;
        uint32_t* os = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int h = 8 * c + 2 * e;
            const float p0 = ok ? ex2(y[h]) : 0.0f;
            const float p1 = ok ? ex2(y[h + 1]) : 0.0f;
            const __half2 hv = __floats2half2_rn(p0, p1);
            const float2 back = __half22float2(hv);
            y[h] = back.x;
            y[h + 1] = back.y;
            os[e] = *reinterpret_cast<const uint32_t*>(&hv);
        }
        *reinterpret_cast<uint4*>(prow_base + sw128(row, c0 + c)) = o;
    }
}

__device__ void role_softmax(Smem& sm, const AttnBatch& ab, int splits, int tps, uint32_t tbase) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int quad = warp & 3;                 // TMEM lane quadrant of this warp
    const int row = 32 * quad + lane;          // item row (S^T) / latent row (O^T) of this thread
    const int st = threadIdx.x - 32 * kWarpSoft;  // 0 .. 127: per-head work for st < 64
    const uint32_t tl = tbase + ((uint32_t)(32 * quad) << 16);
    const int H = ab.H;
    const bool partial = splits > 1;
    bool alive = true;
    uint32_t it = 0, ku = 0;
    Unit u;
    for (int k = 0; unit_at(ab, splits, tps, k, u); ++k) {
        if (u.t0 >= u.t1) {  // a split without tiles: an empty partial
            if (partial && st < H) {
                ab.part_ml[((int64_t)u.unit * H + st) * 2 + 0] = -INFINITY;
                ab.part_ml[((int64_t)u.unit * H + st) * 2 + 1] = 0.0f;
            }
            continue;
        }
        if (st < kHp) sm.mu2[st] = -INFINITY;
        alive = wait_bar_warp(sm, &sm.q_ready[ku & 1], (ku >> 1) & 1u) && alive;
        named_bar(kBarSoft, 32 * kSoftWarps);
        const float* a2 = sm.a2[ku & 1];
        for (int t = u.t0; t < u.t1; ++t, ++it) {
            const int buf = it & 1;
            alive = wait_bar_warp(sm, &sm.lk_full[buf], (it >> 1) & 1u) && alive;
            const bool ok = sm.kind[buf][row] != 0;
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.lk_empty[buf]);
            alive = wait_bar_warp(sm, &sm.s_full, it & 1u) && alive;
            tc_fence_after();
            float y0[32], y1[32];
            // log2-domain exponent of every head against its reference maximum
            auto load_y = [&]() {
                tmem_ld_32x32b_x32(tl + kColS, y0);
                tmem_ld_32x32b_x32(tl + kColS + 32, y1);
#pragma unroll
                for (int h = 0; h < 32; ++h) {
                    y0[h] = y0[h] * a2[h] - sm.mu2[h];
                    y1[h] = y1[h] * a2[32 + h] - sm.mu2[32 + h];
                }
            };
            load_y();
            bool need = false;  // does this item move a head's maximum?
#pragma unroll
            for (int h = 0; h < 32; ++h) need |= (y0[h] > kGap2) | (y1[h] > kGap2);
            if (named_bar_or(kBarSoft, 32 * kSoftWarps, (ok && need) || !alive)) {
                // rare: the tile's maximum per head over the valid items (S^T reloaded)
                tmem_ld_32x32b_x32(tl + kColS, y0);
#pragma unroll
                for (int h = 0; h < 32; ++h) y0[h] = ok ? y0[h] * a2[h] : -INFINITY;
                sm.red[quad][lane] = warp_reduce_scatter32<true>(y0);
                tmem_ld_32x32b_x32(tl + kColS + 32, y1);
#pragma unroll
                for (int h = 0; h < 32; ++h) y1[h] = ok ? y1[h] * a2[32 + h] : -INFINITY;
                sm.red[quad][32 + lane] = warp_reduce_scatter32<true>(y1);
                named_bar(kBarSoft, 32 * kSoftWarps);
                bool resc = false;
                if (st < kHp) {
                    const float mt = fmaxf(fmaxf(sm.red[0][st], sm.red[1][st]), fmaxf(sm.red[2][st], sm.red[3][st]));
                    const float mo = sm.mu2[st];
                    float a = 1.0f;
                    if (mt > mo + kGap2 || (mo == -INFINITY && mt != -INFINITY)) {
                        a = (mo == -INFINITY) ? 0.0f : ex2(mo - mt);
                        sm.mu2[st] = mt;
                        resc = mo != -INFINITY;
                    }
                    sm.alpha[st] = a;
                }
                if (named_bar_or(kBarSoft, 32 * kSoftWarps, resc)) {
                    // rescale the earlier tiles' O^T and row sums (the previous tile's O complete)
                    alive = wait_bar_warp(sm, &sm.o_blk[3], (it - 1) & 1u) && alive;
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < 10; ++c) {  // four O^T blocks, then the row sums, 32 columns at a time
                        const uint32_t col = (c < 8 ? kColO + 32 * c : kColL + 32 * (c - 8));
                        const int h0 = 32 * (c & 1);
                        float o[32];
                        tmem_ld_32x32b_x32(tl + col, o);
#pragma unroll
                        for (int h = 0; h < 32; ++h) o[h] *= sm.alpha[h0 + h];
                        tmem_st_32x32b_x32(tl + col, o);
                    }
                }
                load_y();  // against the updated maxima
            }
            // P^T is free once the previous tile's O has completed
            if (it > 0) alive = wait_bar_warp(sm, &sm.o_blk[3], (it - 1) & 1u) && alive;
            store_p(sm.p, row, 0, ok, y0);
            store_p(sm.p, row, 4, ok, y1);
            // this lane's running row sums (of the rounded p) in TMEM
            if (t == u.t0) {
                tmem_st_32x32b_x32(tl + kColL, y0);
                tmem_st_32x32b_x32(tl + kColL + 32, y1);
            } else {
                float l[32];
                tmem_ld_32x32b_x32(tl + kColL, l);
#pragma unroll
                for (int h = 0; h < 32; ++h) l[h] += y0[h];
                tmem_st_32x32b_x32(tl + kColL, l);
                tmem_ld_32x32b_x32(tl + kColL + 32, l);
#pragma unroll
                for (int h = 0; h < 32; ++h) l[h] += y1[h];
                tmem_st_32x32b_x32(tl + kColL + 32, l);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.p_full);
        }

        // ---- end of the unit: row sums over the items, then O^T out
        alive = wait_bar_warp(sm, &sm.o_blk[3], (it - 1) & 1u) && alive;
        tc_fence_after();
        {
            float l[32];
            tmem_ld_32x32b_x32(tl + kColL, l);
            sm.red[quad][lane] = warp_reduce_scatter32<false>(l);
            tmem_ld_32x32b_x32(tl + kColL + 32, l);
            sm.red[quad][32 + lane] = warp_reduce_scatter32<false>(l);
        }
        named_bar(kBarSoft, 32 * kSoftWarps);
        if (st < kHp) {
            const float l = (sm.red[0][st] + sm.red[1][st]) + (sm.red[2][st] + sm.red[3][st]);
            sm.lfin[st] = partial ? l : (l > 0.0f ? 1.0f / l : 0.0f);
        }
        named_bar(kBarSoft, 32 * kSoftWarps);
        if (alive) {
            float* dst = partial ? ab.part_o + (int64_t)u.unit * H * D : ab.p[u.prob].out + (int64_t)u.b * H * D;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                const int lat = 128 * c + row;  // O^T block c, lane = latent channel
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float o[32];
                    tmem_ld_32x32b_x32(tl + kColO + 64 * c + 32 * half, o);
#pragma unroll
                    for (int h = 0; h < 32; ++h) {
                        const int hd = 32 * half + h;
                        if (hd < H) dst[(int64_t)hd * D + lat] = partial ? o[h] : o[h] * sm.lfin[hd];
                    }
                }
            }
            if (partial && st < H) {
                const float m2 = sm.mu2[st];
                ab.part_ml[((int64_t)u.unit * H + st) * 2 + 0] = m2 == -INFINITY ? -INFINITY : m2 * kLn2;
                ab.part_ml[((int64_t)u.unit * H + st) * 2 + 1] = sm.lfin[st];
            }
        }
        // mu2, red and lfin are reused by the next unit
        named_bar(kBarSoft, 32 * kSoftWarps);
        ++ku;
    }
}

// ---------------------------------------------------------------- kernel

__global__ void __launch_bounds__(kThreads, 1)
    k_attn_mma(const __grid_constant__ AttnBatch ab, const __grid_constant__ AttnMaps maps, int splits, int tps) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.lk_full[i], 1);
            mbar_init(&sm.lk_empty[i], kGathWarps + kSoftWarps);
            mbar_init(&sm.q_ready[i], kGathWarps);
        }
        mbar_init(&sm.q_empty, 1);
        mbar_init(&sm.w_full, 1);
        for (int c = 0; c < 4; ++c) {
            mbar_init(&sm.it_full[c], 2);
            mbar_init(&sm.o_blk[c], 1);
        }
        mbar_init(&sm.s_full, 1);
        mbar_init(&sm.p_full, kSoftWarps);
        mbar_init(&sm.drained, 1);
        sm.abort = 0;
        fence_mbar_init();
    }
    if (warp == kWarpProd) {
        for (int i = lane; i < ab.n; i += 32)
            if (!ab.p[i].win_fp8) prefetch_tmap(&maps.win[i]);
        Unit u0;
        if (lane == 0 && unit_at(ab, splits, tps, 0, u0) && u0.t0 < u0.t1)
            bulk_prefetch_l2(ab.p[u0.prob].q + (int64_t)u0.b * ab.H * D, (uint32_t)(ab.H * D * 2));
    }
    if (warp == kWarpMma) tmem_alloc(&sm.tmem_base, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // lane 0's copy: a value the compiler knows is warp-uniform
    const uint32_t tbase = __shfl_sync(0xffffffffu, sm.tmem_base, 0);

    if (warp == kWarpMma)
        role_mma(sm, ab, splits, tps, tbase);
    else if (warp == kWarpProd)
        role_producer(sm, ab, splits, tps);
    else if (warp < kWarpGath)
        role_softmax(sm, ab, splits, tps, tbase);
    else
        role_gather(sm, ab, maps, splits, tps);

    __syncthreads();
    if (sm.abort && tid == 0) {  // report on the first of this CTA's units that has a cache
        Unit u;
        for (int k = 0; unit_at(ab, splits, tps, k, u); ++k)
            if (ab.p[u.prob].K > 0) {
                atomicOr(ab.p[u.prob].cache.status, CSA2_DEVERR_TIMEOUT);
                break;
            }
    }
    // every MMA of warp 0 has completed before TMEM is freed
    if (warp == kWarpMma) {
        tc_commit_w(&sm.drained);
        (void)mbar_wait_warp(&sm.drained, 0);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
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
    const int units = ab.n * ab.batch * splits;
    const int grid = std::min(units, device_sm_count());
    const size_t smem = sizeof(Smem) + 1024;
    static std::atomic<uint64_t> attr_done{0};
    const cudaError_t ea = smem_opt_in(reinterpret_cast<const void*>(k_attn_mma), (int)smem, attr_done);
    if (ea != cudaSuccess) return ea;
    k_attn_mma<<<grid, kThreads, smem, st>>>(ab, maps, splits, tps);
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
