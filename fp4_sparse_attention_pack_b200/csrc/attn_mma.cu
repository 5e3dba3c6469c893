// Sparse + window attention on the 5th-generation tensor cores (tcgen05.mma
// kind::f16, fp16 operands, fp32 accumulation in TMEM).
//
// Per (problem, sequence) the items are the K selected entries (dequantised
// from E2M1 x E4M3: exact in fp16) and the valid window tokens (bf16 -> fp16,
// exact for |x| in fp16's normal range, saturated at +-65504; E4M3 -> fp16,
// always exact, for an FP8 window); the latent item is key and value.  The
// unit's bf16 query is multiplied by a power of two 2^k that brings its largest
// magnitude into [2^14, 2^15) before it is rounded to fp16 (exact for every
// bf16 value within 2^28 of that maximum), and 2^-k is folded into the softmax
// scale, so no query magnitude overflows.
// Items go through 128-item tiles with an online softmax:
//
//   S^T[128 items x 64 heads] = Items . Q^T            (M = 128, N = 64, K = 512)
//   P^T = exp(scale 2^-k S^T - m_h)                    (fp16, per item lane)
//   O^T[4 x 128 latent x 64 heads] += Items^T . P^T    (M = 128, N = 64, K = 128)
//
// One shared-memory image of the tile serves both MMAs: 128-byte-swizzled
// slabs of 64 latent channels, read as the K-major A operand of S^T and as the
// MN-major A operand of O^T.  The reference maximum m_h only moves when a
// tile's maximum exceeds it by more than 8 (so p <= e^8 fits fp16); the O
// rescale that a move needs is rare, and a tile that moves no maximum needs no
// cross-item reduction at all: every thread forms its item's P^T with the
// current maxima while testing the item against them, one barrier ORs the
// tests, and only a tile that moves a maximum is formed again.
//
// Persistent CTAs (one per SM, 480 threads) walk their units (problem,
// sequence, split of tiles) tile by tile; warps specialise and hand work over
// through mbarriers, never through a block-wide barrier:
//   warp 0      issues the MMAs (one elected lane): S^T of a tile slab pair by
//               slab pair as the pairs are written, then O^T block by block;
//   warp 1      resolves each tile's 128 items (selected index -> page -> entry
//               row, or window slot) two tiles ahead, and prefetches the window
//               rows and the next unit's query into L2;
//   warps 2-5   softmax: thread = item row (TMEM lane), all 64 heads; P^T into
//               shared memory; the per-lane partial row sums (two buffers: a
//               tile reads one and writes the other) and a per-lane copy of the
//               64 reference maxima live in TMEM, so a tile's softmax reads no
//               shared memory but its item's kind; at the end of a unit the
//               O^T readout, normalised (or the split's partial);
//   warps 6-13  gather: all eight write each slab pair of a tile (an O block's
//               operand) together, pair after pair, as soon as the previous
//               tile's O block that reads it has completed; each tile's entry
//               bytes are loaded into registers before the first pair's wait;
//               bf16 window rows are converted in place once their TMA lands;
//               the unit's query is converted in the slab layout;
//   warp 14     window: loads each tile's bf16 window rows by TMA, slab pair by
//               slab pair as the O blocks complete, so a pair's copy is in
//               flight while the gather converts the pair before it.
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
constexpr int kWarpWin = kWarpGath + kGathWarps;         // window TMA issuer
constexpr int kThreads = 32 * (kWarpWin + 1);             // 480
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;      // O^T: 4 blocks x 64 heads
constexpr uint32_t kColS = 256;    // S^T: 64 heads
constexpr uint32_t kColL = 320;    // per-lane partial row sums of P: 64 heads
constexpr uint32_t kColM = 384;    // per-lane copy of the reference maxima: 64 heads
constexpr uint32_t kColL2 = 448;   // the row sums' second buffer (a tile reads one, writes the other)
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
    float a2[2];                   // per unit parity: scale * 2^-k * log2(e)
    uint32_t qmax[2][kGathWarps];  // per unit parity and slab: largest |q| bf16 magnitude bits
    float mu2[kHp];                // reference maximum per head (log2 units)
    float alpha[kHp];              // O / row-sum rescale factor of a move
    float red[4][kHp];             // per-quadrant partial max / sum
    float lfin[kHp];               // row sum of the unit
    uint64_t lk_full[2], lk_empty[2];  // item lookups: producer -> gather + softmax warps
    uint64_t q_ready[2][4];        // the unit's query slab pair c converted (per unit parity)
    uint64_t q_empty[4];           // every S^T MMA of the unit that reads query slab pair c completed
    uint64_t w_full[4];            // window TMA of slab pair c landed
    uint64_t it_full[4];           // slab pair c of the tile written (every gather warp)
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

constexpr int kMaxTail = 256;  // units left after the full rounds: fewer than the CTAs

// Host-computed work plan (a kernel parameter): problems in decreasing order of
// tile count; with one split, the units left after the full rounds over the
// CTAs (r < n_tail): problem and sequence (prob << 16 | b) and first piece.
struct AttnOrder {
    int prob[kMaxProblems];
    int n_tail;
    int tail_pb[kMaxTail];
    int tail_first[kMaxTail + 1];
};

__device__ __forceinline__ int tiles_of(const AttnBatch& ab, int prob) { return (ab.p[prob].K + WIN + kT - 1) / kT; }

// The work item a CTA takes k-th: tiles [t0, t1) of (problem, sequence), the
// whole output or a partial (O, m, l) in slot `unit` of the workspace.
//  - splits > 1 (few units): unit = (problem, sequence, split), strided over
//    the CTAs, every split a partial;
//  - one split: whole units, problems in decreasing tile count, in full rounds
//    of one unit per CTA; then the remaining units' tiles one by one (a unit
//    of one tile whole, the tiles of a longer unit as partials, slot = the
//    piece's number), so no CTA runs a whole unit more than the others.
struct Unit {
    int unit, prob, b, t0, t1;
    bool partial;
};

__device__ __noinline__ bool unit_at(const AttnOrder& ord, const AttnBatch& ab, int splits, int tps, int k, Unit& u) {
    if (splits > 1) {
        const int unit = blockIdx.x + k * gridDim.x;
        if (unit >= ab.n * ab.batch * splits) return false;
        const int split = unit % splits, pb = unit / splits;
        u.unit = unit;
        u.b = pb % ab.batch;
        u.prob = pb / ab.batch;
        u.t0 = split * tps;
        u.t1 = min(tiles_of(ab, u.prob), u.t0 + tps);
        u.partial = true;
        return true;
    }
    const int G = gridDim.x, units = ab.n * ab.batch, rounds = units / G;
    if (k < rounds) {
        const int v = blockIdx.x + k * G;
        u.prob = ord.prob[v / ab.batch];
        u.b = v % ab.batch;
        u.t0 = 0;
        u.t1 = tiles_of(ab, u.prob);
        u.partial = false;
        u.unit = -1;
        return true;
    }
    const int piece = blockIdx.x + (k - rounds) * G;
    if (piece >= ord.tail_first[ord.n_tail]) return false;
    int lo = 0, hi = ord.n_tail - 1;  // the unit r with tail_first[r] <= piece < tail_first[r + 1]
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (ord.tail_first[mid] <= piece) lo = mid; else hi = mid - 1;
    }
    const int T = ord.tail_first[lo + 1] - ord.tail_first[lo];
    u.prob = ord.tail_pb[lo] >> 16;
    u.b = ord.tail_pb[lo] & 0xFFFF;
    u.t0 = piece - ord.tail_first[lo];
    u.t1 = u.t0 + 1;
    u.partial = T > 1;
    u.unit = piece;
    return true;
}

// Valid window tokens of sequence b.
__device__ __forceinline__ int window_len(const AttnProblem& P, int b) {
    const int c = P.win_count[b];
    return c < 0 ? 0 : (c < WIN ? c : WIN);
}

// ---------------------------------------------------------------- warp 1: items and window

__device__ void role_producer(Smem& sm, const AttnBatch& ab, const AttnOrder& ord, int splits, int tps) {
    const int lane = threadIdx.x & 31;
    bool alive = true;
    uint32_t it = 0;
    Unit u;
    if (lane == 0 && unit_at(ord, ab, splits, tps, 0, u) && u.t0 < u.t1)
        bulk_prefetch_l2(ab.p[u.prob].q + (int64_t)u.b * ab.H * D, (uint32_t)(ab.H * D * 2));
    for (int k = 0; unit_at(ord, ab, splits, tps, k, u); ++k) {
        // the next unit's query into L2 while this unit runs
        Unit nu;
        if (lane == 0 && unit_at(ord, ab, splits, tps, k + 1, nu) && nu.t0 < nu.t1)
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

__device__ void role_mma(Smem& sm, const AttnBatch& ab, const AttnOrder& ord, int splits, int tps, uint32_t tbase) {
    const uint32_t idesc_s = idesc_f16(128, kHp, 0, 0, 0);
    const uint32_t idesc_o = idesc_f16(128, kHp, 0, 1, 1);
    const uint64_t desc_items = smem_desc(sm.items[0], 16, 1024, kLayoutSw128);
    const uint64_t desc_q = smem_desc(sm.q[0], 16, 1024, kLayoutSw128);
    const uint64_t desc_vt = smem_desc(sm.items[0], 16384, 1024, kLayoutSw128);
    const uint64_t desc_p = smem_desc(sm.p, 16384, 1024, kLayoutSw128);
    bool alive = true;
    uint32_t it = 0, ku = 0;
    Unit u;
    for (int k = 0; unit_at(ord, ab, splits, tps, k, u); ++k) {
        if (u.t0 >= u.t1) continue;
        for (int t = u.t0; t < u.t1; ++t, ++it) {
            // S^T = Items . Q^T, slab pair by slab pair as the gather warps finish them
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                alive = wait_bar_warp(sm, &sm.it_full[c], it & 1u) && alive;
                // the unit's query slab pair c (converted pair by pair as the previous
                // unit's last S^T releases it)
                if (t == u.t0) alive = wait_bar_warp(sm, &sm.q_ready[ku & 1][c], (ku >> 1) & 1u) && alive;
                tc_fence_after();
                if (alive) {
                    // rolled: unrolled, the compiler hoists all 64 descriptors of a
                    // tile into registers the other warps need
#pragma unroll 1
                    for (int kk = 0; kk < 8; ++kk) {  // 16 latent channels per MMA
                        const int ks = 8 * c + kk;
                        const uint32_t off = (uint32_t)((ks >> 2) * (kT * 128) + (ks & 3) * 32) >> 4;
                        const uint32_t offq = (uint32_t)((ks >> 2) * (kHp * 128) + (ks & 3) * 32) >> 4;
                        tc_mma_f16_w(tbase + kColS, desc_items + off, desc_q + offq, idesc_s, ks > 0 ? 1u : 0u);
                    }
                    // the unit's last S^T frees query slab pair c for the next unit
                    if (t + 1 == u.t1) tc_commit_w(&sm.q_empty[c]);
                }
            }
            if (alive) tc_commit_w(&sm.s_full);
            // O^T += Items^T . P^T, one commit per 128-channel block (slabs 2c, 2c + 1)
            alive = wait_bar_warp(sm, &sm.p_full, it & 1u) && alive;
            tc_fence_after();
            if (alive) {
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
#pragma unroll 1
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
// scaled by 2^k and rounded to fp16.  Eight lanes cover a head row's 128 bytes
// of the slab (lane: chunk l & 7 of heads 4i + l / 8), so a load instruction
// reads four whole lines.  k brings the query's largest bf16 magnitude into
// [2^14, 2^15): a first pass finds it, a second (from L1 / L2) converts, once
// the previous unit's last S^T has read the slab's pair (the first pass runs
// before: the conversion of a unit's query overlaps the end of the previous
// unit).
__device__ bool convert_query(Smem& sm, const AttnBatch& ab, const Unit& u, int g, uint32_t ku, bool alive) {
    const int lane = threadIdx.x & 31;
    const int H = ab.H;
    const int c = lane & 7, h0 = lane >> 3;
    const uint4* qb = reinterpret_cast<const uint4*>(ab.p[u.prob].q + (int64_t)u.b * H * D + 64 * g) + c;
    uint32_t m = 0;
#pragma unroll 4
    for (int i = 0; i < kHp / 4; ++i) {
        const int h = 4 * i + h0;
        if (h < H) {
            const uint4 w = __ldg(qb + (int64_t)h * (D / 8));
            m = __vmaxu2(m, w.x & 0x7FFF7FFFu);
            m = __vmaxu2(m, w.y & 0x7FFF7FFFu);
            m = __vmaxu2(m, w.z & 0x7FFF7FFFu);
            m = __vmaxu2(m, w.w & 0x7FFF7FFFu);
        }
    }
    m = __reduce_max_sync(0xffffffffu, max(m & 0xFFFFu, m >> 16));
    if (lane == 0) sm.qmax[ku & 1][g] = m;
    named_bar(kBarGath, 32 * kGathWarps);
    uint32_t mq = 0;
#pragma unroll
    for (int j = 0; j < kGathWarps; ++j) mq = max(mq, sm.qmax[ku & 1][j]);
    // bf16 magnitude bits: exponent field E = mq >> 7; the maximum lies in
    // [2^(E-127), 2^(E-126)), so k = 141 - E puts it in [2^14, 2^15)
    const int E = (int)(mq >> 7);
    const int kx = mq == 0 ? 0 : min(126, 141 - E);
    const float mul = __uint_as_float((uint32_t)(127 + kx) << 23);
    if (g == 0 && lane == 0) sm.a2[ku & 1] = ab.scale * __uint_as_float((uint32_t)(127 - kx) << 23) * kLog2e;
    // slab g is free once the previous unit's last S^T has read its pair
    if (ku > 0) alive = wait_bar_warp(sm, &sm.q_empty[g >> 1], (ku - 1) & 1u) && alive;
#pragma unroll 4
    for (int i = 0; i < kHp / 4; ++i) {
        const int h = 4 * i + h0;
        const uint4 w = h < H ? __ldg(qb + (int64_t)h * (D / 8)) : make_uint4(0, 0, 0, 0);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
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
    // qmax[ku & 1] is written again two units on, after every gather warp has
    // passed the next unit's barrier, so after every read above
    return alive;
}

// bf16 pair -> f16x2 (round to nearest), saturated to fp16's finite range: one
// conversion instruction whose .satfinite clamps a result beyond +-65504 to it
__device__ __forceinline__ uint32_t bf16x2_to_h2_sat(uint32_t w) {
    uint32_t d;
    asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;"
        : "=r"(d)
        : "f"(__uint_as_float(w & 0xFFFF0000u)), "f"(__uint_as_float(w << 16)));  // (high, low)
    return d;
}

// The eight gather warps write every slab pair of a tile together, pair after
// pair, each as soon as the previous tile's O block that reads it has
// completed, so a pair is ready about a thousand cycles after its block: thread
// (g, l) owns half h = l % 2 of row 16 g + l / 2 of every pair c, i.e. slab
// 2 c + h of that row (64 channels: 32 code bytes, four scale bytes, one
// 128-byte line of the image).  Odd lanes store their chunks four on, so that
// every eight lanes of a store hit distinct banks.  All of a tile's entry bytes
// are loaded into registers before the first pair's wait.
__device__ void role_gather(Smem& sm, const AttnBatch& ab, const AttnOrder& ord, int splits, int tps) {
    const int lane = threadIdx.x & 31;
    const int g = (threadIdx.x >> 5) - kWarpGath;
    const int r = 16 * g + (lane >> 1);  // item row
    const int hf = lane & 1;             // slab 2 c + hf of pair c
    bool alive = true;
    uint32_t it = 0, ku = 0, wn = 0;
    Unit u;
    for (int k = 0; unit_at(ord, ab, splits, tps, k, u); ++k) {
        if (u.t0 >= u.t1) continue;
        // the problem's fields in registers for the unit (a dynamically indexed
        // kernel-parameter read per tile would miss the constant cache)
        const uint8_t* const main_codes = ab.p[u.prob].cache.main_codes;
        const uint8_t* const main_scales = ab.p[u.prob].cache.main_scales;
        const uint8_t* const win8 = static_cast<const uint8_t*>(ab.p[u.prob].win);
        const int PK = ab.p[u.prob].K;
        for (int t = u.t0; t < u.t1; ++t, ++it) {
            const int buf = it & 1;
            if (t == u.t0) {
                // the unit's query (before this tile's entry loads, so their
                // registers are not live across the conversion)
                alive = convert_query(sm, ab, u, g, ku, alive);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.q_ready[ku & 1][g >> 1]);
            }
            alive = wait_bar_warp(sm, &sm.lk_full[buf], (it >> 1) & 1u) && alive;
            // this row's kind, and (an entry) its code words and scale bytes of
            // every pair's half
            const int kind = sm.kind[buf][r];
            uint4 cw[4][2];
            uint32_t sc[4];
            if (kind == 1) {
                const int64_t rw = sm.src_row[buf][r];
                const uint8_t* codes = main_codes + rw * MCB + 32 * hf;
                const uint8_t* scl = main_scales + rw * MSB + 4 * hf;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    cw[c][0] = __ldg(reinterpret_cast<const uint4*>(codes + 64 * c));
                    cw[c][1] = __ldg(reinterpret_cast<const uint4*>(codes + 64 * c + 16));
                    sc[c] = __ldg(reinterpret_cast<const uint32_t*>(scl + 8 * c));
                }
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    cw[c][0] = cw[c][1] = make_uint4(0, 0, 0, 0);
                    sc[c] = 0;
                }
            }
            const bool win = sm.tile_win[buf] != 0;
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.lk_empty[buf]);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                // pair c is free once the previous tile's O block c has completed
                // (every gather warp waits for every block of every tile in order,
                // so the parity never aliases an older phase)
                if (it > 0) alive = wait_bar_warp(sm, &sm.o_blk[c], (it - 1) & 1u) && alive;
                // bf16 window rows of the pair arrive by TMA (the window warp's);
                // rows that are not window tokens are rewritten below, after it lands
                if (win) alive = wait_bar_warp(sm, &sm.w_full[c], wn & 1u) && alive;
                uint8_t* line = sm.items[2 * c + hf];
                if (alive) {
                    if (kind == 1) {
                        // E2M1 codes x E4M3 scale (one per 16 channels) -> fp16, exact:
                        // chunk w holds channels 8 w .. 8 w + 7 (code word w, scale w / 2)
                        const uint32_t w8[8] = {cw[c][0].x, cw[c][0].y, cw[c][0].z, cw[c][0].w,
                                                cw[c][1].x, cw[c][1].y, cw[c][1].z, cw[c][1].w};
                        __half2 s2[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) s2[j] = __float2half2_rn(e4m3_decode_pos((sc[c] >> (8 * j)) & 0xFFu));
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const int w0 = kk, w1 = (kk + 4) & 7;  // odd lanes: four chunks on
                            const uint32_t word = hf ? w8[w1] : w8[w0];
                            const __half2 s = hf ? s2[w1 >> 1] : s2[w0 >> 1];
                            uint4 o;
                            uint32_t* os = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const uint32_t hh = e2m1x2_to_h2((word >> (8 * e)) & 0xFFu);
                                const __half2 v = __hmul2(*reinterpret_cast<const __half2*>(&hh), s);
                                os[e] = *reinterpret_cast<const uint32_t*>(&v);
                            }
                            *reinterpret_cast<uint4*>(line + sw128(r, hf ? w1 : w0)) = o;
                        }
                    } else if (kind == 2) {
                        // bf16 window row, landed by TMA in the slab layout: to fp16 in place
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            uint4* ptr = reinterpret_cast<uint4*>(line + sw128(r, hf ? ((kk + 4) & 7) : kk));
                            const uint4 x = *ptr;
                            *ptr = make_uint4(bf16x2_to_h2_sat(x.x), bf16x2_to_h2_sat(x.y), bf16x2_to_h2_sat(x.z),
                                              bf16x2_to_h2_sat(x.w));
                        }
                    } else if (kind == 3) {
                        // E4M3 window row (slot t * 128 + r - K of the ring): 64 codes -> fp16 (exact)
                        const int64_t rw = (int64_t)u.b * WIN + (t * kT + r - PK);
                        const uint4* src = reinterpret_cast<const uint4*>(win8 + rw * D + 128 * c + 64 * hf);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {  // 16 codes: chunks 2 q, 2 q + 1
                            const uint4 x = __ldg(src + (hf ? ((q + 2) & 3) : q));
                            const int c0 = hf ? ((2 * q + 4) & 7) : 2 * q;
                            *reinterpret_cast<uint4*>(line + sw128(r, c0)) =
                                make_uint4(e4m3x2_to_h2(x.x & 0xFFFFu), e4m3x2_to_h2(x.x >> 16),
                                           e4m3x2_to_h2(x.y & 0xFFFFu), e4m3x2_to_h2(x.y >> 16));
                            *reinterpret_cast<uint4*>(line + sw128(r, c0 + 1)) =
                                make_uint4(e4m3x2_to_h2(x.z & 0xFFFFu), e4m3x2_to_h2(x.z >> 16),
                                           e4m3x2_to_h2(x.w & 0xFFFFu), e4m3x2_to_h2(x.w >> 16));
                        }
                    } else {
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            *reinterpret_cast<uint4*>(line + sw128(r, kk)) = make_uint4(0, 0, 0, 0);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.it_full[c]);
            }
            if (win) ++wn;
        }
        ++ku;
    }
}

// The window warp: for every tile, in order, waits for the previous tile's O
// block c and (a tile with bf16 window tokens) loads slab pair c of the window
// rows by TMA: two 64-channel boxes over the tile's 128 rows, so the copy of a
// pair is in flight while the gather warps convert the pair before it.
__device__ void role_window(Smem& sm, const AttnBatch& ab, const AttnMaps& maps, const AttnOrder& ord, int splits,
                            int tps) {
    const int lane = threadIdx.x & 31;
    bool alive = true;
    uint32_t it = 0;
    uint32_t wiss = 0, wpar = 0;  // bit c: a copy of pair c was issued; parity of their count
    Unit u;
    for (int k = 0; unit_at(ord, ab, splits, tps, k, u); ++k) {
        if (u.t0 >= u.t1) continue;
        const AttnProblem& P = ab.p[u.prob];
        const int wlen = window_len(P, u.b);
        for (int t = u.t0; t < u.t1; ++t, ++it) {
            // the lookup warp's test for kind-2 rows: window slots t kT - K .. + kT - 1
            // that are below the window length
            const bool win = !P.win_fp8 && wlen > 0 && t * kT + kT > P.K && t * kT < P.K + wlen;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                // every block of every tile in order (the parity never aliases)
                if (it > 0) alive = wait_bar_warp(sm, &sm.o_blk[c], (it - 1) & 1u) && alive;
                if (win && alive) {
                    if (lane == 0) {
                        mbar_expect_tx(&sm.w_full[c], 2 * kT * 128);
                        tma_load_3d(sm.items[2 * c], &maps.win[u.prob], 128 * c, t * kT - P.K, u.b, &sm.w_full[c]);
                        tma_load_3d(sm.items[2 * c + 1], &maps.win[u.prob], 128 * c + 64, t * kT - P.K, u.b,
                                    &sm.w_full[c]);
                    }
                    wiss |= 1u << c;
                    wpar ^= 1u << c;
                }
            }
        }
    }
    // copies that were issued but not waited for land before the CTA exits
    if (!alive && lane == 0) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
            if ((wiss >> c) & 1u) (void)mbar_wait(&sm.w_full[c], ((wpar >> c) & 1u) ^ 1u);
    }
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

__device__ void role_softmax(Smem& sm, const AttnBatch& ab, const AttnOrder& ord, int splits, int tps,
                             uint32_t tbase) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int quad = warp & 3;                 // TMEM lane quadrant of this warp
    const int row = 32 * quad + lane;          // item row (S^T) / latent row (O^T) of this thread
    const int st = threadIdx.x - 32 * kWarpSoft;  // 0 .. 127: per-head work for st < 64
    const uint32_t tl = tbase + ((uint32_t)(32 * quad) << 16);
    const int H = ab.H;
    bool alive = true;
    uint32_t it = 0, ku = 0;
    uint32_t lsel = 0;  // which row-sum buffer holds the sums so far
    Unit u;
    for (int k = 0; unit_at(ord, ab, splits, tps, k, u); ++k) {
        const bool partial = u.partial;
        if (u.t0 >= u.t1) {  // a split without tiles: an empty partial
            if (partial && st < H) {
                ab.part_ml[((int64_t)u.unit * H + st) * 2 + 0] = -INFINITY;
                ab.part_ml[((int64_t)u.unit * H + st) * 2 + 1] = 0.0f;
            }
            continue;
        }
        if (st < kHp) sm.mu2[st] = -INFINITY;
        {
            float v[32];
#pragma unroll
            for (int h = 0; h < 32; ++h) v[h] = -INFINITY;
            tmem_st_32x32b_x32(tl + kColM, v);
            tmem_st_32x32b_x32(tl + kColM + 32, v);
        }
        // the unit's scale (written by the gather warp of query slab 0 before its
        // arrival on pair 0)
        alive = wait_bar_warp(sm, &sm.q_ready[ku & 1][0], (ku >> 1) & 1u) && alive;
        named_bar(kBarSoft, 32 * kSoftWarps);
        const float a2 = sm.a2[ku & 1];
        for (int t = u.t0; t < u.t1; ++t, ++it) {
            const int buf = it & 1;
            alive = wait_bar_warp(sm, &sm.lk_full[buf], (it >> 1) & 1u) && alive;
            const bool ok = sm.kind[buf][row] != 0;
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.lk_empty[buf]);
            alive = wait_bar_warp(sm, &sm.s_full, it & 1u) && alive;
            tc_fence_after();
            const bool first = t == u.t0;
            const uint32_t lcur = lsel ? kColL2 : kColL, lnext = lsel ? kColL : kColL2;
            // p = exp2(scale 2^-k s - m) into P^T (fp16), and the lane's running row
            // sums of the rounded p: read from lcur, written to lnext (so that a
            // pass whose maxima turn out stale leaves them intact).  need: does
            // this item move a head's maximum (by more than the gap)?
            auto p_pass = [&](bool acc, bool& need) {
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    uint32_t sv[32], mv[32];
                    tmem_ld_x32_nowait(tl + kColS + 32 * half, sv);
                    tmem_ld_x32_nowait(tl + kColM + 32 * half, mv);
                    tmem_wait_ld2(sv, mv);
                    float y[32];
#pragma unroll
                    for (int h = 0; h < 32; ++h) {
                        y[h] = fmaf(__uint_as_float(sv[h]), a2, -__uint_as_float(mv[h]));
                        need |= y[h] > kGap2;
                    }
                    store_p(sm.p, row, 4 * half, ok, y);
                    if (acc) {
                        float l[32];
                        tmem_ld_32x32b_x32(tl + lcur + 32 * half, l);
#pragma unroll
                        for (int h = 0; h < 32; ++h) y[h] += l[h];
                    }
                    tmem_st_32x32b_x32(tl + lnext + 32 * half, y);
                }
            };
            // P^T is free once the previous tile's O has completed
            if (it > 0) alive = wait_bar_warp(sm, &sm.o_blk[3], (it - 1) & 1u) && alive;
            // a unit's first tile always sets the maxima; a later one is computed
            // with the current maxima at once, and again only if one of them moves
            // (one loop, so the pass is compiled once)
            bool update = first;
#pragma unroll 1
            while (true) {
                if (update) {
                    // the tile's maximum per head over the valid items
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        float z[32];
                        tmem_ld_32x32b_x32(tl + kColS + 32 * half, z);
#pragma unroll
                        for (int h = 0; h < 32; ++h) z[h] = ok ? z[h] * a2 : -INFINITY;
                        sm.red[quad][32 * half + lane] = warp_reduce_scatter32<true>(z);
                    }
                    named_bar(kBarSoft, 32 * kSoftWarps);
                    bool resc = false;
                    if (st < kHp) {
                        const float mt =
                            fmaxf(fmaxf(sm.red[0][st], sm.red[1][st]), fmaxf(sm.red[2][st], sm.red[3][st]));
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
                        tc_fence_after();
#pragma unroll 1
                        for (int c = 0; c < 10; ++c) {  // four O^T blocks, then the row sums, 32 columns at a time
                            const uint32_t col = (c < 8 ? kColO + 32 * c : lcur + 32 * (c - 8));
                            const int h0 = 32 * (c & 1);
                            float o[32];
                            tmem_ld_32x32b_x32(tl + col, o);
#pragma unroll
                            for (int h = 0; h < 32; ++h) o[h] *= sm.alpha[h0 + h];
                            tmem_st_32x32b_x32(tl + col, o);
                        }
                    }
                    // this lane's TMEM copy of the updated maxima
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        float v[32];
#pragma unroll
                        for (int h = 0; h < 32; ++h) v[h] = sm.mu2[32 * half + h];
                        tmem_st_32x32b_x32(tl + kColM + 32 * half, v);
                    }
                }
                bool need = false;
                p_pass(!first, need);
                if (update || !named_bar_or(kBarSoft, 32 * kSoftWarps, (ok && need) || !alive)) break;
                update = true;
            }
            lsel ^= 1u;
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.p_full);
        }

        // ---- end of the unit: row sums over the items, then O^T out
        alive = wait_bar_warp(sm, &sm.o_blk[3], (it - 1) & 1u) && alive;
        tc_fence_after();
        {
            const uint32_t lfinal = lsel ? kColL2 : kColL;  // the buffer the unit's last tile wrote
            float l[32];
            tmem_ld_32x32b_x32(tl + lfinal, l);
            sm.red[quad][lane] = warp_reduce_scatter32<false>(l);
            tmem_ld_32x32b_x32(tl + lfinal + 32, l);
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
            for (int h0 = 0; h0 < H; h0 += 16) {
                float lf[16];  // the normalisers of these 16 heads, in registers
#pragma unroll
                for (int h = 0; h < 16; ++h) lf[h] = partial ? 1.0f : sm.lfin[h0 + h];
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    const int lat = 128 * c + row;  // O^T block c, lane = latent channel
                    float o[16];
                    tmem_ld_32x32b_x16(tl + kColO + 64 * c + h0, o);
                    float* d = dst + (int64_t)h0 * D + lat;
#pragma unroll
                    for (int h = 0; h < 16; ++h)
                        if (h0 + h < H) d[(int64_t)h * D] = o[h] * lf[h];
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
    k_attn_mma(const __grid_constant__ AttnBatch ab, const __grid_constant__ AttnMaps maps,
               const __grid_constant__ AttnOrder ord, int splits, int tps) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.lk_full[i], 1);
            mbar_init(&sm.lk_empty[i], kGathWarps + kSoftWarps);
            for (int c = 0; c < 4; ++c) mbar_init(&sm.q_ready[i][c], 2);
        }
        for (int c = 0; c < 4; ++c) mbar_init(&sm.q_empty[c], 1);
        for (int c = 0; c < 4; ++c) mbar_init(&sm.w_full[c], 1);
        for (int c = 0; c < 4; ++c) {
            mbar_init(&sm.it_full[c], kGathWarps);
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
    }
    if (warp == kWarpMma) tmem_alloc(&sm.tmem_base, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // lane 0's copy: a value the compiler knows is warp-uniform
    const uint32_t tbase = __shfl_sync(0xffffffffu, sm.tmem_base, 0);

    if (warp == kWarpMma)
        role_mma(sm, ab, ord, splits, tps, tbase);
    else if (warp == kWarpProd)
        role_producer(sm, ab, ord, splits, tps);
    else if (warp < kWarpGath)
        role_softmax(sm, ab, ord, splits, tps, tbase);
    else if (warp < kWarpWin)
        role_gather(sm, ab, ord, splits, tps);
    else
        role_window(sm, ab, maps, ord, splits, tps);

    __syncthreads();
    if (sm.abort && tid == 0) {  // report on the first of this CTA's units that has a cache
        Unit u;
        for (int k = 0; unit_at(ord, ab, splits, tps, k, u); ++k)
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

// out[j] = sum_s O_s[j] e^(m_s - M) / sum_s l_s e^(m_s - M) over the partials in
// slots slot0 .. slot0 + n - 1 of head h (threadIdx.x: channels x, x + 128, ...).
__device__ void merge_partials(const AttnBatch& ab, int64_t slot0, int n, int h, float* o) {
    const int H = ab.H;
    float M = -INFINITY;
    for (int s = 0; s < n; ++s) M = fmaxf(M, ab.part_ml[((slot0 + s) * H + h) * 2]);
    float L = 0.0f;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (M != -INFINITY) {
        for (int s = 0; s < n; ++s) {
            const float m = ab.part_ml[((slot0 + s) * H + h) * 2];
            const float l = ab.part_ml[((slot0 + s) * H + h) * 2 + 1];
            if (m == -INFINITY || l == 0.0f) continue;
            const float f = expf(m - M);
            L += l * f;
            const float* po = ab.part_o + ((slot0 + s) * H + h) * D;
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[i] = fmaf(f, po[threadIdx.x + 128 * i], acc[i]);
        }
    }
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) o[threadIdx.x + 128 * i] = acc[i] * inv;
}

// Every split of (problem, sequence) is a partial: merge them.
__global__ void k_attn_mma_combine(const __grid_constant__ AttnBatch ab, int splits) {
    const int h = blockIdx.x, b = blockIdx.y, prob = blockIdx.z;
    merge_partials(ab, ((int64_t)prob * ab.batch + b) * splits, splits, h,
                   ab.p[prob].out + ((int64_t)b * ab.H + h) * D);
}

// One split: the units after the full rounds ran tile by tile; merge the
// pieces of each such unit longer than one tile (blockIdx.y: the r-th of them).
__global__ void k_attn_mma_combine_tail(const __grid_constant__ AttnBatch ab, const __grid_constant__ AttnOrder ord,
                                        int G) {
    (void)G;
    const int h = blockIdx.x, r = blockIdx.y;
    const int p0 = ord.tail_first[r], T = ord.tail_first[r + 1] - p0;
    if (T == 1) return;  // written whole by its CTA
    const int prob = ord.tail_pb[r] >> 16, b = ord.tail_pb[r] & 0xFFFF;
    merge_partials(ab, p0, T, h, ab.p[prob].out + ((int64_t)b * ab.H + h) * D);
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

// CTAs of a launch over `units` work units: one per SM, at most one per unit
// (and at most kMaxTail, the size of the plan's tail table).
static int attn_grid(int units) { return std::min(std::min(units, device_sm_count()), kMaxTail); }

// Partial slots of a launch: every split, or (one split) at most every tile of
// the units left after the full rounds over the CTAs.
static size_t attn_mma_slots(int n_problems, int batch, int Kmax) {
    const int splits = attn_mma_splits(n_problems, batch, Kmax);
    const int units = n_problems * batch;
    if (splits > 1) return (size_t)units * splits;
    const int G = attn_grid(units);
    const int rem = G > 0 ? units % G : 0;
    return (size_t)rem * ((Kmax + WIN + kT - 1) / kT);
}

size_t attn_mma_workspace_bytes(int n_problems, int batch, int H, int Kmax) {
    const size_t slots = attn_mma_slots(n_problems, batch, Kmax);
    return slots * H * D * sizeof(float) + slots * H * 2 * sizeof(float);
}

namespace {

// The work plan of a launch on G CTAs: problems in decreasing tile count (ties
// in problem order) and, with one split, the units left after the full rounds.
AttnOrder attn_order(const AttnBatch& ab, int splits, int G) {
    AttnOrder o;
    std::memset(&o, 0, sizeof(o));
    for (int i = 0; i < ab.n; ++i) o.prob[i] = i;
    std::stable_sort(o.prob, o.prob + ab.n, [&](int a, int b) { return ab.p[a].K > ab.p[b].K; });
    if (splits == 1 && G > 0) {
        const int units = ab.n * ab.batch, rounds = units / G;
        int first = 0;
        for (int v = rounds * G; v < units; ++v) {
            const int r = o.n_tail++;
            const int prob = o.prob[v / ab.batch];
            o.tail_pb[r] = prob << 16 | (v % ab.batch);
            o.tail_first[r] = first;
            first += (ab.p[prob].K + WIN + kT - 1) / kT;
        }
        o.tail_first[o.n_tail] = first;
    }
    return o;
}

// Does a unit of the tail have more than one tile (so the tail merge runs)?
bool attn_tail_merge(const AttnOrder& o) {
    for (int r = 0; r < o.n_tail; ++r)
        if (o.tail_first[r + 1] - o.tail_first[r] > 1) return true;
    return false;
}

}  // namespace

int attn_mma_launches(const AttnBatch& ab) {
    const int splits = attn_mma_splits(ab.n, ab.batch, ab.Kmax);
    if (splits > 1) return 2;
    const int units = ab.n * ab.batch;
    return 1 + (attn_tail_merge(attn_order(ab, 1, attn_grid(units))) ? 1 : 0);
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
    const size_t slots = attn_mma_slots(ab.n, ab.batch, ab.Kmax);
    if (slots > 0) ab.part_ml = ab.part_o + slots * ab.H * D;
    const int units = ab.n * ab.batch * splits;
    const int grid = attn_grid(units);
    const AttnOrder ord = attn_order(ab, splits, grid);
    const size_t smem = sizeof(Smem) + 1024;
    static std::atomic<uint64_t> attr_done{0};
    const cudaError_t ea = smem_opt_in(reinterpret_cast<const void*>(k_attn_mma), (int)smem, attr_done);
    if (ea != cudaSuccess) return ea;
    k_attn_mma<<<grid, kThreads, smem, st>>>(ab, maps, ord, splits, tps);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (ev) cudaEventRecord(ev[0], st);
    if (splits > 1) {
        dim3 g(ab.H, ab.batch, ab.n);
        k_attn_mma_combine<<<g, 128, 0, st>>>(ab, splits);
        e = cudaGetLastError();
    } else if (attn_tail_merge(ord)) {
        dim3 g(ab.H, ord.n_tail);
        k_attn_mma_combine_tail<<<g, 128, 0, st>>>(ab, ord, grid);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess && ev) cudaEventRecord(ev[1], st);
    return e;
}

}  // namespace csa2
