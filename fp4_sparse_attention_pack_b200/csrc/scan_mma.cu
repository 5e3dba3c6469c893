// Indexer scan on the 5th-generation tensor cores: tcgen05.mma kind::mxf4
// (E2M1 operands, one E8M0 scale per 32 channels applied by the hardware,
// fp32 accumulation in TMEM).
//
//   score[b][e] = sum_h w[b][h] * max(0, qhat[b][h] . khat[b][e])
//
// With 64 indexer heads every key meets 64 x 128 MXFP4 products: a dense
// contraction that CUDA cores cannot keep up with at HBM speed.  Several scan
// problems (the Full and Reindex layers of one source) read the same keys, so
// the kernel groups them: a work item is (subset of up to kMaxSub problems
// over one cache, sequence, chunk of tiles), and each 128-entry key tile is
// loaded once and multiplied by the queries of every problem of the subset,
// two problems (128 query rows) per MMA pass:
//   D[128 entries x 128 rows] = K[128 x 128] . [Q_a; Q_b]^T
// (two MMAs of K = 64 each).  The epilogue applies ReLU, the head weights and
// the head sum, one thread per (entry row, problem).
//
// Persistent, warp-specialised CTA (640 threads, one CTA per SM):
//   warps 0, 19  producers: TMA tile loads of the keys (one 64-entry page per
//           box, 64-byte swizzle) and bulk copies of their E8M0 scales into an
//           8-stage ring, the two warps taking alternate tiles; warp 0 also
//           loads per work item the query tiles, scales and head weights of
//           every problem of the subset (double-buffered).  Keys stream with an
//           L2 evict-first policy.  Copies are issued by several lanes at once
//           (a lane per page, per problem or per pool block): issued one by one
//           from a single lane of a single warp, they set the pace of the whole
//           pipeline when a subset holds one problem.
//   warp 1  MMA issuer: per tile issues one MMA pass per
//           problem pair into one of three TMEM accumulators (pass p into
//           p % 3), committing each pass to its epilogue group.  Its only
//           commits are those: the epilogue warp that sees a tile's last pass
//           complete hands the key stage back to the producer, and the
//           epilogue's arrivals after an item's last pass free the query
//           buffer.  Three accumulators let the next pass run while both
//           groups drain theirs.
//   warps 2-17 epilogue, two groups of eight; group g drains the passes p with
//           p % 2 == g.  Warp w of a group reads TMEM lane quadrant
//           w % 4 and problem (w / 4) % 2 of the pass: tcgen05.ld of the 64 head
//           columns of its entry, ReLU, weight, sum, one score store.
//           A subset that scans a pool (hierarchical indexer) instead gathers
//           each tile as 16 boxes of 8 rows, one per pool block, each into its
//           own 512-byte slot, so the swizzled layout is that of a whole page.
//   warp 18 scale warp: rearranges the E8M0 scales that landed in shared memory
//           into the 32x128-bit layout tcgen05.cp reads (per item for the
//           queries, per stage for the keys), copies them into TMEM and commits
//           the copies to the ready barriers the MMA issuer waits on, keeping
//           the transposition, its proxy fence and the copies off the issuer's
//           path (one tcgen05 instruction costs the issuing warp about a hundred
//           cycles).
// Every wait is bounded; a timeout sets CSA2_DEVERR_TIMEOUT in the problem's
// status word and the CTA drains and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace csa2 {

namespace {

using namespace sm100;

constexpr int kHeads = 64;        // query rows per problem
constexpr int kPass = 2;          // problems per MMA pass (N = 128)
constexpr int kMaxSub = 12;       // problems per work item
constexpr int kMaxPasses = kMaxSub / kPass;
constexpr int kStages = 8;
constexpr int kTile = 128;        // entries per MMA tile (MMA M)
constexpr int kMaxChunk = 16;     // tiles per work item at most (32 pages: one per producer lane)
constexpr int kGroups = 2;        // epilogue groups
constexpr int kAcc = 3;           // TMEM accumulators: pass p lands in p % kAcc, group p % kGroups drains it
constexpr int kEpiWarps = 8 * kGroups;
constexpr int kSfWarp = 2 + kEpiWarps;
constexpr int kProducer1Warp = kSfWarp + 1;  // second producer: the odd tiles
constexpr int kThreads = 32 * (kProducer1Warp + 1);
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColAcc = 0;                            // kAcc x 128 accumulator columns
constexpr uint32_t kColSfa = 128 * kAcc;                   // kStages x 4 scale columns (keys)
constexpr uint32_t kColSfb = kColSfa + 4 * kStages;        // 2 x kMaxPasses x 4 (queries)
static_assert(kColSfb + 2 * kMaxPasses * 4 <= kTmemCols, "TMEM columns");
constexpr int kMaxSources = CSA2_MAX_SOURCES;

// Problems that read one cache, scanned together.
struct ScanSub {
    int src;      // keys[] map index
    int n;        // problems
    int chunk;    // tiles per work item
    int chunks;   // work items per sequence
    int item0;    // first work item
    int pool;     // the problems scan the same pool (positions instead of entries)
    int8_t prob[kMaxSub];
};

struct MmaScanMaps {
    CUtensorMap keys[kMaxSources];  // per distinct cache: idx codes [num_pages*64][64 B]
    CUtensorMap keys8[kMaxSources]; // the same with 8-row boxes (pool blocks)
    CUtensorMap queries;            // [n * batch * 64][64 B]
    ScanSub sub[kMaxProblems];
    int n_sub;
    int n_items;
};

struct __align__(1024) Smem {
    uint8_t a[kStages][kTile * 64];          // key codes, 64B-swizzled rows
    uint8_t b[2][kMaxSub * kHeads * 64];     // query codes of the subset, 64B-swizzled rows
    uint8_t sfa_raw[kStages][kTile * 4];
    uint8_t sfa_tc[kStages][512];            // 32 rows x 16 B for tcgen05.cp
    uint8_t sfb_raw[2][kMaxSub * kHeads * 4];
    uint8_t sfb_tc[2][kMaxPasses][512];
    float w[2][kMaxSub][kHeads];
    float* rows[2][kMaxSub];                 // score row of the item's sequence, per problem
    int prow[2][kMaxChunk * 16];             // pool items, per producer: first physical key row of each slot
    uint64_t full[kStages], empty[kStages], sfa_ready[kStages];
    uint64_t bfull[2], bempty[2], sfb_ready[2];
    uint64_t tfull[kAcc], tempty[kAcc];
    uint64_t drained, sdrained;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory beyond the 227 KB per-block limit");


struct Item {
    int s, b, t0, t1, n;
};

__device__ __forceinline__ bool item_at(const ScanBatch& sb, const MmaScanMaps& mp, int id, Item& it) {
    int s = 0;
    while (s + 1 < mp.n_sub && id >= mp.sub[s + 1].item0) ++s;
    const ScanSub& S = mp.sub[s];
    const int r = id - S.item0;
    it.s = s;
    it.b = r / S.chunks;
    const int c = r - it.b * S.chunks;
    const ScanProblem& P0 = sb.p[S.prob[0]];
    it.n = S.pool ? min(max(P0.pool_n[it.b], 0), kPoolBlock * P0.pool_blocks) : entries_of(P0.cache, it.b);
    const int tiles = (it.n + kTile - 1) / kTile;
    it.t0 = c * S.chunk;
    it.t1 = min(it.t0 + S.chunk, tiles);
    // Lane 0's values for the whole warp: the compiler then sees every loop
    // bound and ring index derived from them as warp-uniform, so the tcgen05
    // operands built from them need no per-lane handling at issue.
    it.n = __shfl_sync(0xffffffffu, it.n, 0);
    it.t1 = __shfl_sync(0xffffffffu, it.t1, 0);
    return it.t0 < it.t1;
}

__device__ __forceinline__ void raise_abort(Smem& sm, uint32_t* status) {
    atomicOr(status, CSA2_DEVERR_TIMEOUT);
    *reinterpret_cast<volatile int*>(&sm.abort) = 1;
}

__device__ __forceinline__ bool aborted(Smem& sm) {
    return *reinterpret_cast<volatile int*>(&sm.abort) != 0;
}

// 128 rows of 4 scale bytes (one 32-bit word per row) -> the 32x128-bit layout
// of tcgen05.cp: lane r holds rows r, 32 + r, 64 + r, 96 + r (one per column).
__device__ __forceinline__ void scales_to_tc(const uint8_t* raw, uint8_t* tc, int lane) {
    const uint32_t* src = reinterpret_cast<const uint32_t*>(raw);
    reinterpret_cast<uint4*>(tc)[lane] = make_uint4(src[lane], src[32 + lane], src[64 + lane], src[96 + lane]);
}

// d = a * b + c on two fp32 lanes (each lane an IEEE fma).
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    uint64_t d, ua, ub, uc;
    asm("mov.b64 %0, {%1, %2};" : "=l"(ua) : "f"(a.x), "f"(a.y));
    asm("mov.b64 %0, {%1, %2};" : "=l"(ub) : "f"(b.x), "f"(b.y));
    asm("mov.b64 %0, {%1, %2};" : "=l"(uc) : "f"(c.x), "f"(c.y));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(ua), "l"(ub), "l"(uc));
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(d));
    return r;
}

__global__ void __launch_bounds__(kThreads, 1)
    k_scan_mma(const __grid_constant__ ScanBatch sb, const __grid_constant__ MmaScanMaps mp) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int batch = sb.p[0].cache.batch;
    const int n_items = mp.n_items;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);  // the epilogue warp that sees the tile's last pass complete
            mbar_init(&sm.sfa_ready[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.bfull[i], 1);
            mbar_init(&sm.bempty[i], kEpiWarps);  // after the item's last pass: its MMAs are done
            mbar_init(&sm.sfb_ready[i], 1);
        }
        for (int a = 0; a < kAcc; ++a) {
            mbar_init(&sm.tfull[a], 1);
            mbar_init(&sm.tempty[a], 8);  // the eight warps of the group that drains it
        }
        mbar_init(&sm.drained, 1);
        mbar_init(&sm.sdrained, 1);
        sm.abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&sm.tmem_base, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = __shfl_sync(0xffffffffu, sm.tmem_base, 0);  // warp-uniform (see item_at)

    if (warp == 0 || warp == kProducer1Warp) {
        // ------------------------------------------------------------ producers
        // Two warps walk the same items; the CTA's tiles are numbered in order (g)
        // and producer pw loads the tiles with g % 2 == pw into stage g % kStages
        // (kStages is even, so every use of a stage belongs to one producer).
        // Producer 0 also loads each item's queries.  Lanes fetch the item's page
        // ids (2 per tile, up to 32) in one round; barrier arms come from one
        // elected lane, and the copies of a tile or an item are issued by several
        // lanes at once.
        const uint32_t pw = warp == 0 ? 0u : 1u;
        const uint64_t pol_stream = policy_evict_first();
        const uint64_t pol_keep = policy_evict_last();
        if (lane == 0 && pw == 0) prefetch_tmap(&mp.queries);
        uint32_t g = 0, bslot = 0, bphase = 0;
        uint32_t issued = 0, issued_par = 0;  // per stage: a copy was issued, and its phase
        for (int id = blockIdx.x; id < n_items && !__any_sync(0xffffffffu, aborted(sm)); id += gridDim.x) {
            Item it;
            if (!item_at(sb, mp, id, it)) continue;
            const ScanSub& S = mp.sub[it.s];
            const CacheView& c = sb.p[S.prob[0]].cache;
            const int used_pages = (it.n + PAGE - 1) / PAGE;
            const int li = 2 * it.t0 + lane;  // logical page this lane looks up
            int my_pg = -1;
            if (!S.pool && lane < 2 * (it.t1 - it.t0) && li < used_pages) {
                const int pp = c.page_table[(int64_t)it.b * c.max_pages + li];
                if (pp >= 0 && pp < c.num_pages)
                    my_pg = pp;
                else
                    atomicOr(c.status, CSA2_DEVERR_PAGE);
            }
            bool stop = false;
            if (pw != 0) {
                // queries are producer 0's
            } else if (!mbar_wait_warp(&sm.bempty[bslot], bphase ^ 1)) {
                if (lane == 0) raise_abort(sm, c.status);
                stop = true;
            } else {
                if (lane < S.n) sm.rows[bslot][lane] = sb.p[S.prob[lane]].scores + (int64_t)it.b * sb.score_stride;
                __syncwarp();
                mbar_expect_tx_w(&sm.bfull[bslot], S.n * (kHeads * 64 + kHeads * 4 + kHeads * 4));
                __syncwarp();
                // lane j issues problem j's copies: one warp instruction per kind of copy
                if (lane < S.n) {
                    const int p = S.prob[lane];
                    const int64_t qrow = ((int64_t)p * batch + it.b) * kHeads;
                    tma_load_2d(sm.b[bslot] + lane * kHeads * 64, &mp.queries, 0, (int)qrow, &sm.bfull[bslot], pol_keep);
                    bulk_load(sm.sfb_raw[bslot] + lane * kHeads * 4, sb.qs + qrow * ISB, kHeads * 4, &sm.bfull[bslot],
                              pol_keep);
                    bulk_load(sm.w[bslot][lane], sb.p[p].w + (int64_t)it.b * kHeads, kHeads * 4, &sm.bfull[bslot],
                              pol_keep);
                }
                __syncwarp();
            }
            if (++bslot == 2) bslot = 0, bphase ^= 1;
            const CUtensorMap* kmap = &mp.keys[S.src];
            if (S.pool) {
                // physical first row of every pool block of the item (positions
                // below it.n are valid, so their blocks lie below n_entries)
                const ScanProblem& P0 = sb.p[S.prob[0]];
                const int slots = (it.n + kPoolBlock - 1) / kPoolBlock;
                const int n_slot = 16 * (it.t1 - it.t0);  // <= 32 * kSlotsPerLane
                constexpr int kSlotsPerLane = kMaxChunk * 16 / 32;
                __syncwarp();  // the previous item's reads of prow are done
                // all of a lane's block ids, then all their page ids: two rounds of
                // independent loads instead of a chain of dependent pairs
                int blk[kSlotsPerLane], pg[kSlotsPerLane];
#pragma unroll
                for (int j = 0; j < kSlotsPerLane; ++j) {
                    const int i = lane + 32 * j, slot = 16 * it.t0 + i;
                    blk[j] = (i < n_slot && slot < slots) ? P0.pool[(int64_t)it.b * P0.pool_blocks + slot] : -1;
                    if (blk[j] >= c.max_pages * (PAGE / kPoolBlock)) blk[j] = -1;  // never past the table
                }
#pragma unroll
                for (int j = 0; j < kSlotsPerLane; ++j)
                    pg[j] = blk[j] >= 0 ? c.page_table[(int64_t)it.b * c.max_pages + kPoolBlock * blk[j] / PAGE] : -1;
#pragma unroll
                for (int j = 0; j < kSlotsPerLane; ++j) {
                    const int i = lane + 32 * j;
                    if (i >= n_slot) continue;
                    int r = -1;
                    if (blk[j] >= 0) {
                        if (pg[j] >= 0 && pg[j] < c.num_pages)
                            r = pg[j] * PAGE + kPoolBlock * blk[j] % PAGE;
                        else
                            atomicOr(c.status, CSA2_DEVERR_PAGE);
                    }
                    sm.prow[pw][i] = r;
                }
                __syncwarp();
            }
            for (int t = it.t0; t < it.t1 && !stop; ++t, ++g) {
                if ((g & 1u) != pw) continue;
                const uint32_t stage = g % kStages, sphase = (g / kStages) & 1u;
                const int pg0 = __shfl_sync(0xffffffffu, my_pg, 2 * (t - it.t0));
                const int pg1 = __shfl_sync(0xffffffffu, my_pg, 2 * (t - it.t0) + 1);
                const int prow = S.pool && lane < 16 ? sm.prow[pw][16 * (t - it.t0) + lane] : -1;
                const unsigned have = __ballot_sync(0xffffffffu, prow >= 0);
                if (!mbar_wait_warp(&sm.empty[stage], sphase ^ 1)) {
                    if (lane == 0) raise_abort(sm, c.status);
                    stop = true;
                    break;
                }
                if (S.pool) {
                    if (have == 0) {
                        mbar_arrive_w(&sm.full[stage]);
                    } else {
                        mbar_expect_tx_w(&sm.full[stage], __popc(have) * kPoolBlock * (ICB + ISB));
                        __syncwarp();
                        if (prow >= 0) {
                            tma_load_2d(sm.a[stage] + lane * kPoolBlock * ICB, &mp.keys8[S.src], 0, prow,
                                        &sm.full[stage], pol_stream);
                            bulk_load(sm.sfa_raw[stage] + lane * kPoolBlock * ISB, c.idx_scales + (int64_t)prow * ISB,
                                      kPoolBlock * ISB, &sm.full[stage], pol_stream);
                        }
                    }
                    issued |= 1u << stage;
                    issued_par = (issued_par & ~(1u << stage)) | (sphase << stage);
                    continue;
                }
                const uint32_t bytes = (pg0 >= 0 ? PAGE * (ICB + ISB) : 0) + (pg1 >= 0 ? PAGE * (ICB + ISB) : 0);
                if (bytes == 0) {
                    mbar_arrive_w(&sm.full[stage]);
                } else {
                    mbar_expect_tx_w(&sm.full[stage], bytes);
                    __syncwarp();
                    // lanes 0, 1 load the two pages' key codes, lanes 2, 3 their scales
                    const int h = lane & 1;
                    const int pg = h ? pg1 : pg0;
                    if (lane < 4 && pg >= 0) {
                        if (lane < 2)
                            tma_load_2d(sm.a[stage] + h * PAGE * ICB, kmap, 0, pg * PAGE, &sm.full[stage], pol_stream);
                        else
                            bulk_load(sm.sfa_raw[stage] + h * PAGE * ISB, c.idx_scales + (int64_t)pg * PAGE * ISB,
                                      PAGE * ISB, &sm.full[stage], pol_stream);
                    }
                    __syncwarp();
                }
                issued |= 1u << stage;
                issued_par = (issued_par & ~(1u << stage)) | (sphase << stage);
            }
            if (stop) break;
        }
        // never leave with copies in flight
        if (lane == 0)
            for (int s = 0; s < kStages; ++s)
                if ((issued >> s) & 1u) (void)mbar_wait(&sm.full[s], (issued_par >> s) & 1u);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        uint32_t stage = 0, sphase = 0, bslot = 0, bphase = 0, acc = 0, aphase = 0;
        for (int id = blockIdx.x; id < n_items && !__any_sync(0xffffffffu, aborted(sm)); id += gridDim.x) {
            Item it;
            if (!item_at(sb, mp, id, it)) continue;
            const ScanSub& S = mp.sub[it.s];
            uint32_t* status = sb.p[S.prob[0]].cache.status;
            const int passes = (S.n + kPass - 1) / kPass;
            // the query scales of the item are in TMEM once sfb_ready completes
            if (!mbar_wait_warp(&sm.sfb_ready[bslot], bphase)) { raise_abort(sm, status); break; }
            bool stop = false;
            for (int t = it.t0; t < it.t1; ++t) {
                // ... and the stage's key scales once sfa_ready completes
                if (!mbar_wait_warp(&sm.sfa_ready[stage], sphase)) { raise_abort(sm, status); stop = true; break; }
                const uint32_t sfa = tbase + kColSfa + 4 * stage;
                tc_fence_after();
                const uint64_t adesc = smem_desc(sm.a[stage], 16, 512, kLayoutSw64);
                for (int k = 0; k < passes; ++k) {
                    if (!mbar_wait_warp(&sm.tempty[acc], aphase ^ 1)) { raise_abort(sm, status); stop = true; break; }
                    tc_fence_after();
                    const uint32_t n_rows = (uint32_t)min(kPass, S.n - kPass * k) * kHeads;
                    const uint32_t sfb = tbase + kColSfb + (bslot * kMaxPasses + k) * 4;
                    const uint32_t d = tbase + kColAcc + 128 * acc;
                    const uint64_t bdesc = smem_desc(sm.b[bslot] + k * kPass * kHeads * 64, 16, 512, kLayoutSw64);
                    // K = 0..63 (scale bytes 0, 1), then K = 64..127 (bytes 2, 3): +32 B start
                    tc_mma_mxf4_w(d, adesc, bdesc, idesc_mxf4(n_rows, 0, 0), sfa, sfb, 0u);
                    tc_mma_mxf4_w(d, adesc + 2, bdesc + 2, idesc_mxf4(n_rows, 2, 2), sfa, sfb, 1u);
                    tc_commit_w(&sm.tfull[acc]);
                    if (++acc == kAcc) acc = 0, aphase ^= 1;
                }
                if (stop) break;
                if (++stage == kStages) stage = 0, sphase ^= 1;
            }
            if (++bslot == 2) bslot = 0, bphase ^= 1;
            if (stop) break;
        }
        // every tcgen05 operation of this thread has completed before TMEM is freed
        tc_commit_w(&sm.drained);
        (void)mbar_wait_warp(&sm.drained, 0);
    } else if (warp < kSfWarp) {
        // ------------------------------------------------------------ epilogue
        const int ew = warp - 2;
        const int grp = ew >> 3;
        const int jp = (ew >> 2) & 1;     // problem of the pass this warp reads
        const int quad = warp & 3;        // TMEM lane quadrant of this warp
        const int row = quad * 32 + lane;
        uint32_t bslot = 0, bphase = 0, pass_no = 0, stage = 0;
        for (int id = blockIdx.x; id < n_items && !__any_sync(0xffffffffu, aborted(sm)); id += gridDim.x) {
            Item it;
            if (!item_at(sb, mp, id, it)) continue;
            const ScanSub& S = mp.sub[it.s];
            const int passes = (S.n + kPass - 1) / kPass;
            uint32_t* status = sb.p[S.prob[0]].cache.status;
            if (!mbar_wait_warp(&sm.bfull[bslot], bphase)) { raise_abort(sm, status); break; }
            bool stop = false;
            for (int t = it.t0; t < it.t1 && !stop; ++t, stage = stage + 1 == kStages ? 0 : stage + 1) {
                for (int k = 0; k < passes; ++k, ++pass_no) {
                    if ((int)(pass_no % kGroups) != grp) continue;
                    const int acc = (int)(pass_no % kAcc);
                    if (!mbar_wait_warp(&sm.tfull[acc], (pass_no / kAcc) & 1u)) {
                        raise_abort(sm, status);
                        stop = true;
                        break;
                    }
                    // the tile's last pass has completed, and every MMA before it:
                    // its key stage goes back to the producer
                    if (k == passes - 1 && (ew & 7) == 0 && lane == 0) mbar_arrive(&sm.empty[stage]);
                    tc_fence_after();
                    const int j = kPass * k + jp;
                    if (j < S.n) {
                        const uint32_t taddr = tbase + ((uint32_t)(quad * 32) << 16) + kColAcc + 128 * acc + 64 * jp;
                        const float* w = sm.w[bslot][j];
                        float2 acc2[4];  // eight chains: heads h = 8i + c go to chain c
#pragma unroll
                        for (int c = 0; c < 4; ++c) acc2[c] = make_float2(0.0f, 0.0f);
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            float v[32];
                            tmem_ld_32x32b_x32(taddr + 32 * half, v);
                            if (half == 1) {
                                tc_fence_before();
                                __syncwarp();
                                if (lane == 0) mbar_arrive(&sm.tempty[acc]);
                            }
#pragma unroll
                            for (int h = 0; h < 32; h += 8) {
                                const float4 wa = *reinterpret_cast<const float4*>(w + 32 * half + h);
                                const float4 wb = *reinterpret_cast<const float4*>(w + 32 * half + h + 4);
                                acc2[0] = fma2(make_float2(wa.x, wa.y), make_float2(fmaxf(v[h], 0.0f), fmaxf(v[h + 1], 0.0f)),
                                               acc2[0]);
                                acc2[1] = fma2(make_float2(wa.z, wa.w),
                                               make_float2(fmaxf(v[h + 2], 0.0f), fmaxf(v[h + 3], 0.0f)), acc2[1]);
                                acc2[2] = fma2(make_float2(wb.x, wb.y),
                                               make_float2(fmaxf(v[h + 4], 0.0f), fmaxf(v[h + 5], 0.0f)), acc2[2]);
                                acc2[3] = fma2(make_float2(wb.z, wb.w),
                                               make_float2(fmaxf(v[h + 6], 0.0f), fmaxf(v[h + 7], 0.0f)), acc2[3]);
                            }
                        }
                        const float s = ((acc2[0].x + acc2[0].y) + (acc2[1].x + acc2[1].y)) +
                                        ((acc2[2].x + acc2[2].y) + (acc2[3].x + acc2[3].y));
                        const int e = t * kTile + row;
                        if (e < it.n) sm.rows[bslot][j][e] = s;
                    } else {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sm.tempty[acc]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.bempty[bslot]);
            if (++bslot == 2) bslot = 0, bphase ^= 1;
            if (stop) break;
        }
    } else {
        // ------------------------------------------------------------ scale warp
        uint32_t stage = 0, sphase = 0, bslot = 0, bphase = 0;
        for (int id = blockIdx.x; id < n_items && !__any_sync(0xffffffffu, aborted(sm)); id += gridDim.x) {
            Item it;
            if (!item_at(sb, mp, id, it)) continue;
            const ScanSub& S = mp.sub[it.s];
            uint32_t* status = sb.p[S.prob[0]].cache.status;
            const int passes = (S.n + kPass - 1) / kPass;
            if (!mbar_wait_warp(&sm.bfull[bslot], bphase)) { if (lane == 0) raise_abort(sm, status); break; }
            // bfull implies the MMAs of the item two back, which read these TMEM
            // columns, have completed (bempty follows its last pass's completion)
            tc_fence_after();
            for (int k = 0; k < passes; ++k) scales_to_tc(sm.sfb_raw[bslot] + k * 512, sm.sfb_tc[bslot][k], lane);
            fence_proxy_async_smem();
            __syncwarp();
            for (int k = 0; k < passes; ++k)
                tc_cp_32x128b_x4_w(tbase + kColSfb + (bslot * kMaxPasses + k) * 4,
                                   smem_desc(sm.sfb_tc[bslot][k], 16, 128, kLayoutNone));
            tc_commit_w(&sm.sfb_ready[bslot]);
            if (++bslot == 2) bslot = 0, bphase ^= 1;
            bool stop = false;
            for (int t = it.t0; t < it.t1; ++t) {
                if (!mbar_wait_warp(&sm.full[stage], sphase)) {
                    if (lane == 0) raise_abort(sm, status);
                    stop = true;
                    break;
                }
                // full implies the MMAs that last read this stage's scale columns
                // have completed (the stage's empty arrival follows them)
                tc_fence_after();
                scales_to_tc(sm.sfa_raw[stage], sm.sfa_tc[stage], lane);
                fence_proxy_async_smem();
                __syncwarp();
                tc_cp_32x128b_x4_w(tbase + kColSfa + 4 * stage, smem_desc(sm.sfa_tc[stage], 16, 128, kLayoutNone));
                tc_commit_w(&sm.sfa_ready[stage]);
                if (++stage == kStages) stage = 0, sphase ^= 1;
            }
            if (stop) break;
        }
        // every scale copy of this warp has completed before TMEM is freed
        tc_commit_w(&sm.sdrained);
        (void)mbar_wait_warp(&sm.sdrained, 0);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, kTmemCols);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// Rows of 64 bytes, boxes of box_rows rows, 64-byte swizzle.
bool make_rows64_map(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {64, rows};
    cuuint64_t strides[1] = {64};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


}  // namespace

bool scan_mma_supported(const ScanBatch& sb) {
    if (sb.H_idx != kHeads || sb.n < 1) return false;
    int srcs = 0;
    const uint8_t* seen[kMaxSources];
    for (int i = 0; i < sb.n; ++i) {
        bool found = false;
        for (int j = 0; j < srcs; ++j) found |= (seen[j] == sb.p[i].cache.idx_codes);
        if (!found) {
            if (srcs == kMaxSources) return false;
            seen[srcs++] = sb.p[i].cache.idx_codes;
        }
    }
    return encode_fn() != nullptr;
}

cudaError_t launch_scan_mma(const ScanBatch& sb, cudaStream_t st) {
    MmaScanMaps mp;
    std::memset(&mp, 0, sizeof(mp));
    const int batch = sb.p[0].cache.batch;
    // distinct caches -> key maps; problems of one cache -> subsets of <= kMaxSub
    int srcs = 0;
    const uint8_t* seen[kMaxSources];
    int src_of[kMaxProblems];
    int cap_tiles[kMaxSources];
    bool have8[kMaxSources] = {};
    for (int i = 0; i < sb.n; ++i) {
        const CacheView& c = sb.p[i].cache;
        int j = 0;
        for (; j < srcs; ++j)
            if (seen[j] == c.idx_codes) break;
        if (j == srcs) {
            seen[srcs] = c.idx_codes;
            if (!make_rows64_map(&mp.keys[srcs], c.idx_codes, (uint64_t)c.num_pages * PAGE, PAGE))
                return cudaErrorInvalidValue;
            cap_tiles[srcs] = (c.max_pages * PAGE + kTile - 1) / kTile;
            ++srcs;
        }
        src_of[i] = j;
        if (sb.p[i].pool && !have8[j]) {
            if (!make_rows64_map(&mp.keys8[j], c.idx_codes, (uint64_t)c.num_pages * PAGE, kPoolBlock))
                return cudaErrorInvalidValue;
            have8[j] = true;
        }
    }
    // groups: problems over one cache that scan the same pool (or none)
    bool grouped[kMaxProblems] = {};
    int sub_tiles[kMaxProblems];
    for (int i0 = 0; i0 < sb.n; ++i0) {
        if (grouped[i0]) continue;
        int members[kMaxProblems], m = 0;
        for (int i = i0; i < sb.n; ++i)
            if (!grouped[i] && src_of[i] == src_of[i0] && sb.p[i].pool == sb.p[i0].pool) {
                members[m++] = i;
                grouped[i] = true;
            }
        const bool pool = sb.p[i0].pool != nullptr;
        const int tiles = pool ? (kPoolBlock * sb.p[i0].pool_blocks + kTile - 1) / kTile : cap_tiles[src_of[i0]];
        // split into near-equal subsets of at most kMaxSub problems
        const int parts = (m + kMaxSub - 1) / kMaxSub;
        for (int q = 0, k0 = 0; q < parts; ++q) {
            const int cnt = (m - k0) / (parts - q);
            sub_tiles[mp.n_sub] = tiles;
            ScanSub& S = mp.sub[mp.n_sub++];
            S.src = src_of[i0];
            S.pool = pool ? 1 : 0;
            S.n = cnt;
            for (int k = 0; k < cnt; ++k) S.prob[k] = (int8_t)members[k0 + k];
            k0 += cnt;
        }
    }
    // Tiles per work item: about 64 tile-problems of work each (so subsets of
    // different sizes cost about the same per item), fewer when the items would
    // not fill the grid a few times over.
    const int grid_max = device_sm_count();
    int items = 0;
    for (int base = 64;; base /= 2) {
        items = 0;
        for (int s = 0; s < mp.n_sub; ++s) {
            ScanSub& S = mp.sub[s];
            S.chunk = std::max(2, std::min(kMaxChunk, base / S.n));
            S.chunks = (sub_tiles[s] + S.chunk - 1) / S.chunk;
            S.item0 = items;
            items += batch * S.chunks;
        }
        if (items >= 3 * grid_max || base <= 4) break;
    }
    if (!make_rows64_map(&mp.queries, sb.qc, (uint64_t)sb.n * batch * kHeads, kHeads))
        return cudaErrorInvalidValue;
    mp.n_items = items;
    const int grid = std::min(items, grid_max);
    const size_t smem = sizeof(Smem) + 1024;
    static std::atomic<uint64_t> attr_done{0};
    const cudaError_t ea = smem_opt_in(reinterpret_cast<const void*>(k_scan_mma), (int)smem, attr_done);
    if (ea != cudaSuccess) return ea;
    k_scan_mma<<<grid, kThreads, smem, st>>>(sb, mp);
    return cudaGetLastError();
}

}  // namespace csa2
