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
// A pass costs the tensor core 128 cycles and the epilogue's ReLU, weight and
// sum over its 16,384 accumulators about twice that on the CUDA cores.  The
// pass rate is bound by the hand-off between the two: measured on this GPU,
// the commit of a pass becomes visible to a waiting warp ~600 cycles after the
// MMAs were issued, so with three 128-column accumulators (what TMEM holds
// beside the scale factors) and the epilogue's TMEM loads in the loop, a pass
// costs ~300-450 cycles even with an empty epilogue.  Two alternating
// epilogue groups keep the loads of one pass off the critical path of the next.
//
// Persistent, warp-specialised CTA (608 threads, one CTA per SM):
//   warps 0, 18  producers: warp 0 decodes the CTA's work items into a
//           descriptor in shared memory per query buffer and loads per item the
//           query tiles, query scales and head weights of every problem of the
//           subset (double-buffered); both load the key tiles, alternately, into
//           an 8-stage ring: the key codes by TMA (one 64-entry page per box,
//           64-byte swizzle) and their E8M0 scales by bulk copy.  Keys stream
//           with an L2 evict-first policy.  Tile copies are issued by one lane
//           with warp-uniform operands.
//   warp 1  MMA issuer: rearranges each stage's and each item's E8M0 scales into
//           the 32x128-bit layout tcgen05.cp reads and copies them into TMEM, then
//           issues one MMA pass per problem pair into one of three TMEM
//           accumulators (pass p into p % 3), each pass committed to its
//           accumulator's barrier; after a tile's passes a commit hands the key
//           stage back to the producer, after an item's a commit releases the
//           query buffer.  Copies and MMAs of one thread run in issue order, so
//           no barrier separates a scale copy from the MMAs that read it.
//   warps 2-17 epilogue, two groups of eight; group g drains the passes p with
//           p % 2 == g.  Warp w of a group reads TMEM lane quadrant w % 4 and
//           problem (w / 4) % 2 of the pass: two tcgen05.ld of 32 head columns
//           each (the accumulator is released after the second), ReLU, weight,
//           sum, one coalesced score store per 32 entries.  The ReLU is x + |x|
//           (exactly twice max(x, 0), halved once at the end) on the FMA pipe:
//           fmaxf would fill the half-rate ALU pipe, and busy ALU warps delay
//           the tcgen05 instructions of the MMA warp on the same sub-partition.
// A subset that scans a pool (hierarchical indexer) gathers each tile as 16
// boxes of 8 rows, one per pool block, each into its own 512-byte slot, so the
// swizzled layout is that of a whole page.
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
constexpr int kAcc = 3;           // TMEM accumulators: pass p lands in p % kAcc
constexpr int kGroups = 2;        // epilogue groups: group g drains the passes p with p % 2 == g
constexpr int kEpiWarps = 8 * kGroups;  // per group one per (TMEM lane quadrant, problem of the pass)
constexpr int kEpi0 = 2;          // first epilogue warp
constexpr int kProd1 = kEpi0 + kEpiWarps;  // second producer warp: the odd tiles
constexpr int kThreads = 32 * (kProd1 + 1);
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

// A work item as the producer decodes it for the other roles (shared memory,
// one per query buffer): the MMA and epilogue warps never touch the kernel
// parameters inside their loops, whose dynamically indexed reads miss the
// constant cache.
struct ItemDesc {
    int b, t0, t1, n;        // sequence, tile range, valid positions
    int nprob;               // problems of the subset; 0 ends the CTA's work
    uint32_t* status;        // status word of the cache
    float* rows[kMaxSub];    // each problem's score row of sequence b
};

struct __align__(1024) Smem {
    uint8_t a[kStages][kTile * 64];          // key codes, 64B-swizzled rows
    uint8_t b[2][kMaxSub * kHeads * 64];     // query codes of the subset, 64B-swizzled rows
    uint8_t sfa_raw[kStages][kTile * 4];
    uint8_t sfa_tc[kStages][512];            // 32 rows x 16 B for tcgen05.cp
    uint8_t sfb_raw[2][kMaxSub * kHeads * 4];
    uint8_t sfb_tc[2][kMaxPasses][512];
    float w[2][kMaxSub][kHeads];
    ItemDesc desc[2];
    int prow[2][kMaxChunk * 16];             // pool items, per producer: first physical key row of each slot
    uint64_t full[kStages], empty[kStages];
    uint64_t qfull[2], qempty[2];
    uint64_t tfull[kAcc], tempty[kAcc];
    uint64_t drained;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory beyond the 227 KB per-block limit");


struct Item {
    int s, b, t0, t1, n;
};

// Work item id -> (subset, sequence, tile range).  Every lane of the warp must
// call it.  Lane 0's entry count is shuffled to the whole warp, so the
// compiler knows every loop bound, ring index and copy operand derived from
// the item is warp-uniform.
__device__ __forceinline__ bool item_at(const ScanBatch& sb, const MmaScanMaps& mp, int id, Item& it) {
    int s = 0;
    while (s + 1 < mp.n_sub && id >= mp.sub[s + 1].item0) ++s;
    const ScanSub& S = mp.sub[s];
    const int r = id - S.item0;
    it.s = s;
    it.b = r / S.chunks;
    const int c = r - it.b * S.chunks;
    const ScanProblem& P0 = sb.p[S.prob[0]];
    int n = S.pool ? min(max(P0.pool_n[it.b], 0), kPoolBlock * P0.pool_blocks) : entries_of(P0.cache, it.b);
    n = __shfl_sync(0xffffffffu, n, 0);
    const int tiles = (n + kTile - 1) / kTile;
    it.n = n;
    it.t0 = c * S.chunk;
    it.t1 = min(it.t0 + S.chunk, tiles);
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

// 2 max(x, 0), exactly: x + |x| is 2x or 0.  One add with an absolute-value
// operand on the FMA pipe, where fmaxf would occupy the half-rate ALU pipe that
// the MMA and producer warps need for their own instructions.
__device__ __forceinline__ float relu2(float x) { return x + fabsf(x); }

// acc += w[h] * 2 max(v[h], 0) over N heads: head h goes to fp32 chain h % 8
// (four packed pairs).  The caller halves the fixed pairwise sum of the
// chains at the end (exact), so the score equals the one formed with max(v, 0).
template <int N>
__device__ __forceinline__ void relu_weighted_acc(const float (&v)[N], const float* w, float2 (&acc2)[4]) {
#pragma unroll
    for (int h = 0; h < N; h += 8) {
        const float4 wa = *reinterpret_cast<const float4*>(w + h);
        const float4 wb = *reinterpret_cast<const float4*>(w + h + 4);
        float x[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = relu2(v[h + i]);
        acc2[0] = fma2(make_float2(wa.x, wa.y), make_float2(x[0], x[1]), acc2[0]);
        acc2[1] = fma2(make_float2(wa.z, wa.w), make_float2(x[2], x[3]), acc2[1]);
        acc2[2] = fma2(make_float2(wb.x, wb.y), make_float2(x[4], x[5]), acc2[2]);
        acc2[3] = fma2(make_float2(wb.z, wb.w), make_float2(x[6], x[7]), acc2[3]);
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    k_scan_mma(const __grid_constant__ ScanBatch sb, const __grid_constant__ MmaScanMaps mp) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_items = mp.n_items;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);  // the MMA warp's commit after the tile's last pass
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.qfull[i], 1);
            mbar_init(&sm.qempty[i], 1 + kEpiWarps);  // the MMA warp's commit + every epilogue warp
        }
        for (int a = 0; a < kAcc; ++a) {
            mbar_init(&sm.tfull[a], 1);
            mbar_init(&sm.tempty[a], 8);  // the eight warps of the group that drains it
        }
        mbar_init(&sm.drained, 1);
        sm.abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&sm.tmem_base, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = __shfl_sync(0xffffffffu, sm.tmem_base, 0);

    if (warp == 0 || warp == kProd1) {
        // ------------------------------------------------------------ producers
        // Both warps walk the same items and number the CTA's tiles in order (g);
        // producer pw loads the tiles with g % 2 == pw into stage g % kStages
        // (kStages is even, so every use of a stage belongs to one producer).
        // Producer 0 also decodes each item's descriptor and loads its queries:
        // a tile of one problem costs one warp ~1,000 cycles of copy issue,
        // more than the MMA warp's pass.
        const uint32_t pw = warp == 0 ? 0u : 1u;
        const int batch = sb.p[0].cache.batch;
        const uint64_t pol_stream = policy_evict_first();
        const uint64_t pol_keep = policy_evict_last();
        if (lane == 0 && pw == 0) prefetch_tmap(&mp.queries);
        uint32_t g = 0, bslot = 0, bphase = 0;
        uint32_t issued = 0, issued_par = 0;  // per stage: a copy was issued, and its phase
        bool stop = false;
        for (int id = blockIdx.x; id < n_items && !stop; id += gridDim.x) {
            Item it;
            if (!item_at(sb, mp, id, it)) continue;
            const ScanSub& S = mp.sub[it.s];
            const int nprob = S.n, src = S.src, pool = S.pool;
            const ScanProblem& P0 = sb.p[S.prob[0]];
            const int32_t* page_table = P0.cache.page_table + (int64_t)it.b * P0.cache.max_pages;
            const int max_pages = P0.cache.max_pages, num_pages = P0.cache.num_pages;
            const uint8_t* idx_scales = P0.cache.idx_scales;
            uint32_t* status = P0.cache.status;
            // the item's page ids, one per lane (two pages a tile, at most 32)
            const int used_pages = (it.n + PAGE - 1) / PAGE;
            const int li = 2 * it.t0 + lane;
            int my_pg = -1;
            if (!pool && lane < 2 * (it.t1 - it.t0) && li < used_pages) {
                const int pp = page_table[li];
                if (pp >= 0 && pp < num_pages)
                    my_pg = pp;
                else
                    atomicOr(status, CSA2_DEVERR_PAGE);
            }
            // the query buffer (and its item descriptor) is free once the item two
            // back is done: its MMAs completed and every epilogue warp left it
            if (pw == 0) {
            if (!mbar_wait_warp(&sm.qempty[bslot], bphase ^ 1)) {
                if (lane == 0) raise_abort(sm, status);
                break;
            }
            ItemDesc& D = sm.desc[bslot];
            if (lane < nprob) D.rows[lane] = sb.p[S.prob[lane]].scores + (int64_t)it.b * sb.score_stride;
            if (lane == 0) {
                D.b = it.b;
                D.t0 = it.t0;
                D.t1 = it.t1;
                D.n = it.n;
                D.nprob = nprob;
                D.status = status;
            }
            __syncwarp();
            // queries, scales and head weights of the subset's problems (the
            // arrival also publishes the descriptor)
            mbar_expect_tx_w(&sm.qfull[bslot], nprob * (kHeads * 64 + kHeads * 4 + kHeads * 4));
            __syncwarp();
            if (lane < nprob) {  // lane j: problem j's three copies
                const int p = S.prob[lane];
                const int64_t qrow = ((int64_t)p * batch + it.b) * kHeads;
                tma_load_2d(sm.b[bslot] + lane * kHeads * 64, &mp.queries, 0, (int)qrow, &sm.qfull[bslot], pol_keep);
                bulk_load(sm.sfb_raw[bslot] + lane * kHeads * 4, sb.qs + qrow * ISB, kHeads * 4, &sm.qfull[bslot],
                          pol_keep);
                bulk_load(sm.w[bslot][lane], sb.p[p].w + (int64_t)it.b * kHeads, kHeads * 4, &sm.qfull[bslot],
                          pol_keep);
            }
            __syncwarp();
            if (++bslot == 2) bslot = 0, bphase ^= 1;
            }  // producer 0's descriptor and queries
            const CUtensorMap* kmap = pool ? &mp.keys8[src] : &mp.keys[src];
            if (pool) {
                // physical first row of every pool block of the item (positions
                // below it.n are valid, so their blocks lie below n_entries)
                const int32_t* pool_ids = P0.pool + (int64_t)it.b * P0.pool_blocks;
                const int slots = (it.n + kPoolBlock - 1) / kPoolBlock;
                const int n_slot = 16 * (it.t1 - it.t0);
                constexpr int kSlotsPerLane = kMaxChunk * 16 / 32;
                __syncwarp();  // the previous item's reads of prow are done
                int blk[kSlotsPerLane], pg[kSlotsPerLane];
#pragma unroll
                for (int j = 0; j < kSlotsPerLane; ++j) {
                    const int i = lane + 32 * j, slot = 16 * it.t0 + i;
                    blk[j] = (i < n_slot && slot < slots) ? pool_ids[slot] : -1;
                    if (blk[j] >= max_pages * (PAGE / kPoolBlock)) blk[j] = -1;  // never past the table
                }
#pragma unroll
                for (int j = 0; j < kSlotsPerLane; ++j) pg[j] = blk[j] >= 0 ? page_table[kPoolBlock * blk[j] / PAGE] : -1;
#pragma unroll
                for (int j = 0; j < kSlotsPerLane; ++j) {
                    const int i = lane + 32 * j;
                    if (i >= n_slot) continue;
                    int r = -1;
                    if (blk[j] >= 0) {
                        if (pg[j] >= 0 && pg[j] < num_pages)
                            r = pg[j] * PAGE + kPoolBlock * blk[j] % PAGE;
                        else
                            atomicOr(status, CSA2_DEVERR_PAGE);
                    }
                    sm.prow[pw][i] = r;
                }
                __syncwarp();
            }
            for (int t = it.t0; t < it.t1; ++t, ++g) {
                if ((g & 1u) != pw) continue;  // the other producer's tile
                const uint32_t stage = g % kStages, sphase = (g / kStages) & 1u;
                if (!mbar_wait_warp(&sm.empty[stage], sphase ^ 1)) {
                    if (lane == 0) raise_abort(sm, status);
                    stop = true;
                    break;
                }
                if (pool) {
                    const int prow = lane < 16 ? sm.prow[pw][16 * (t - it.t0) + lane] : -1;
                    const unsigned have = __ballot_sync(0xffffffffu, prow >= 0);
                    if (have == 0) {
                        mbar_arrive_w(&sm.full[stage]);
                    } else {
                        mbar_expect_tx_w(&sm.full[stage], __popc(have) * kPoolBlock * (ICB + ISB));
                        __syncwarp();
                        if (prow >= 0) {
                            tma_load_2d(sm.a[stage] + lane * kPoolBlock * ICB, kmap, 0, prow, &sm.full[stage],
                                        pol_stream);
                            bulk_load(sm.sfa_raw[stage] + lane * kPoolBlock * ISB, idx_scales + (int64_t)prow * ISB,
                                      kPoolBlock * ISB, &sm.full[stage], pol_stream);
                        }
                        __syncwarp();
                    }
                } else {
                    const int pg0 = __shfl_sync(0xffffffffu, my_pg, 2 * (t - it.t0));
                    const int pg1 = __shfl_sync(0xffffffffu, my_pg, 2 * (t - it.t0) + 1);
                    const uint32_t bytes = (pg0 >= 0 ? PAGE * (ICB + ISB) : 0) + (pg1 >= 0 ? PAGE * (ICB + ISB) : 0);
                    if (bytes == 0) {
                        mbar_arrive_w(&sm.full[stage]);
                    } else if (lane == 0) {
                        mbar_expect_tx(&sm.full[stage], bytes);
                        if (pg0 >= 0) {
                            tma_load_2d(sm.a[stage], kmap, 0, pg0 * PAGE, &sm.full[stage], pol_stream);
                            bulk_load(sm.sfa_raw[stage], idx_scales + (int64_t)pg0 * PAGE * ISB, PAGE * ISB,
                                      &sm.full[stage], pol_stream);
                        }
                        if (pg1 >= 0) {
                            tma_load_2d(sm.a[stage] + PAGE * ICB, kmap, 0, pg1 * PAGE, &sm.full[stage], pol_stream);
                            bulk_load(sm.sfa_raw[stage] + PAGE * ISB, idx_scales + (int64_t)pg1 * PAGE * ISB,
                                      PAGE * ISB, &sm.full[stage], pol_stream);
                        }
                    }
                    __syncwarp();
                }
                issued |= 1u << stage;
                issued_par = (issued_par & ~(1u << stage)) | (sphase << stage);
            }
            stop = stop || __any_sync(0xffffffffu, aborted(sm));
        }
        // the end of the CTA's work: a descriptor with no problems
        if (pw == 0 && !stop && mbar_wait_warp(&sm.qempty[bslot], bphase ^ 1)) {
            if (lane == 0) {
                sm.desc[bslot].nprob = 0;
                mbar_arrive(&sm.qfull[bslot]);
            }
        }
        // never leave with copies in flight
        if (lane == 0)
            for (int s = 0; s < kStages; ++s)
                if ((issued >> s) & 1u) (void)mbar_wait(&sm.full[s], (issued_par >> s) & 1u);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // The pass loop keeps its per-pass work to the MMAs: the accumulator ring
        // index and phase, the query descriptor and the scale column advance by
        // constant steps, and the instruction descriptors are constants (this
        // warp's issue rate, shared with busy epilogue warps, sets the pace).
        uint32_t stage = 0, sphase = 0, bslot = 0, bphase = 0;
        uint32_t acc = 0, aphase = 0;  // accumulator of the next pass, and its ring phase
        constexpr uint32_t kIdesc2a = idesc_mxf4(kPass * kHeads, 0, 0), kIdesc2b = idesc_mxf4(kPass * kHeads, 2, 2);
        constexpr uint32_t kIdesc1a = idesc_mxf4(kHeads, 0, 0), kIdesc1b = idesc_mxf4(kHeads, 2, 2);
        uint32_t* status = sb.p[0].cache.status;
        while (true) {
            if (!mbar_wait_warp(&sm.qfull[bslot], bphase)) {
                if (lane == 0) raise_abort(sm, status);
                break;
            }
            const ItemDesc& D = sm.desc[bslot];
            // lane 0's copies: warp-uniform to the compiler, so the loops below
            // and the tcgen05 operands derived from their counters need no
            // per-lane handling at issue
            const int nprob = __shfl_sync(0xffffffffu, D.nprob, 0);
            const int t0 = __shfl_sync(0xffffffffu, D.t0, 0), t1 = __shfl_sync(0xffffffffu, D.t1, 0);
            if (nprob == 0) break;
            status = D.status;
            const int passes = (nprob + kPass - 1) / kPass;
            static_assert(kPass == 2, "a pass holds two problems, the last pass of an odd subset one");
            const bool odd = (nprob & 1) != 0;
            const uint64_t bdesc0 = smem_desc(sm.b[bslot], 16, 512, kLayoutSw64);
            const uint32_t sfb0 = tbase + kColSfb + bslot * kMaxPasses * 4;
            // the item's query scales into TMEM (the columns' previous reader, the
            // item two back, has completed: its commit preceded this buffer's reload)
            tc_fence_after();
            for (int k = 0; k < passes; ++k) scales_to_tc(sm.sfb_raw[bslot] + k * 512, sm.sfb_tc[bslot][k], lane);
            fence_proxy_async_smem();
            __syncwarp();
            for (int k = 0; k < passes; ++k)
                tc_cp_32x128b_x4_w(tbase + kColSfb + (bslot * kMaxPasses + k) * 4,
                                   smem_desc(sm.sfb_tc[bslot][k], 16, 128, kLayoutNone));
            bool stop = false;
            for (int t = t0; t < t1; ++t) {
                if (!mbar_wait_warp(&sm.full[stage], sphase)) {
                    if (lane == 0) raise_abort(sm, status);
                    stop = true;
                    break;
                }
                // the stage's key scales into TMEM (their previous reader, the tile
                // eight back, completed before the producer could refill the stage)
                tc_fence_after();
                scales_to_tc(sm.sfa_raw[stage], sm.sfa_tc[stage], lane);
                fence_proxy_async_smem();
                __syncwarp();
                const uint32_t sfa = tbase + kColSfa + 4 * stage;
                tc_cp_32x128b_x4_w(sfa, smem_desc(sm.sfa_tc[stage], 16, 128, kLayoutNone));
                const uint64_t adesc = smem_desc(sm.a[stage], 16, 512, kLayoutSw64);
                uint64_t bdesc = bdesc0;  // pass k: the queries of problems kPass k, kPass k + 1
                uint32_t sfb = sfb0;      // and their scale columns
#pragma unroll 1
                for (int k = 0; k < passes; ++k) {
                    if (!mbar_wait_warp(&sm.tempty[acc], aphase ^ 1u)) {
                        if (lane == 0) raise_abort(sm, status);
                        stop = true;
                        break;
                    }
                    tc_fence_after();
                    const bool one = odd && k + 1 == passes;  // an odd subset's last pass: one problem (N = 64)
                    const uint32_t d = tbase + kColAcc + 128 * acc;
                    // K = 0..63 (scale bytes 0, 1), then K = 64..127 (bytes 2, 3): +32 B start
                    tc_mma_mxf4_w(d, adesc, bdesc, one ? kIdesc1a : kIdesc2a, sfa, sfb, 0u);
                    tc_mma_mxf4_w(d, adesc + 2, bdesc + 2, one ? kIdesc1b : kIdesc2b, sfa, sfb, 1u);
                    tc_commit_w(&sm.tfull[acc]);
                    bdesc += (uint64_t)((kPass * kHeads * 64) >> 4);
                    sfb += 4;
                    if (++acc == (uint32_t)kAcc) acc = 0, aphase ^= 1u;
                }
                if (stop) break;
                tc_commit_w(&sm.empty[stage]);  // the stage is free once these MMAs complete
                if (++stage == kStages) stage = 0, sphase ^= 1;
            }
            if (stop) break;
            tc_commit_w(&sm.qempty[bslot]);  // the item's MMAs no longer read its queries
            if (++bslot == 2) bslot = 0, bphase ^= 1;
        }
        // every tcgen05 operation of this thread has completed before TMEM is freed
        tc_commit_w(&sm.drained);
        (void)mbar_wait_warp(&sm.drained, 0);
    } else {
        // ------------------------------------------------------------ epilogue
        // Two groups of eight warps; group g drains the passes p with p % 2 == g.
        // Warp w of a group reads TMEM lane quadrant w % 4 (entries 32 (w % 4) ..
        // + 31 of the tile) and problem (w / 4) % 2 of the pass: two loads of 32
        // head columns (the accumulator is released after the second), ReLU,
        // weight and head sum, one coalesced store per 32 entries.
        const int ew = warp - kEpi0;
        const uint32_t grp = (uint32_t)(ew >> 3);
        const int jp = (ew >> 2) & 1;
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t tlane = tbase + ((uint32_t)(quad * 32) << 16) + kColAcc + 64 * jp;
        uint32_t bslot = 0, bphase = 0, pass_no = 0;
        uint32_t* status = sb.p[0].cache.status;
        while (true) {
            if (!mbar_wait_warp(&sm.qfull[bslot], bphase)) {
                if (lane == 0) raise_abort(sm, status);
                break;
            }
            const ItemDesc& D = sm.desc[bslot];
            const int nprob = __shfl_sync(0xffffffffu, D.nprob, 0);  // warp-uniform, as in the MMA warp
            const int t0 = __shfl_sync(0xffffffffu, D.t0, 0), t1 = __shfl_sync(0xffffffffu, D.t1, 0);
            const int n = D.n;
            if (nprob == 0) break;
            status = D.status;
            const int passes = (nprob + kPass - 1) / kPass;
            bool stop = false;
            for (int t = t0; t < t1 && !stop; ++t) {
                const int e = t * kTile + row;
                for (int k = 0; k < passes; ++k, ++pass_no) {
                    if (pass_no % kGroups != grp) continue;
                    const uint32_t acc = pass_no % kAcc;
                    if (!mbar_wait_warp(&sm.tfull[acc], (pass_no / kAcc) & 1u)) {
                        if (lane == 0) raise_abort(sm, status);
                        stop = true;
                        break;
                    }
                    tc_fence_after();
                    const int j = kPass * k + jp;
                    if (j < nprob) {
                        const float* w = sm.w[bslot][j];
                        float2 acc2[4];
#pragma unroll
                        for (int c = 0; c < 4; ++c) acc2[c] = make_float2(0.0f, 0.0f);
                        {
                            float v0[32];
                            tmem_ld_32x32b_x32(tlane + 128 * acc, v0);
                            relu_weighted_acc(v0, w, acc2);
                        }
                        {
                            float v1[32];
                            tmem_ld_32x32b_x32(tlane + 128 * acc + 32, v1);
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&sm.tempty[acc]);
                            relu_weighted_acc(v1, w + 32, acc2);
                        }
                        const float s = 0.5f * (((acc2[0].x + acc2[0].y) + (acc2[1].x + acc2[1].y)) +
                                                ((acc2[2].x + acc2[2].y) + (acc2[3].x + acc2[3].y)));
                        if (e < n) D.rows[j][e] = s;
                    } else {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sm.tempty[acc]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.qempty[bslot]);
            if (++bslot == 2) bslot = 0, bphase ^= 1;
            if (stop) break;
        }
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
