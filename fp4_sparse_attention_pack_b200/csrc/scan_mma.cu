// Indexer scan on the 5th-generation tensor cores: tcgen05.mma kind::mxf4
// (E2M1 operands, one E8M0 scale per 32 channels applied by the hardware,
// fp32 accumulation in TMEM).
//
//   score[b][e] = sum_h w[b][h] * max(0, qhat[b][h] . khat[b][e])
//
// With 64 indexer heads every key meets 64 x 128 MXFP4 products: a dense
// contraction (about 240 flop per key byte) that CUDA cores cannot keep up
// with at HBM speed, while the FP4 tensor cores need well under half the HBM
// time.  Per 128-entry tile: D[128 entries x 64 heads] = K[128 x 128] . Q^T,
// two MMAs of K = 64 each; the epilogue applies ReLU, the head weights and the
// head sum, one thread per entry row.
//
// Persistent, warp-specialised CTA (320 threads, two CTAs per SM):
//   warp 0  producer: TMA tile loads of the keys (one 64-entry page per box,
//           64-byte swizzle) and bulk copies of their E8M0 scales into an
//           8-stage ring; per work item also the query tile, its scales and
//           the head weights.  Keys stream with an L2 evict-first policy.
//   warp 1  MMA issuer: rearranges each stage's scales into the 32x128-bit
//           layout tcgen05.cp copies into TMEM, then issues the two MMAs into
//           one of two TMEM accumulators and commits the stage back.
//   warps 2-9 epilogue, two groups of four (one TMEM lane quadrant per warp);
//           group g drains accumulator g (every other tile): tcgen05.ld of the
//           64 head columns of its entry, ReLU, weight, sum, one score store.
// Work item = (problem, sequence, chunk of kChunkTiles tiles), round-robin over
// the grid.  Every wait is bounded; a timeout sets CSA2_DEVERR_TIMEOUT in the
// problem's status word and the CTA drains and exits.
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

constexpr int kHeads = 64;        // MMA N (indexer heads)
constexpr int kStages = 8;
constexpr int kTile = 128;        // entries per MMA tile (MMA M)
constexpr int kChunkTiles = 16;   // tiles per work item
constexpr int kThreads = 320;     // producer, MMA issuer, 2 x 4 epilogue warps
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColAcc = 0;         // 2 x 64 accumulator columns
constexpr uint32_t kColSfa = 128;       // kStages x 4 scale columns (A)
constexpr uint32_t kColSfb = 128 + 4 * kStages;  // 2 x 4 scale columns (B)
constexpr int kMaxSources = CSA2_MAX_SOURCES;

struct MmaScanMaps {
    CUtensorMap keys[kMaxSources];  // per distinct cache: idx codes [num_pages*64][64 B]
    CUtensorMap queries;            // [n * batch * 64][64 B]
    int src_of[kMaxProblems];       // problem -> keys[] index
    int chunks;                     // work items per (problem, sequence)
};

struct __align__(1024) Smem {
    uint8_t a[kStages][kTile * 64];     // key codes, 64B-swizzled rows
    uint8_t b[2][kHeads * 64];          // query codes, 64B-swizzled rows
    uint8_t sfa_raw[kStages][kTile * 4];
    uint8_t sfa_tc[kStages][512];       // 32 rows x 16 B for tcgen05.cp
    uint8_t sfb_raw[2][kHeads * 4];
    uint8_t sfb_tc[2][512];
    float w[2][kHeads];
    uint64_t full[kStages], empty[kStages];
    uint64_t bfull[2], bempty[2];
    uint64_t tfull[2], tempty[2];
    uint64_t drained;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory beyond the 227 KB per-block limit");


struct Item {
    int p, b, t0, t1, n;
};

__device__ __forceinline__ bool item_at(const ScanBatch& sb, const MmaScanMaps& mp, int id, Item& it) {
    const int batch = sb.p[0].cache.batch;
    const int per_p = batch * mp.chunks;
    it.p = id / per_p;
    const int r = id - it.p * per_p;
    it.b = r / mp.chunks;
    const int c = r - it.b * mp.chunks;
    it.n = entries_of(sb.p[it.p].cache, it.b);
    const int tiles = (it.n + kTile - 1) / kTile;
    it.t0 = c * kChunkTiles;
    it.t1 = min(it.t0 + kChunkTiles, tiles);
    return it.t0 < it.t1;
}

__device__ __forceinline__ void raise_abort(Smem& sm, uint32_t* status) {
    atomicOr(status, CSA2_DEVERR_TIMEOUT);
    *reinterpret_cast<volatile int*>(&sm.abort) = 1;
}

__device__ __forceinline__ bool aborted(Smem& sm) {
    return *reinterpret_cast<volatile int*>(&sm.abort) != 0;
}

__global__ void __launch_bounds__(kThreads, 2)
    k_scan_mma(const __grid_constant__ ScanBatch sb, const __grid_constant__ MmaScanMaps mp) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int batch = sb.p[0].cache.batch;
    const int n_items = sb.n * batch * mp.chunks;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.bfull[i], 1);
            mbar_init(&sm.bempty[i], 1 + 8);
            mbar_init(&sm.tfull[i], 1);
            mbar_init(&sm.tempty[i], 4);  // the four warps of epilogue group i
        }
        mbar_init(&sm.drained, 1);
        sm.abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&sm.tmem_base, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = sm.tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        // Lanes fetch the item's page ids (2 per tile, up to 32) in one round;
        // lane 0 issues every copy.
        const uint64_t pol_stream = policy_evict_first();
        const uint64_t pol_keep = policy_evict_last();
        if (lane == 0) prefetch_tmap(&mp.queries);
        uint32_t stage = 0, sphase = 0, bslot = 0, bphase = 0;
        int issued[kStages];
        uint32_t issued_par[kStages];
        for (int s = 0; s < kStages; ++s) issued[s] = 0, issued_par[s] = 0;
        for (int id = blockIdx.x; id < n_items && !__any_sync(0xffffffffu, aborted(sm)); id += gridDim.x) {
            Item it;
            if (!item_at(sb, mp, id, it)) continue;
            const ScanProblem& P = sb.p[it.p];
            const CacheView& c = P.cache;
            const int used_pages = (it.n + PAGE - 1) / PAGE;
            const int li = 2 * it.t0 + lane;  // logical page this lane looks up
            int my_pg = -1;
            if (lane < 2 * (it.t1 - it.t0) && li < used_pages) {
                const int pp = c.page_table[(int64_t)it.b * c.max_pages + li];
                if (pp >= 0 && pp < c.num_pages)
                    my_pg = pp;
                else
                    atomicOr(c.status, CSA2_DEVERR_PAGE);
            }
            bool stop = false;
            if (lane == 0) {
                if (!mbar_wait(&sm.bempty[bslot], bphase ^ 1)) {
                    raise_abort(sm, c.status);
                    stop = true;
                } else {
                    const int64_t qrow = ((int64_t)it.p * batch + it.b) * kHeads;
                    mbar_expect_tx(&sm.bfull[bslot], kHeads * 64 + kHeads * 4 + kHeads * 4);
                    tma_load_2d(sm.b[bslot], &mp.queries, 0, (int)qrow, &sm.bfull[bslot], pol_keep);
                    bulk_load(sm.sfb_raw[bslot], sb.qs + qrow * ISB, kHeads * 4, &sm.bfull[bslot], pol_keep);
                    bulk_load(sm.w[bslot], P.w + (int64_t)it.b * kHeads, kHeads * 4, &sm.bfull[bslot], pol_keep);
                }
            }
            if (++bslot == 2) bslot = 0, bphase ^= 1;
            const CUtensorMap* kmap = &mp.keys[mp.src_of[it.p]];
            for (int t = it.t0; t < it.t1 && !__any_sync(0xffffffffu, stop); ++t) {
                const int pg0 = __shfl_sync(0xffffffffu, my_pg, 2 * (t - it.t0));
                const int pg1 = __shfl_sync(0xffffffffu, my_pg, 2 * (t - it.t0) + 1);
                if (lane == 0) {
                    if (!mbar_wait(&sm.empty[stage], sphase ^ 1)) {
                        raise_abort(sm, c.status);
                        stop = true;
                    } else {
                        const int pg[2] = {pg0, pg1};
                        const uint32_t bytes = (pg0 >= 0 ? PAGE * (ICB + ISB) : 0) + (pg1 >= 0 ? PAGE * (ICB + ISB) : 0);
                        if (bytes == 0) {
                            mbar_arrive(&sm.full[stage]);
                        } else {
                            mbar_expect_tx(&sm.full[stage], bytes);
                            for (int h = 0; h < 2; ++h) {
                                if (pg[h] < 0) continue;
                                tma_load_2d(sm.a[stage] + h * PAGE * ICB, kmap, 0, pg[h] * PAGE, &sm.full[stage],
                                            pol_stream);
                                bulk_load(sm.sfa_raw[stage] + h * PAGE * ISB,
                                          c.idx_scales + (int64_t)pg[h] * PAGE * ISB, PAGE * ISB, &sm.full[stage],
                                          pol_stream);
                            }
                        }
                        issued[stage] = 1;
                        issued_par[stage] = sphase;
                    }
                }
                if (++stage == kStages) stage = 0, sphase ^= 1;
            }
            if (__any_sync(0xffffffffu, stop)) break;
        }
        // never leave with copies in flight
        if (lane == 0)
            for (int s = 0; s < kStages; ++s)
                if (issued[s]) (void)mbar_wait(&sm.full[s], issued_par[s]);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        uint32_t stage = 0, sphase = 0, bslot = 0, bphase = 0, acc = 0, aphase = 0;
        const uint32_t idesc_lo = idesc_mxf4(kHeads, 0, 0);
        const uint32_t idesc_hi = idesc_mxf4(kHeads, 2, 2);
        for (int id = blockIdx.x; id < n_items && !__any_sync(0xffffffffu, aborted(sm)); id += gridDim.x) {
            Item it;
            if (!item_at(sb, mp, id, it)) continue;
            uint32_t* status = sb.p[it.p].cache.status;
            if (!mbar_wait_warp(&sm.bfull[bslot], bphase)) { raise_abort(sm, status); break; }
            {   // query scales -> 32x128b layout: row r holds heads r and 32 + r
                const uint32_t* src = reinterpret_cast<const uint32_t*>(sm.sfb_raw[bslot]);
                uint4 v = make_uint4(src[lane], src[32 + lane], 0u, 0u);
                reinterpret_cast<uint4*>(sm.sfb_tc[bslot])[lane] = v;
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tc_fence_after();
                    tc_cp_32x128b_x4(tbase + kColSfb + 4 * bslot, smem_desc(sm.sfb_tc[bslot], 16, 128, kLayoutNone));
                }
                __syncwarp();
            }
            const uint64_t bdesc = smem_desc(sm.b[bslot], 16, 512, kLayoutSw64);
            bool stop = false;
            for (int t = it.t0; t < it.t1; ++t) {
                if (!mbar_wait_warp(&sm.full[stage], sphase)) { raise_abort(sm, status); stop = true; break; }
                {   // key scales -> 32x128b layout: row r holds entries r, 32+r, 64+r, 96+r
                    const uint32_t* src = reinterpret_cast<const uint32_t*>(sm.sfa_raw[stage]);
                    uint4 v = make_uint4(src[lane], src[32 + lane], src[64 + lane], src[96 + lane]);
                    reinterpret_cast<uint4*>(sm.sfa_tc[stage])[lane] = v;
                    fence_proxy_async_smem();
                }
                __syncwarp();
                if (!mbar_wait_warp(&sm.tempty[acc], aphase ^ 1)) { raise_abort(sm, status); stop = true; break; }
                if (lane == 0) {
                    tc_fence_after();
                    const uint32_t sfa = tbase + kColSfa + 4 * stage;
                    const uint32_t sfb = tbase + kColSfb + 4 * bslot;
                    const uint32_t d = tbase + kColAcc + kHeads * acc;
                    tc_cp_32x128b_x4(sfa, smem_desc(sm.sfa_tc[stage], 16, 128, kLayoutNone));
                    const uint64_t adesc = smem_desc(sm.a[stage], 16, 512, kLayoutSw64);
                    // K = 0..63 (scale bytes 0, 1), then K = 64..127 (bytes 2, 3): +32 B start
                    tc_mma_mxf4(d, adesc, bdesc, idesc_lo, sfa, sfb, 0u);
                    tc_mma_mxf4(d, adesc + 2, bdesc + 2, idesc_hi, sfa, sfb, 1u);
                    tc_commit(&sm.empty[stage]);
                    tc_commit(&sm.tfull[acc]);
                }
                __syncwarp();
                if (++stage == kStages) stage = 0, sphase ^= 1;
                acc ^= 1;
                if (acc == 0) aphase ^= 1;
            }
            if (lane == 0) tc_commit(&sm.bempty[bslot]);
            __syncwarp();
            if (++bslot == 2) bslot = 0, bphase ^= 1;
            if (stop) break;
        }
        // every tcgen05 operation of this thread has completed before TMEM is freed
        if (lane == 0) {
            tc_commit(&sm.drained);
            (void)mbar_wait(&sm.drained, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        // Group g = (warp - 2) / 4 drains accumulator g, i.e. every other tile.
        const int grp = (warp - 2) >> 2;
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        uint32_t bslot = 0, bphase = 0, aphase = 0, tile_no = 0;
        for (int id = blockIdx.x; id < n_items && !__any_sync(0xffffffffu, aborted(sm)); id += gridDim.x) {
            Item it;
            if (!item_at(sb, mp, id, it)) continue;
            const ScanProblem& P = sb.p[it.p];
            if (!mbar_wait_warp(&sm.bfull[bslot], bphase)) { raise_abort(sm, P.cache.status); break; }
            const float* w = sm.w[bslot];
            float* out = P.scores + (int64_t)it.b * sb.score_stride;
            bool stop = false;
            for (int t = it.t0; t < it.t1; ++t, ++tile_no) {
                if ((int)(tile_no & 1u) != grp) continue;
                if (!mbar_wait_warp(&sm.tfull[grp], aphase)) { raise_abort(sm, P.cache.status); stop = true; break; }
                aphase ^= 1;
                tc_fence_after();
                float v[64];
                tmem_ld_32x32b_x64(tbase + ((uint32_t)(quad * 32) << 16) + kColAcc + kHeads * grp, v);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.tempty[grp]);
                float part[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // four independent chains
#pragma unroll
                for (int h = 0; h < kHeads; h += 4) {
                    const float4 w4 = *reinterpret_cast<const float4*>(w + h);
                    part[0] = fmaf(w4.x, fmaxf(v[h], 0.0f), part[0]);
                    part[1] = fmaf(w4.y, fmaxf(v[h + 1], 0.0f), part[1]);
                    part[2] = fmaf(w4.z, fmaxf(v[h + 2], 0.0f), part[2]);
                    part[3] = fmaf(w4.w, fmaxf(v[h + 3], 0.0f), part[3]);
                }
                const float s = (part[0] + part[1]) + (part[2] + part[3]);
                const int e = t * kTile + row;
                if (e < it.n) out[e] = s;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.bempty[bslot]);
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

int sm_count() {
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
    int srcs = 0;
    const uint8_t* seen[kMaxSources];
    int cap = 0;
    for (int i = 0; i < sb.n; ++i) {
        const CacheView& c = sb.p[i].cache;
        cap = max(cap, c.max_pages * PAGE);
        int j = 0;
        for (; j < srcs; ++j)
            if (seen[j] == c.idx_codes) break;
        if (j == srcs) {
            seen[srcs] = c.idx_codes;
            if (!make_rows64_map(&mp.keys[srcs], c.idx_codes, (uint64_t)c.num_pages * PAGE, PAGE))
                return cudaErrorInvalidValue;
            ++srcs;
        }
        mp.src_of[i] = j;
    }
    if (!make_rows64_map(&mp.queries, sb.qc, (uint64_t)sb.n * batch * kHeads, kHeads))
        return cudaErrorInvalidValue;
    const int tiles = (cap + kTile - 1) / kTile;
    mp.chunks = (tiles + kChunkTiles - 1) / kChunkTiles;
    const long n_items = (long)sb.n * batch * mp.chunks;
    const int grid = (int)std::min<long>(n_items, 2L * sm_count());
    const size_t smem = sizeof(Smem) + 1024;
    static const bool attr = [smem] {
        cudaFuncSetAttribute(k_scan_mma, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        return true;
    }();
    (void)attr;
    k_scan_mma<<<grid, kThreads, smem, st>>>(sb, mp);
    return cudaGetLastError();
}

}  // namespace csa2
