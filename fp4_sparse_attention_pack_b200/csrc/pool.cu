// Hierarchical sparse indexer ("DeepSeek-V4.1-Flash, expliqué pas à pas", CSA2
// chapter, hierarchical indexer paragraph; the video-summary page gives the
// candidate pool as blocks of 8 positions, 2,048 blocks at a million tokens,
// assembled by the first decoder layer).  The page's step list did not survive;
// this library reads it as: the Full layer's scores are reduced to one maximum
// per block of 8 consecutive entries, the pool is the Top-pool_blocks of those
// maxima (block ids, increasing), and a deeper Reindex layer of the same source
// scores only the pool's entries and keeps its Top-K among them.
//
// The pool build is k_block_max followed by the ordinary Top-K kernel over the
// block-maximum rows.  k_pool_count turns a pool into the number of its valid
// positions, which the restricted scan and its Top-K read on the device.
#include "common.cuh"
#include "kernels.cuh"

namespace csa2 {

namespace {

constexpr int kThreads = 256;

// One thread per block of 8 entries: two 16-byte loads, the maximum of the
// entries below n_entries.
__global__ void __launch_bounds__(kThreads) k_block_max(const __grid_constant__ ScanBatch sb, float* bmax,
                                                        int64_t bstride) {
    const ScanProblem& P = sb.p[blockIdx.z];
    const int b = blockIdx.y;
    const int n = entries_of(P.cache, b);
    const int j = blockIdx.x * kThreads + threadIdx.x;
    if (kPoolBlock * j >= n) return;
    const float* row = P.scores + (int64_t)b * sb.score_stride + kPoolBlock * j;
    float m;
    if (kPoolBlock * j + kPoolBlock <= n) {
        const float4 u = reinterpret_cast<const float4*>(row)[0];
        const float4 v = reinterpret_cast<const float4*>(row)[1];
        m = fmaxf(fmaxf(fmaxf(u.x, u.y), fmaxf(u.z, u.w)), fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
    } else {
        m = row[0];
        for (int r = 1; kPoolBlock * j + r < n; ++r) m = fmaxf(m, row[r]);
    }
    bmax[((int64_t)blockIdx.z * P.cache.batch + b) * bstride + j] = m;
}

// pool_n[b] = the first position 8s + r whose block id is negative or whose
// entry is at or beyond n_entries (8 * pool_blocks when there is none).  For an
// increasing, -1 padded pool every position before it is valid and every one
// after it is not.
__global__ void __launch_bounds__(kThreads) k_pool_count(const __grid_constant__ ScanBatch sb) {
    const ScanProblem& P = sb.p[blockIdx.y];
    if (!P.pool) return;
    const int b = blockIdx.x;
    const int n = entries_of(P.cache, b);
    const int32_t* pool = P.pool + (int64_t)b * P.pool_blocks;
    __shared__ int first;
    if (threadIdx.x == 0) first = kPoolBlock * P.pool_blocks;
    __syncthreads();
    int mine = kPoolBlock * P.pool_blocks;
    for (int s = threadIdx.x; s < P.pool_blocks; s += kThreads) {
        const int64_t e0 = (int64_t)kPoolBlock * pool[s];
        const int64_t left = pool[s] < 0 ? 0 : (int64_t)n - e0;
        const int cnt = (int)(left < 0 ? 0 : (left > kPoolBlock ? kPoolBlock : left));
        if (cnt < kPoolBlock) mine = min(mine, kPoolBlock * s + cnt);
    }
    atomicMin(&first, mine);
    __syncthreads();
    if (threadIdx.x == 0) P.pool_n[b] = first;
}

}  // namespace

cudaError_t launch_block_max(const ScanBatch& sb, float* bmax, int64_t bstride, cudaStream_t st) {
    const int batch = sb.p[0].cache.batch;
    int cap = 0;
    for (int i = 0; i < sb.n; ++i) cap = max(cap, sb.p[i].cache.max_pages * PAGE);
    const int blocks = (cap + kPoolBlock - 1) / kPoolBlock;
    dim3 grid((blocks + kThreads - 1) / kThreads, batch, sb.n);
    k_block_max<<<grid, kThreads, 0, st>>>(sb, bmax, bstride);
    return cudaGetLastError();
}

cudaError_t launch_pool_count(const ScanBatch& sb, cudaStream_t st) {
    const int batch = sb.p[0].cache.batch;
    dim3 grid(batch, sb.n);
    k_pool_count<<<grid, kThreads, 0, st>>>(sb);
    return cudaGetLastError();
}

}  // namespace csa2
