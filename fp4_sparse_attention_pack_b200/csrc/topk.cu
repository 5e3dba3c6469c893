// Per-sequence Top-K of the indexer scores: block-level radix select.
//
// Scores map to order-preserving uint32 keys.  Three MSB-first passes with
// 11/11/10-bit digits find the key T of the K-th largest score and how many
// elements equal to T are still needed; a final pass compacts, in index order,
// every element with key > T and the first `need` elements with key == T
// (equal scores: lower index first).  The output is therefore sorted by index.
// One CTA of 1024 threads per (problem, sequence).
#include "common.cuh"
#include "kernels.cuh"

namespace csa2 {

namespace {

constexpr int kThreads = 1024;

// Exclusive prefix sum of one int per thread over the block; returns the total.
__device__ __forceinline__ int block_excl_scan(int v, int* s_warp, int* excl) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[wid] = x;
    __syncthreads();
    if (wid == 0) {
        int t = s_warp[lane];
        int u = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, u, o);
            if (lane >= o) u += y;
        }
        s_warp[lane] = u - t;       // exclusive warp offsets
        if (lane == 31) s_warp[32] = u;  // total
    }
    __syncthreads();
    *excl = s_warp[wid] + x - v;
    const int total = s_warp[32];
    __syncthreads();
    return total;
}

__global__ void __launch_bounds__(kThreads) k_topk(ScanBatch sb) {
    __shared__ int hist[2048];
    __shared__ int s_warp[33];
    __shared__ int s_sel[2];
    const ScanProblem& P = sb.p[blockIdx.y];
    const int b = blockIdx.x;
    const int K = sb.K;
    const int n = entries_of(P.cache, b);
    const float* row = P.scores + (int64_t)b * sb.score_stride;
    int32_t* io = P.idx_out + (int64_t)b * K;
    float* so = P.score_out ? P.score_out + (int64_t)b * K : nullptr;
    const int tid = threadIdx.x;

    if (n <= K) {
        for (int i = tid; i < K; i += kThreads) {
            io[i] = i < n ? i : -1;
            if (so) so[i] = i < n ? row[i] : 0.0f;
        }
        return;
    }

    uint32_t prefix = 0, mask = 0;
    int remaining = K;
    const int shifts[3] = {21, 10, 0};
    const int widths[3] = {11, 11, 10};
    for (int pass = 0; pass < 3; ++pass) {
        const int sh = shifts[pass], nb = 1 << widths[pass];
        for (int i = tid; i < 2048; i += kThreads) hist[i] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += kThreads) {
            const uint32_t k = f32_order_key(row[i]);
            if ((k & mask) == prefix) atomicAdd(&hist[(k >> sh) & (nb - 1)], 1);
        }
        __syncthreads();
        // suffix counts: thread t owns bins [2t, 2t+1]; scan from the top bin
        const int t_hi = kThreads - 1 - tid;  // reversed owner so the scan runs top-down
        int c0 = 0, c1 = 0;
        if (2 * t_hi + 1 < nb) c1 = hist[2 * t_hi + 1];
        if (2 * t_hi < nb) c0 = hist[2 * t_hi];
        int above;
        block_excl_scan(c0 + c1, s_warp, &above);  // count in bins above 2*t_hi+1
        // the digit where the running count from the top reaches `remaining`
        if (2 * t_hi + 1 < nb && above < remaining && above + c1 >= remaining) {
            s_sel[0] = 2 * t_hi + 1;
            s_sel[1] = remaining - above;
        } else if (2 * t_hi < nb && above + c1 < remaining && above + c1 + c0 >= remaining) {
            s_sel[0] = 2 * t_hi;
            s_sel[1] = remaining - above - c1;
        }
        __syncthreads();
        prefix |= (uint32_t)s_sel[0] << sh;
        mask |= (uint32_t)(nb - 1) << sh;
        remaining = s_sel[1];
        __syncthreads();
    }
    const uint32_t T = prefix;
    const int need_eq = remaining;  // elements equal to T still to take

    int base = 0, eq_seen = 0;
    for (int start = 0; start < n; start += kThreads) {
        const int i = start + tid;
        const float f = i < n ? row[i] : 0.0f;
        const uint32_t k = f32_order_key(f);
        const int gt = (i < n) && (k > T);
        const int eq = (i < n) && (k == T);
        int eq_rank;
        const int eq_tot = block_excl_scan(eq, s_warp, &eq_rank);
        const int take = gt || (eq && (eq_seen + eq_rank) < need_eq);
        int pos;
        const int take_tot = block_excl_scan(take, s_warp, &pos);
        if (take && base + pos < K) {
            io[base + pos] = i;
            if (so) so[base + pos] = f;
        }
        base += take_tot;
        eq_seen += eq_tot;
        if (base >= K) break;
    }
}

}  // namespace

cudaError_t launch_topk(const ScanBatch& sb, cudaStream_t st) {
    const int batch = sb.p[0].cache.batch;
    dim3 grid(batch, sb.n);
    k_topk<<<grid, kThreads, 0, st>>>(sb);
    return cudaGetLastError();
}

}  // namespace csa2
