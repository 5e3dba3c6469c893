// Per-sequence Top-K of the indexer scores (the pages' indexer keeps the 512
// best-scoring entries: "DeepSeek-V4.1-Flash, expliqué pas à pas", attention
// taxonomy).
//
// Scores map to order-preserving uint32 keys; the K largest are kept, equal
// scores lower index first, and written in increasing index order.  A row is a
// problem's score row (entries), its pool positions (hierarchical indexer: the
// winners are written as the entries they stand for), or its block maxima
// (pool build: the winners are block ids).
//
// One CTA of 512 threads per (problem, sequence):
//   1. Threshold guess: 2,048 samples of the row (256 evenly spaced runs of 8
//      consecutive scores); a radix select in shared memory finds the leading
//      16 bits of the sample key ranked ~2K * 2048 / n, so that about 2K of the
//      n scores lie at or above it.
//   2. One pass over the row compacts every score at or above the guess, in
//      index order, into shared memory (at most kCap).  If fewer than K or more
//      than kCap qualify, the CTA falls back to an exact radix select over the
//      whole row (two or more passes), so the result never depends on the guess.
//   3. Exact radix select among the candidates (8-bit digits, warp-aggregated
//      shared-memory histograms), then an ordered compaction of the keys above
//      the K-th key plus the first `need` keys equal to it.
// A key equal to the K-th largest is >= the guess whenever >= K keys are, so
// every member of the Top-K (ties included) is among the candidates.
#include "common.cuh"
#include "kernels.cuh"

namespace csa2 {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kSamples = 2048;
constexpr int kCap = 4096;  // candidates kept in shared memory (the guess targets about 2K + 1 %)
constexpr int kRun = 8;   // contiguous scores per thread per pass
constexpr int kSampleRun = 8;  // consecutive scores per sample run (one 32-byte sector)

struct TopkSmem {
    uint32_t key[kCap];
    int32_t idx[kCap];
    int hist[256];
    int warp_tot[33];
    int sel[2];
    int flag;
};
static_assert(sizeof(TopkSmem) + 1024 <= 232448, "shared memory beyond the 227 KB per-block limit");


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
        int t = lane < kWarps ? s_warp[lane] : 0;
        int u = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, u, o);
            if (lane >= o) u += y;
        }
        s_warp[lane] = u - t;
        if (lane == 31) s_warp[32] = u;
    }
    __syncthreads();
    *excl = s_warp[wid] + x - v;
    const int total = s_warp[32];
    __syncthreads();
    return total;
}

// Add one to hist[d] for every active lane with d < 256, one atomic per distinct d.
__device__ __forceinline__ void hist_add(int* hist, uint32_t d) {
    const unsigned act = __activemask();
    const unsigned same = __match_any_sync(act, d);
    if (d < 256 && (threadIdx.x & 31) == (__ffs(same) - 1)) atomicAdd(&hist[d], __popc(same));
}

// Exact radix select: the k-th largest key among key(i), i < cnt (k <= cnt), and
// how many keys equal to it belong to the top k.  8-bit digits, MSB first.
// With passes < 4 the result is the k-th largest key's leading 8 * passes bits
// with the rest zero, a lower bound of it (need is then meaningless).
template <class KeyAt>
__device__ void radix_select(KeyAt key_at, int cnt, int k, TopkSmem& sm, uint32_t* kth, int* need, int passes = 4) {
    uint32_t prefix = 0, mask = 0;
    int remaining = k;
    const int tid = threadIdx.x;
    for (int pass = 0; pass < passes; ++pass) {
        const int sh = 24 - 8 * pass;
        if (tid < 256) sm.hist[tid] = 0;
        __syncthreads();
        for (int i0 = 0; i0 < cnt; i0 += kThreads) {
            const int i = i0 + tid;
            uint32_t d = 256;
            if (i < cnt) {
                const uint32_t kk = key_at(i);
                if ((kk & mask) == prefix) d = (kk >> sh) & 255u;
            }
            hist_add(sm.hist, d);
        }
        __syncthreads();
        // bins in decreasing digit order: thread t owns digit 255 - t
        const int c = tid < 256 ? sm.hist[255 - tid] : 0;
        int above;
        block_excl_scan(c, sm.warp_tot, &above);
        if (tid < 256 && above < remaining && above + c >= remaining) {
            sm.sel[0] = 255 - tid;
            sm.sel[1] = remaining - above;
        }
        __syncthreads();
        prefix |= (uint32_t)sm.sel[0] << sh;
        mask |= 255u << sh;
        remaining = sm.sel[1];
        __syncthreads();
    }
    *kth = prefix;
    *need = remaining;
}

// Ordered compaction of the Top-K: keys above kth, then (in index order) the
// first `need` keys equal to it.  Writes out positions [0, K), each as
// out_of(row position).  Each thread takes a contiguous run of kRun keys per round.
template <class KeyAt, class IdxAt, class OutOf>
__device__ void emit_topk(KeyAt key_at, IdxAt idx_at, OutOf out_of, int cnt, uint32_t kth, int need, int K,
                          TopkSmem& sm, int32_t* io, float* so) {
    int base_out = 0, eq_seen = 0;
    for (int base = 0; base < cnt; base += kThreads * kRun) {
        const int i0 = base + threadIdx.x * kRun;
        uint32_t kk[kRun];
        int gt = 0, eq = 0;
#pragma unroll
        for (int v = 0; v < kRun; ++v) {
            kk[v] = (i0 + v < cnt) ? key_at(i0 + v) : 0u;
            gt += (i0 + v < cnt) && (kk[v] > kth);
            eq += (i0 + v < cnt) && (kk[v] == kth);
        }
        int eq_rank;
        const int eq_tot = block_excl_scan(eq, sm.warp_tot, &eq_rank);
        // equal keys this thread may take: those whose rank among equals is < need
        const int eq_take = max(0, min(eq, need - (eq_seen + eq_rank)));
        int pos;
        const int take_tot = block_excl_scan(gt + eq_take, sm.warp_tot, &pos);
        int o = base_out + pos, e_left = eq_take;
#pragma unroll
        for (int v = 0; v < kRun; ++v) {
            if (i0 + v >= cnt) continue;
            bool take = kk[v] > kth;
            if (kk[v] == kth && e_left > 0) {
                take = true;
                --e_left;
            }
            if (take) {
                if (o < K) {
                    io[o] = out_of(idx_at(i0 + v));
                    if (so) so[o] = order_key_f32(kk[v]);
                }
                ++o;
            }
        }
        base_out += take_tot;
        eq_seen += eq_tot;
        if (base_out >= K) break;
    }
}

__global__ void __launch_bounds__(kThreads, 4) k_topk(const __grid_constant__ ScanBatch sb) {
    extern __shared__ uint8_t smem_raw[];
    TopkSmem& sm = *reinterpret_cast<TopkSmem*>(smem_raw);
    const ScanProblem& P = sb.p[blockIdx.y];
    const int b = blockIdx.x;
    const int K = P.K > 0 ? P.K : sb.K;
    const int n = row_len(P, b);
    const float* row = P.scores + (int64_t)b * (P.row_stride > 0 ? P.row_stride : sb.score_stride);
    int32_t* io = P.idx_out + (int64_t)b * K;
    float* so = P.score_out ? P.score_out + (int64_t)b * K : nullptr;
    const int tid = threadIdx.x;
    auto out_of = [&](int i) { return row_entry(P, b, i); };

    if (n <= K) {
        for (int i = tid; i < K; i += kThreads) {
            io[i] = i < n ? out_of(i) : -1;
            if (so) so[i] = i < n ? row[i] : 0.0f;
        }
        return;
    }

    // 1. threshold guess from sampled scores (all scores qualify when they fit):
    // about 2K candidates, at most halfway from K to kCap
    uint32_t guess = 0;
    if (n > kCap && K < kCap) {
        // 256 evenly spaced runs of 8 consecutive scores, one 32-byte sector
        // each: single samples every n / 2048 scores would touch every cache
        // line of a 65,536-entry row and cost the memory traffic of the row
        for (int i = tid; i < kSamples; i += kThreads) {
            const int r = i / kSampleRun, j = i % kSampleRun;
            const int64_t start = ((int64_t)r * n / (kSamples / kSampleRun)) & ~(int64_t)(kSampleRun - 1);
            sm.key[i] = f32_order_key(row[min(start + j, (int64_t)n - 1)]);
        }
        __syncthreads();
        const int64_t target = min((int64_t)2 * K, (int64_t)(K + kCap) / 2);
        const int rank = min(kSamples, (int)((target * kSamples + n - 1) / n) + 16);
        // the sample's leading 16 bits suffice: the guess only has to lie at or
        // below the rank-th sample (within 1/128 of it for positive scores)
        int unused;
        radix_select([&](int i) { return sm.key[i]; }, kSamples, rank, sm, &guess, &unused, 2);
    }

    // 2. one pass: ordered compaction of the scores at or above the guess.  Each
    // thread takes a contiguous run of kRun scores, so a chunk of kThreads * kRun
    // scores costs four vector loads and one block scan per thread.
    int cnt = 0;
    bool fits = K < kCap;  // with K >= kCap the candidates never fit: straight to the exact select
    for (int base = 0; fits && base < n; base += kThreads * kRun) {
        const int i0 = base + tid * kRun;
        uint32_t kk[kRun];
        if (i0 + kRun <= n) {
#pragma unroll
            for (int v = 0; v < kRun / 4; ++v) {
                const float4 f = *reinterpret_cast<const float4*>(row + i0 + 4 * v);
                kk[4 * v] = f32_order_key(f.x);
                kk[4 * v + 1] = f32_order_key(f.y);
                kk[4 * v + 2] = f32_order_key(f.z);
                kk[4 * v + 3] = f32_order_key(f.w);
            }
        } else {
#pragma unroll
            for (int v = 0; v < kRun; ++v) kk[v] = (i0 + v < n) ? f32_order_key(row[i0 + v]) : 0u;
        }
        int c = 0;
#pragma unroll
        for (int v = 0; v < kRun; ++v) c += (i0 + v < n) && (kk[v] >= guess);
        int pos;
        const int tot = block_excl_scan(c, sm.warp_tot, &pos);
        if (cnt + tot <= kCap) {
            int o = cnt + pos;
#pragma unroll
            for (int v = 0; v < kRun; ++v)
                if ((i0 + v < n) && (kk[v] >= guess)) {
                    sm.key[o] = kk[v];
                    sm.idx[o] = i0 + v;
                    ++o;
                }
        }
        cnt += tot;
        if (cnt > kCap) {
            fits = false;
            break;
        }
    }
    __syncthreads();

    uint32_t kth;
    int need;
    if (fits && cnt >= K) {
        // 3. exact selection among the candidates (already in index order)
        radix_select([&](int i) { return sm.key[i]; }, cnt, K, sm, &kth, &need);
        emit_topk([&](int i) { return sm.key[i]; }, [&](int i) { return sm.idx[i]; }, out_of, cnt, kth, need, K,
                  sm, io, so);
    } else {
        // the guess failed: exact radix select over the whole row
        auto gkey = [&](int i) { return f32_order_key(row[i]); };
        radix_select(gkey, n, K, sm, &kth, &need);
        emit_topk(gkey, [](int i) { return i; }, out_of, n, kth, need, K, sm, io, so);
    }
}

}  // namespace

cudaError_t launch_topk(const ScanBatch& sb, cudaStream_t st) {
    const int batch = sb.p[0].cache.batch;
    const size_t smem = sizeof(TopkSmem);
    static std::atomic<uint64_t> attr_done{0};
    const cudaError_t ea = smem_opt_in(reinterpret_cast<const void*>(k_topk), (int)smem, attr_done);
    if (ea != cudaSuccess) return ea;
    dim3 grid(batch, sb.n);
    k_topk<<<grid, kThreads, smem, st>>>(sb);
    return cudaGetLastError();
}

}  // namespace csa2
