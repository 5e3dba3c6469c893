// Internal launchers of the CSA2 kernels (host side of csrc/*.cu).
#pragma once

#include <atomic>

#include "common.cuh"

namespace csa2 {

// Opt `func` into `bytes` of dynamic shared memory on the current device.  The
// attribute is per device, so it is set once per device (bit d of `done`) and
// its error is returned; devices 64 and up set it on every call.
inline cudaError_t smem_opt_in(const void* func, int bytes, std::atomic<uint64_t>& done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

// Host-side checks of a cache descriptor made before any launch: CSA2_OK, or
// CSA2_ERR_INVALID_ARG (a null pointer, a bad size or ratio), CSA2_ERR_ALIGN (a
// pointer not 16-byte aligned) or CSA2_ERR_UNSUPPORTED (capacity beyond 2^30).
int check_cache(const csa2_cache* c);

// Host-side fault injection for tests of callers' error paths: true when the
// environment variable CSA2_INJECT_FAULT names `entry` (a comma-separated list
// of entry-point names, or "*" for all).  The entry point then returns
// CSA2_ERR_CUDA after its argument checks and before its first launch, as if
// the launch had failed.  Unset (the default), it costs one getenv per call.
bool inject_fault(const char* entry);

// Multiprocessors of the current device (148 when the query fails).
inline int device_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    return n;
}

// ---- cache write: the same T new tokens per sequence for each listed source
constexpr int kMaxPackSources = 8;
struct PackBatch {
    CacheView cache[kMaxPackSources];
    const void* x[kMaxPackSources];      // [batch][T][512] bf16 or fp32
    const float* gates[kMaxPackSources]; // [batch][T]
    const float* W[kMaxPackSources];     // [512][128]
    int n;
};
cudaError_t launch_pack(const PackBatch& pb, bool x_f32, int T, cudaStream_t st);

// ---- indexer
// One scan problem: one indexer query set over one cache, for all sequences.
struct ScanProblem {
    CacheView cache;
    const uint16_t* q_idx;  // bf16 [batch][H_idx][128]
    const float* w;         // fp32 [batch][H_idx]
    float* scores;          // workspace: fp32 [batch][score_stride]
    int32_t* idx_out;       // [batch][K]
    float* score_out;       // nullable [batch][K]
    // Hierarchical indexer.  pool (nullable): [batch][pool_blocks] ids of
    // 8-entry blocks, increasing, -1 padded.  The problem then scores only the
    // pool's entries: position i of its score row is entry 8 * pool[i / 8] + i % 8,
    // and pool_n[b] (written by launch_pool_count) is the number of valid
    // positions, a prefix of the row.
    const int32_t* pool;
    int32_t* pool_n;        // [batch]
    int pool_blocks;
    int block_rows;         // the score row holds block maxima: ceil(n_entries / 8) of them
    int K;                  // Top-K of this row (0: the batch's K)
    int64_t row_stride;     // floats between sequences' score rows (0: the batch's score_stride)
};

constexpr int kMaxProblems = 64;
struct ScanBatch {
    ScanProblem p[kMaxProblems];
    uint8_t* qc;            // workspace: MXFP4 query codes [n][batch][H_idx][64]
    uint8_t* qs;            // workspace: E8M0 query scales [n][batch][H_idx][4]
    int64_t score_stride;   // entries per score row (>= every problem's capacity)
    int n;
    int H_idx;
    int K;
};

constexpr int kPoolBlock = 8;  // entries per hierarchical-indexer block

// Length of problem P's score row for sequence b.
__device__ __forceinline__ int row_len(const ScanProblem& P, int b) {
    if (P.pool) return P.pool_n[b];
    const int n = entries_of(P.cache, b);
    return P.block_rows ? (n + kPoolBlock - 1) / kPoolBlock : n;
}

// Entry (or block id) at position i of problem P's score row for sequence b.
__device__ __forceinline__ int row_entry(const ScanProblem& P, int b, int i) {
    return P.pool ? kPoolBlock * P.pool[(int64_t)b * P.pool_blocks + i / kPoolBlock] + i % kPoolBlock : i;
}

// Bytes of scan workspace for n problems.
size_t scan_workspace_bytes(int n_problems, int batch, int max_entries, int H_idx);
// Point sb.qc / sb.qs / every problem's scores into ws (sb.n must be set).
void carve_scan_workspace(ScanBatch& sb, uint8_t* ws, int batch, int max_entries);

// ev (nullable): events recorded after query quantisation, after the scan and
// after Top-K (three cudaEvent_t).
cudaError_t launch_index_topk(const ScanBatch& sb, cudaStream_t st, cudaEvent_t* ev = nullptr);
// The same without the Top-K (ev: two events).
cudaError_t launch_quant_scan(const ScanBatch& sb, cudaStream_t st, cudaEvent_t* ev = nullptr);
// Kernel launches one launch_index_topk(sb) call makes.
int index_topk_launches(const ScanBatch& sb);

// Top-K of every problem's score row (row_len positions), P.K (else sb.K) per row.
cudaError_t launch_topk(const ScanBatch& sb, cudaStream_t st);

// pool_n of every pool problem of sb: the valid prefix of its positions.
cudaError_t launch_pool_count(const ScanBatch& sb, cudaStream_t st);

// Block maxima of every problem's score row: bmax[(i * batch + b) * bstride + j]
// = max of entries 8j .. 8j + 7 (below n_entries) of problem i, sequence b.
// bstride is a multiple of 4.
cudaError_t launch_block_max(const ScanBatch& sb, float* bmax, int64_t bstride, cudaStream_t st);
inline int64_t block_row_stride(int max_entries) {
    return ((int64_t)(max_entries + kPoolBlock - 1) / kPoolBlock + 3) / 4 * 4;
}

// ---- attention
struct AttnProblem {
    CacheView cache;          // valid when K > 0
    const uint16_t* q;        // bf16 [batch][H][512]
    const int32_t* idx;       // [batch][K] or null (K == 0)
    const void* win;          // bf16 or E4M3 (win_fp8) [batch][128][512]
    const int32_t* win_count; // [batch]
    int win_fp8;
    float* out;               // fp32 [batch][H][512]
    int K;                    // 0 for window-only layers
};

struct AttnBatch {
    AttnProblem p[kMaxProblems];
    int n;
    int batch;
    int H;
    int Kmax;
    float scale;
    float* part_o;   // workspace partial outputs
    float* part_ml;  // workspace partial (max, sum)
};

size_t attn_workspace_bytes(int n_problems, int batch, int H, int Kmax);
// ev (nullable): events recorded after the split kernel and after the combine.
// Kernel launches one launch_sparse_attn(ab) call makes.
int sparse_attn_launches(const AttnBatch& ab);
cudaError_t launch_sparse_attn(const AttnBatch& ab, cudaStream_t st, cudaEvent_t* ev = nullptr);

// ---- window
struct WinAppend {
    void* tokens[kMaxProblems];      // bf16 or E4M3 (fp8[l]) rings
    int32_t* count[kMaxProblems];
    const uint16_t* tok[kMaxProblems];
    int fp8[kMaxProblems];
    int n;
    int batch;
};
cudaError_t launch_window_append(const WinAppend& wa, cudaStream_t st);

}  // namespace csa2
