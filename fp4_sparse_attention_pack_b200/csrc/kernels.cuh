// Internal launchers of the CSA2 kernels (host side of csrc/*.cu).
#pragma once

#include "common.cuh"

namespace csa2 {

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

// Bytes of scan workspace for n problems.
size_t scan_workspace_bytes(int n_problems, int batch, int max_entries, int H_idx);
// Point sb.qc / sb.qs / every problem's scores into ws (sb.n must be set).
void carve_scan_workspace(ScanBatch& sb, uint8_t* ws, int batch, int max_entries);

// ev (nullable): events recorded after query quantisation, after the scan and
// after Top-K (three cudaEvent_t).
cudaError_t launch_index_topk(const ScanBatch& sb, cudaStream_t st, cudaEvent_t* ev = nullptr);

// ---- attention
struct AttnProblem {
    CacheView cache;          // valid when K > 0
    const uint16_t* q;        // bf16 [batch][H][512]
    const int32_t* idx;       // [batch][K] or null (K == 0)
    const uint16_t* win;      // bf16 [batch][128][512]
    const int32_t* win_count; // [batch]
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
    uint16_t* tokens[kMaxProblems];
    int32_t* count[kMaxProblems];
    const uint16_t* tok[kMaxProblems];
    int n;
    int batch;
};
cudaError_t launch_window_append(const WinAppend& wa, cudaStream_t st);

}  // namespace csa2
