// Indexer scan + Top-K for callers that cannot allocate device memory.
//
// csa2_index_topk needs a caller-provided workspace for its scratch (the
// MXFP4-quantised queries and one fp32 score per cached entry).  Some callers
// cannot provide one: a serving engine that reserves all of its device memory
// in a fixed pool before decoding starts and allows no allocation on the decode
// path (cudaMalloc there can stall the device, fail under memory pressure or
// fragment the pool), or a plugin interface whose fixed signature has no
// workspace argument.  csa2_index_topk_noalloc runs the same kernels with their
// scratch in one static device array that is part of this library's image, so
// the call itself allocates nothing (no cudaMalloc, no cudaFree, no allocating
// library routine).
//
// The array holds kNoAllocBytes (8 MiB) on every device that loads the library,
// until the process exits.  Requests that need more scratch are refused with
// CSA2_ERR_UNSUPPORTED.  Host code cannot use the array's name as a device
// address, so the first call on each device looks the address up with
// cudaGetSymbolAddress while that device is current and keeps it.  Nothing in
// the array has to start at zero: every byte a kernel reads was written earlier
// in the same call.  All calls share the array, so calls whose kernels overlap
// on the GPU (other streams, other host threads) race; callers serialise them.
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace {

constexpr size_t kNoAllocBytes = CSA2_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocBytes];

std::mutex g_addr_mutex;
void* g_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
int scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return CSA2_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return CSA2_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_addr_mutex);
    if (!g_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return CSA2_ERR_CUDA;
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return CSA2_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int csa2_index_topk_noalloc(const csa2_cache* cache, const uint16_t* q_idx, const float* w,
                                       int H_idx, int K, int32_t* idx_out, float* score_out,
                                       csa2_stream stream) {
    using namespace csa2;
    // the same checks, in the same order, as csa2_index_topk; then the size limit
    int rc0 = check_cache(cache);
    if (rc0) return rc0;
    if (H_idx < 1 || H_idx > CSA2_MAX_H_IDX || K < 1 || K > CSA2_MAX_K) return CSA2_ERR_INVALID_ARG;
    if (!q_idx || !w || !idx_out) return CSA2_ERR_INVALID_ARG;
    if (!aligned16(q_idx) || !aligned16(w) || !aligned16(idx_out) || (score_out && !aligned16(score_out)))
        return CSA2_ERR_ALIGN;
    const int cap = cache->max_pages * PAGE;
    if (scan_workspace_bytes(1, cache->batch, cap, H_idx) > kNoAllocBytes) return CSA2_ERR_UNSUPPORTED;
    if (inject_fault("csa2_index_topk_noalloc")) return CSA2_ERR_CUDA;
    void* scratch = nullptr;
    const int rc = scratch_address(&scratch);
    if (rc) return rc;

    ScanBatch sb;
    std::memset(&sb, 0, sizeof(sb));
    sb.n = 1;
    sb.H_idx = H_idx;
    sb.K = K;
    ScanProblem& P = sb.p[0];
    P.cache = view_of(*cache);
    P.q_idx = q_idx;
    P.w = w;
    P.idx_out = idx_out;
    P.score_out = score_out;
    carve_scan_workspace(sb, static_cast<uint8_t*>(scratch), cache->batch, cap);
    return launch_index_topk(sb, (cudaStream_t)stream) == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}
