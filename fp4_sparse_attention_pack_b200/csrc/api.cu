// C ABI of the CSA2 library: argument validation, workspace layout and the
// per-step schedule of the Full / Reindex / Reuse mode table ("Résumé
// exécutif", CSA2 table: Full computes cache, keys and indices; Reindex reuses
// cache and keys and recomputes indices; Reuse reuses all three).
//
// Everything is validated before the first launch, so an error return means
// nothing was enqueued.  Nothing is allocated and nothing synchronises, so
// every entry point can be captured in a CUDA graph.
#include <atomic>
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

using namespace csa2;

namespace {
std::atomic<int> g_injected_faults{0};
}  // namespace

bool csa2::inject_fault(const char* entry) {
    const char* v = std::getenv("CSA2_INJECT_FAULT");
    if (!v || !*v) return false;
    const size_t n = std::strlen(entry);
    bool hit = false;
    for (const char* p = v; *p && !hit;) {
        const char* e = std::strchr(p, ',');
        const size_t len = e ? (size_t)(e - p) : std::strlen(p);
        hit = (len == 1 && p[0] == '*') || (len == n && std::strncmp(p, entry, n) == 0);
        p = e ? e + 1 : p + len;
    }
    if (hit) g_injected_faults.fetch_add(1, std::memory_order_relaxed);
    return hit;
}

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }
inline bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

int csa2::check_cache(const csa2_cache* c) {
    if (!c) return CSA2_ERR_INVALID_ARG;
    if (!c->main_codes || !c->main_scales || !c->idx_codes || !c->idx_scales || !c->page_table ||
        !c->n_entries || !c->pend_x || !c->pend_g || !c->pend_valid || !c->status)
        return CSA2_ERR_INVALID_ARG;
    if (c->batch < 1 || c->max_pages < 1 || c->num_pages < 1 || (c->ratio != 1 && c->ratio != 2))
        return CSA2_ERR_INVALID_ARG;
    if ((int64_t)c->max_pages * PAGE > (int64_t)1 << 30) return CSA2_ERR_UNSUPPORTED;
    if (!a16(c->main_codes) || !a16(c->main_scales) || !a16(c->idx_codes) || !a16(c->idx_scales) ||
        !a16(c->page_table) || !a16(c->n_entries) || !a16(c->pend_x) || !a16(c->pend_g) ||
        !a16(c->pend_valid) || !a16(c->status))
        return CSA2_ERR_ALIGN;
    return CSA2_OK;
}

namespace {

int check_window(const csa2_window* w, int batch) {
    if (!w || !w->tokens || !w->count || w->batch != batch) return CSA2_ERR_INVALID_ARG;
    if (w->dtype != CSA2_WIN_BF16 && w->dtype != CSA2_WIN_FP8) return CSA2_ERR_INVALID_ARG;
    if (!a16(w->tokens) || !a16(w->count)) return CSA2_ERR_ALIGN;
    return CSA2_OK;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA; }

size_t topk_ws_one(int batch, int max_entries, int H_idx) {
    return scan_workspace_bytes(1, batch, max_entries, H_idx);
}

}  // namespace

extern "C" {

int csa2_version(void) { return (0 << 16) | 1; }

int csa2_injected_faults(void) { return g_injected_faults.load(std::memory_order_relaxed); }

namespace {

// One thread waits on a barrier that no thread arrives at: the bounded wait
// gives up after limit_ns and reports it, as every kernel's waits do.
__global__ void k_selftest_wait_timeout(uint32_t* status, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    csa2::sm100::mbar_init(&bar, 1);
    csa2::sm100::fence_mbar_init();
    if (!csa2::sm100::mbar_wait_ns(&bar, 0, limit_ns)) atomicOr(status, CSA2_DEVERR_TIMEOUT);
}

}  // namespace

int csa2_selftest_wait_timeout(uint32_t* status, unsigned timeout_us, csa2_stream stream) {
    if (!status || (reinterpret_cast<uintptr_t>(status) & 3u)) return CSA2_ERR_INVALID_ARG;
    const uint64_t us = timeout_us < 1u ? 1u : (timeout_us > 2000000u ? 2000000u : timeout_us);
    k_selftest_wait_timeout<<<1, 32, 0, (cudaStream_t)stream>>>(status, us * 1000ull);
    return cudaGetLastError() == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

const char* csa2_strerror(int status) {
    switch (status) {
        case CSA2_OK: return "ok";
        case CSA2_ERR_INVALID_ARG: return "invalid argument";
        case CSA2_ERR_ALIGN: return "device pointer not 16-byte aligned";
        case CSA2_ERR_UNSUPPORTED: return "size not supported by this build";
        case CSA2_ERR_CUDA: return "CUDA launch or runtime error";
        case CSA2_ERR_TIMEOUT: return "bounded device wait timed out";
        case CSA2_ERR_WORKSPACE: return "workspace missing or too small";
        default: return "unknown status";
    }
}

int csa2_pack_cache(const csa2_cache* cache, const void* x, int x_dtype, const float* gates,
                    const float* w_idx, int T_new, csa2_stream stream) {
    int rc = check_cache(cache);
    if (rc) return rc;
    if (T_new < 0 || (x_dtype != CSA2_DTYPE_BF16 && x_dtype != CSA2_DTYPE_F32))
        return CSA2_ERR_INVALID_ARG;
    if (T_new == 0) return CSA2_OK;
    if (!x || !gates || !w_idx) return CSA2_ERR_INVALID_ARG;
    if (!a16(x) || !a16(w_idx)) return CSA2_ERR_ALIGN;
    if ((int64_t)T_new > (int64_t)cache->max_pages * PAGE * 2) return CSA2_ERR_INVALID_ARG;
    PackBatch pb;
    std::memset(&pb, 0, sizeof(pb));
    pb.n = 1;
    pb.cache[0] = view_of(*cache);
    pb.x[0] = x;
    pb.gates[0] = gates;
    pb.W[0] = w_idx;
    if (inject_fault("csa2_pack_cache")) return CSA2_ERR_CUDA;
    return cuda_status(launch_pack(pb, x_dtype == CSA2_DTYPE_F32, T_new, (cudaStream_t)stream));
}

size_t csa2_index_topk_workspace(int batch, int max_entries, int H_idx, int K) {
    (void)K;
    if (batch < 1 || max_entries < 0 || H_idx < 1) return 0;
    return topk_ws_one(batch, max_entries, H_idx);
}

int csa2_index_topk(const csa2_cache* cache, const uint16_t* q_idx, const float* w, int H_idx, int K,
                    int32_t* idx_out, float* score_out, void* ws, size_t ws_bytes,
                    csa2_stream stream) {
    int rc = check_cache(cache);
    if (rc) return rc;
    if (H_idx < 1 || H_idx > CSA2_MAX_H_IDX || K < 1 || K > CSA2_MAX_K) return CSA2_ERR_INVALID_ARG;
    if (!q_idx || !w || !idx_out) return CSA2_ERR_INVALID_ARG;
    if (!a16(q_idx) || !a16(w) || !a16(idx_out) || (score_out && !a16(score_out)) || (ws && !a16(ws)))
        return CSA2_ERR_ALIGN;
    const int cap = cache->max_pages * PAGE;
    const size_t need = topk_ws_one(cache->batch, cap, H_idx);
    if (!ws || ws_bytes < need) return CSA2_ERR_WORKSPACE;
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
    carve_scan_workspace(sb, static_cast<uint8_t*>(ws), cache->batch, cap);
    if (inject_fault("csa2_index_topk")) return CSA2_ERR_CUDA;
    return cuda_status(launch_index_topk(sb, (cudaStream_t)stream));
}

// ---------------------------------------------------------------- hierarchical indexer

namespace {

// Workspace of the standalone pool calls: one scan problem whose score rows hold
// max(max_entries, 8 * pool_blocks) floats, the block-maximum rows, pool_n.
struct PoolWs {
    size_t scan, bmax, count, total;
    int rows;
    int64_t bstride;
};

PoolWs pool_ws(int batch, int max_entries, int H_idx, int pool_blocks) {
    PoolWs w;
    w.rows = std::max(max_entries, kPoolBlock * pool_blocks);
    w.bstride = block_row_stride(max_entries);
    w.scan = align_up(topk_ws_one(batch, w.rows, H_idx));
    w.bmax = align_up((size_t)batch * w.bstride * sizeof(float));
    w.count = align_up((size_t)batch * sizeof(int32_t));
    w.total = w.scan + w.bmax + w.count;
    return w;
}

int check_scan_args(const csa2_cache* cache, const uint16_t* q_idx, const float* w, int H_idx, int K,
                    const int32_t* idx_out, const float* score_out, int pool_blocks, const int32_t* pool,
                    const void* ws) {
    int rc = check_cache(cache);
    if (rc) return rc;
    if (H_idx < 1 || H_idx > CSA2_MAX_H_IDX || K < 1 || K > CSA2_MAX_K) return CSA2_ERR_INVALID_ARG;
    if (pool_blocks < 1 || pool_blocks > CSA2_MAX_POOL_BLOCKS) return CSA2_ERR_INVALID_ARG;
    if (!q_idx || !w || !idx_out || !pool) return CSA2_ERR_INVALID_ARG;
    if (!a16(q_idx) || !a16(w) || !a16(idx_out) || (score_out && !a16(score_out)) || !a16(pool) ||
        (ws && !a16(ws)))
        return CSA2_ERR_ALIGN;
    return CSA2_OK;
}

}  // namespace

size_t csa2_index_pool_workspace(int batch, int max_entries, int H_idx, int K, int pool_blocks) {
    (void)K;
    if (batch < 1 || max_entries < 0 || H_idx < 1 || pool_blocks < 1 || pool_blocks > CSA2_MAX_POOL_BLOCKS)
        return 0;
    return pool_ws(batch, max_entries, H_idx, pool_blocks).total;
}

int csa2_index_topk_pool(const csa2_cache* cache, const uint16_t* q_idx, const float* w, int H_idx, int K,
                         int32_t* idx_out, float* score_out, int pool_blocks, int32_t* pool_out, void* ws,
                         size_t ws_bytes, csa2_stream stream) {
    int rc = check_scan_args(cache, q_idx, w, H_idx, K, idx_out, score_out, pool_blocks, pool_out, ws);
    if (rc) return rc;
    const int cap = cache->max_pages * PAGE;
    const PoolWs pw = pool_ws(cache->batch, cap, H_idx, pool_blocks);
    if (!ws || ws_bytes < pw.total) return CSA2_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    uint8_t* wsp = static_cast<uint8_t*>(ws);
    ScanBatch sb;
    std::memset(&sb, 0, sizeof(sb));
    sb.n = 1;
    sb.H_idx = H_idx;
    sb.K = K;
    sb.p[0].cache = view_of(*cache);
    sb.p[0].q_idx = q_idx;
    sb.p[0].w = w;
    sb.p[0].idx_out = idx_out;
    sb.p[0].score_out = score_out;
    carve_scan_workspace(sb, wsp, cache->batch, pw.rows);
    if (inject_fault("csa2_index_topk_pool")) return CSA2_ERR_CUDA;
    rc = cuda_status(launch_quant_scan(sb, st));
    if (rc) return rc;
    float* bmax = reinterpret_cast<float*>(wsp + pw.scan);
    rc = cuda_status(launch_block_max(sb, bmax, pw.bstride, st));
    if (rc) return rc;
    // one Top-K launch: the entries (K) and the block maxima (pool_blocks)
    ScanProblem& B = sb.p[1];
    B.cache = sb.p[0].cache;
    B.scores = bmax;
    B.row_stride = pw.bstride;
    B.block_rows = 1;
    B.K = pool_blocks;
    B.idx_out = pool_out;
    sb.n = 2;
    return cuda_status(launch_topk(sb, st));
}

int csa2_index_topk_in_pool(const csa2_cache* cache, const uint16_t* q_idx, const float* w, int H_idx, int K,
                            const int32_t* pool, int pool_blocks, int32_t* idx_out, float* score_out, void* ws,
                            size_t ws_bytes, csa2_stream stream) {
    int rc = check_scan_args(cache, q_idx, w, H_idx, K, idx_out, score_out, pool_blocks, pool, ws);
    if (rc) return rc;
    const int cap = cache->max_pages * PAGE;
    const PoolWs pw = pool_ws(cache->batch, cap, H_idx, pool_blocks);
    if (!ws || ws_bytes < pw.total) return CSA2_ERR_WORKSPACE;
    uint8_t* wsp = static_cast<uint8_t*>(ws);
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
    P.pool = pool;
    P.pool_blocks = pool_blocks;
    P.pool_n = reinterpret_cast<int32_t*>(wsp + pw.scan + pw.bmax);
    carve_scan_workspace(sb, wsp, cache->batch, pw.rows);
    if (inject_fault("csa2_index_topk_in_pool")) return CSA2_ERR_CUDA;
    return cuda_status(launch_index_topk(sb, (cudaStream_t)stream));
}

size_t csa2_sparse_attn_workspace(int batch, int H, int K) {
    if (batch < 1 || H < 1 || K < 0) return 0;
    return attn_workspace_bytes(1, batch, H, K);
}

int csa2_sparse_attn(const csa2_cache* cache, const uint16_t* q, int H, const int32_t* idx, int K,
                     const csa2_window* win, float scale, float* out, void* ws, size_t ws_bytes,
                     csa2_stream stream) {
    if (H < 1 || H > CSA2_MAX_H || K < 0 || K > CSA2_MAX_K || !q || !out || !win)
        return CSA2_ERR_INVALID_ARG;
    int batch = win->batch;
    if (K > 0) {
        int rc = check_cache(cache);
        if (rc) return rc;
        if (!idx) return CSA2_ERR_INVALID_ARG;
        if (!a16(idx)) return CSA2_ERR_ALIGN;
        if (cache->batch != batch) return CSA2_ERR_INVALID_ARG;
    }
    int rc = check_window(win, batch);
    if (rc) return rc;
    if (batch < 1) return CSA2_ERR_INVALID_ARG;
    if (!a16(q) || !a16(out) || (ws && !a16(ws))) return CSA2_ERR_ALIGN;
    const size_t need = attn_workspace_bytes(1, batch, H, K);
    if (need > 0 && (!ws || ws_bytes < need)) return CSA2_ERR_WORKSPACE;
    AttnBatch ab;
    std::memset(&ab, 0, sizeof(ab));
    ab.n = 1;
    ab.batch = batch;
    ab.H = H;
    ab.Kmax = K;
    ab.scale = scale;
    const size_t units = need / ((D + 2) * sizeof(float));
    ab.part_o = static_cast<float*>(ws);
    ab.part_ml = ab.part_o + units * D;  // CUDA-core layout; the tensor-core path re-derives it
    AttnProblem& P = ab.p[0];
    if (K > 0) P.cache = view_of(*cache);
    P.q = q;
    P.idx = idx;
    P.win = win->tokens;
    P.win_fp8 = win->dtype == CSA2_WIN_FP8;
    P.win_count = win->count;
    P.out = out;
    P.K = K;
    if (inject_fault("csa2_sparse_attn")) return CSA2_ERR_CUDA;
    return cuda_status(launch_sparse_attn(ab, (cudaStream_t)stream));
}

int csa2_window_append(const csa2_window* win, const uint16_t* tok, csa2_stream stream) {
    if (!win || !tok) return CSA2_ERR_INVALID_ARG;
    int rc = check_window(win, win->batch);
    if (rc) return rc;
    if (win->batch < 1) return CSA2_ERR_INVALID_ARG;
    if (!a16(tok)) return CSA2_ERR_ALIGN;
    WinAppend wa;
    std::memset(&wa, 0, sizeof(wa));
    wa.n = 1;
    wa.batch = win->batch;
    wa.tokens[0] = win->tokens;
    wa.fp8[0] = win->dtype == CSA2_WIN_FP8;
    wa.count[0] = win->count;
    wa.tok[0] = tok;
    if (inject_fault("csa2_window_append")) return CSA2_ERR_CUDA;
    return cuda_status(launch_window_append(wa, (cudaStream_t)stream));
}

// ---------------------------------------------------------------- layer step

namespace {

int check_model(const csa2_model* m) {
    if (!m || m->n_layers < 1 || m->n_layers > CSA2_MAX_LAYERS || m->n_sources < 1 ||
        m->n_sources > CSA2_MAX_SOURCES || !m->mode || !m->src || !m->idx_src || !m->caches ||
        !m->w_idx || !m->windows)
        return CSA2_ERR_INVALID_ARG;
    if (m->batch < 1 || m->H < 1 || m->H > CSA2_MAX_H || m->H_idx < 1 || m->H_idx > CSA2_MAX_H_IDX ||
        m->K < 1 || m->K > CSA2_MAX_K || m->pool_blocks < 0 || m->pool_blocks > CSA2_MAX_POOL_BLOCKS)
        return CSA2_ERR_INVALID_ARG;
    int full_of[CSA2_MAX_SOURCES];
    for (int s = 0; s < m->n_sources; ++s) full_of[s] = -1;
    for (int l = 0; l < m->n_layers; ++l) {
        const int md = m->mode[l], s = m->src[l];
        if (md < CSA2_MODE_SWA_ONLY || md > CSA2_MODE_REUSE) return CSA2_ERR_INVALID_ARG;
        if (md == CSA2_MODE_SWA_ONLY) continue;
        if (s < 0 || s >= m->n_sources) return CSA2_ERR_INVALID_ARG;
        if (md == CSA2_MODE_FULL) {
            if (full_of[s] >= 0 || m->idx_src[l] != l) return CSA2_ERR_INVALID_ARG;
            full_of[s] = l;
        } else if (md == CSA2_MODE_REINDEX) {
            if (full_of[s] < 0 || m->idx_src[l] != l) return CSA2_ERR_INVALID_ARG;
        } else {
            const int j = m->idx_src[l];
            if (j < 0 || j >= l || m->src[j] != s ||
                (m->mode[j] != CSA2_MODE_FULL && m->mode[j] != CSA2_MODE_REINDEX))
                return CSA2_ERR_INVALID_ARG;
        }
    }
    for (int s = 0; s < m->n_sources; ++s) {
        if (full_of[s] < 0) return CSA2_ERR_INVALID_ARG;
        int rc = check_cache(&m->caches[s]);
        if (rc) return rc;
        if (m->caches[s].batch != m->batch || !m->w_idx[s]) return CSA2_ERR_INVALID_ARG;
        if (!a16(m->w_idx[s])) return CSA2_ERR_ALIGN;
    }
    for (int l = 0; l < m->n_layers; ++l) {
        int rc = check_window(&m->windows[l], m->batch);
        if (rc) return rc;
    }
    return CSA2_OK;
}

int max_entries(const csa2_model* m) {
    int cap = 0;
    for (int s = 0; s < m->n_sources; ++s) cap = std::max(cap, m->caches[s].max_pages * PAGE);
    return cap;
}

int n_scans(const csa2_model* m) {
    int n = 0;
    for (int l = 0; l < m->n_layers; ++l)
        n += (m->mode[l] == CSA2_MODE_FULL || m->mode[l] == CSA2_MODE_REINDEX);
    return n;
}

int n_mode(const csa2_model* m, int mode) {
    int n = 0;
    for (int l = 0; l < m->n_layers; ++l) n += m->mode[l] == mode;
    return n;
}

// Step workspace, in order: scan workspace (one region; with pools one for the
// FULL layers and one for the REINDEX layers), attention partials, and with
// pools the pools [n_sources][batch][pool_blocks], the block-maximum rows of the
// FULL layers and pool_n of the REINDEX layers.
struct StepWs {
    size_t scan1, scan2, attn, pools, bmax, count, total;
    int rows;
    int64_t bstride;
};

StepWs step_ws(const csa2_model* m) {
    StepWs w{};
    const int cap = max_entries(m), B = m->batch, PB = m->pool_blocks;
    w.rows = PB > 0 ? std::max(cap, kPoolBlock * PB) : cap;
    w.bstride = block_row_stride(cap);
    if (PB == 0) {
        w.scan1 = align_up(scan_workspace_bytes(n_scans(m), B, cap, m->H_idx));
    } else {
        w.scan1 = align_up(scan_workspace_bytes(n_mode(m, CSA2_MODE_FULL), B, w.rows, m->H_idx));
        w.scan2 = align_up(scan_workspace_bytes(n_mode(m, CSA2_MODE_REINDEX), B, w.rows, m->H_idx));
        w.pools = align_up((size_t)m->n_sources * B * PB * sizeof(int32_t));
        w.bmax = align_up((size_t)n_mode(m, CSA2_MODE_FULL) * B * w.bstride * sizeof(float));
        w.count = align_up((size_t)n_mode(m, CSA2_MODE_REINDEX) * B * sizeof(int32_t));
    }
    w.attn = align_up(attn_workspace_bytes(m->n_layers, B, m->H, m->K));
    w.total = w.scan1 + w.scan2 + w.attn + w.pools + w.bmax + w.count;
    return w;
}

}  // namespace

size_t csa2_layer_step_workspace(const csa2_model* m) {
    if (check_model(m)) return 0;
    return step_ws(m).total;
}

namespace {

// The attention batch of one step (shapes and caches; pointers filled by the caller).
void model_attn_batch(const csa2_model* m, AttnBatch& ab) {
    std::memset(&ab, 0, sizeof(ab));
    ab.n = m->n_layers;
    ab.batch = m->batch;
    ab.H = m->H;
    ab.Kmax = m->K;
    ab.scale = m->scale;
    for (int l = 0; l < m->n_layers; ++l) {
        AttnProblem& P = ab.p[l];
        if (m->mode[l] == CSA2_MODE_SWA_ONLY) {
            P.K = 0;
        } else {
            P.K = m->K;
            P.cache = view_of(m->caches[m->src[l]]);
        }
    }
}

int layer_step_impl(const csa2_model* m, const csa2_step_in* in, const csa2_step_out* out, void* ws,
                    size_t ws_bytes, csa2_stream stream, cudaEvent_t* ev) {
    int rc = check_model(m);
    if (rc) return rc;
    if (!in || !out || !in->x_new || !in->g_new || !in->q || !in->win_tok || !out->out)
        return CSA2_ERR_INVALID_ARG;
    const int L = m->n_layers, B = m->batch;
    for (int l = 0; l < L; ++l) {
        if (!in->q[l] || !in->win_tok[l] || !out->out[l]) return CSA2_ERR_INVALID_ARG;
        if (!a16(in->q[l]) || !a16(in->win_tok[l]) || !a16(out->out[l])) return CSA2_ERR_ALIGN;
        const int md = m->mode[l];
        if (md == CSA2_MODE_FULL || md == CSA2_MODE_REINDEX) {
            if (!in->q_idx || !in->w || !out->idx || !in->q_idx[l] || !in->w[l] || !out->idx[l])
                return CSA2_ERR_INVALID_ARG;
            if (!a16(in->q_idx[l]) || !a16(in->w[l]) || !a16(out->idx[l])) return CSA2_ERR_ALIGN;
        }
    }
    for (int s = 0; s < m->n_sources; ++s) {
        if ((in->x_new[s] == nullptr) != (in->g_new[s] == nullptr)) return CSA2_ERR_INVALID_ARG;
        if (in->x_new[s] && !a16(in->x_new[s])) return CSA2_ERR_ALIGN;
    }
    const size_t need = csa2_layer_step_workspace(m);
    if (!ws || ws_bytes < need) return CSA2_ERR_WORKSPACE;
    if (!a16(ws)) return CSA2_ERR_ALIGN;
    if (inject_fault(ev ? "csa2_layer_step_profiled" : "csa2_layer_step")) return CSA2_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    if (ev) cudaEventRecord(ev[0], st);

    // (1) every layer's window takes its token
    WinAppend wa;
    std::memset(&wa, 0, sizeof(wa));
    wa.n = L;
    wa.batch = B;
    for (int l = 0; l < L; ++l) {
        wa.tokens[l] = m->windows[l].tokens;
        wa.fp8[l] = m->windows[l].dtype == CSA2_WIN_FP8;
        wa.count[l] = m->windows[l].count;
        wa.tok[l] = in->win_tok[l];
    }
    rc = cuda_status(launch_window_append(wa, st));
    if (rc) return rc;
    if (ev) cudaEventRecord(ev[1], st);

    // (2) the Full layer of each source writes its new token into the cache
    PackBatch pb;
    std::memset(&pb, 0, sizeof(pb));
    for (int s = 0; s < m->n_sources; ++s) {
        if (!in->x_new[s]) continue;
        pb.cache[pb.n] = view_of(m->caches[s]);
        pb.x[pb.n] = in->x_new[s];
        pb.gates[pb.n] = in->g_new[s];
        pb.W[pb.n] = m->w_idx[s];
        ++pb.n;
    }
    if (pb.n > 0) {
        rc = cuda_status(launch_pack(pb, false, 1, st));
        if (rc) return rc;
    }
    if (ev) cudaEventRecord(ev[2], st);

    // (3) every Full / Reindex layer scans its source with its own query; with
    // pools the Full layers go first and build their sources' pools
    uint8_t* wsp = static_cast<uint8_t*>(ws);
    const StepWs sw = step_ws(m);
    const int PB = m->pool_blocks;
    ScanBatch sb;
    std::memset(&sb, 0, sizeof(sb));
    sb.H_idx = m->H_idx;
    sb.K = m->K;
    for (int l = 0; l < L; ++l) {
        const int md = m->mode[l];
        if (md != CSA2_MODE_FULL && (md != CSA2_MODE_REINDEX || PB > 0)) continue;
        ScanProblem& P = sb.p[sb.n++];
        P.cache = view_of(m->caches[m->src[l]]);
        P.q_idx = in->q_idx[l];
        P.w = in->w[l];
        P.idx_out = out->idx[l];
        P.score_out = nullptr;
    }
    carve_scan_workspace(sb, wsp, B, sw.rows);
    if (sb.n > 0 && PB == 0) {
        rc = cuda_status(launch_index_topk(sb, st, ev ? ev + 3 : nullptr));
        if (rc) return rc;
    } else if (PB == 0 && ev) {
        for (int i = 3; i < 6; ++i) cudaEventRecord(ev[i], st);
    }
    if (PB > 0) {
        uint8_t* region = wsp + sw.scan1 + sw.scan2 + sw.attn;
        int32_t* pools = reinterpret_cast<int32_t*>(region);
        float* bmax = reinterpret_cast<float*>(region + sw.pools);
        int32_t* pool_n = reinterpret_cast<int32_t*>(region + sw.pools + sw.bmax);
        // the Full layers' scans, then the pool of each source: the block maxima of
        // its Full layer's scores; one Top-K launch over the Full layers' entries
        // (K) and their block maxima (pool_blocks)
        rc = cuda_status(launch_quant_scan(sb, st, ev ? ev + 3 : nullptr));
        if (rc) return rc;
        rc = cuda_status(launch_block_max(sb, bmax, sw.bstride, st));
        if (rc) return rc;
        const int n_full = sb.n;
        int li = 0;
        for (int l = 0; l < L; ++l) {
            if (m->mode[l] != CSA2_MODE_FULL) continue;
            ScanProblem& P = sb.p[n_full + li];
            P.cache = sb.p[li].cache;
            P.scores = bmax + (int64_t)li * B * sw.bstride;
            P.row_stride = sw.bstride;
            P.block_rows = 1;
            P.K = PB;
            P.idx_out = pools + (int64_t)m->src[l] * B * PB;
            ++li;
        }
        sb.n = 2 * n_full;
        rc = cuda_status(launch_topk(sb, st));
        if (rc) return rc;
        // the Reindex layers over their sources' pools
        ScanBatch sr;
        std::memset(&sr, 0, sizeof(sr));
        sr.H_idx = m->H_idx;
        sr.K = m->K;
        for (int l = 0; l < L; ++l) {
            if (m->mode[l] != CSA2_MODE_REINDEX) continue;
            ScanProblem& P = sr.p[sr.n];
            P.cache = view_of(m->caches[m->src[l]]);
            P.q_idx = in->q_idx[l];
            P.w = in->w[l];
            P.idx_out = out->idx[l];
            P.pool = pools + (int64_t)m->src[l] * B * PB;
            P.pool_blocks = PB;
            P.pool_n = pool_n + (int64_t)sr.n * B;
            ++sr.n;
        }
        if (sr.n > 0) {
            carve_scan_workspace(sr, wsp + sw.scan1, B, sw.rows);
            rc = cuda_status(launch_index_topk(sr, st));
            if (rc) return rc;
        }
        if (ev) cudaEventRecord(ev[5], st);  // the indexer phase ends after the pool scans
    }
    wsp += sw.scan1 + sw.scan2;

    // (4) every layer attends; Reuse layers read the indices of idx_src
    AttnBatch ab;
    model_attn_batch(m, ab);
    const size_t units = attn_workspace_bytes(L, B, m->H, m->K) / ((D + 2) * sizeof(float));  // in wsp
    ab.part_o = reinterpret_cast<float*>(wsp);
    ab.part_ml = ab.part_o + units * D;
    for (int l = 0; l < L; ++l) {
        AttnProblem& P = ab.p[l];
        P.q = in->q[l];
        P.win = m->windows[l].tokens;
        P.win_fp8 = m->windows[l].dtype == CSA2_WIN_FP8;
        P.win_count = m->windows[l].count;
        P.out = out->out[l];
        P.idx = m->mode[l] == CSA2_MODE_SWA_ONLY ? nullptr : out->idx[m->idx_src[l]];
    }
    return cuda_status(launch_sparse_attn(ab, st, ev ? ev + 6 : nullptr));
}

}  // namespace

int csa2_layer_step(const csa2_model* m, const csa2_step_in* in, const csa2_step_out* out, void* ws,
                    size_t ws_bytes, csa2_stream stream) {
    return layer_step_impl(m, in, out, ws, ws_bytes, stream, nullptr);
}

int csa2_layer_step_profiled(const csa2_model* m, const csa2_step_in* in, const csa2_step_out* out,
                             void* ws, size_t ws_bytes, csa2_stream stream, void* const* events) {
    if (!events) return CSA2_ERR_INVALID_ARG;
    cudaEvent_t ev[CSA2_STEP_EVENTS];
    for (int i = 0; i < CSA2_STEP_EVENTS; ++i) {
        if (!events[i]) return CSA2_ERR_INVALID_ARG;
        ev[i] = (cudaEvent_t)events[i];
    }
    return layer_step_impl(m, in, out, ws, ws_bytes, stream, ev);
}

int csa2_layer_step_launches(const csa2_model* m, const csa2_step_in* in) {
    const int rc = check_model(m);
    if (rc) return rc;
    if (!in || !in->x_new) return CSA2_ERR_INVALID_ARG;
    int n = 1;  // window append
    for (int s = 0; s < m->n_sources; ++s)
        if (in->x_new[s]) {
            n += 2;  // cache write: entries, then the pending slots
            break;
        }
    if (n_scans(m) > 0) n += 3;  // query quantisation, scan, Top-K
    if (m->pool_blocks > 0) {
        n += 1;                                        // block maxima (the pool Top-K shares a launch)
        if (n_mode(m, CSA2_MODE_REINDEX) > 0) n += 4;  // pool count, quantisation, scan, Top-K
    }
    AttnBatch ab;
    model_attn_batch(m, ab);
    return n + sparse_attn_launches(ab);
}

}  // extern "C"
