/*
 * csa2.h -- C ABI of the CSA2 sparse-decode library for NVIDIA B200 (sm_100a).
 *
 * CSA2 ("DeepSeek-V4.1-Flash, expliqué pas à pas", CSA2 chapter; "Résumé
 * exécutif", section "CSA2 -- le partage du cache entre couches") gives each
 * layer a global branch over a compressed, shared cache and a local 128-token
 * sliding-window (SWA) branch.  This library implements the decode hot path:
 *
 *   csa2_pack_cache   cache write: disjoint token groups of m = 2 (or m = 1)
 *                     compressed into one entry, stored as E2M1 with one E4M3
 *                     scale per 16 channels (288 B), plus an indexer key
 *                     projected from that entry and stored as OCP MXFP4
 *                     (E2M1 + one E8M0 scale per 32 channels, 68 B);
 *   csa2_index_topk   indexer scan: score every entry from an MXFP4 indexer
 *                     query, keep the K best per sequence;
 *   csa2_sparse_attn  attention of the main query over the K selected entries
 *                     (dequantised) joined with the layer's own window;
 *   csa2_window_append  SWA ring write of the current token;
 *   csa2_layer_step   one decode step of a whole stack of layers under the
 *                     static Full / Reindex / Reuse mode table.
 *
 * Conventions (all entry points):
 *   - Every tensor is caller-owned DEVICE memory unless stated otherwise; the
 *     library allocates nothing and keeps no pointer after a call returns.
 *     Scratch memory is a caller-provided workspace whose size the matching
 *     *_workspace function reports (0 is a valid answer).
 *   - Calls are asynchronous on the caller's CUDA stream (NULL = the legacy
 *     default stream) and never synchronise the device, so they may be
 *     captured in a CUDA graph.  Host-side descriptor structs are read during
 *     the call only.
 *   - Return value: CSA2_OK (0) or a negative csa2_status.  Arguments are
 *     validated before anything is launched: on an error return nothing has
 *     been enqueued.  No call aborts, throws or traps.
 *   - Conditions only the device can see (a full cache, a page id outside the
 *     pool) never fault: the kernel skips the write and ORs a CSA2_DEVERR_*
 *     bit into the cache's sticky status word, which the caller reads back.
 *   - Device pointers must be 16-byte aligned (CSA2_ERR_ALIGN otherwise).
 *   - bf16 tensors are passed as uint16_t bit patterns.
 *   - Fixed dimensions: latent D = 512, indexer dim 128, window 128,
 *     page = 64 entries.
 */
#ifndef CSA2_H
#define CSA2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* csa2_stream; /* same type as cudaStream_t */

enum {
    CSA2_D = 512,                 /* main latent channels */
    CSA2_D_IDX = 128,             /* indexer query / key dim */
    CSA2_WIN = 128,               /* sliding window (n_win) */
    CSA2_PAGE = 64,               /* entries per cache page */
    CSA2_MAIN_CODE_BYTES = 256,   /* 512 E2M1 codes */
    CSA2_MAIN_SCALE_BYTES = 32,   /* 32 E4M3 scales (one per 16 channels) */
    CSA2_IDX_CODE_BYTES = 64,     /* 128 E2M1 codes */
    CSA2_IDX_SCALE_BYTES = 4,     /* 4 E8M0 scales (one per 32 channels) */
    CSA2_MAX_K = 2048,
    CSA2_MAX_H = 128,
    CSA2_MAX_H_IDX = 64,
    CSA2_MAX_LAYERS = 64,
    CSA2_MAX_SOURCES = 8
};

typedef enum {
    CSA2_OK = 0,
    CSA2_ERR_INVALID_ARG = -1, /* null pointer, size out of range, bad mode table */
    CSA2_ERR_ALIGN = -2,       /* a device pointer is not 16-byte aligned */
    CSA2_ERR_UNSUPPORTED = -3, /* a size this build does not handle */
    CSA2_ERR_CUDA = -4,        /* a CUDA launch or runtime call failed */
    CSA2_ERR_TIMEOUT = -5,     /* a bounded device wait gave up (reported via status) */
    CSA2_ERR_WORKSPACE = -6    /* ws is NULL or smaller than the *_workspace size */
} csa2_status;

typedef enum {
    CSA2_MODE_SWA_ONLY = 0, /* window only (layers 0 and 1 of the model) */
    CSA2_MODE_FULL = 1,     /* computes main cache, indexer keys and Top-K */
    CSA2_MODE_REINDEX = 2,  /* reuses cache and keys, recomputes Top-K */
    CSA2_MODE_REUSE = 3     /* reuses cache, keys and Top-K indices */
} csa2_mode;

typedef enum { CSA2_DTYPE_BF16 = 0, CSA2_DTYPE_F32 = 1 } csa2_dtype;

/* Sticky device error bits (csa2_cache.status). */
#define CSA2_DEVERR_CAPACITY 0x1u /* an append would exceed max_pages * 64 entries */
#define CSA2_DEVERR_PAGE 0x2u     /* a page-table entry is outside [0, num_pages) */
#define CSA2_DEVERR_COUNT 0x4u    /* n_entries outside [0, max_pages * 64] */
#define CSA2_DEVERR_TIMEOUT 0x8u  /* a bounded device wait gave up */
#define CSA2_DEVERR_IMAGE 0x10u   /* a sequence image's header does not fit the cache (see import) */

/*
 * One source layer's compressed cache for `batch` sequences, paged.
 * ("Le cache KV en FP4": main entry = 512 E2M1 values + one E4M3 scale per 16
 * channels = 256 + 32 B; indexer key = 128 E2M1 + one E8M0 per 32 = 64 + 4 B.)
 *
 * Logical entry e of sequence b lives in physical page
 * p = page_table[b * max_pages + e / 64], slot e % 64, and its bytes are
 *   main_codes [p][slot][256]  channel 2i in the low nibble of byte i,
 *                              channel 2i+1 in the high nibble;
 *   main_scales[p][slot][32]   E4M3, byte j scales channels 16j..16j+15;
 *   idx_codes  [p][slot][64]   same nibble order over the 128 key channels;
 *   idx_scales [p][slot][4]    E8M0, byte j scales channels 32j..32j+31.
 * Each pool is num_pages * 64 * (bytes per entry) long.
 *
 * Ratio-2 sources keep one pending token per sequence (pend_x fp32[512],
 * pend_g, pend_valid) until its pair arrives.  `status` is a device uint32
 * the kernels OR CSA2_DEVERR_* bits into; the caller clears it.
 */
typedef struct {
    uint8_t* main_codes;
    uint8_t* main_scales;
    uint8_t* idx_codes;
    uint8_t* idx_scales;
    const int32_t* page_table; /* [batch][max_pages] */
    int32_t* n_entries;        /* [batch] entries stored */
    float* pend_x;             /* [batch][512] */
    float* pend_g;             /* [batch] */
    int32_t* pend_valid;       /* [batch] 0 or 1 */
    uint32_t* status;          /* [1] */
    int32_t batch;
    int32_t max_pages;         /* pages per sequence (page-table row length) */
    int32_t num_pages;         /* pages in each pool */
    int32_t ratio;             /* tokens per entry: 2 (encoder) or 1 (decoder) */
} csa2_cache;

/*
 * One layer's SWA window for `batch` sequences (CSA2 chapter of "DeepSeek-V4.1-
 * Flash, expliqué pas à pas": a local SWA branch keeps the KV of the last 128
 * tokens): a ring of 128 tokens of 512 channels.  Token number t (0-based, counted per sequence) sits in slot
 * t % 128; count[b] tokens were appended, the first min(count[b], 128) slots
 * are valid.  Attention is order-free, so the ring needs no rotation.
 *
 * dtype CSA2_WIN_BF16: tokens are bf16 [batch][128][512] (1,024 B a token).
 * dtype CSA2_WIN_FP8 ("Le cache KV en FP4": the SWA KV stays in FP8, being more
 * sensitive to quantisation): tokens are E4M3 codes uint8 [batch][128][512]
 * (512 B a token, half the bf16 ring).  The pages give no scale for it, and
 * the FP8 main entry of V4 they cite is 512 bytes for 512 channels, so none is
 * kept: each channel is the nearest finite E4M3 value of the bf16 input (ties
 * to the even code, saturating at +-448, a negative value rounding to zero
 * keeps its sign).  E4M3 values are exact in fp16 and fp32.
 */
#define CSA2_WIN_BF16 0
#define CSA2_WIN_FP8 1
typedef struct {
    void* tokens;     /* bf16 or E4M3 [batch][128][512], per dtype */
    int32_t* count;   /* [batch] */
    int32_t batch;
    int32_t dtype;    /* CSA2_WIN_BF16 or CSA2_WIN_FP8 */
} csa2_window;

/* Library version, (major << 16) | minor. */
int csa2_version(void);

/*
 * Host-side fault injection, for testing a caller's error paths without a GPU
 * fault.  (The pages have no counterpart.)  When the environment variable
 * CSA2_INJECT_FAULT holds a comma-separated list of entry-point names (or "*"
 * for all of them), each listed entry point that launches work returns
 * CSA2_ERR_CUDA after its argument checks and before anything is enqueued, as
 * if its launch had failed; argument errors still take precedence.  Unset, it
 * does nothing.  csa2_injected_faults() counts the injected failures of the
 * process so far.
 */
int csa2_injected_faults(void);

/*
 * Self-test of the kernels' bounded waits (the pages have no counterpart).
 * Every wait of every kernel of this library on an mbarrier (a copy landing, an
 * MMA completing, another warp's hand-over) gives up after a time bound, ORs
 * CSA2_DEVERR_TIMEOUT into a status word and lets the kernel return instead of
 * hanging.  This entry point launches one small kernel that makes such a wait
 * run out on purpose: it waits on a barrier nothing arrives at, with a bound of
 * timeout_us microseconds (clamped to [1, 2,000,000]), then ORs
 * CSA2_DEVERR_TIMEOUT into *status and returns; no memory but *status is
 * touched and the context stays usable.
 *   status   device pointer to one uint32 (4-byte aligned), caller-owned.
 * Returns CSA2_ERR_INVALID_ARG for a NULL status, CSA2_ERR_CUDA if the launch
 * fails; asynchronous on `stream` like every entry point.
 */
int csa2_selftest_wait_timeout(uint32_t* status, unsigned timeout_us, csa2_stream stream);

/* Static string for a csa2_status value (never NULL). */
const char* csa2_strerror(int status);

/*
 * Cache write ("DeepSeek-V4.1-Flash, expliqué pas à pas", CSA2 chapter: token
 * groups no longer overlap, and the indexer key is a plain projection of the
 * main KV; chapter "Le cache KV en FP4" for the formats).  Appends T_new tokens
 * to every sequence of `cache`:
 *   x       [batch][T_new][512] tokens, bf16 or fp32 per x_dtype (the
 *           post-RoPE latent of the source layer);
 *   gates   fp32 [batch][T_new], one gate logit per token;
 *   w_idx   fp32 [512][128] row-major indexer projection of this source.
 * Ratio 2: tokens pair up in arrival order with the pending token first; each
 * pair (x0, x1) becomes e = w0*x0 + w1*x1, (w0, w1) = softmax(g0, g1), in fp32
 * with the library's fixed exp (Cody-Waite reduction + degree-7 Taylor).  Ratio
 * 1: each token is an entry.  Each entry is packed (per 16 channels:
 * s = E4M3(amax/6) nearest-even, codes = E2M1(e/s) nearest-even saturating),
 * its indexer key is k_o = sum_c w_idx[c][o] * deq_c accumulated in fp32 fma
 * order c = 0..511, and k is packed to MXFP4 (per 32: X = floor(log2 amax)-2,
 * codes = E2M1(k * 2^-X)).  Updates n_entries and the pending slot.
 * Errors: INVALID_ARG (null, T_new < 0 or above twice the capacity
 * max_pages * 64, bad dtype/ratio), ALIGN, CUDA.  An append that does not fit
 * a sequence's remaining capacity sets CSA2_DEVERR_CAPACITY and leaves that
 * sequence unchanged.
 */
int csa2_pack_cache(const csa2_cache* cache, const void* x, int x_dtype, const float* gates,
                    const float* w_idx, int T_new, csa2_stream stream);

/* Workspace bytes csa2_index_topk needs for these sizes. */
size_t csa2_index_topk_workspace(int batch, int max_entries, int H_idx, int K);

/*
 * Indexer scan + Top-K (CSA2 chapter of "DeepSeek-V4.1-Flash, expliqué pas à
 * pas": a light indexer scores every main-KV entry from an indexer query and
 * an indexer key and keeps the best 512; indexer queries and keys in OCP
 * MXFP4).  For every sequence b:
 *   score[e] = sum_h w[b][h] * max(0, qhat[b][h] . khat[e]),  e < n_entries[b],
 * qhat = MXFP4 of q_idx (same rule as the keys), khat the stored keys.
 * The K highest scores are kept (equal scores: lower index first); idx_out
 * [batch][K] receives them in increasing index order followed by -1 padding
 * when n_entries < K.  score_out (nullable) [batch][K] receives the matching
 * fp32 scores (0 for padding).
 *   q_idx  bf16 [batch][H_idx][128];  w fp32 [batch][H_idx].
 * H_idx in 1..64, K in 1..2048.  ws must hold
 * csa2_index_topk_workspace(batch, max_pages*64, H_idx, K) bytes.
 */
int csa2_index_topk(const csa2_cache* cache, const uint16_t* q_idx, const float* w, int H_idx,
                    int K, int32_t* idx_out, float* score_out, void* ws, size_t ws_bytes,
                    csa2_stream stream);

/*
 * Hierarchical sparse indexer ("DeepSeek-V4.1-Flash, expliqué pas à pas",
 * CSA2 chapter, hierarchical indexer paragraph: the shallow indexer's result
 * restricts what the deeper indexers may consider, and only the first Full
 * layer keeps scanning the whole context; the video-summary page sizes the
 * candidate pool at 2,048 blocks of 8 positions for a million tokens).  The
 * page's step list did not survive; this library's reading:
 *   - a block is 8 consecutive entries of a sequence (block j = entries
 *     8j .. 8j + 7, the last block of a sequence possibly shorter);
 *   - its score is the largest score of its entries under the Full layer's
 *     indexer query (the csa2_index_topk score);
 *   - the pool is the pool_blocks highest-scoring blocks (equal scores: lower
 *     block first), written as block ids in increasing order, -1 padded when
 *     the sequence has fewer blocks;
 *   - a deeper layer scores only the entries of the pool's blocks (below
 *     n_entries) and keeps the K best of them (equal scores: lower entry
 *     first), written in increasing entry order, -1 padded.
 * pool_blocks in 1..CSA2_MAX_POOL_BLOCKS.
 */
#define CSA2_MAX_POOL_BLOCKS 8192

/* Workspace bytes of csa2_index_topk_pool and csa2_index_topk_in_pool. */
size_t csa2_index_pool_workspace(int batch, int max_entries, int H_idx, int K, int pool_blocks);

/*
 * The Full layer's scan: exactly csa2_index_topk (idx_out, score_out), and in
 * addition the pool of every sequence, pool_out int32 [batch][pool_blocks].
 * ws must hold csa2_index_pool_workspace(batch, max_pages*64, H_idx, K,
 * pool_blocks) bytes.  Errors as csa2_index_topk, plus INVALID_ARG for
 * pool_blocks out of range or a NULL pool_out.
 */
int csa2_index_topk_pool(const csa2_cache* cache, const uint16_t* q_idx, const float* w, int H_idx,
                         int K, int32_t* idx_out, float* score_out, int pool_blocks,
                         int32_t* pool_out, void* ws, size_t ws_bytes, csa2_stream stream);

/*
 * A deeper layer's scan restricted to a pool: scores as csa2_index_topk but
 * only for the entries of the blocks pool[b][0..pool_blocks), then the Top-K
 * among them into idx_out [batch][K] (and score_out, nullable) as described
 * above.  `pool` must be as csa2_index_topk_pool writes it (increasing valid
 * block ids, then -1); block ids that are negative or at or beyond the
 * sequence's blocks end the pool early.  A pool in another order gives a
 * selection among its blocks' entries whose order and tie rule are not
 * specified, and a block listed twice can give an index twice.  Same
 * workspace and errors as csa2_index_topk_pool (INVALID_ARG for a NULL pool).
 */
int csa2_index_topk_in_pool(const csa2_cache* cache, const uint16_t* q_idx, const float* w,
                            int H_idx, int K, const int32_t* pool, int pool_blocks,
                            int32_t* idx_out, float* score_out, void* ws, size_t ws_bytes,
                            csa2_stream stream);

/* Workspace bytes csa2_sparse_attn needs for these sizes. */
size_t csa2_sparse_attn_workspace(int batch, int H, int K);

/*
 * Sparse + window attention ("DeepSeek-V4.1-Flash, expliqué pas à pas", CSA2
 * chapter, main attention: the main query reads the selected entries together
 * with the layer's local SWA KV, and the FP4 entries are decompressed before
 * attention).  For every sequence b and head h:
 *   items = dequantised entries idx[b][0..K) (index -1 skipped; indices at or
 *           beyond n_entries[b] skipped) followed by the valid window tokens;
 *   out[b][h] = sum_j softmax_j(scale * q[b][h] . item_j) * item_j
 * (the latent serves as key and value).  No items gives zeros.
 *   q     bf16 [batch][H][512];  idx int32 [batch][K] (may be NULL when K = 0);
 *   out   fp32 [batch][H][512].
 * H in 1..128, K in 0..2048.  `cache` may be NULL when K = 0.
 * Kernels: 1..64 heads run on the tensor cores (fp16 operands: the query is
 * scaled by a power of two per (sequence, layer) before its fp16 rounding, so
 * any bf16 query is exact within 2^28 of its largest magnitude; bf16 window
 * values beyond +-65504 saturate there); other head counts, or every head count
 * when the environment variable CSA2_ATTN_CUDA_CORE is "1" at the call (and at
 * the workspace query), run on the CUDA cores with bf16 kept exact.
 */
int csa2_sparse_attn(const csa2_cache* cache, const uint16_t* q, int H, const int32_t* idx, int K,
                     const csa2_window* win, float scale, float* out, void* ws, size_t ws_bytes,
                     csa2_stream stream);

/* SWA ring write: tok bf16 [batch][512] goes to slot count % 128 (as E4M3 codes
 * for an FP8 window); count += 1.  INVALID_ARG for an unknown dtype. */
int csa2_window_append(const csa2_window* win, const uint16_t* tok, csa2_stream stream);

/*
 * A stack of layers and its static mode table (CSA2 chapter of "DeepSeek-V4.1-
 * Flash, expliqué pas à pas": each layer is given one of the three modes once,
 * statically; "Résumé exécutif", mode table):
 *   mode[l]     csa2_mode of layer l;
 *   src[l]      the source cache layer l reads (ignored for SWA_ONLY);
 *   idx_src[l]  for REUSE: the earlier FULL/REINDEX layer of the same source
 *               whose indices it reuses; for FULL/REINDEX: l itself.
 * Every source is written by exactly one FULL layer.  Host arrays; the caches,
 * w_idx pointers and windows they list are device memory as above.
 */
typedef struct {
    int32_t n_layers;
    int32_t n_sources;
    const int32_t* mode;            /* host [n_layers] */
    const int32_t* src;             /* host [n_layers] */
    const int32_t* idx_src;         /* host [n_layers] */
    const csa2_cache* caches;       /* host [n_sources] */
    const float* const* w_idx;      /* host [n_sources] -> device fp32 [512][128] */
    const csa2_window* windows;     /* host [n_layers] */
    int32_t batch;
    int32_t H;                      /* main query heads */
    int32_t H_idx;                  /* indexer heads */
    int32_t K;                      /* Top-K */
    float scale;                    /* softmax scale (1/sqrt(512) in the tests) */
    int32_t pool_blocks;            /* 0: every REINDEX layer scans its whole source;
                                       1..CSA2_MAX_POOL_BLOCKS: hierarchical indexer, the
                                       FULL layer of each source builds a pool of this many
                                       blocks (csa2_index_topk_pool) and the REINDEX layers
                                       of that source scan only it (csa2_index_topk_in_pool) */
} csa2_model;

/* Per-step inputs: host arrays of device pointers. */
typedef struct {
    const uint16_t* const* x_new; /* [n_sources] -> bf16 [batch][512]: the new token */
    const float* const* g_new;    /* [n_sources] -> fp32 [batch]: its gate logit */
    const uint16_t* const* q;     /* [n_layers] -> bf16 [batch][H][512] */
    const uint16_t* const* q_idx; /* [n_layers] -> bf16 [batch][H_idx][128] (FULL/REINDEX) */
    const float* const* w;        /* [n_layers] -> fp32 [batch][H_idx] (FULL/REINDEX) */
    const uint16_t* const* win_tok; /* [n_layers] -> bf16 [batch][512]: this token's SWA KV */
} csa2_step_in;

/* Per-step outputs: host arrays of device pointers. */
typedef struct {
    float* const* out;   /* [n_layers] -> fp32 [batch][H][512] */
    int32_t* const* idx; /* [n_layers] -> int32 [batch][K] for FULL/REINDEX layers (others
                            unused and may be NULL) */
} csa2_step_out;

/* Workspace bytes csa2_layer_step needs for this model. */
size_t csa2_layer_step_workspace(const csa2_model* model);

/*
 * One decode step of every layer.  Order: (1) each layer's window takes its
 * token; (2) each source takes its new token (an entry is written when a
 * ratio-2 pair completes); (3) every FULL/REINDEX layer scans its source with
 * its own indexer query and keeps the Top-K (with pool_blocks > 0: the FULL
 * layers first, each building its source's pool, then the REINDEX layers over
 * the pools); (4) every layer attends: REUSE
 * layers over the indices of idx_src, SWA_ONLY layers over the window only.
 * Errors as the per-op calls; INVALID_ARG for an inconsistent mode table.
 */
int csa2_layer_step(const csa2_model* model, const csa2_step_in* in, const csa2_step_out* out,
                    void* ws, size_t ws_bytes, csa2_stream stream);

/*
 * csa2_index_topk for callers that cannot allocate device memory.  (The pages
 * have no counterpart; this is an interface of this library only.)
 *
 * Some callers cannot give the library a workspace: an engine whose device
 * memory is a fixed pool reserved before decoding, with no allocation allowed
 * on the decode path, or a plugin interface without a workspace argument.
 * This call computes exactly what csa2_index_topk computes, with the same
 * kernels and arguments, but keeps its scratch (quantised queries and one fp32
 * score per entry) in a static array inside the library's device image:
 * CSA2_NOALLOC_SCRATCH_BYTES (8 MiB) on every device that loads the library,
 * held until the process exits.  The call itself allocates nothing.
 *   - Size limit: the scratch needed, about batch * max_pages * 64 * 4 +
 *     batch * H_idx * 68 bytes, must fit in 8 MiB; larger requests return
 *     CSA2_ERR_UNSUPPORTED before anything is launched.
 *   - Set-up: the first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and keeps it for the
 *     life of the process.  Make that first call before any stream capture.
 *     The kept address belongs to the device's current context: after a
 *     cudaDeviceReset of that device it is stale, so do not call this entry
 *     point on a device that has been reset.
 *   - Sharing: every call uses the same array and leaves its contents behind
 *     (nothing in it needs to start at zero).  Calls whose kernels overlap on
 *     the GPU -- other streams or other host threads -- race; serialise them.
 * Errors: as csa2_index_topk, plus CSA2_ERR_UNSUPPORTED for the size limit.
 */
#define CSA2_NOALLOC_SCRATCH_BYTES (8u << 20)
int csa2_index_topk_noalloc(const csa2_cache* cache, const uint16_t* q_idx, const float* w,
                            int H_idx, int K, int32_t* idx_out, float* score_out,
                            csa2_stream stream);

/*
 * Measurement variant of csa2_layer_step: identical work, and in addition
 * records CUDA events on `stream` at the phase boundaries.  `events` is a host
 * array of CSA2_STEP_EVENTS cudaEvent_t handles (as void*) created by the caller
 * with timing enabled:
 *   [0] start            [1] after window append  [2] after cache write
 *   [3] after query quantisation                  [4] after the indexer scan
 *   [5] after Top-K      [6] after attention      [7] after the split combine
 * With pool_blocks > 0, [3] and [4] follow the FULL layers' query
 * quantisation and scan, and [5] follows everything else of the indexer: the
 * FULL layers' Top-K, the pool build and the REINDEX layers' pool scans.
 * A phase with nothing to do gives two events with no work between them.
 */
#define CSA2_STEP_EVENTS 8
int csa2_layer_step_profiled(const csa2_model* model, const csa2_step_in* in,
                             const csa2_step_out* out, void* ws, size_t ws_bytes,
                             csa2_stream stream, void* const* events);

/*
 * Prefix-cache export / import of one sequence ("DeepSeek-V4.1-Flash,
 * expliqué pas à pas": the introduction names the prefix cache, a session's
 * cache reloaded instead of recomputed; the FP4-cache section keeps the global
 * cache whole in the persistent store).  The pages give the feature, not a
 * format; this image format is this library's own.
 *
 * A sequence image with room for `capacity` entries is, in order:
 *   header   int32 n_entries, int32 pend_valid, float pend_g, int32 ratio (16 B)
 *   pend_x   fp32[512]
 *   main_codes [capacity][256], main_scales [capacity][32],
 *   idx_codes  [capacity][64],  idx_scales  [capacity][4]
 * with entries in logical order (entry e of the sequence at row e), the byte
 * layout of each row as in csa2_cache.  csa2_seq_image_bytes(capacity) is its
 * size: 2,064 + 356 * capacity bytes.
 *
 * csa2_cache_export copies sequence `seq` of `cache` into `image`: the header,
 * the pending slot and the first n = n_entries[seq] rows; when n > capacity only
 * `capacity` rows are copied, the header records that many, and
 * CSA2_DEVERR_CAPACITY is set.  csa2_cache_import writes an image back into
 * sequence `seq` of a cache (any page table, same ratio): its n rows go to the
 * pages the page table gives, and n_entries and the pending slot are set.  An
 * image whose ratio differs from the cache's, or whose n is negative or larger
 * than min(capacity, max_pages * 64), is not imported (nothing written) and
 * CSA2_DEVERR_IMAGE is set.  Rows whose page id is outside the pool are skipped
 * with CSA2_DEVERR_PAGE.
 *
 * `image` is caller-owned memory the device can address (device memory, or
 * pinned host memory mapped into the device address space), 16-byte aligned.
 * Both calls are asynchronous on `stream`, read n_entries and the header on the
 * device (no host synchronisation) and may be captured in a CUDA graph.
 * Returns CSA2_ERR_INVALID_ARG for a NULL pointer, seq outside [0, batch) or
 * capacity < 0; CSA2_ERR_ALIGN for an unaligned image.
 */
size_t csa2_seq_image_bytes(int capacity);
int csa2_cache_export(const csa2_cache* cache, int seq, void* image, int capacity, csa2_stream stream);
int csa2_cache_import(const csa2_cache* cache, int seq, const void* image, int capacity, csa2_stream stream);

/*
 * Number of kernel launches one csa2_layer_step(model, in, ...) call enqueues
 * on the current device (the measurement variant adds none): the window
 * append, two for the cache write when any source takes a token, three for the
 * indexer (query quantisation, scan, Top-K) when any layer scans -- with
 * pool_blocks > 0 plus one for the block maxima (their Top-K shares the FULL
 * layers' Top-K launch) and,
 * when REINDEX layers exist, four for their pool scans (pool count, query
 * quantisation, scan, Top-K) -- and one or two
 * for attention (a second one combines split tiles when there are fewer
 * (layer, sequence) pairs than SMs).  Returns a negative csa2_status when the
 * model table is invalid or `in` is NULL.  Enqueues nothing.
 */
int csa2_layer_step_launches(const csa2_model* model, const csa2_step_in* in);

#ifdef __cplusplus
}
#endif
#endif /* CSA2_H */
