/*
 * CSA2 CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously correct restatement of what the CSA2 decode path
 * computes, used to check the CUDA library.  Only the tests, the smoke check
 * and the benchmark's CPU-baseline / reference leg may load it.  It shares no
 * code, header, table or constant with the CUDA path.
 *
 * Sources ("DeepSeek-V4.1-Flash, expliqué pas à pas", chapter "Le cache KV en
 * FP4" and the CSA2 chapter; "Résumé exécutif", section "Le cache principal en
 * FP4"; the OCP Microscaling Formats (MX) v1.0 specification that the pages
 * name for the indexer format):
 *   - main entry: 512 channels E2M1 + one E4M3 scale per 16 channels (288 B);
 *   - indexer key: 128 channels E2M1 + one E8M0 scale per 32 channels (68 B),
 *     obtained by a plain projection of the main entry;
 *   - indexer: score every entry from an indexer query and keep the best k;
 *   - attention: the main query reads the selected entries plus the layer's
 *     own 128-token sliding window.
 * Readings the pages leave open are stated at each function.
 */
#ifndef CSA2_REF_H
#define CSA2_REF_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* formats */
double ref_e2m1_value(unsigned code);
double ref_e4m3_value(unsigned code);
double ref_e8m0_value(unsigned code);
unsigned ref_e2m1_encode(float v);
unsigned ref_e4m3_encode(float v);
void ref_window_fp8(const float* x, int n, uint8_t* codes);
int ref_mx_shared_exp(float amax);
float ref_spec_exp(float x);

/* cache write */
void ref_compress_pair(const float* x0, float g0, const float* x1, float g1, float* e);
void ref_pack_main(const float* e, uint8_t* codes, uint8_t* scales);
void ref_dequant_main(const uint8_t* codes, const uint8_t* scales, float* out);
void ref_mxfp4_quant(const float* v, int n, uint8_t* codes, uint8_t* scales);
void ref_index_key(const uint8_t* codes, const uint8_t* scales, const float* W, uint8_t* kc,
                   uint8_t* ks);
int ref_append_tokens(int ratio, const float* x, const float* g, int T, const float* W,
                      int32_t* pend_valid, float* pend_x, float* pend_g, uint8_t* mc, uint8_t* ms,
                      uint8_t* kc, uint8_t* ks, int n_entries, int cap);

/* indexer */
void ref_index_scores(const uint8_t* kc, const uint8_t* ks, int N, const uint8_t* qc,
                      const uint8_t* qs, const float* w, int H, double* out);
void ref_topk(const double* scores, int N, int K, int32_t* out);

/* attention */
int ref_gather_items(const uint8_t* mc, const uint8_t* ms, int n_entries, const int32_t* idx, int K,
                     const uint16_t* win, int win_len, float* items);
void ref_attention(const float* q, int H, const float* items, int M, double scale, float* out);

int ref_threads(void);

#ifdef __cplusplus
}
#endif
#endif
