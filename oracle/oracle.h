/*
 * oracle.h -- entry points of the CPU oracle (test infrastructure; see oracle.c).
 * The constants are the oracle's own statement of the CSA2 decode shapes.
 */
#ifndef CSA2_ORACLE_H
#define CSA2_ORACLE_H
#include <stdint.h>

#define CSA2O_D 512  /* main-KV latent width (shared K = V) */
#define CSA2O_HQ 16  /* attention query heads */
#define CSA2O_HI 4   /* indexer heads */
#define CSA2O_DI 64  /* indexer key / query width */
#define CSA2O_S 8    /* positions per pool block */

double oracle_e2m1_decode(uint8_t code);
uint8_t oracle_e2m1_encode(float r);
double oracle_e4m3_decode(uint8_t code);
uint8_t oracle_e4m3_encode(float v);
void oracle_e4m3_encode_array(const float *v, int64_t n, uint8_t *out);
void oracle_e2m1_encode_array(const float *v, int64_t n, uint8_t *out);

void oracle_mxfp4_quantize_f32(const float *x, uint8_t *codes, uint8_t *scales);
void oracle_ced_project(const uint16_t *h, const uint16_t *w, int64_t M, int d, double *c,
                        double *absdot);
void oracle_mxfp4_quantize_entry(const uint16_t *x, uint8_t *codes, uint8_t *scales);
void oracle_mxfp4_dequantize_entry(const uint8_t *codes, const uint8_t *scales, double *out);
void oracle_swa_quantize_token(const uint16_t *x, uint8_t *e, float *scale);
uint16_t oracle_f64_to_bf16(double x);
void oracle_swa_replay(const uint16_t *h, const uint16_t *w, int B, int Wr, int d,
                       const int32_t *N, uint8_t *swa_e4m3, float *swa_scale, int W);
int oracle_append(const uint16_t *x, const uint16_t *ik, int B, int n, const int32_t *pos,
                  int n_cap, uint8_t *codes, uint8_t *scales, uint16_t *ik_cache,
                  uint8_t *swa_e4m3, float *swa_scale, int W);

double oracle_index_score(const uint16_t *iq, const float *w, const uint16_t *k);
double oracle_index_score_tol(const uint16_t *iq, const float *w, const uint16_t *k);
void oracle_index_scores(const uint16_t *iq, const float *w, const uint16_t *ik_rows, int64_t n,
                         double *score_out, double *tol_out);
int oracle_topk(const double *score, const int64_t *index, int64_t n, int k, int64_t *out);
int oracle_index_full_seq(const uint16_t *iq, const float *w, const uint16_t *ik_rows, int64_t N,
                          int K, int P, double *score_out, double *blockmax_out, int64_t *topk,
                          int64_t *pool);
int oracle_index_reindex_seq(const uint16_t *iq, const float *w, const uint16_t *ik_rows,
                             const int64_t *pool, int64_t L, int K, double *score_out,
                             int64_t *topk);
int oracle_attend_seq(const uint16_t *q, float softmax_scale, const uint8_t *codes_rows,
                      const uint8_t *scales_rows, const int64_t *idx, int K,
                      const uint8_t *swa_rows, const float *swa_scale, int swa_len, float *out,
                      float *lse, double *weights_out);
#endif
