/*
 * oracle.c -- plain, slow CPU restatement of the CSA2 decode path.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's CPU-baseline arm
 * load this file's library. It shares no code, header, table or constant generator with the
 * CUDA library, and it never reads a value that the CUDA library produced as an expected value.
 *
 * Sources (the pages give no code, no formulas and no worked examples; every definition below is
 * the plainest reading of what they say):
 *   [T1] "DeepSeek V4.1 Flash 拆解：KV Cache 压掉 3/4 的工程胜利，与它没解决的三个问题"
 *        (austincafe.tech/?p=406), section 一. It names the three CSA2 layer modes (Full computes
 *        its own main KV and indexer and emits a new Top-K; Reindex reuses the main KV and the
 *        indexer keys and rescoring with its own indexer query picks its own Top-K; Reuse also
 *        reuses the Top-K and runs sparse attention directly), the hierarchical sparse indexer
 *        (the first decoder layer picks a Top-512, then a candidate pool of 2048 blocks x 8
 *        positions = 16,384 positions that later layers score), the MXFP4 main KV (E2M1 values
 *        with one E4M3 scale per 16 channels) and the FP8 sliding-window (SWA) KV.
 *   [A]  "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression", abstract: CSA2
 *        cross-layer KV reuse plus an FP4 KV cache.
 *   [OCP-MX]  OCP Microscaling Formats (MX) v1.0: the E2M1 element format.
 *   [OCP-FP8] OCP 8-bit Floating Point (OFP8): the E4M3 format (bias 7, no infinities, one NaN
 *             pattern per sign, largest finite 448).
 *
 * Readings taken where the pages are silent (each is restated next to the code that uses it):
 *   - indexer score I_t = sum_h w_h * ReLU(q_h . k_t), one 64-wide key per entry shared by the
 *     4 indexer heads;
 *   - block score = max of I over the block's 8 positions (positions past N excluded);
 *   - Top-K ranks by (score descending, index ascending); -0 == +0;
 *   - MXFP4 scale = E4M3 round-to-nearest-even (saturating) of the fp32 quotient amax/6; element
 *     code = E2M1 round-to-nearest-even (saturating at 6) of the fp32 quotient x/scale; the sign
 *     bit is the sign of x; a zero scale gives all-zero codes;
 *   - SWA: per-token fp32 scale amax/448, element = E4M3 RNE-saturating of the fp32 quotient;
 *   - attention: K = V = dequantised entry, softmax over the selected entries and the valid SWA
 *     rows together, out = sum p_t v_t, lse = log sum exp(z_t); empty set -> out 0, lse -inf.
 *
 * Precision: dot products, the softmax and the outputs are accumulated in double. The codecs are
 * exact: they compare the real value of their fp32 input with midpoints of the format's grid.
 * fp32 arithmetic appears only where the reading above defines a quantity as an fp32 quotient.
 * Single-threaded on purpose.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "oracle.h"

/* ------------------------------------------------------------------------------------------ */
/* bf16 / fp32 bit helpers                                                                     */
/* ------------------------------------------------------------------------------------------ */

/* bf16 is the top half of an IEEE binary32. */
static float bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

static int f32_signbit(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return (int)(u >> 31);
}

/* ------------------------------------------------------------------------------------------ */
/* E2M1 [OCP-MX]: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit, no inf/NaN.           */
/* Codes 0..7 (sign 0) have the magnitudes below; code | 8 is the negative of code.            */
/* ------------------------------------------------------------------------------------------ */
static const double kE2M1Mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double oracle_e2m1_decode(uint8_t code) {
  double m = kE2M1Mag[code & 7];
  return (code & 8) ? -m : m;
}

/* Index of the nearest grid point to a >= 0 on an ascending grid; an exact midpoint goes to
 * the even index (round-to-nearest-even, since an even index is an even trailing mantissa bit
 * in both formats used here); a at or above the top point saturates to the top index. */
static int round_to_grid_rne_sat(double a, const double *grid, int n) {
  if (a >= grid[n - 1]) return n - 1;
  for (int i = 0; i + 1 < n; ++i) {
    double mid = 0.5 * (grid[i] + grid[i + 1]); /* exact: both are short dyadic numbers */
    if (a < mid) return i;
    if (a == mid) return (i % 2 == 0) ? i : i + 1;
  }
  return n - 1; /* not reached */
}

uint8_t oracle_e2m1_encode(float r) {
  double a = fabs((double)r);
  uint8_t mag = (uint8_t)round_to_grid_rne_sat(a, kE2M1Mag, 8);
  return (uint8_t)(mag | (f32_signbit(r) ? 8 : 0));
}

/* ------------------------------------------------------------------------------------------ */
/* E4M3 [OCP-FP8] (the "fn" variant): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits.      */
/* exponent 0 -> subnormal m/8 * 2^-6; exponent 15 with mantissa 7 -> NaN; no infinities.     */
/* ------------------------------------------------------------------------------------------ */
double oracle_e4m3_decode(uint8_t code) {
  int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) v = ldexp((double)m / 8.0, -6);
  else v = ldexp(1.0 + (double)m / 8.0, e - 7);
  return s ? -v : v;
}

/* Magnitudes of codes 0..126 (all non-negative finite values) in ascending order; code order is
 * magnitude order for a fixed sign. */
static double g_e4m3_grid[127];

/* Filled once when the library is loaded, before any caller's thread can use it, so that
 * concurrent callers never see a partly built table. */
__attribute__((constructor)) static void e4m3_grid_init(void) {
  for (int c = 0; c < 127; ++c) g_e4m3_grid[c] = oracle_e4m3_decode((uint8_t)c);
}

static const double *e4m3_grid(void) { return g_e4m3_grid; }

/* Round-to-nearest-even with saturation to +-448 ("satfinite"); the sign bit is kept, so a
 * negative input that rounds to zero gives 0x80. NaN in -> 0x7F. */
uint8_t oracle_e4m3_encode(float v) {
  if (isnan(v)) return 0x7F;
  double a = fabs((double)v);
  uint8_t mag = (uint8_t)round_to_grid_rne_sat(a, e4m3_grid(), 127);
  return (uint8_t)(mag | (f32_signbit(v) ? 0x80 : 0));
}

void oracle_e4m3_encode_array(const float *v, int64_t n, uint8_t *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(v[i]);
}

void oracle_e2m1_encode_array(const float *v, int64_t n, uint8_t *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_e2m1_encode(v[i]);
}

/* ------------------------------------------------------------------------------------------ */
/* MXFP4 main-KV entry [T1 FP4 KV Cache paragraph]: 512 channels, 32 groups of 16 channels.    */
/* ------------------------------------------------------------------------------------------ */
void oracle_mxfp4_quantize_entry(const uint16_t *x, uint8_t *codes, uint8_t *scales) {
  for (int g = 0; g < CSA2O_D / 16; ++g) {
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) {
      float a = fabsf(bf16_to_f32(x[16 * g + i]));
      if (a > amax) amax = a;
    }
    /* scale: E4M3 RNE-saturating of the fp32 quotient amax / 6 (6 = largest E2M1 magnitude) */
    float q = amax / 6.0f;
    uint8_t sc = oracle_e4m3_encode(q);
    scales[g] = sc;
    double s = oracle_e4m3_decode(sc);
    uint8_t c[16];
    for (int i = 0; i < 16; ++i) {
      if (s == 0.0) {
        c[i] = 0; /* zero scale: every code of the group is 0x0 */
      } else {
        float r = bf16_to_f32(x[16 * g + i]) / (float)s; /* fp32 quotient */
        c[i] = oracle_e2m1_encode(r);
      }
    }
    /* two codes per byte: channel 2j in the low nibble, channel 2j+1 in the high nibble */
    for (int j = 0; j < 8; ++j) codes[8 * g + j] = (uint8_t)(c[2 * j] | (c[2 * j + 1] << 4));
  }
}

/* The same quantisation of a 512-channel row given as fp32 values (the CED projection output):
 * scale = E4M3 RNE-saturating of the fp32 quotient amax / 6, code = E2M1 RNE-saturating of the
 * fp32 quotient |x| / scale with the sign bit of x, all codes 0 for a zero scale. */
void oracle_mxfp4_quantize_f32(const float *x, uint8_t *codes, uint8_t *scales) {
  for (int g = 0; g < CSA2O_D / 16; ++g) {
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) {
      float a = fabsf(x[16 * g + i]);
      if (a > amax) amax = a;
    }
    float q = amax / 6.0f;
    uint8_t sc = oracle_e4m3_encode(q);
    scales[g] = sc;
    float s = (float)oracle_e4m3_decode(sc); /* every E4M3 value is exact in fp32 */
    uint8_t c[16];
    for (int i = 0; i < 16; ++i) {
      if (s == 0.0f) {
        c[i] = 0;
      } else {
        float r = fabsf(x[16 * g + i]) / s; /* fp32 quotient */
        c[i] = (uint8_t)(oracle_e2m1_encode(r) | (f32_signbit(x[16 * g + i]) << 3));
      }
    }
    for (int j = 0; j < 8; ++j) codes[8 * g + j] = (uint8_t)(c[2 * j] | (c[2 * j + 1] << 4));
  }
}

/* Dequantised channel i of an MXFP4 entry: E2M1 value times the group's E4M3 scale. */
static double mxfp4_value(const uint8_t *codes, const uint8_t *scales, int i) {
  uint8_t byte = codes[i / 2];
  uint8_t c = (i % 2 == 0) ? (byte & 15) : (byte >> 4);
  return oracle_e2m1_decode(c) * oracle_e4m3_decode(scales[i / 16]);
}

void oracle_mxfp4_dequantize_entry(const uint8_t *codes, const uint8_t *scales, double *out) {
  for (int i = 0; i < CSA2O_D; ++i) out[i] = mxfp4_value(codes, scales, i);
}

/* ------------------------------------------------------------------------------------------ */
/* FP8 SWA token [T1: the SWA KV is quantisation-sensitive and stays FP8].                     */
/* Reading: one fp32 scale per token, amax/448, elements E4M3 RNE-saturating of x/scale.       */
/* ------------------------------------------------------------------------------------------ */
void oracle_swa_quantize_token(const uint16_t *x, uint8_t *e, float *scale) {
  float amax = 0.0f;
  for (int i = 0; i < CSA2O_D; ++i) {
    float a = fabsf(bf16_to_f32(x[i]));
    if (a > amax) amax = a;
  }
  float s = amax / 448.0f; /* fp32 quotient */
  *scale = s;
  for (int i = 0; i < CSA2O_D; ++i) {
    if (s == 0.0f) e[i] = 0;
    else e[i] = oracle_e4m3_encode(bf16_to_f32(x[i]) / s);
  }
}

/* ------------------------------------------------------------------------------------------ */
/* Append: write n new entries per sequence at rows pos[b] .. pos[b]+n-1.                      */
/* ------------------------------------------------------------------------------------------ */
int oracle_append(const uint16_t *x, const uint16_t *ik, int B, int n, const int32_t *pos,
                  int n_cap, uint8_t *codes, uint8_t *scales, uint16_t *ik_cache,
                  uint8_t *swa_e4m3, float *swa_scale, int W) {
  for (int b = 0; b < B; ++b) {
    for (int i = 0; i < n; ++i) {
      int64_t p = (int64_t)pos[b] + i;
      if (p < 0 || p >= n_cap) return -1;
      const uint16_t *xr = x + ((int64_t)b * n + i) * CSA2O_D;
      int64_t row = (int64_t)b * n_cap + p;
      oracle_mxfp4_quantize_entry(xr, codes + row * (CSA2O_D / 2), scales + row * (CSA2O_D / 16));
      if (ik && ik_cache)
        memcpy(ik_cache + row * CSA2O_DI, ik + ((int64_t)b * n + i) * CSA2O_DI,
               CSA2O_DI * sizeof(uint16_t));
      if (swa_e4m3 && W > 0) {
        /* the ring holds the most recent W tokens: token at position p lives in slot p mod W;
         * writing in order lets later tokens overwrite earlier ones */
        int64_t slot = (int64_t)b * W + (p % W);
        oracle_swa_quantize_token(xr, swa_e4m3 + slot * CSA2O_D, swa_scale + slot);
      }
    }
  }
  return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* Indexer score: I_t = sum_h w_h * ReLU(q_h . k_t), double accumulation.                      */
/* ------------------------------------------------------------------------------------------ */
double oracle_index_score(const uint16_t *iq, const float *w, const uint16_t *k) {
  double total = 0.0;
  for (int h = 0; h < CSA2O_HI; ++h) {
    double dot = 0.0;
    for (int i = 0; i < CSA2O_DI; ++i)
      dot += (double)bf16_to_f32(iq[h * CSA2O_DI + i]) * (double)bf16_to_f32(k[i]);
    double relu = dot > 0.0 ? dot : 0.0;
    total += (double)w[h] * relu;
  }
  return total;
}

/* Bound on the fp32 rounding of one score: 2^-16 * sum_h |w_h| * sum_i |q_hi * k_i|. */
double oracle_index_score_tol(const uint16_t *iq, const float *w, const uint16_t *k) {
  double total = 0.0;
  for (int h = 0; h < CSA2O_HI; ++h) {
    double s = 0.0;
    for (int i = 0; i < CSA2O_DI; ++i)
      s += fabs((double)bf16_to_f32(iq[h * CSA2O_DI + i]) * (double)bf16_to_f32(k[i]));
    total += fabs((double)w[h]) * s;
  }
  return ldexp(total, -16);
}

/* Scores (and optionally their tolerance bounds) of n consecutive key rows. */
void oracle_index_scores(const uint16_t *iq, const float *w, const uint16_t *ik_rows, int64_t n,
                         double *score_out, double *tol_out) {
  for (int64_t t = 0; t < n; ++t) {
    if (score_out) score_out[t] = oracle_index_score(iq, w, ik_rows + t * CSA2O_DI);
    if (tol_out) tol_out[t] = oracle_index_score_tol(iq, w, ik_rows + t * CSA2O_DI);
  }
}

/* ------------------------------------------------------------------------------------------ */
/* Top-K by (score descending, index ascending), output ascending by index, -1 padded.         */
/* ------------------------------------------------------------------------------------------ */
typedef struct {
  double score;
  int64_t index;
} ranked_t;

static int cmp_rank(const void *pa, const void *pb) {
  const ranked_t *a = (const ranked_t *)pa, *b = (const ranked_t *)pb;
  if (a->score > b->score) return -1; /* higher score first; -0 == +0 compares equal */
  if (a->score < b->score) return 1;
  if (a->index < b->index) return -1; /* tie: lower index first */
  if (a->index > b->index) return 1;
  return 0;
}

static int cmp_i64(const void *pa, const void *pb) {
  int64_t a = *(const int64_t *)pa, b = *(const int64_t *)pb;
  return (a > b) - (a < b);
}

/* Select the first min(k, n) items of the (score desc, index asc) order; their indices are
 * written ascending into out[0..k) and the rest of out is -1. items is reordered. */
static void topk_ascending(ranked_t *items, int64_t n, int k, int64_t *out) {
  qsort(items, (size_t)n, sizeof(ranked_t), cmp_rank);
  int64_t take = n < k ? n : k;
  for (int64_t i = 0; i < take; ++i) out[i] = items[i].index;
  qsort(out, (size_t)take, sizeof(int64_t), cmp_i64);
  for (int64_t i = take; i < k; ++i) out[i] = -1;
}

int oracle_topk(const double *score, const int64_t *index, int64_t n, int k, int64_t *out) {
  ranked_t *items = (ranked_t *)malloc(sizeof(ranked_t) * (size_t)(n > 0 ? n : 1));
  if (!items) return -1;
  for (int64_t i = 0; i < n; ++i) {
    items[i].score = score[i];
    items[i].index = index ? index[i] : i;
  }
  topk_ascending(items, n, k, out);
  free(items);
  return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* CED KV projection [T1 CED paragraph]: the decoder layers' global KV is projected from the   */
/* middle layer's hidden state, C_l = H_{L/2} W^KV_l. Here C[m][j] = sum_k h[m][k] w[j][k]    */
/* (w holds one row per latent channel), summed in double; absdot[m][j] = sum_k |h w|, the   */
/* scale of any fp32 accumulation error of the same sum.                                      */
/* ------------------------------------------------------------------------------------------ */
void oracle_ced_project(const uint16_t *h, const uint16_t *w, int64_t M, int d, double *c,
                        double *absdot) {
  for (int64_t m = 0; m < M; ++m) {
    const uint16_t *hr = h + m * d;
    for (int j = 0; j < CSA2O_D; ++j) {
      const uint16_t *wr = w + (int64_t)j * d;
      double acc = 0.0, aacc = 0.0;
      for (int k = 0; k < d; ++k) {
        double p = (double)bf16_to_f32(hr[k]) * (double)bf16_to_f32(wr[k]);
        acc += p;
        aacc += fabs(p);
      }
      c[m * CSA2O_D + j] = acc;
      if (absdot) absdot[m * CSA2O_D + j] = aacc;
    }
  }
}

/* ------------------------------------------------------------------------------------------ */
/* Rounding of a double to bf16, nearest-even, by its definition: with |x| = m 2^e, m in       */
/* [0.5, 1), a normal bf16 keeps 8 significant bits (fewer below 2^-126, where the spacing     */
/* stays 2^-133); the scaled significand is rounded to an integer with ties to even, once.     */
/* Values above the largest finite bf16 after rounding become infinities.                      */
/* ------------------------------------------------------------------------------------------ */
uint16_t oracle_f64_to_bf16(double x) {
  const int neg = signbit(x) != 0;
  double a = fabs(x);
  uint16_t out;
  if (isnan(x)) return 0x7FC0;
  if (a == 0.0 || isinf(a)) {
    out = a == 0.0 ? 0x0000 : 0x7F80;
  } else {
    int e;
    double m = frexp(a, &e);                   /* a = m * 2^e, m in [0.5, 1) */
    int bits = 8;                              /* significant bits kept */
    if (e - 1 < -126) bits -= (-126 - (e - 1)); /* bf16 subnormal: spacing 2^-133 */
    double r;
    if (bits < 0) {
      r = 0.0;                                 /* below half the smallest subnormal */
    } else {
      double q = ldexp(m, bits);               /* exact */
      double f = floor(q), d = q - f;
      r = f;
      if (d > 0.5 || (d == 0.5 && fmod(f, 2.0) != 0.0)) r = f + 1.0;
    }
    double v = ldexp(r, e - bits);             /* the rounded value, exact in double */
    if (v > 3.3895313892515355e38) {           /* (2 - 2^-7) * 2^127 */
      out = 0x7F80;
    } else {
      float fv = (float)v;                     /* exact: v has at most 8 significant bits */
      uint32_t u;
      memcpy(&u, &fv, sizeof u);
      out = (uint16_t)(u >> 16);
    }
  }
  return (uint16_t)(out | (neg ? 0x8000 : 0));
}

/* ------------------------------------------------------------------------------------------ */
/* SWA bounded replay [A: "SWA Bounded Replay" keeps the persistent (host / SSD) KV cache at   */
/* about 1/8 of DeepSeek-V4-Flash's; Juju Radar's note on the report: the persistent cache      */
/* rebuilds the local sliding-window state instead of storing it; T1 "最后的结果": persistent   */
/* KV cache (SSD / host memory) about 1/8].                                                     */
/* Reading: the persisted copy of a sequence holds its global KV (MXFP4 codes and scales) and   */
/* its indexer keys; a restore copies those rows back and rebuilds the FP8 SWA ring from the    */
/* hidden states of the last Wr tokens: token r of sequence b sits at position                 */
/* p = N[b] - Wr + r (rows with p < 0 do not exist and are skipped); its SWA row is             */
/* x[j] = bf16_RNE(sum_k h[k] w[j][k]) (w holds one row per SWA channel; the sum is exact up to */
/* double rounding), quantised with the SWA codec into ring slot p mod W -- the row an append   */
/* of x at position p writes. Slots of other positions are left as they are.                   */
/* ------------------------------------------------------------------------------------------ */
void oracle_swa_replay(const uint16_t *h, const uint16_t *w, int B, int Wr, int d,
                       const int32_t *N, uint8_t *swa_e4m3, float *swa_scale, int W) {
  uint16_t x[CSA2O_D];
  for (int b = 0; b < B; ++b) {
    for (int r = 0; r < Wr; ++r) {
      int64_t p = (int64_t)N[b] - Wr + r;
      if (p < 0) continue;
      const uint16_t *hr = h + ((int64_t)b * Wr + r) * d;
      for (int j = 0; j < CSA2O_D; ++j) {
        const uint16_t *wr = w + (int64_t)j * d;
        double acc = 0.0;
        for (int k = 0; k < d; ++k) acc += (double)bf16_to_f32(hr[k]) * (double)bf16_to_f32(wr[k]);
        x[j] = oracle_f64_to_bf16(acc);
      }
      int64_t slot = (int64_t)b * W + (p % W);
      oracle_swa_quantize_token(x, swa_e4m3 + slot * CSA2O_D, swa_scale + slot);
    }
  }
}

/* ------------------------------------------------------------------------------------------ */
/* Full-mode indexer for one sequence [T1 hierarchical sparse indexer]:                        */
/*   scores over all N entries; Top-K positions; block maxima over 8-position blocks;          */
/*   Top-P blocks; pool = the selected blocks' positions in ascending block order, -1 past N.  */
/* ------------------------------------------------------------------------------------------ */
int oracle_index_full_seq(const uint16_t *iq, const float *w, const uint16_t *ik_rows, int64_t N,
                          int K, int P, double *score_out, double *blockmax_out, int64_t *topk,
                          int64_t *pool) {
  int64_t nb = (N + CSA2O_S - 1) / CSA2O_S;
  ranked_t *items = (ranked_t *)malloc(sizeof(ranked_t) * (size_t)(N > 0 ? N : 1));
  ranked_t *blocks = (ranked_t *)malloc(sizeof(ranked_t) * (size_t)(nb > 0 ? nb : 1));
  int64_t *sel_blocks = (int64_t *)malloc(sizeof(int64_t) * (size_t)P);
  if (!items || !blocks || !sel_blocks) {
    free(items);
    free(blocks);
    free(sel_blocks);
    return -1;
  }
  for (int64_t t = 0; t < N; ++t) {
    double s = oracle_index_score(iq, w, ik_rows + t * CSA2O_DI);
    if (score_out) score_out[t] = s;
    items[t].score = s;
    items[t].index = t;
  }
  for (int64_t j = 0; j < nb; ++j) {
    double m = -INFINITY;
    for (int64_t t = j * CSA2O_S; t < (j + 1) * CSA2O_S && t < N; ++t)
      if (items[t].score > m) m = items[t].score;
    if (blockmax_out) blockmax_out[j] = m;
    blocks[j].score = m;
    blocks[j].index = j;
  }
  topk_ascending(items, N, K, topk);
  topk_ascending(blocks, nb, P, sel_blocks);
  for (int i = 0; i < P; ++i) {
    for (int r = 0; r < CSA2O_S; ++r) {
      int64_t p = sel_blocks[i] < 0 ? -1 : sel_blocks[i] * CSA2O_S + r;
      pool[(int64_t)i * CSA2O_S + r] = (p >= 0 && p < N) ? p : -1;
    }
  }
  free(items);
  free(blocks);
  free(sel_blocks);
  return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* Reindex-mode indexer for one sequence [T1 Reindex mode]: the layer's own query and weights  */
/* score only the pool positions (-1 slots skipped); Top-K by (score desc, position asc).      */
/* ------------------------------------------------------------------------------------------ */
int oracle_index_reindex_seq(const uint16_t *iq, const float *w, const uint16_t *ik_rows,
                             const int64_t *pool, int64_t L, int K, double *score_out,
                             int64_t *topk) {
  ranked_t *items = (ranked_t *)malloc(sizeof(ranked_t) * (size_t)(L > 0 ? L : 1));
  if (!items) return -1;
  int64_t n = 0;
  for (int64_t i = 0; i < L; ++i) {
    if (pool[i] < 0) {
      if (score_out) score_out[i] = NAN;
      continue;
    }
    double s = oracle_index_score(iq, w, ik_rows + pool[i] * CSA2O_DI);
    if (score_out) score_out[i] = s;
    items[n].score = s;
    items[n].index = pool[i];
    ++n;
  }
  topk_ascending(items, n, K, topk);
  free(items);
  return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* Sparse attention for one sequence [T1 Reuse mode: sparse attention directly over the        */
/* selected entries; T1 FP8 SWA KV], all 16 heads. K = V = the dequantised entry. The selected */
/* MXFP4 entries (idx != -1) and the SWA slots 0..swa_len-1 enter one softmax.                 */
/* ------------------------------------------------------------------------------------------ */
int oracle_attend_seq(const uint16_t *q, float softmax_scale, const uint8_t *codes_rows,
                      const uint8_t *scales_rows, const int64_t *idx, int K,
                      const uint8_t *swa_rows, const float *swa_scale, int swa_len, float *out,
                      float *lse, double *weights_out) {
  int n = 0;
  for (int j = 0; j < K; ++j) n += idx[j] >= 0;
  n += swa_len;
  double *v = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * CSA2O_D);
  double *z = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  if (!v || !z) {
    free(v);
    free(z);
    return -1;
  }
  /* dequantised value rows, selected entries first, then SWA slots */
  int r = 0;
  for (int j = 0; j < K; ++j) {
    if (idx[j] < 0) continue;
    oracle_mxfp4_dequantize_entry(codes_rows + idx[j] * (CSA2O_D / 2),
                                  scales_rows + idx[j] * (CSA2O_D / 16), v + (int64_t)r * CSA2O_D);
    ++r;
  }
  for (int u = 0; u < swa_len; ++u, ++r)
    for (int i = 0; i < CSA2O_D; ++i)
      v[(int64_t)r * CSA2O_D + i] =
          oracle_e4m3_decode(swa_rows[(int64_t)u * CSA2O_D + i]) * (double)swa_scale[u];

  for (int h = 0; h < CSA2O_HQ; ++h) {
    const uint16_t *qh = q + (int64_t)h * CSA2O_D;
    float *oh = out + (int64_t)h * CSA2O_D;
    if (n == 0) {
      for (int i = 0; i < CSA2O_D; ++i) oh[i] = 0.0f;
      if (lse) lse[h] = -INFINITY;
      continue;
    }
    double m = -INFINITY;
    for (int t = 0; t < n; ++t) {
      double dot = 0.0;
      for (int i = 0; i < CSA2O_D; ++i)
        dot += (double)bf16_to_f32(qh[i]) * v[(int64_t)t * CSA2O_D + i];
      z[t] = (double)softmax_scale * dot;
      if (z[t] > m) m = z[t];
    }
    double l = 0.0;
    for (int t = 0; t < n; ++t) l += exp(z[t] - m);
    for (int t = 0; t < n; ++t) z[t] = exp(z[t] - m) / l; /* z now holds the softmax weights */
    for (int i = 0; i < CSA2O_D; ++i) {
      double acc = 0.0;
      for (int t = 0; t < n; ++t) acc += z[t] * v[(int64_t)t * CSA2O_D + i];
      oh[i] = (float)acc;
    }
    if (lse) lse[h] = (float)(m + log(l));
    if (weights_out)
      for (int t = 0; t < n; ++t) weights_out[(int64_t)h * n + t] = z[t];
  }
  free(v);
  free(z);
  return n;
}
