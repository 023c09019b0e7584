/*
 * qlora_oracle.c -- plain, slow CPU oracle for the QLoRA linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark load this file's library.  The product path
 * (the CUDA library and its Python binding) never includes, links or calls
 * anything here, and this file includes nothing from the product.
 *
 * Every step is the plain definition from the source pages, evaluated one
 * element at a time:
 *   - floats the format stores are fp32; each fp32 step below is a single
 *     IEEE round-to-nearest-even operation evaluated as written
 *     (build with -ffp-contract=off so that no FMA contraction happens);
 *   - dot products accumulate in fp64, sequentially, in index order;
 *   - every weight is decoded from its nibble and its block scale inside
 *     the sums (no dequantized matrix is formed by fwd/bwd).
 *
 * Sources (page title, section):
 *   [NF4]   "QLoRA Fine-Tuning" (Riftco Transformer how-to), section
 *           "NF4 representation": blockwise absmax, nearest codebook entry,
 *           low nibble first, all-zero block -> scale 0 and the zero code,
 *           legacy and double-quantized scale formulas, payload sizes.
 *   [FWD]   same page, section "Forward and backward": Y and dL/dX sums.
 *   [LAYER] "QLoRA on Mac -- fine-tuning larger open models on 48 GB",
 *           section "Design / Q-LoRA layer": base + (alpha/r)(x A^T) B^T.
 *   [TOY]   "QLoRA: Fine-Tuning Under Memory Constraints", section
 *           "See how a scale can hide small values" (2-bit absmax example).
 *   [NFC]   same page, section "Understand what NF4 chooses": levels follow
 *           a normal distribution.  The 16 values are not printed on the
 *           pages, which fix them as the canonical bitsandbytes mapping
 *           ("QLoRA Fine-Tuning", "NF4 representation");
 *           oracle_nf4_codebook() builds that table from the normal
 *           quantile construction evaluated in single precision.
 *   [EXPORT] "QLoRA Fine-Tuning", section "Training lifecycle" (step 5:
 *           dequantize the packed weights, add the trained LoRA deltas,
 *           restore an ordinary fp32 matrix).
 *   [ADAM]  same page, sections "Training lifecycle" (only the adapter
 *           factors are trained, with Adam) and "Current scope" (paged
 *           Adam state: pages of at most page_size elements).
 *   [AFF]   "LoRA vs QLoRA on Apple Silicon: memory/quality tradeoffs in
 *           MLX", sections "Method" and "Honest caveats": affine group-wise
 *           integer quantization with fp32 scale and bias (formula not
 *           printed; the plain min/max affine scheme is used).
 *
 * Readings where the pages are silent (each also listed in the design
 * notes): flat row-major block order; ties between two codebook entries go
 * to the lower index; w/s_b is a true fp32 division; the mean mu sums block
 * scales in fp64 sequentially inside each group of C blocks, then the group
 * partials sequentially; "round" is round-half-away-from-zero; odd N leaves
 * the last high nibble 0; an empty tensor has mu = 0; the adapter optimizer
 * is Adam with bias correction, eps added after the square root and no
 * weight decay; the merged weight adds s B A to the decoded weight.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_NONFINITE 1
#define ORACLE_ERR_ARG 2

#define ORACLE_FMT_NF4_DQ 0
#define ORACLE_FMT_NF4_FP32SCALE 1
#define ORACLE_FMT_AFFINE 2

/* ------------------------------------------------------------------------ */
/* Standard normal quantile (needed only to build the NF4 levels).           */
/* ------------------------------------------------------------------------ */

static double std_normal_cdf(double x) { return 0.5 * erfc(-x / sqrt(2.0)); }

/* Inverse of the standard normal CDF by bisection on the monotone CDF. */
double oracle_norm_ppf(double p) {
  if (!(p > 0.0 && p < 1.0)) return NAN;
  double lo = -40.0, hi = 40.0;
  for (int it = 0; it < 400; ++it) {
    double mid = 0.5 * (lo + hi);
    if (mid <= lo || mid >= hi) break;
    if (std_normal_cdf(mid) < p)
      lo = mid;
    else
      hi = mid;
  }
  return 0.5 * (lo + hi);
}

/*
 * [NFC] + [NF4] NF4 levels.  The pages fix the table as the canonical
 * mapping of the bitsandbytes implementation ("NF4 representation") and say
 * the levels follow a normal distribution ("Understand what NF4 chooses").
 * That table is the normal-quantile construction evaluated in single
 * precision:
 *   - offset delta = 0.9677083 (the midpoint of 1 - 1/30 and 1 - 1/32,
 *     written to seven decimals), as an fp32 number;
 *   - n evenly spaced fp32 probabilities from delta to 1/2 (n = 9 for the
 *     positive side, n = 8 for the negative side), 1/2 itself dropped:
 *     step = fp32((1/2 - delta) / (n - 1)); the first half of the sequence
 *     steps up from delta (delta + j step), the second half down from 1/2
 *     (1/2 - (n - 1 - j) step), every product and sum rounded to fp32;
 *   - the standard normal quantile of each probability (fp64), rounded to
 *     fp32: 8 positive levels, 7 negated ones, and an exact zero;
 *   - sorted ascending and divided (fp32) by the largest.
 * out32 is the table the quantized format uses; out64 holds the same values
 * widened to fp64.
 */
static void nf4_probabilities(int n, float* p) {
  const float delta = 0.9677083f, half = 0.5f;
  const float step = (half - delta) / (float)(n - 1);
  for (int j = 0; j < n; ++j) {
    if (j < n / 2) {
      const float t = (float)j * step;
      p[j] = delta + t;
    } else {
      const float t = (float)(n - 1 - j) * step;
      p[j] = half - t;
    }
  }
}

void oracle_nf4_codebook(double out64[16], float out32[16]) {
  float pp[9], pn[8], v[16];
  nf4_probabilities(9, pp);
  nf4_probabilities(8, pn);
  int n = 0;
  for (int j = 0; j < 8; ++j) v[n++] = (float)oracle_norm_ppf((double)pp[j]);
  v[n++] = 0.0f;
  for (int j = 0; j < 7; ++j) v[n++] = (float)(-oracle_norm_ppf((double)pn[j]));
  for (int a = 1; a < 16; ++a) { /* insertion sort, ascending */
    float key = v[a];
    int b = a - 1;
    while (b >= 0 && v[b] > key) {
      v[b + 1] = v[b];
      --b;
    }
    v[b + 1] = key;
  }
  const float mx = v[15];
  for (int k = 0; k < 16; ++k) {
    out32[k] = v[k] / mx;
    out64[k] = (double)out32[k];
  }
}

/* ------------------------------------------------------------------------ */
/* Nearest level of a sorted codebook.                                       */
/* ------------------------------------------------------------------------ */

/*
 * [NF4] each normalized weight takes its closest level.  code = number of midpoints
 * (c_k + c_{k+1})/2 (exact in fp64) strictly below x, which is argmin_k
 * |x - c_k| with the lower index kept on a tie.
 */
static int nearest_level(double x, const double* levels, int L) {
  int code = 0;
  for (int k = 0; k + 1 < L; ++k) {
    double mid = 0.5 * (levels[k] + levels[k + 1]);
    if (x > mid) ++code;
  }
  return code;
}

/*
 * [TOY] Generic absmax block quantizer with an arbitrary sorted codebook
 * (levels in [-1, 1]).  Writes one code per weight (unpacked) and the
 * block scale; W_hat receives level*scale.  Used by the tests to replay the
 * pages' 2-bit teaching example with the same absmax + nearest-level steps
 * the NF4 path takes.
 */
int oracle_quantize_levels(const float* w, int64_t n, int64_t B, const double* levels, int L,
                           uint8_t* codes, float* scales, double* w_hat) {
  if (B <= 0 || L < 2) return ORACLE_ERR_ARG;
  for (int64_t i = 0; i < n; ++i)
    if (!isfinite(w[i])) return ORACLE_ERR_NONFINITE;
  int zero = nearest_level(0.0, levels, L);
  for (int64_t lo = 0, b = 0; lo < n; lo += B, ++b) {
    int64_t hi = lo + B < n ? lo + B : n;
    float s = 0.0f;
    for (int64_t i = lo; i < hi; ++i)
      if (fabsf(w[i]) > s) s = fabsf(w[i]);
    scales[b] = s;
    for (int64_t i = lo; i < hi; ++i) {
      int c = (s == 0.0f) ? zero : nearest_level((double)(w[i] / s), levels, L);
      codes[i] = (uint8_t)c;
      w_hat[i] = levels[c] * (double)s;
    }
  }
  return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* NF4 with double-quantized scales.                                         */
/* ------------------------------------------------------------------------ */

/*
 * [NF4] Encode W (N fp32 values, flat row-major) with block size B and
 * scale-group size C.
 *   codes  : ceil(N/2) bytes, value 2j in the low nibble of byte j
 *   qcodes : M = ceil(N/B) centred unsigned-byte scale codes
 *   t      : S = ceil(M/C) fp32 second-level absmax values t_g
 *   mu     : the one fp32 mean of the block scales
 *   s_out  : (nullable) the exact fp32 block absmax values s_b
 */
int oracle_quantize_nf4(const float* W, int64_t N, int32_t B, int32_t C, uint8_t* codes,
                        uint8_t* qcodes, float* t, float* mu, float* s_out) {
  if (N < 0 || B <= 0 || C <= 0) return ORACLE_ERR_ARG;
  for (int64_t i = 0; i < N; ++i)
    if (!isfinite(W[i])) return ORACLE_ERR_NONFINITE;
  double c64[16];
  float c32[16];
  oracle_nf4_codebook(c64, c32);
  double lv[16];
  for (int k = 0; k < 16; ++k) lv[k] = (double)c32[k];
  const int64_t M = (N + B - 1) / B;
  const int64_t S = (M + C - 1) / C;
  float* s = (float*)malloc(sizeof(float) * (size_t)(M > 0 ? M : 1));
  if (!s) return ORACLE_ERR_ARG;
  memset(codes, 0, (size_t)((N + 1) / 2));

  /* block absmax, then the nearest code of w / s_b */
  for (int64_t b = 0; b < M; ++b) {
    int64_t lo = b * B, hi = lo + B < N ? lo + B : N;
    float sb = 0.0f;
    for (int64_t i = lo; i < hi; ++i)
      if (fabsf(W[i]) > sb) sb = fabsf(W[i]);
    s[b] = sb;
    for (int64_t i = lo; i < hi; ++i) {
      int code;
      if (sb == 0.0f) {
        code = 7; /* the exact-zero entry */
      } else {
        float x = W[i] / sb;
        code = nearest_level((double)x, lv, 16);
      }
      if (i & 1)
        codes[i >> 1] |= (uint8_t)(code << 4);
      else
        codes[i >> 1] |= (uint8_t)code;
    }
  }

  /* the shared mean of the block scales */
  double total = 0.0;
  for (int64_t g = 0; g < S; ++g) {
    double part = 0.0;
    int64_t lo = g * C, hi = lo + C < M ? lo + C : M;
    for (int64_t b = lo; b < hi; ++b) part += (double)s[b];
    total += part;
  }
  float m = (M > 0) ? (float)(total / (double)M) : 0.0f;
  *mu = m;

  /* second-level absmax per group, then the centred byte codes */
  for (int64_t g = 0; g < S; ++g) {
    int64_t lo = g * C, hi = lo + C < M ? lo + C : M;
    float tg = 0.0f;
    for (int64_t b = lo; b < hi; ++b) {
      float d = s[b] - m;
      if (fabsf(d) > tg) tg = fabsf(d);
    }
    t[g] = tg;
  }
  for (int64_t b = 0; b < M; ++b) {
    float tg = t[b / C];
    int q;
    if (tg == 0.0f) {
      q = 128; /* zero range */
    } else {
      float d = s[b] - m;
      float num = 127.0f * d;
      float v = num / tg;
      float rv = roundf(v);
      if (rv < -127.0f) rv = -127.0f;
      if (rv > 127.0f) rv = 127.0f;
      q = 128 + (int)rv;
    }
    qcodes[b] = (uint8_t)q;
  }
  if (s_out)
    for (int64_t b = 0; b < M; ++b) s_out[b] = s[b];
  free(s);
  return ORACLE_OK;
}

/* [NF4] Decoded block scale: clamp(mu + t_g (q_b - 128)/127, 0, FLT_MAX). */
float oracle_decode_scale(uint8_t q, float t, float mu) {
  float k = (float)((int)q - 128);
  float a = t * k;
  float b = a / 127.0f;
  float s = mu + b;
  if (s < 0.0f) s = 0.0f;
  if (s > FLT_MAX) s = FLT_MAX;
  return s;
}

/* ------------------------------------------------------------------------ */
/* Affine group-wise integer quantization.                                   */
/* ------------------------------------------------------------------------ */

/*
 * [AFF] Group g = G consecutive weights.  scale = (max - min)/(2^bits - 1),
 * bias = min, code = round((w - bias)/scale) clamped to [0, 2^bits - 1]
 * (0 when scale is 0); 4-bit codes pack low nibble first, 8-bit codes use
 * one byte each.
 */
int oracle_quantize_affine(const float* W, int64_t N, int32_t bits, int32_t G, uint8_t* codes,
                           float* scale, float* bias) {
  if (N < 0 || G <= 0 || (bits != 4 && bits != 8)) return ORACLE_ERR_ARG;
  for (int64_t i = 0; i < N; ++i)
    if (!isfinite(W[i])) return ORACLE_ERR_NONFINITE;
  const int levels = (1 << bits) - 1;
  const int64_t ng = (N + G - 1) / G;
  if (bits == 4) memset(codes, 0, (size_t)((N + 1) / 2));
  for (int64_t g = 0; g < ng; ++g) {
    int64_t lo = g * G, hi = lo + G < N ? lo + G : N;
    float mn = W[lo], mx = W[lo];
    for (int64_t i = lo; i < hi; ++i) {
      if (W[i] < mn) mn = W[i];
      if (W[i] > mx) mx = W[i];
    }
    float sc = (mx - mn) / (float)levels;
    if (!isfinite(sc)) return ORACLE_ERR_NONFINITE;
    scale[g] = sc;
    bias[g] = mn;
    for (int64_t i = lo; i < hi; ++i) {
      int q = 0;
      if (sc != 0.0f) {
        float v = (W[i] - mn) / sc;
        float rv = roundf(v);
        if (rv < 0.0f) rv = 0.0f;
        if (rv > (float)levels) rv = (float)levels;
        q = (int)rv;
      }
      if (bits == 8)
        codes[i] = (uint8_t)q;
      else if (i & 1)
        codes[i >> 1] |= (uint8_t)(q << 4);
      else
        codes[i >> 1] |= (uint8_t)q;
    }
  }
  return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Per-element decode of a quantized weight.                                 */
/* ------------------------------------------------------------------------ */

typedef struct {
  int32_t fmt; /* ORACLE_FMT_NF4_DQ, ORACLE_FMT_NF4_FP32SCALE or ORACLE_FMT_AFFINE */
  int64_t O, I;
  int32_t block; /* B (NF4) or G (affine) */
  int32_t group; /* C (NF4) */
  int32_t bits;  /* 4 or 8 (affine); 4 for NF4 */
  const uint8_t* codes;
  const uint8_t* qcodes;
  const float* t;
  float mu;
  const float* scale;
  const float* bias;
} OracleWeight;

static float g_cb[16];
static int g_cb_ready = 0;

static void ensure_codebook(void) {
  if (!g_cb_ready) {
    double c64[16];
    oracle_nf4_codebook(c64, g_cb);
    g_cb_ready = 1;
  }
}

/* w_hat at flat index n: codebook entry of its nibble times its block scale. */
static float weight_at(const OracleWeight* w, int64_t n) {
  if (w->fmt == ORACLE_FMT_NF4_DQ) {
    uint8_t byte = w->codes[n >> 1];
    int code = (n & 1) ? (byte >> 4) : (byte & 15);
    int64_t b = n / w->block;
    int64_t g = b / w->group;
    float s = oracle_decode_scale(w->qcodes[b], w->t[g], w->mu);
    return g_cb[code] * s;
  } else if (w->fmt == ORACLE_FMT_NF4_FP32SCALE) {
    /* [NF4] legacy scales: the block absmax s_b itself, one fp32 per block */
    uint8_t byte = w->codes[n >> 1];
    int code = (n & 1) ? (byte >> 4) : (byte & 15);
    return g_cb[code] * w->scale[n / w->block];
  } else {
    int q;
    if (w->bits == 8) {
      q = w->codes[n];
    } else {
      uint8_t byte = w->codes[n >> 1];
      q = (n & 1) ? (byte >> 4) : (byte & 15);
    }
    int64_t g = n / w->block;
    float a = w->scale[g] * (float)q;
    return a + w->bias[g];
  }
}

/* Diagnostic dequantization of the whole matrix to fp32. */
void oracle_dequantize(const OracleWeight* w, float* W_hat) {
  ensure_codebook();
  const int64_t N = w->O * w->I;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) W_hat[n] = weight_at(w, n);
}

/* ------------------------------------------------------------------------ */
/* The QLoRA linear layer.                                                   */
/* ------------------------------------------------------------------------ */

static double lora_scale(float alpha, int32_t r) { return (double)(alpha / (float)r); }

/*
 * [FWD], [LAYER]  Y = X W_hat^T + s (X A^T) B^T,  s = alpha / r.
 * X [R x I] (fp32 values; bf16 inputs arrive already widened), A [r x I],
 * Bm [O x r].  rows (nullable) selects nrows of the R rows; the outputs
 * hold only those rows: Y [nrows x O], U [nrows x r].
 */
void oracle_linear_fwd(const OracleWeight* w, const float* X, int64_t R, const int64_t* rows,
                       int64_t nrows, const float* A, const float* Bm, int32_t r, float alpha,
                       double* Y, double* U) {
  ensure_codebook();
  (void)R;
  const int64_t O = w->O, I = w->I;
  const double s = lora_scale(alpha, r);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < nrows; ++j) {
    const float* x = X + (rows ? rows[j] : j) * I;
    for (int32_t k = 0; k < r; ++k) {
      double acc = 0.0;
      for (int64_t i = 0; i < I; ++i) acc += (double)x[i] * (double)A[k * I + i];
      U[j * r + k] = acc;
    }
  }
#pragma omp parallel
  {
    double* wrow = (double*)malloc(sizeof(double) * (size_t)(I > 0 ? I : 1));
#pragma omp for schedule(dynamic, 4)
    for (int64_t o = 0; o < O; ++o) {
      for (int64_t i = 0; i < I; ++i) wrow[i] = (double)weight_at(w, o * I + i);
      for (int64_t j = 0; j < nrows; ++j) {
        const float* x = X + (rows ? rows[j] : j) * I;
        double acc = 0.0;
        for (int64_t i = 0; i < I; ++i) acc += (double)x[i] * wrow[i];
        double ad = 0.0;
        for (int32_t k = 0; k < r; ++k) ad += U[j * r + k] * (double)Bm[o * r + k];
        Y[j * O + o] = acc + s * ad;
      }
    }
    free(wrow);
  }
}

/*
 * [FWD] input gradient and the LoRA chain rule (no weight gradient: the base
 * is frozen).
 *   V  = dY B                 (all R rows)
 *   U  = X A^T                (all R rows)
 *   dX = dY W_hat + s V A     (rows selected by `rows`, nrows of them)
 *   dA = s V^T X              [r x I], full reduction over R
 *   dB = s dY^T U             [O x r], full reduction over R
 * Any of dX, dA, dB may be NULL to skip it.
 */
void oracle_linear_bwd(const OracleWeight* w, const float* X, const float* dY, int64_t R,
                       const int64_t* rows, int64_t nrows, const float* A, const float* Bm,
                       int32_t r, float alpha, double* dX, double* dA, double* dB) {
  ensure_codebook();
  const int64_t O = w->O, I = w->I;
  const double s = lora_scale(alpha, r);
  double* V = (double*)calloc((size_t)(R > 0 ? R : 1) * (size_t)(r > 0 ? r : 1), sizeof(double));
  double* U = (double*)calloc((size_t)(R > 0 ? R : 1) * (size_t)(r > 0 ? r : 1), sizeof(double));
#pragma omp parallel for schedule(static)
  for (int64_t rr = 0; rr < R; ++rr) {
    for (int32_t k = 0; k < r; ++k) {
      double v = 0.0, u = 0.0;
      for (int64_t o = 0; o < O; ++o) v += (double)dY[rr * O + o] * (double)Bm[o * r + k];
      for (int64_t i = 0; i < I; ++i) u += (double)X[rr * I + i] * (double)A[k * I + i];
      V[rr * r + k] = v;
      U[rr * r + k] = u;
    }
  }
  if (dX) {
    const int64_t CH = 64;
    const int64_t nch = (I + CH - 1) / CH;
#pragma omp parallel
    {
      double* acc = (double*)malloc(sizeof(double) * (size_t)(nrows > 0 ? nrows : 1) * CH);
      double wv[64];
#pragma omp for schedule(dynamic, 1)
      for (int64_t c = 0; c < nch; ++c) {
        int64_t i0 = c * CH, i1 = i0 + CH < I ? i0 + CH : I;
        for (int64_t q = 0; q < nrows * CH; ++q) acc[q] = 0.0;
        for (int64_t o = 0; o < O; ++o) {
          for (int64_t i = i0; i < i1; ++i) wv[i - i0] = (double)weight_at(w, o * I + i);
          for (int64_t j = 0; j < nrows; ++j) {
            double g = (double)dY[(rows ? rows[j] : j) * O + o];
            for (int64_t i = i0; i < i1; ++i) acc[j * CH + (i - i0)] += g * wv[i - i0];
          }
        }
        for (int64_t j = 0; j < nrows; ++j) {
          int64_t rj = rows ? rows[j] : j;
          for (int64_t i = i0; i < i1; ++i) {
            double ad = 0.0;
            for (int32_t k = 0; k < r; ++k) ad += V[rj * r + k] * (double)A[k * I + i];
            dX[j * I + i] = acc[j * CH + (i - i0)] + s * ad;
          }
        }
      }
      free(acc);
    }
  }
  if (dA) {
    const int64_t CH = 256;
    const int64_t nch = (I + CH - 1) / CH;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t c = 0; c < nch; ++c) {
      int64_t i0 = c * CH, i1 = i0 + CH < I ? i0 + CH : I;
      for (int32_t k = 0; k < r; ++k)
        for (int64_t i = i0; i < i1; ++i) dA[k * I + i] = 0.0;
      for (int64_t rr = 0; rr < R; ++rr)
        for (int32_t k = 0; k < r; ++k) {
          double v = V[rr * r + k];
          for (int64_t i = i0; i < i1; ++i) dA[k * I + i] += v * (double)X[rr * I + i];
        }
      for (int32_t k = 0; k < r; ++k)
        for (int64_t i = i0; i < i1; ++i) dA[k * I + i] *= s;
    }
  }
  if (dB) {
    const int64_t CH = 256;
    const int64_t nch = (O + CH - 1) / CH;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t c = 0; c < nch; ++c) {
      int64_t o0 = c * CH, o1 = o0 + CH < O ? o0 + CH : O;
      for (int64_t o = o0; o < o1; ++o)
        for (int32_t k = 0; k < r; ++k) dB[o * r + k] = 0.0;
      for (int64_t rr = 0; rr < R; ++rr)
        for (int64_t o = o0; o < o1; ++o) {
          double g = (double)dY[rr * O + o];
          for (int32_t k = 0; k < r; ++k) dB[o * r + k] += g * U[rr * r + k];
        }
      for (int64_t o = o0; o < o1; ++o)
        for (int32_t k = 0; k < r; ++k) dB[o * r + k] *= s;
    }
  }
  free(V);
  free(U);
}

/* ------------------------------------------------------------------------ */
/* Export and the adapter optimizer step.                                    */
/* ------------------------------------------------------------------------ */

/*
 * [EXPORT]  W_merged = W_hat + s B A,  s = alpha / r.  A [r x I], Bm [O x r];
 * out [O x I] in fp64.  The export step of the training lifecycle
 * dequantizes every packed weight and adds its trained LoRA delta, giving
 * an ordinary floating-point matrix; the delta of element (o, i) is the
 * rank-r sum over k of B[o,k] A[k,i], the same product the forward applies
 * to X (Y = X W_merged^T).  The delta is summed in fp64, in k order.
 */
void oracle_merge(const OracleWeight* w, const float* A, const float* Bm, int32_t r, float alpha,
                  double* out) {
  ensure_codebook();
  const int64_t O = w->O, I = w->I;
  const double s = lora_scale(alpha, r);
#pragma omp parallel for schedule(static)
  for (int64_t o = 0; o < O; ++o) {
    for (int64_t i = 0; i < I; ++i) {
      double delta = 0.0;
      for (int32_t k = 0; k < r; ++k) delta += (double)Bm[o * r + k] * (double)A[k * I + i];
      out[o * I + i] = (double)weight_at(w, o * I + i) + s * delta;
    }
  }
}

/*
 * [ADAM]  One Adam step on n adapter parameters (the adapter factors are the
 * only optimizer inputs; the packed base never is).  The pages name Adam but
 * print no update rule; this is Adam with bias correction, step t >= 1:
 *   m' = beta1 m + (1 - beta1) g
 *   v' = beta2 v + (1 - beta2) g^2
 *   p' = p - lr (m' / (1 - beta1^t)) / (sqrt(v' / (1 - beta2^t)) + eps)
 * Inputs are the fp32 state; everything is evaluated in fp64 and p', m', v'
 * are returned in fp64.  Paging the state (pages of at most page_size
 * elements, one page update at a time) changes when each element is
 * updated, not what it becomes, so the oracle has no page argument.
 */
void oracle_adam_step(const float* p, const float* g, const float* m, const float* v, int64_t n,
                      int64_t t, float lr, float beta1, float beta2, float eps, double* p_out,
                      double* m_out, double* v_out) {
  const double b1 = (double)beta1, b2 = (double)beta2;
  const double bc1 = 1.0 - pow(b1, (double)t);
  const double bc2 = 1.0 - pow(b2, (double)t);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < n; ++j) {
    const double gj = (double)g[j];
    const double mj = b1 * (double)m[j] + (1.0 - b1) * gj;
    const double vj = b2 * (double)v[j] + (1.0 - b2) * gj * gj;
    const double mhat = mj / bc1;
    const double vhat = vj / bc2;
    p_out[j] = (double)p[j] - (double)lr * mhat / (sqrt(vhat) + (double)eps);
    m_out[j] = mj;
    v_out[j] = vj;
  }
}

/* Threads OpenMP will use (reported beside the CPU timings). */
#ifdef _OPENMP
#include <omp.h>
int oracle_num_threads(void) { return omp_get_max_threads(); }
#else
int oracle_num_threads(void) { return 1; }
#endif
