/*
 * Oracle for block-causal attention with cross-step prefix K/V reuse.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file: only the test suite, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or helper with the CUDA
 * library, and it includes nothing from it.
 *
 * A plain, slow, obviously correct fp64 CPU restatement of what the hot path
 * computes.  Every function below is the definition written out, with no
 * blocking, fusion or reordering beyond what the definition states.
 *
 * Sources (web pages; cited by page title and section):
 *  - "Qwen-Image-2.1 + vLLM-Omni day-0" (thakicloud.com, English), sections
 *    "What is Qwen-Image-2.1" (the DiT uses block-causal attention) and
 *    "Serving architecture: the cross-step prefix KV cache" (prefix K/V from the
 *    first denoising step is exact for later steps; rebuilt per request).
 *  - "Qwen/Qwen-Image-2.1" (recipes.vllm.ai), section "Prefix KV cache" (exact,
 *    per generation; "fp8_v" quantises V only, "fp8" quantises K too).
 *  - OCP 8-bit Floating Point Specification (OFP8), E4M3 encoding: 1 sign bit,
 *    4 exponent bits (bias 7), 3 mantissa bits, no infinities, S.1111.111 = NaN,
 *    largest finite magnitude 448.
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes): blocks are contiguous and ordered, block b sees blocks 0..b
 * (so row i sees keys j < end of its block); MHA with head_dim d; activations
 * are [tokens, H, d]; a cache is [H, cap, d]; per-(head, K|V) absmax scales
 * s = fp32(amax) / 448 (s = 1 when amax = 0), code = e4m3_rne_satfinite(fp32(x / s)),
 * dequantised value = fp32(decode(code) * s).
 *
 * All inputs arrive as raw bf16 bit patterns (uint16) or e4m3 codes (uint8);
 * bf16 -> fp64 widening is exact.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* Number formats                                                            */
/* ------------------------------------------------------------------------ */

/* bf16 is the top half of an IEEE binary32: widen exactly. */
double bca_oracle_bf16_to_f64(uint16_t bits) {
  uint32_t w = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &w, sizeof f);
  return (double)f;
}

/* OFP8 E4M3 decode, straight from the bit-field definition.
 * exponent field 0 -> subnormal m * 2^-9; otherwise (1 + m/8) * 2^(e-7);
 * S.1111.111 is NaN (there are no infinities). */
double bca_oracle_e4m3_decode(uint8_t code) {
  int sign = (code >> 7) & 1;
  int e = (code >> 3) & 0xF;
  int m = code & 0x7;
  double mag;
  if (e == 0xF && m == 0x7) return NAN;
  if (e == 0)
    mag = ldexp((double)m, -9);
  else
    mag = ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -mag : mag;
}

/* OFP8 E4M3 encode with round-to-nearest-even and saturation to the largest
 * finite magnitude (448).  Brute force: compare |x| exactly against every one of
 * the 127 non-negative finite magnitudes (codes 0x00..0x7E) and take the
 * nearest; on an exact tie take the code whose mantissa LSB is 0 (the even
 * one).  The sign bit is copied, so a negative value that rounds to zero gives
 * 0x80.  Precondition: x is finite. */
uint8_t bca_oracle_e4m3_encode(float x) {
  double ax = fabs((double)x);
  uint8_t sign = signbit(x) ? 0x80 : 0x00;
  int best = 0;
  double best_err = INFINITY;
  if (ax >= 448.0) return (uint8_t)(sign | 0x7E);
  for (int c = 0; c <= 0x7E; ++c) {
    double err = fabs(bca_oracle_e4m3_decode((uint8_t)c) - ax);
    if (err < best_err) {
      best_err = err;
      best = c;
    } else if (err == best_err && (c & 1) == 0 && (best & 1) == 1) {
      best = c; /* tie: prefer the even mantissa */
    }
  }
  return (uint8_t)(sign | best);
}

/* The same encode applied to n values (a loop, for test throughput). */
void bca_oracle_e4m3_encode_n(const float* x, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = bca_oracle_e4m3_encode(x[i]);
}

/* Per-(head, tensor) scale: s = fp32(amax) / 448 rounded to binary32 (amax is a
 * bf16 value, hence exactly a float; the fp64 quotient rounded to fp32 equals the
 * correctly rounded fp32 quotient because 53 >= 2*24 + 2).  s = 1 when amax = 0.
 * x points at row 0 of a [n_rows, d] view whose rows are row_stride elements apart. */
float bca_oracle_absmax_scale(const uint16_t* x, int64_t n_rows, int64_t row_stride, int64_t d) {
  double amax = 0.0;
  for (int64_t t = 0; t < n_rows; ++t)
    for (int64_t c = 0; c < d; ++c) {
      double a = fabs(bca_oracle_bf16_to_f64(x[t * row_stride + c]));
      if (a > amax) amax = a;
    }
  if (amax == 0.0) return 1.0f;
  return (float)(amax / 448.0);
}

/* Quantise the prefix rows [0, P) of one [tokens, H, d] bf16 tensor (token rows
 * `row_stride` elements apart) into a [H, cap, d] e4m3 cache plus scales[H].
 * Rows [P, cap) of the cache are left untouched. */
void bca_oracle_quantize_prefix(const uint16_t* x, int64_t P, int64_t H, int64_t d,
                                int64_t row_stride, int64_t cap, uint8_t* codes,
                                float* scales) {
  for (int64_t h = 0; h < H; ++h) {
    float s = bca_oracle_absmax_scale(x + h * d, P, row_stride, d);
    scales[h] = s;
    for (int64_t t = 0; t < P; ++t)
      for (int64_t c = 0; c < d; ++c) {
        double v = bca_oracle_bf16_to_f64(x[t * row_stride + h * d + c]);
        float q = (float)(v / (double)s);
        codes[(h * cap + t) * d + c] = bca_oracle_e4m3_encode(q);
      }
  }
}

/* ------------------------------------------------------------------------ */
/* Key/value sources                                                         */
/* ------------------------------------------------------------------------ */

enum { SRC_BF16 = 0, SRC_E4M3 = 1 };

/* A list of n rows of length d.  Row j starts at element j*row_stride of base.
 * For e4m3 rows the element value is fp32(decode(code) * scale) (the dequantised
 * value a reader of the cache sees). */
typedef struct {
  const void* base;
  int kind;
  int64_t row_stride;
  int64_t n;
  float scale;
} kv_src;

static double src_elem(const kv_src* s, int64_t j, int64_t c) {
  int64_t idx = j * s->row_stride + c;
  if (s->kind == SRC_BF16) return bca_oracle_bf16_to_f64(((const uint16_t*)s->base)[idx]);
  float dq = (float)bca_oracle_e4m3_decode(((const uint8_t*)s->base)[idx]) * s->scale;
  return (double)dq;
}

/* One output row: softmax(q . k_j * scale) over the keys of the sources, in
 * order (source 0 rows 0..n0-1, then source 1 rows 0..n1-1, ...), applied to the
 * matching values.  q[s] is the query row that meets source s's keys (the same
 * row for every source, except where the query is quantised for one of them).
 * Keys not listed are simply absent from the sum (that is the mask).  scores[] is
 * caller scratch of length >= total keys. */
static void attend_row(const double* const* q, int64_t d, const kv_src* ks, const kv_src* vs,
                       int nsrc, double scale, double* scores, double* out) {
  int64_t nk = 0;
  double m = -INFINITY;
  for (int s = 0; s < nsrc; ++s)
    for (int64_t j = 0; j < ks[s].n; ++j) {
      double dot = 0.0;
      for (int64_t c = 0; c < d; ++c) dot += q[s][c] * src_elem(&ks[s], j, c);
      double sc = scale * dot;
      scores[nk++] = sc;
      if (sc > m) m = sc;
    }
  double l = 0.0;
  for (int64_t j = 0; j < nk; ++j) {
    scores[j] = exp(scores[j] - m);
    l += scores[j];
  }
  for (int64_t c = 0; c < d; ++c) out[c] = 0.0;
  nk = 0;
  for (int s = 0; s < nsrc; ++s)
    for (int64_t j = 0; j < vs[s].n; ++j) {
      double p = scores[nk++] / l;
      for (int64_t c = 0; c < d; ++c) out[c] += p * src_elem(&vs[s], j, c);
    }
}

static int check_blocks(const int32_t* off, int n_blocks, int64_t S) {
  if (n_blocks < 1 || off[0] != 0 || off[n_blocks] != S) return 0;
  for (int b = 0; b < n_blocks; ++b)
    if (off[b + 1] <= off[b]) return 0;
  return 1;
}

/* End offset of the block that holds row i (its key limit). */
static int64_t block_end(const int32_t* off, int n_blocks, int64_t i) {
  for (int b = 0; b < n_blocks; ++b)
    if (i < off[b + 1]) return off[b + 1];
  return off[n_blocks];
}

static void set_threads(int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
}

int bca_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Step 1: block-causal attention over the whole sequence                    */
/* ------------------------------------------------------------------------ */
/* q, k, v: [S, H, d] bf16 bits.  Blocks: offsets[0] = 0 < offsets[1] < ... <
 * offsets[n_blocks] = S.  Row i attends to keys j < end of its block, with full
 * attention inside the block.  rows: the n_rows query rows to compute (NULL means
 * all S rows in order).  out: [n_rows, H, d] fp64.  Returns 0, or -1 on bad
 * arguments. */
int bca_oracle_prefill(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t S,
                       int64_t H, int64_t d, const int32_t* offsets, int n_blocks,
                       double scale, const int64_t* rows, int64_t n_rows, double* out,
                       int nthreads) {
  if (S < 1 || H < 1 || d < 1 || !check_blocks(offsets, n_blocks, S)) return -1;
  if (!rows) n_rows = S;
  for (int64_t r = 0; r < n_rows; ++r)
    if (rows && (rows[r] < 0 || rows[r] >= S)) return -1;
  set_threads(nthreads);
#pragma omp parallel
  {
    double* scores = (double*)malloc(sizeof(double) * (size_t)S);
    double* qrow = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 1)
    for (int64_t rh = 0; rh < n_rows * H; ++rh) {
      int64_t r = rh / H, h = rh % H;
      int64_t i = rows ? rows[r] : r;
      int64_t lim = block_end(offsets, n_blocks, i);
      kv_src ks = {k + h * d, SRC_BF16, H * d, lim, 1.0f};
      kv_src vs = {v + h * d, SRC_BF16, H * d, lim, 1.0f};
      for (int64_t c = 0; c < d; ++c) qrow[c] = bca_oracle_bf16_to_f64(q[(i * H + h) * d + c]);
      const double* qs[1] = {qrow};
      attend_row(qs, d, &ks, &vs, 1, scale, scores, out + (r * H + h) * d);
    }
    free(scores);
    free(qrow);
  }
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Steps 2..N: target rows over [cached prefix ; own K/V]                     */
/* ------------------------------------------------------------------------ */
/* q_t, k_t, v_t: [T, H, d] bf16 bits (one request's target rows).
 * k_cache, v_cache: [H, cap, d]; rows [0, P) are used.  kind 0 = bf16 bits,
 * kind 1 = e4m3 codes dequantised with k_scale[h] / v_scale[h].
 * Every target row attends to all P cached keys and all T target keys (the
 * target is the last block), in that order.  rows: target rows to compute
 * (NULL = all).  out: [n_rows, H, d] fp64.
 * q_codes, q_scale (both NULL, or both given): the e4m3-Q reading of the cached
 * step -- the request's Q quantised per head like a cache tensor (codes [H, T, d],
 * scales [H], the same encoder and scale rule), and the scores against the cached
 * keys taken with the dequantised Q, fp32(decode(code) * scale); the scores
 * against the target's own keys keep the bf16 Q. */
int bca_oracle_cached_step(const uint16_t* q_t, const uint16_t* k_t, const uint16_t* v_t,
                           int64_t T, int64_t H, int64_t d, const void* k_cache, int k_kind,
                           const float* k_scale, const void* v_cache, int v_kind,
                           const float* v_scale, int64_t P, int64_t cap, double scale,
                           const int64_t* rows, int64_t n_rows, double* out, int nthreads,
                           const uint8_t* q_codes, const float* q_scale) {
  if (T < 1 || H < 1 || d < 1 || P < 0 || cap < P) return -1;
  if (P > 0 && (!k_cache || !v_cache)) return -1;
  if ((k_kind == SRC_E4M3 && !k_scale) || (v_kind == SRC_E4M3 && !v_scale)) return -1;
  if ((q_codes == NULL) != (q_scale == NULL)) return -1;
  if (!rows) n_rows = T;
  for (int64_t r = 0; r < n_rows; ++r)
    if (rows && (rows[r] < 0 || rows[r] >= T)) return -1;
  set_threads(nthreads);
#pragma omp parallel
  {
    double* scores = (double*)malloc(sizeof(double) * (size_t)(P + T));
    double* qrow = (double*)malloc(sizeof(double) * (size_t)d);
    double* q8row = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 1)
    for (int64_t rh = 0; rh < n_rows * H; ++rh) {
      int64_t r = rh / H, h = rh % H;
      int64_t i = rows ? rows[r] : r;
      size_t ke = k_kind == SRC_E4M3 ? 1 : 2, ve = v_kind == SRC_E4M3 ? 1 : 2;
      kv_src ks[2] = {
          {P ? (const char*)k_cache + (size_t)(h * cap * d) * ke : NULL, k_kind, d, P,
           k_kind == SRC_E4M3 ? k_scale[h] : 1.0f},
          {k_t + h * d, SRC_BF16, H * d, T, 1.0f}};
      kv_src vs[2] = {
          {P ? (const char*)v_cache + (size_t)(h * cap * d) * ve : NULL, v_kind, d, P,
           v_kind == SRC_E4M3 ? v_scale[h] : 1.0f},
          {v_t + h * d, SRC_BF16, H * d, T, 1.0f}};
      for (int64_t c = 0; c < d; ++c) qrow[c] = bca_oracle_bf16_to_f64(q_t[(i * H + h) * d + c]);
      if (q_codes) {
        kv_src qs = {q_codes + (size_t)(h * T * d), SRC_E4M3, d, T, q_scale[h]};
        for (int64_t c = 0; c < d; ++c) q8row[c] = src_elem(&qs, i, c);
      }
      /* source 0 = the cached keys, source 1 = the target's own keys */
      const double* qsrc[2] = {q_codes ? q8row : qrow, qrow};
      attend_row(qsrc, d, ks, vs, 2, scale, scores, out + (r * H + h) * d);
    }
    free(scores);
    free(qrow);
    free(q8row);
  }
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Q/K RMS norm and rotary embedding                                         */
/* ------------------------------------------------------------------------ */
/* "SGLang-Diffusion stöder Qwen-Image-2.1 på dag noll" (orcarouter.ai), section
 * "Siffrorna, och vad de inte säger", names a Q/K-norm change next to the DiT's
 * attention but gives no formula.  Reading taken: RMS norm over the head dimension
 * with one weight vector per tensor, then the rotary embedding of consecutive
 * channel pairs by caller-given angles (as cos/sin tables).  fp64 throughout; the
 * fp32 weights and tables are widened exactly. */

/* One vector: y[c] = x[c] / sqrt(mean_c' x[c']^2 + eps) * gamma[c]. */
static void rms_norm_vec(const double* x, int64_t d, const float* gamma, double eps, double* y) {
  double ss = 0.0;
  for (int64_t c = 0; c < d; ++c) ss += x[c] * x[c];
  double inv = 1.0 / sqrt(ss / (double)d + eps);
  for (int64_t c = 0; c < d; ++c) y[c] = x[c] * inv * (double)gamma[c];
}

/* One vector: pair (2i, 2i+1) turned by the angle whose cos/sin are cs[i], sn[i]. */
static void rope_vec(const double* y, int64_t d, const float* cs, const float* sn, double* out) {
  for (int64_t i = 0; i < d / 2; ++i) {
    double c = (double)cs[i], s = (double)sn[i];
    out[2 * i] = y[2 * i] * c - y[2 * i + 1] * s;
    out[2 * i + 1] = y[2 * i] * s + y[2 * i + 1] * c;
  }
}

/* y[v, c] = x[v, c] / sqrt(mean_c' x[v, c']^2 + eps) * gamma[c], for n_vec vectors
 * of d bf16 values each. */
void bca_oracle_rms_norm(const uint16_t* x, int64_t n_vec, int64_t d, const float* gamma,
                         double eps, double* y) {
  double* xv = (double*)malloc(sizeof(double) * (size_t)d);
  for (int64_t v = 0; v < n_vec; ++v) {
    for (int64_t c = 0; c < d; ++c) xv[c] = bca_oracle_bf16_to_f64(x[v * d + c]);
    rms_norm_vec(xv, d, gamma, eps, y + v * d);
  }
  free(xv);
}

/* Rotate every pair (2i, 2i+1) of y [rows, H, d] by the angle of row t and pair i:
 * out_{2i} = y_{2i} cos - y_{2i+1} sin, out_{2i+1} = y_{2i} sin + y_{2i+1} cos,
 * with cos/sin [rows, d/2].  out may not alias y. */
void bca_oracle_rope(const double* y, int64_t rows, int64_t H, int64_t d, const float* cos_t,
                     const float* sin_t, double* out) {
  for (int64_t t = 0; t < rows; ++t)
    for (int64_t h = 0; h < H; ++h)
      rope_vec(y + (t * H + h) * d, d, cos_t + t * (d / 2), sin_t + t * (d / 2),
               out + (t * H + h) * d);
}

/* ------------------------------------------------------------------------ */
/* Q/K/V projection with the Q/K norm and rotary embedding                   */
/* ------------------------------------------------------------------------ */
/* The same page and section place the Q/K-norm change between the projection of
 * the target rows and the attention.  Reading taken: one linear projection (no
 * bias) of the rows x [T, D] by w [3*H*d, D] (the torch Linear layout: output
 * features Q heads 0..H-1, then K heads, then V heads, d = head_dim each), then the
 * RMS norm + rotary embedding above on every Q and K head vector; V as projected.
 *   y[t, n]    = sum_c x[t, c] * w[n, c]                       (fp64)
 *   q[t, h, :] = rope(rms_norm(y[t, h*d .. h*d+d-1], gamma_q), cos[t], sin[t])
 *   k[t, h, :] = rope(rms_norm(y[t, (H+h)*d ..], gamma_k), cos[t], sin[t])
 *   v[t, h, :] = y[t, (2H+h)*d ..]
 * rows: the rows to compute (NULL: all T); outputs [n_rows, H, d] fp64. */
int bca_oracle_qkv_project(const uint16_t* x, int64_t T, int64_t D, const uint16_t* w, int64_t H,
                           int64_t d, const float* gamma_q, const float* gamma_k,
                           const float* cos_t, const float* sin_t, double eps,
                           const int64_t* rows, int64_t n_rows, double* q, double* k, double* v,
                           int nthreads) {
  if (T < 1 || D < 1 || H < 1 || d < 2 || (d & 1)) return -1;
  if (!rows) n_rows = T;
  for (int64_t r = 0; r < n_rows; ++r)
    if (rows && (rows[r] < 0 || rows[r] >= T)) return -1;
  const int64_t N = 3 * H * d;
  set_threads(nthreads);
#pragma omp parallel
  {
    double* xr = (double*)malloc(sizeof(double) * (size_t)D);
    double* y = (double*)malloc(sizeof(double) * (size_t)N);
    double* nrm = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
      int64_t t = rows ? rows[r] : r;
      for (int64_t c = 0; c < D; ++c) xr[c] = bca_oracle_bf16_to_f64(x[t * D + c]);
      for (int64_t n = 0; n < N; ++n) {
        double acc = 0.0;
        for (int64_t c = 0; c < D; ++c) acc += xr[c] * bca_oracle_bf16_to_f64(w[n * D + c]);
        y[n] = acc;
      }
      const float* cs = cos_t + t * (d / 2);
      const float* sn = sin_t + t * (d / 2);
      for (int64_t h = 0; h < H; ++h) {
        rms_norm_vec(y + h * d, d, gamma_q, eps, nrm);
        rope_vec(nrm, d, cs, sn, q + (r * H + h) * d);
        rms_norm_vec(y + (H + h) * d, d, gamma_k, eps, nrm);
        rope_vec(nrm, d, cs, sn, k + (r * H + h) * d);
        for (int64_t c = 0; c < d; ++c) v[(r * H + h) * d + c] = y[(2 * H + h) * d + c];
      }
    }
    free(xr);
    free(y);
    free(nrm);
  }
  return 0;
}
