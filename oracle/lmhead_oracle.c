/*
 * CPU oracle for the LM-head logits projection -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg may load or call
 * this file. The product path (the CUDA library) never does, and the two share no code.
 *
 * What is computed, written out as the plain definition, in double precision:
 *
 *   S[r, v]  = sum over k = 0 .. H-1, ascending, of dec(hidden[r, k]) * dec(W[v, k])
 *   fp32 head:   logits[r, v] = RN_fp32( alpha * (S[r, v] + dec(bias[v])) )   (bias optional)
 *   NVFP4 head:  W[v, k] = e2m1(code[v, k]) * e4m3(scale[v, k / 16]) * g
 *                logits[r, v] = RN_bf16( alpha * S[r, v] )          (one rounding, from double)
 *
 * Sources (the pages this library follows):
 *  - "[Model] Honor fp32 head_dtype in Inkling muP logits (target + MTP draft)", sections
 *    "Purpose" and "muP is folded into the fp32 GEMM (not a bypass)": out = alpha * (hidden @ w.t())
 *    with alpha = 1/mup, bf16 inputs accumulated into fp32 without an fp32 weight copy, fp32 output.
 *  - "FP32 LM head skip FP32 cast" (SGLang PR #32370 summary), sections on function/motivation and
 *    the implementation breakdown: torch.mm(hidden, W.T, out_dtype=float32), a bf16 x bf16 -> fp32
 *    product with an fp32 accumulator; the path's predicate admits float16 as well as bfloat16
 *    hidden states, of the same dtype as the weight.
 *  - The first page's "Purpose" lists the embedding bias among the cases the fused multiply does
 *    not cover; there the head projects with its bias and then multiplies every logit by
 *    1/mup, read here as alpha * (hidden @ w.t() + bias), the bias in the weight's dtype.
 *  - lm_head_nvfp4_rows.rs, module doc and lm_head_nvfp4_rows_run: the NVFP4 head kept at the
 *    W4A16 precision its checkpoint declares (16-bit activations, never cast to E4M3), bf16
 *    logits[rows, vocab], row-major layouts (row offsets done*h*2 and done*v*2 bytes), values
 *    independent of the row count.
 *
 * Readings where the pages are silent (the NVFP4 layout is not printed anywhere):
 *  - bf16 decode: the 16 bits are the top half of an IEEE binary32.
 *  - fp16 decode: IEEE binary16 (1 sign bit, 5 exponent bits with bias 15, 10 fraction bits;
 *    exponent 0 is subnormal, fraction * 2^-24; exponent 31 is infinity or NaN).
 *  - E2M1: bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa; exponent 0 is subnormal
 *    (value 0.5 * m). Element 2j of a row is the LOW nibble of byte j, element 2j+1 the high one.
 *  - E4M3 (the "fn" variant): bit 7 sign, bits 6..3 exponent (bias 7), bits 2..0 mantissa, no
 *    infinities, 0x7F / 0xFF are NaN, exponent 0 is subnormal (m * 2^-9).
 *  - Block scales are a plain row-major [V, H/16] byte array; scale j of row v covers k in
 *    [16j, 16j+16). g is the per-tensor decode multiplier (w = q * s * g).
 *  - Rounding is IEEE round-to-nearest-even, done once from double.
 *
 * Log-probabilities of given tokens (oracle_logprobs_f32). The first page's "Purpose" wants fp32
 * logits for RL training-inference consistency and for speculative decoding, where the logits
 * drive rejection sampling; what those consume is the log-softmax. Reading: with z[r, v] the fp32
 * logits above (bias and alpha applied, rounded to fp32),
 *   lse[r] = log sum_v exp(z[r, v]),   logprob[r] = z[r, target[r]] - lse[r]
 * computed in double from the fp32 z (max-shifted), each rounded once to fp32; a target outside
 * [0, V) gives NaN.
 *
 * NVFP4 quantiser (oracle_nvfp4_quantize). lm_head_nvfp4_rows.rs and mtp_head/new_bf16_moe.rs
 * name it (`quantize_to_nvfp4`, handed an absmax kernel and an encode kernel) but print no
 * rules. Reading, with every step one IEEE binary32 operation so that
 * a GPU implementation can take the same decisions bit for bit:
 *   amax = max |w| over the tensor;  g = amax / 2688 (= 6 * 448), or 1 when amax = 0
 *   per 16-element block: t = bmax / (6 * g);  s = RN_e4m3(t), saturating at 448
 *   per element: d = e4m3(s) * g;  x = w / d (0 when d = 0);  q = RN_e2m1(x), saturating at 6,
 *   sign kept only when the magnitude is not zero. RN = nearest, ties to the even code.
 *
 * Why double is exact enough: a bf16 x bf16 product has at most 16 significant bits and an
 * e2m1 * e4m3 * g * bf16 product at most 2+4+24+8 = 38, so every product is exact in double;
 * the double sum's error is below H * 2^-53 * sum|p|, far inside any fp32 tolerance.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "lmhead_oracle.h"

/* ---------------------------------------------------------------- element decoders */

double oracle_bf16_value(uint16_t bits) {
  /* bf16 is the upper half of a binary32: widen, reinterpret, convert (all exact). */
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

double oracle_f16_value(uint16_t bits) {
  int sign = (bits >> 15) & 1;
  int expo = (bits >> 10) & 31;
  int frac = bits & 1023;
  double mag;
  if (expo == 31) {
    mag = frac ? NAN : INFINITY;
  } else if (expo == 0) {
    mag = ldexp((double)frac, -24); /* subnormal: (frac / 1024) * 2^-14 */
  } else {
    mag = ldexp(1.0 + (double)frac / 1024.0, expo - 15);
  }
  return sign ? -mag : mag;
}

static double decode16(uint16_t bits, int dtype) {
  return dtype == 1 ? oracle_f16_value(bits) : oracle_bf16_value(bits);
}

double oracle_e2m1_value(uint8_t code) {
  int sign = (code >> 3) & 1;
  int expo = (code >> 1) & 3;
  int mant = code & 1;
  double mag;
  if (expo == 0) {
    mag = 0.5 * (double)mant; /* subnormal: 0 or 0.5 */
  } else {
    mag = ldexp(1.0 + 0.5 * (double)mant, expo - 1);
  }
  return sign ? -mag : mag;
}

double oracle_e4m3_value(uint8_t code) {
  int sign = (code >> 7) & 1;
  int expo = (code >> 3) & 15;
  int mant = code & 7;
  double mag;
  if (expo == 15 && mant == 7) return NAN; /* the only NaN encodings: 0x7F, 0xFF */
  if (expo == 0) {
    mag = ldexp((double)mant, -9); /* subnormal: (m/8) * 2^-6 */
  } else {
    mag = ldexp(1.0 + (double)mant / 8.0, expo - 7);
  }
  return sign ? -mag : mag;
}

/* ---------------------------------------------------------------- one rounding from double */

float oracle_round_f32(double x) {
  /* C's double -> float conversion is IEEE round-to-nearest-even in the default mode. */
  return (float)x;
}

uint16_t oracle_round_bf16(double x) {
  /* Direct double -> bf16 round-to-nearest-even (never via float, which would round twice). */
  uint16_t sign = signbit(x) ? 0x8000u : 0u;
  double a = fabs(x);
  if (isnan(x)) return (uint16_t)(sign | 0x7FC0u);
  /* Largest finite bf16 is (2 - 2^-7) * 2^127; the halfway point to 2^128 and beyond rounds
   * to infinity (the tie goes to the even neighbour, which is 2^128). */
  if (a >= ldexp(2.0 - ldexp(1.0, -8), 127)) return (uint16_t)(sign | 0x7F80u);
  if (a == 0.0) return sign;
  int e2;
  frexp(a, &e2); /* a in [2^(e2-1), 2^e2) */
  int e = e2 - 1;          /* a in [2^e, 2^(e+1)) */
  if (e < -126) e = -126;  /* below the normal range the spacing stays 2^-133 */
  double ulp = ldexp(1.0, e - 7);
  double q = a / ulp;      /* exact: division by a power of two */
  double n = nearbyint(q); /* ties to even in the default rounding mode */
  double r = n * ulp;      /* a bf16 value, exactly representable as float */
  float rf = (float)r;
  uint32_t u;
  memcpy(&u, &rf, sizeof u);
  return (uint16_t)(sign | (uint16_t)(u >> 16));
}

/* ---------------------------------------------------------------- the head, fp32 output */

int oracle_logits_f32(const uint16_t* hidden, int dtype, int64_t rows, int64_t H,
                      const uint16_t* W, int64_t V, float alpha, const uint16_t* bias,
                      float* logits, double* abs_sum, int threads) {
  if (rows < 0 || H <= 0 || V <= 0 || (dtype != 0 && dtype != 1)) return 1;
  if (rows == 0) return 0;
  if (!hidden || !W || !logits) return 1;
  const double a = (double)alpha;
  /* hidden decoded once: hd[r * H + k] = dec(hidden[r, k]) */
  double* hd = (double*)malloc((size_t)rows * (size_t)H * sizeof(double));
  if (!hd) return 2;
  for (int64_t i = 0; i < rows * H; ++i) hd[i] = decode16(hidden[i], dtype);
  int failed = 0;
#pragma omp parallel num_threads(threads > 0 ? threads : 1)
  {
    double* wv = (double*)malloc((size_t)H * sizeof(double));
    if (!wv) {
#pragma omp atomic write
      failed = 1;
    }
#pragma omp for schedule(static)
    for (int64_t v = 0; v < V; ++v) {
      if (!wv) continue;
      for (int64_t k = 0; k < H; ++k) wv[k] = decode16(W[v * H + k], dtype);
      const double b = bias ? decode16(bias[v], dtype) : 0.0;
      for (int64_t r = 0; r < rows; ++r) {
        const double* h = hd + r * H;
        double s = 0.0, sa = 0.0;
        for (int64_t k = 0; k < H; ++k) {
          double p = h[k] * wv[k];
          s += p;
          sa += fabs(p);
        }
        logits[r * V + v] = oracle_round_f32(a * (s + b));
        if (abs_sum) abs_sum[r * V + v] = fabs(a) * (sa + fabs(b));
      }
    }
    free(wv);
  }
  free(hd);
  return failed ? 2 : 0;
}

int oracle_logits_bf16_f32(const uint16_t* hidden, int64_t rows, int64_t H, const uint16_t* W,
                           int64_t V, float alpha, float* logits, double* abs_sum, int threads) {
  return oracle_logits_f32(hidden, 0, rows, H, W, V, alpha, NULL, logits, abs_sum, threads);
}

/* ---------------------------------------------------------------- log-probabilities */

int oracle_logprobs_f32(const uint16_t* hidden, int dtype, int64_t rows, int64_t H,
                        const uint16_t* W, int64_t V, float alpha, const uint16_t* bias,
                        const int32_t* targets, float* logprobs, float* lse, int threads) {
  if (rows < 0 || H <= 0 || V <= 0) return 1;
  if (rows == 0) return 0;
  if (!targets || !logprobs) return 1;
  float* z = (float*)malloc((size_t)rows * (size_t)V * sizeof(float));
  if (!z) return 2;
  int rc = oracle_logits_f32(hidden, dtype, rows, H, W, V, alpha, bias, z, NULL, threads);
  if (rc != 0) {
    free(z);
    return rc;
  }
  for (int64_t r = 0; r < rows; ++r) {
    const float* zr = z + r * V;
    double m = -INFINITY;
    for (int64_t v = 0; v < V; ++v)
      if ((double)zr[v] > m) m = (double)zr[v];
    double sum = 0.0;
    for (int64_t v = 0; v < V; ++v) sum += exp((double)zr[v] - m);
    const double l = m + log(sum);
    if (lse) lse[r] = oracle_round_f32(l);
    const int32_t t = targets[r];
    logprobs[r] = (t >= 0 && t < V) ? oracle_round_f32((double)zr[t] - l) : (float)NAN;
  }
  free(z);
  return 0;
}

/* Vocab-parallel split. "FP32 LM head skip FP32 cast" (key source excerpt, _compute_lm_head)
 * takes the head as a VocabParallelEmbedding, whose rows of W are spread over GPUs; the
 * log-softmax above then needs a max and a sum over every slice. The definition is unchanged:
 * the union of the slices' terms, merged here in double. */
int oracle_logprob_shard_stats(const uint16_t* hidden, int dtype, int64_t rows, int64_t H,
                               const uint16_t* W_shard, int64_t V_shard, int64_t v_begin,
                               float alpha, const uint16_t* bias_shard, const int32_t* targets,
                               double* stats, int threads) {
  if (rows < 0 || H <= 0 || V_shard <= 0 || v_begin < 0) return 1;
  if (rows == 0) return 0;
  if (!targets || !stats) return 1;
  float* z = (float*)malloc((size_t)rows * (size_t)V_shard * sizeof(float));
  if (!z) return 2;
  int rc = oracle_logits_f32(hidden, dtype, rows, H, W_shard, V_shard, alpha, bias_shard, z, NULL,
                             threads);
  if (rc != 0) {
    free(z);
    return rc;
  }
  for (int64_t r = 0; r < rows; ++r) {
    const float* zr = z + r * V_shard;
    double m = -INFINITY;
    for (int64_t v = 0; v < V_shard; ++v)
      if ((double)zr[v] > m) m = (double)zr[v];
    double sum = 0.0;
    for (int64_t v = 0; v < V_shard; ++v) sum += exp((double)zr[v] - m);
    const int64_t t = (int64_t)targets[r] - v_begin;
    stats[3 * r] = m;
    stats[3 * r + 1] = sum;
    stats[3 * r + 2] = (t >= 0 && t < V_shard) ? (double)zr[t] : NAN;
  }
  free(z);
  return 0;
}

int oracle_logprob_merge_shards(const double* stats, int64_t shards, int64_t rows,
                                float* logprobs, float* lse) {
  if (shards <= 0 || rows < 0) return 1;
  if (rows == 0) return 0;
  if (!stats || !logprobs) return 1;
  for (int64_t r = 0; r < rows; ++r) {
    double big = -INFINITY;
    for (int64_t g = 0; g < shards; ++g) {
      const double m = stats[3 * (g * rows + r)];
      if (m > big) big = m;
    }
    double sum = 0.0, zt = NAN;
    for (int64_t g = 0; g < shards; ++g) {
      const double* q = stats + 3 * (g * rows + r);
      sum += q[1] * exp(q[0] - big);
      if (isnan(zt) && !isnan(q[2])) zt = q[2];
    }
    const double l = big + log(sum);
    if (lse) lse[r] = oracle_round_f32(l);
    logprobs[r] = isnan(zt) ? (float)NAN : oracle_round_f32(zt - l);
  }
  return 0;
}

/* ---------------------------------------------------------------- the NVFP4 quantiser */

/* Nearest entry of an ascending table of exact values (ties to the even index); x >= 0 finite
 * or +inf. Differences are taken in double: x and the table entries are floats, so a tie (x
 * exactly halfway, itself a short float) is detected exactly. */
static int nearest_even_index(float x, const double* vals, int n) {
  if (!(x > vals[0])) return 0;
  if (x >= vals[n - 1]) return n - 1;
  int hi = 1;
  while (vals[hi] < (double)x) ++hi;
  const int lo = hi - 1;
  const double dlo = (double)x - vals[lo];
  const double dhi = vals[hi] - (double)x;
  if (dhi < dlo) return hi;
  if (dlo < dhi) return lo;
  return (hi % 2 == 0) ? hi : lo;
}

uint8_t oracle_rn_e4m3(float t) {
  static double vals[127];
  static int ready = 0;
  if (!ready) {
    for (int c = 0; c < 127; ++c) vals[c] = oracle_e4m3_value((uint8_t)c);
    ready = 1;
  }
  return (uint8_t)nearest_even_index(t, vals, 127);
}

uint8_t oracle_rn_e2m1(float x) {
  static const double mags[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  const int m = nearest_even_index(fabsf(x), mags, 8);
  return (uint8_t)((x < 0.0f && m != 0) ? (m | 8) : m);
}

int oracle_nvfp4_quantize(const uint16_t* w, int64_t V, int64_t H, uint8_t* packed,
                          uint8_t* scales, float* g_out) {
  if (V <= 0 || H <= 0 || H % 16 != 0 || !w || !packed || !scales || !g_out) return 1;
  float amax = 0.0f;
  for (int64_t i = 0; i < V * H; ++i) {
    const float a = fabsf((float)oracle_bf16_value(w[i]));
    if (a > amax) amax = a;
  }
  const float g = amax > 0.0f ? amax / 2688.0f : 1.0f;
  const float six_g = 6.0f * g;
  for (int64_t v = 0; v < V; ++v) {
    for (int64_t j = 0; j < H / 16; ++j) {
      const uint16_t* blk = w + v * H + j * 16;
      float bmax = 0.0f;
      for (int i = 0; i < 16; ++i) {
        const float a = fabsf((float)oracle_bf16_value(blk[i]));
        if (a > bmax) bmax = a;
      }
      const float t = bmax / six_g;
      const uint8_t s = oracle_rn_e4m3(t);
      scales[v * (H / 16) + j] = s;
      const float d = (float)oracle_e4m3_value(s) * g;
      for (int i = 0; i < 16; i += 2) {
        const float x0 = d > 0.0f ? (float)oracle_bf16_value(blk[i]) / d : 0.0f;
        const float x1 = d > 0.0f ? (float)oracle_bf16_value(blk[i + 1]) / d : 0.0f;
        packed[v * (H / 2) + j * 8 + i / 2] =
            (uint8_t)(oracle_rn_e2m1(x0) | (oracle_rn_e2m1(x1) << 4));
      }
    }
  }
  *g_out = g;
  return 0;
}

/* ---------------------------------------------------------------- the NVFP4 W4A16 head */

double oracle_nvfp4_weight(const uint8_t* packed, const uint8_t* scales, float g, int64_t H,
                           int64_t v, int64_t k) {
  uint8_t byte = packed[v * (H / 2) + k / 2];
  uint8_t code = (k & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0x0F);
  uint8_t sc = scales[v * (H / 16) + k / 16];
  return oracle_e2m1_value(code) * oracle_e4m3_value(sc) * (double)g;
}

int oracle_logits_w4a16_nvfp4(const uint16_t* hidden, int64_t rows, int64_t H,
                              const uint8_t* packed, const uint8_t* scales, float g, int64_t V,
                              float alpha, uint16_t* logits, double* abs_sum, int threads) {
  if (rows < 0 || H <= 0 || V <= 0 || (H % 16) != 0) return 1;
  if (rows == 0) return 0;
  if (!hidden || !packed || !scales || !logits) return 1;
  const double a = (double)alpha;
  double* hd = (double*)malloc((size_t)rows * (size_t)H * sizeof(double));
  if (!hd) return 2;
  for (int64_t i = 0; i < rows * H; ++i) hd[i] = oracle_bf16_value(hidden[i]);
  int failed = 0;
#pragma omp parallel num_threads(threads > 0 ? threads : 1)
  {
    double* wv = (double*)malloc((size_t)H * sizeof(double));
    if (!wv) {
#pragma omp atomic write
      failed = 1;
    }
#pragma omp for schedule(static)
    for (int64_t v = 0; v < V; ++v) {
      if (!wv) continue;
      for (int64_t k = 0; k < H; ++k) wv[k] = oracle_nvfp4_weight(packed, scales, g, H, v, k);
      for (int64_t r = 0; r < rows; ++r) {
        const double* h = hd + r * H;
        double s = 0.0, sa = 0.0;
        for (int64_t k = 0; k < H; ++k) {
          double p = h[k] * wv[k];
          s += p;
          sa += fabs(p);
        }
        logits[r * V + v] = oracle_round_bf16(a * s);
        if (abs_sum) abs_sum[r * V + v] = fabs(a) * sa;
      }
    }
    free(wv);
  }
  free(hd);
  return failed ? 2 : 0;
}
