/*
 * CPU oracle for the LM-head logits projection -- TEST INFRASTRUCTURE ONLY (see
 * lmhead_oracle.c for the definition it computes and the pages it follows). Nothing in the
 * CUDA library includes this header.
 */
#ifndef LMHEAD_ORACLE_H
#define LMHEAD_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exact value of one bf16 / IEEE fp16 / E2M1 (low 4 bits of code) / E4M3fn encoding. */
double oracle_bf16_value(uint16_t bits);
double oracle_f16_value(uint16_t bits);
double oracle_e2m1_value(uint8_t code);
double oracle_e4m3_value(uint8_t code);

/* One IEEE round-to-nearest-even from double. */
float oracle_round_f32(double x);
uint16_t oracle_round_bf16(double x);

/* Decoded NVFP4 weight W[v, k] = e2m1 * e4m3 * g, exact in double. */
double oracle_nvfp4_weight(const uint8_t* packed, const uint8_t* scales, float g, int64_t H,
                           int64_t v, int64_t k);

/*
 * logits[r, v] = RN_fp32(alpha * sum_k hidden[r, k] * W[v, k]), all host arrays, row-major:
 * hidden [rows, H] bf16 bits, W [V, H] bf16 bits, logits [rows, V] fp32. If abs_sum is not
 * NULL it receives |alpha| * sum_k |hidden[r, k] * W[v, k]| (the error-bound scale).
 * Returns 0 on success, 1 on bad arguments, 2 when host memory runs out.
 */
int oracle_logits_bf16_f32(const uint16_t* hidden, int64_t rows, int64_t H, const uint16_t* W,
                           int64_t V, float alpha, float* logits, double* abs_sum, int threads);

/*
 * The same with the input type chosen by dtype (0 = bf16, 1 = IEEE fp16; hidden, W and bias all
 * of it) and an optional bias [V] (NULL = none):
 *   logits[r, v] = RN_fp32(alpha * (sum_k hidden[r, k] * W[v, k] + bias[v])),
 * abs_sum = |alpha| * (sum_k |hidden[r, k] * W[v, k]| + |bias[v]|).
 */
int oracle_logits_f32(const uint16_t* hidden, int dtype, int64_t rows, int64_t H,
                      const uint16_t* W, int64_t V, float alpha, const uint16_t* bias,
                      float* logits, double* abs_sum, int threads);

/*
 * logits[r, v] = RN_bf16(alpha * sum_k hidden[r, k] * e2m1(code[v, k]) * e4m3(scale[v, k/16]) * g)
 * packed [V, H/2] (element 2j = low nibble of byte j), scales [V, H/16] E4M3 bytes,
 * logits [rows, V] bf16 bits. H must be a multiple of 16.
 */
int oracle_logits_w4a16_nvfp4(const uint16_t* hidden, int64_t rows, int64_t H,
                              const uint8_t* packed, const uint8_t* scales, float g, int64_t V,
                              float alpha, uint16_t* logits, double* abs_sum, int threads);

/*
 * Log-probabilities of given tokens: with z the fp32 logits of oracle_logits_f32 (same arguments),
 * lse[r] = log sum_v exp(z[r, v]) and logprobs[r] = z[r, targets[r]] - lse[r], computed in double
 * from the fp32 z and rounded once; NaN for a target outside [0, V). lse may be NULL.
 */
int oracle_logprobs_f32(const uint16_t* hidden, int dtype, int64_t rows, int64_t H,
                        const uint16_t* W, int64_t V, float alpha, const uint16_t* bias,
                        const int32_t* targets, float* logprobs, float* lse, int threads);

/*
 * Vocab-parallel log-probabilities, the same quantities split over slices of W's rows. For the
 * slice W_shard = W[v_begin, v_begin + V_shard), with z its fp32 logits (oracle_logits_f32):
 *   stats[3r] = max_v z[r, v],  stats[3r+1] = sum_v exp(z[r, v] - stats[3r])  (double),
 *   stats[3r+2] = z[r, targets[r]] when the slice holds the target (global id), else NaN.
 * oracle_logprob_merge_shards takes [shards][rows][3] such stats and returns, rounded once,
 *   lse[r] = M + log(sum_g s_g exp(m_g - M)),  M = max_g m_g,   logprobs[r] = z_t - lse[r]
 * with z_t from the shard that holds the target (NaN when none does). lse may be NULL.
 */
int oracle_logprob_shard_stats(const uint16_t* hidden, int dtype, int64_t rows, int64_t H,
                               const uint16_t* W_shard, int64_t V_shard, int64_t v_begin,
                               float alpha, const uint16_t* bias_shard, const int32_t* targets,
                               double* stats, int threads);
int oracle_logprob_merge_shards(const double* stats, int64_t shards, int64_t rows,
                                float* logprobs, float* lse);

/*
 * NVFP4 quantiser (this library's reading; every decision step one IEEE binary32 operation):
 * amax = max|w|, g = amax / 2688 (1 when amax = 0); per 16-element block s = RN_e4m3(bmax / (6g))
 * saturating; per element q = RN_e2m1(w / (e4m3(s) * g)) saturating, sign only on non-zero
 * magnitudes. w is bf16 [V, H] bits, H % 16 == 0; outputs packed [V, H/2], scales [V, H/16], g.
 */
int oracle_nvfp4_quantize(const uint16_t* w, int64_t V, int64_t H, uint8_t* packed,
                          uint8_t* scales, float* g_out);
/* Nearest E4M3 code (non-negative, saturating at 448) / E2M1 code, ties to the even code. */
uint8_t oracle_rn_e4m3(float t);
uint8_t oracle_rn_e2m1(float x);

#ifdef __cplusplus
}
#endif

#endif
