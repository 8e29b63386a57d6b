// NVFP4 quantiser for the W4A16 head's weights: an absmax pass, then an encode pass, the two
// kernels that lm_head_nvfp4_rows.rs / mtp_head/new_bf16_moe.rs hand to `quantize_to_nvfp4`.
// The pages print no rules; this library's reading takes every decision as one IEEE binary32
// operation, so a CPU re-implementation can match it bit for bit:
//   amax = max |w|;  g = amax / 2688 (= 6 * 448), or 1 when amax = 0
//   per 16-element block:  s = RN_e4m3(bmax / (6 * g)), saturating at 448
//   per element:           q = RN_e2m1(w / d), d = e4m3(s) * g, saturating at 6, and 0 where
//                          d is 0; the sign is kept only on a non-zero magnitude
// RN is round to nearest, ties to the even code (the conversions' .rn mode).
//
// Both passes stream W once. The absmax pass is HBM-bound; the encode pass is held by its
// instruction issue (about 8 instructions an element), so its per-block work is trimmed: the
// block maximum on the bf16x2 max, the divisor and reciprocals of every scale code from a
// per-CTA table, four code bytes packed by one vector move. Its divisions are IEEE (div.rn).
#pragma once

#include "lmhead_common.cuh"

namespace lmh {

constexpr int kQuantThreads = 256;
constexpr int kQuantMaxPartials = 1024;  // absmax partials: one 32-bit word per CTA of pass 1

// Largest |bf16| of a 16-byte chunk as its magnitude bits (0x0000..0x7F80 for finite values and
// infinity, ordered like the values).
__device__ __forceinline__ uint32_t chunk_absmax_bits(const uint4& c) {
  const uint32_t m = __vmaxu2(__vmaxu2(c.x & 0x7FFF7FFFu, c.y & 0x7FFF7FFFu),
                              __vmaxu2(c.z & 0x7FFF7FFFu, c.w & 0x7FFF7FFFu));
  return max(m & 0xFFFFu, m >> 16);
}

// Largest |bf16| of a 32-byte block of finite values as magnitude bits, on the bf16x2 max
// (each lane's result has magnitude max(|a|, |b|); the sign bits are cleared at the end).
__device__ __forceinline__ uint32_t block_absmax_bits(const uint4& c0, const uint4& c1) {
  uint32_t a, b, c, d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(a) : "r"(c0.x), "r"(c0.y));
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(b) : "r"(c0.z), "r"(c0.w));
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(c) : "r"(c1.x), "r"(c1.y));
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(c1.z), "r"(c1.w));
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(a) : "r"(a), "r"(b));
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(c) : "r"(c), "r"(d));
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(a) : "r"(a), "r"(c));
  const uint32_t m = a & 0x7FFF7FFFu;
  return max(m & 0xFFFFu, m >> 16);
}

__device__ __forceinline__ uint32_t block_max_u32(uint32_t v, uint32_t* red) {
  v = __reduce_max_sync(0xffffffffu, v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < (int)(blockDim.x >> 5) ? red[lane] : 0u;
    v = __reduce_max_sync(0xffffffffu, v);
    if (lane == 0) red[0] = v;
  }
  __syncthreads();
  const uint32_t r = red[0];
  __syncthreads();
  return r;
}

// Pass 1: partial[blockIdx.x] = largest |w| (magnitude bits) over this CTA's grid-stride share.
__global__ void __launch_bounds__(kQuantThreads)
    nvfp4_absmax_kernel(const uint4* __restrict__ w, int64_t n_chunks, uint32_t* partial) {
  __shared__ uint32_t red[32];
  uint32_t m = 0;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  // Eight independent 16-byte loads in flight per thread (128 B; the grid's 6 CTAs per SM are
  // all resident at 32 registers a thread), to cover the DRAM latency at the HBM rate.
  for (; i + 7 * stride < n_chunks; i += 8 * stride) {
    uint4 c[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) c[k] = __ldcs(w + i + k * stride);
#pragma unroll
    for (int k = 0; k < 8; ++k) m = max(m, chunk_absmax_bits(c[k]));
  }
  for (; i < n_chunks; i += stride) m = max(m, chunk_absmax_bits(__ldcs(w + i)));
  m = block_max_u32(m, red);
  if (threadIdx.x == 0) partial[blockIdx.x] = m;
}

// Nearest E4M3 code of t >= 0 (saturating at 448): the conversion packs two values; both lanes
// get t, so either byte is the answer.
__device__ __forceinline__ uint32_t rn_e4m3_code(float t) {
  uint16_t two;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(two) : "f"(t));
  return two & 0xFFu;
}

// Exact value of an E4M3 code (through the e4m3 -> f16 conversion, which is exact).
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  uint32_t h2;
  const uint16_t both = (uint16_t)(code | (code << 8));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(both));
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// E2M1 codes of two values (saturating at +-6, round to nearest, ties to the even code) as one
// byte: lo in the low nibble, hi in the high one (the conversion puts its first operand in the
// upper half). A zero magnitude may carry a sign bit here; drop_negative_zeros clears it.
__device__ __forceinline__ uint32_t e2m1_pair_code(float lo, float hi) {
  uint16_t two;
  asm("{\n\t.reg .b8 q;\n\tcvt.rn.satfinite.e2m1x2.f32 q, %1, %2;\n\tcvt.u16.u8 %0, q;\n\t}"
      : "=h"(two)
      : "f"(hi), "f"(lo));
  return two & 0xFFu;
}

// E2M1 codes of four pairs (x0, x1) .. (x6, x7) as one word: pair j in byte j, its first value in
// the low nibble (the codes of e2m1_pair_code, packed by one vector move).
__device__ __forceinline__ uint32_t e2m1_quad(float x0, float x1, float x2, float x3, float x4,
                                              float x5, float x6, float x7) {
  uint32_t r;
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
      "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
      : "=r"(r)
      : "f"(x0), "f"(x1), "f"(x2), "f"(x3), "f"(x4), "f"(x5), "f"(x6), "f"(x7));
  return r;
}

// Eight E2M1 codes in a word: clear the sign bit of every nibble whose magnitude is zero. Adding
// 7 to a 3-bit magnitude carries into the nibble's bit 3 exactly when the magnitude is non-zero,
// and never out of the nibble.
__device__ __forceinline__ uint32_t drop_negative_zeros(uint32_t q) {
  const uint32_t mag = q & 0x77777777u;
  return mag | (q & ((mag + 0x77777777u) & 0x88888888u));
}

// Relative guard band of the quotient shortcut in encode_block.
constexpr float kQuotientBand = 0x1p-16f;

// One 16-element block: 32 bytes of W (c0, c1) to 8 bytes of codes and one scale byte.
//
// Each code is that of the correctly rounded quotient x = fl(w / d). Instead of dividing every
// element, the block takes one correctly rounded reciprocal r = fl(1 / d) and converts the two
// products w * fl(r (1 - b)) and w * fl(r (1 + b)), b = 2^-16. Their magnitudes bracket |x|
// strictly: each is within 3 * 2^-24 relative of w / d times (1 -+ b), and x within 2^-24 of it
// wherever a code boundary can lie (|x| >= 1/4, all normal numbers). The code is monotone in the
// magnitude, so when both products give the same code, x has that code as well. Only a pair with
// a quotient within about 2^-16 of a boundary (0.25, 0.75, ..., 5) is divided exactly. d outside
// [2^-120, 2^120], where r could leave the normal range, is always divided exactly.
//
// The divisor d = fl(e4m3(s) g) and the two bracketing reciprocals depend only on the scale
// code s, so each CTA computes them once for all 128 codes (make_scale_entry) into a shared
// table; the conversion saturates at 448 (code 0x7E), so code 0x7F (NaN) is never looked up.
struct ScaleEntry {
  float d, r_lo, r_hi;
  uint32_t shortcut;  // 1 when d is in [2^-120, 2^120]
};

__device__ __forceinline__ ScaleEntry make_scale_entry(uint32_t s, float g) {
  ScaleEntry e;
  e.d = __fmul_rn(e4m3_value(s), g);
  e.shortcut = (e.d >= 0x1p-120f && e.d <= 0x1p120f) ? 1u : 0u;
  const float r = __frcp_rn(e.d);
  e.r_lo = __fmul_rn(r, 1.0f - kQuotientBand);
  e.r_hi = __fmul_rn(r, 1.0f + kQuotientBand);
  return e;
}

__device__ __forceinline__ void encode_block(const uint4& c0, const uint4& c1, float six_g,
                                             const float4* scale_table, uint2* packed,
                                             uint8_t* scale) {
  const float bmax = __uint_as_float(block_absmax_bits(c0, c1) << 16);
  const uint32_t s = rn_e4m3_code(__fdiv_rn(bmax, six_g));
  const float4 te = scale_table[s & 0x7Fu];  // s <= 0x7E: the conversion saturates at 448
  const float d = te.x, r_lo = te.y, r_hi = te.z;
  const bool shortcut = __float_as_uint(te.w) != 0u;
  const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  uint32_t lo[2] = {0u, 0u}, hi[2] = {0u, 0u};
  float pl[16], ph[16];  // the products by r_lo and by r_hi, in element order
#pragma unroll
  for (int i = 0; i < 8; ++i) {  // word i holds elements 2i (low half) and 2i + 1
    const float w0 = __uint_as_float(words[i] << 16);
    const float w1 = __uint_as_float(words[i] & 0xFFFF0000u);
    pl[2 * i] = __fmul_rn(w0, r_lo);
    pl[2 * i + 1] = __fmul_rn(w1, r_lo);
    ph[2 * i] = __fmul_rn(w0, r_hi);
    ph[2 * i + 1] = __fmul_rn(w1, r_hi);
  }
  lo[0] = e2m1_quad(pl[0], pl[1], pl[2], pl[3], pl[4], pl[5], pl[6], pl[7]);
  lo[1] = e2m1_quad(pl[8], pl[9], pl[10], pl[11], pl[12], pl[13], pl[14], pl[15]);
  hi[0] = e2m1_quad(ph[0], ph[1], ph[2], ph[3], ph[4], ph[5], ph[6], ph[7]);
  hi[1] = e2m1_quad(ph[8], ph[9], ph[10], ph[11], ph[12], ph[13], ph[14], ph[15]);
  if (!shortcut || lo[0] != hi[0] || lo[1] != hi[1]) {
    // Some quotient of the block sits near a code boundary (or r is unusable): divide those
    // pairs exactly.
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int sh = 8 * (i & 3);
      const uint32_t a = (lo[i >> 2] >> sh) & 0xFFu;
      if (shortcut && a == ((hi[i >> 2] >> sh) & 0xFFu)) continue;
      const float w0 = __uint_as_float(words[i] << 16);
      const float w1 = __uint_as_float(words[i] & 0xFFFF0000u);
      const uint32_t q = e2m1_pair_code(__fdiv_rn(w0, d), __fdiv_rn(w1, d));
      lo[i >> 2] = (lo[i >> 2] & ~(0xFFu << sh)) | (q << sh);
    }
  }
  // d = 0 when the block's scale code is 0 (a block far below amax), or when e4m3(s) * g
  // underflows (g subnormal): every code is 0.
  const bool zero = !(d > 0.0f);
  *packed = make_uint2(zero ? 0u : drop_negative_zeros(lo[0]),
                       zero ? 0u : drop_negative_zeros(lo[1]));
  *scale = (uint8_t)s;
}

// Pass 2: every CTA reduces the partials to amax (the same value everywhere), then each thread
// encodes 16-element blocks: 32 bytes of W in, 8 bytes of codes and one scale byte out.
// Four CTAs per SM (at most 64 registers a thread): two full waves of the 8-per-SM grid.
__global__ void __launch_bounds__(kQuantThreads, 4)
    nvfp4_encode_kernel(const uint4* __restrict__ w, int64_t n_blocks,
                        const uint32_t* __restrict__ partial, int n_partial, uint2* packed,
                        uint8_t* scales, float* g_out) {
  __shared__ uint32_t red[32];
  __shared__ float4 scale_table[128];
  uint32_t m = 0;
  for (int i = threadIdx.x; i < n_partial; i += blockDim.x) m = max(m, partial[i]);
  m = block_max_u32(m, red);
  const float amax = __uint_as_float(m << 16);
  const float g = amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
  const float six_g = __fmul_rn(6.0f, g);
  if (blockIdx.x == 0 && threadIdx.x == 0) *g_out = g;
  static_assert(kQuantThreads >= 128, "one thread per scale code");
  if (threadIdx.x < 128) {
    const ScaleEntry e = make_scale_entry(threadIdx.x, g);
    scale_table[threadIdx.x] = make_float4(e.d, e.r_lo, e.r_hi, __uint_as_float(e.shortcut));
  }
  __syncthreads();
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  // Two blocks per iteration, their four loads issued together.
  for (; b + stride < n_blocks; b += 2 * stride) {
    const uint4 a0 = __ldcs(w + 2 * b), a1 = __ldcs(w + 2 * b + 1);
    const uint4 b0 = __ldcs(w + 2 * (b + stride)), b1 = __ldcs(w + 2 * (b + stride) + 1);
    encode_block(a0, a1, six_g, scale_table, packed + b, scales + b);
    encode_block(b0, b1, six_g, scale_table, packed + b + stride, scales + b + stride);
  }
  for (; b < n_blocks; b += stride) {
    const uint4 c0 = __ldcs(w + 2 * b);
    const uint4 c1 = __ldcs(w + 2 * b + 1);
    encode_block(c0, c1, six_g, scale_table, packed + b, scales + b);
  }
}

}  // namespace lmh
