// W4A16 NVFP4 LM head: bf16 logits from E2M1 weights with E4M3 block scales and bf16 hidden
// rows that are never quantised (lm_head_nvfp4_rows.rs, module doc: the declared W4A16 head on
// tensor-core row tiles, bf16 logits, a row's logits independent of the row count).
//
// The weight tile is dequantised in registers and written to tensor memory, where the bf16
// tcgen05 MMA reads it as its A operand; the hidden rows (B) come from shared memory as in the
// bf16 head. Keeping A out of shared memory matters: at HBM speed the dequantised tile would
// need more shared-memory bandwidth (write it, then read it back) than an SM has.
//
// Exactness. The value placed in TMEM is w' = e2m1 * e4m3 * 2^-7: it has at most 6 significant
// bits and lies in [2^-17, 21], so it is an exact normal bf16, and every product with a bf16
// hidden value is exact in the fp32 accumulator. The accumulator therefore holds exactly 2^-7
// times what unscaled weights would give (fp32 rounding commutes with a power-of-two scale away
// from the subnormal range), and the epilogue restores it exactly:
//   logits = bf16_rn( fl32( fl32( (acc * 2^7) * g ) * alpha ) ).
//
// Every hand-off covers 4 K steps (256 elements of K). The single-thread roles (TMA producer,
// MMA issuer) share their SM sub-partitions with busy dequantiser warps, so each of their
// instructions is slow; paying one wait and one commit per K step of 64 made them the
// bottleneck.
//   stage (shared memory) 4 K steps of: the packed codes [128 rows x 128 bytes] in one box,
//         their block scales [128 rows x 16 bytes] (TMA when the scale pitch allows, 4-byte
//         async copies otherwise) and the hidden rows [BN x 64] x 4.
//   slot  (tensor memory) the dequantised weights of one stage, [128 x 256] bf16; a ring of 3
//         slots (2 when the row tile is 128), so refilling a slot never waits for the MMAs
//         that were just issued.
// Roles (192 + 128 * kDequantGroups threads):
//   warp 0      producer: fills stages.
//   warp 1      TMEM allocator and MMA issuer: per stage waits for it and for its weight slot,
//               16 x tcgen05.mma with A from TMEM, one commit frees each.
//   warps 2-5   epilogue.
//   warps 6-13  dequantisers: two groups of four warps (one per TMEM lane quarter); group g
//               takes stages g, g + 2, ...; stage i goes to slot i mod slots. Each thread
//               converts one weight row.
#pragma once

#include "lmhead_common.cuh"

namespace lmh {

// Two dequantiser groups of four warps take stages in turn. The slot ring's phase waits assume
// no more groups than TMEM weight slots (a group is never two uses of a slot ahead).
constexpr int kDequantGroups = 2;
constexpr int kDequantWarp0 = 6;
constexpr int kDequantThreads = 128;                    // threads that fill one K step
constexpr int kNvfp4Threads = 32 * kDequantWarp0 + kDequantThreads * kDequantGroups;
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxSlots = 3;         // dequantised weight slots at the top of TMEM
static_assert(kDequantGroups <= 2, "the slot ring may have only 2 slots");
constexpr int kBnMax = 128;          // row tile cap: two accumulators of <= 128 columns

constexpr int kRawK = 4;                                  // K steps per stage
constexpr uint32_t kRawCodeBytes = kBM * kRawK * kBK / 2;  // 16 KB
constexpr uint32_t kRawScaleBytes = kBM * kRawK * 4;       // 2 KB
constexpr uint32_t kSlotCols = kRawK * kBK / 2;            // TMEM columns of one weight slot

struct Nvfp4HeadParams {
  int64_t rows, H, V;
  uint16_t* out;          // bf16 logits
  const uint8_t* scales;  // [V, H/16] E4M3
  float alpha;
  float gscale;
  int32_t bn;
  int32_t hid_rows;       // rows of hidden one TMA box brings (<= bn; MMA columns past it unused)
  TileSched sched;
  int32_t num_kb;         // K steps of 64 per tile (H / 64)
  int32_t stages;
  int32_t slots;          // TMEM weight slots: 3 when 2 * bn + 3 * 128 <= 512, else 2
  int32_t scale_tma;      // 1: block scales by TMA (H % 256 == 0), 0: 4-byte async copies
  WaitCfg wait;
};

// Shared-memory stage (4 K steps): [hidden: 4 sub-tiles of BN x 64 bf16, 128-byte swizzle]
// [codes: 128 rows x 128 bytes, 128-byte swizzle][scales: 128 rows x 16 bytes]
__host__ __device__ constexpr uint32_t nvfp4_hid_sub_bytes(int bn) {
  return (uint32_t)(bn * kBK * 2);
}
__host__ __device__ constexpr uint32_t nvfp4_stage_bytes(int bn) {
  return (uint32_t)kRawK * nvfp4_hid_sub_bytes(bn) + kRawCodeBytes + kRawScaleBytes;
}

__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}

__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, bf16 inputs, fp32 accumulate. Called by a whole converged
// warp; one elected lane issues it, so the operands stay warp-uniform.
__device__ __forceinline__ void mma_bf16_ts_elect(uint32_t d_tmem, uint32_t a_tmem,
                                                  uint64_t b_desc, uint32_t idesc,
                                                  uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// One K step of 64 with A from TMEM: four K = 16 MMAs, A advancing 8 columns and B 32 bytes per
// MMA; only the first may start a fresh accumulator. One elected lane of a converged warp
// issues them.
__device__ __forceinline__ void mma4_bf16_ts_elect(uint32_t d_tmem, uint32_t a_tmem,
                                                   uint64_t b_desc, uint32_t idesc,
                                                   uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t.reg .b32 a1, a2, a3;\n\t.reg .b64 b1, b2, b3;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "add.s32 a1, %1, 8;\n\tadd.s32 a2, %1, 16;\n\tadd.s32 a3, %1, 24;\n\t"
      "add.s64 b1, %2, 2;\n\tadd.s64 b2, %2, 4;\n\tadd.s64 b3, %2, 6;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], b1, %3, 1;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a2], b2, %3, 1;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a3], b3, %3, 1;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// A whole stage (4 K steps of 64 = 16 MMAs) from one asm block: A advances 8 TMEM columns per
// MMA, B 32 bytes per MMA within a sub-tile and `b_sub` bytes (>> 4 in `b_step`) per K step.
// Only the very first MMA may start a fresh accumulator.
__device__ __forceinline__ void mma16_bf16_ts_elect(uint32_t d_tmem, uint32_t a_tmem,
                                                    uint64_t b_desc, uint32_t b_step,
                                                    uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t.reg .b32 a;\n\t.reg .b64 b, bk;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "cvt.u64.u32 bk, %3;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %4, p;\n\t"
      "add.s32 a, %1, 8;\n\tadd.s64 b, %2, 2;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, 1;\n\t"
      "add.s32 a, %1, 16;\n\tadd.s64 b, %2, 4;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, 1;\n\t"
      "add.s32 a, %1, 24;\n\tadd.s64 b, %2, 6;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, 1;\n\t"
      "add.s64 b, %2, bk;\n\t"
      "add.s32 a, %1, 32;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, 1;\n\t"
      "add.s32 a, %1, 40;\n\tadd.s64 b, b, 2;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, 1;\n\t"
      "add.s32 a, %1, 48;\n\tadd.s64 b, b, 2;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, 1;\n\t"
      "add.s32 a, %1, 56;\n\tadd.s64 b, b, 2;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, 1;\n\t"
      "add.s64 bk, bk, bk;\n\tadd.s64 b, %2, bk;\n\t"
      "add.s32 a, %1, 64;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, 1;\n\t"
      "add.s32 a, %1, 72;\n\tadd.s64 b, b, 2;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, 1;\n\t"
      "add.s32 a, %1, 80;\n\tadd.s64 b, b, 2;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, 1;\n\t"
      "add.s32 a, %1, 88;\n\tadd.s64 b, b, 2;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, 1;\n\t"
      "cvt.u64.u32 bk, %3;\n\tmul.lo.u64 bk, bk, 3;\n\tadd.s64 b, %2, bk;\n\t"
      "add.s32 a, %1, 96;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, 1;\n\t"
      "add.s32 a, %1, 104;\n\tadd.s64 b, b, 2;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, 1;\n\t"
      "add.s32 a, %1, 112;\n\tadd.s64 b, b, 2;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, 1;\n\t"
      "add.s32 a, %1, 120;\n\tadd.s64 b, b, 2;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, 1;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(b_step), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// bf16x2 (s', s') with s' = e4m3(code) * 2^119: exact (4 significant bits) and inside bf16's
// normal range for every finite E4M3 (2^-9 .. 448).
__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t code) {
  const uint32_t both = code | (code << 8);
  uint32_t h2;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
      : "=r"(h2)
      : "r"(both));
  const float f = __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu))) * 0x1p119f;
  uint32_t out;
  asm("cvt.rn.bf16x2.f32 %0, %1, %1;" : "=r"(out) : "f"(f));
  return out;
}

// Eight E2M1 codes (one little-endian word: element i in nibble i) times the block scale, as
// four bf16x2 words in natural order (elements 2j, 2j+1 in word j), each value e2m1*e4m3*2^-7.
//   1. A multiply spreads each selected nibble twice: to bits 9..6 (its exponent and mantissa
//      land on bf16 bits 8..6) and to bits 15..12 (its sign lands on bit 15); a mask keeps just
//      those four bits. Read as bf16 that is +-q * 2^-126 -- a bf16 subnormal for q = 0.5,
//      exactly as E2M1 is subnormal there -- and zero for codes 0 / 8. The multiply handles
//      nibbles i and i + 4 together (16 bits apart).
//   2. prmt re-pairs halves into (2j, 2j+1) order.
//   3. One exact bf16x2 multiply by s * 2^119.
__device__ __forceinline__ void dequant8(uint32_t x, uint32_t s2, uint32_t* w) {
  const uint32_t x8 = x >> 8;
  const uint32_t p04 = ((x & 0x000F000Fu) * 0x1040u) & 0x81C081C0u;   // nibbles 0, 4
  const uint32_t p15 = ((x & 0x00F000F0u) * 0x104u) & 0x81C081C0u;    // nibbles 1, 5
  const uint32_t p26 = ((x8 & 0x000F000Fu) * 0x1040u) & 0x81C081C0u;  // nibbles 2, 6
  const uint32_t p37 = ((x8 & 0x00F000F0u) * 0x104u) & 0x81C081C0u;   // nibbles 3, 7
  w[0] = mul_bf16x2(prmt(p04, p15, 0x5410u), s2);
  w[1] = mul_bf16x2(prmt(p26, p37, 0x5410u), s2);
  w[2] = mul_bf16x2(prmt(p04, p15, 0x7632u), s2);
  w[3] = mul_bf16x2(prmt(p26, p37, 0x7632u), s2);
}

__global__ void __launch_bounds__(kNvfp4Threads, 1)
    lmhead_w4a16_nvfp4_kernel(const __grid_constant__ CUtensorMap tmap_q,
                              const __grid_constant__ CUtensorMap tmap_s,
                              const __grid_constant__ CUtensorMap tmap_h,
                              const Nvfp4HeadParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t scale_lut[256];  // E4M3 code -> bf16x2 of its value * 2^119
  uint8_t* smem = align_up_1024(smem_raw);
  // Broadcast from lane 0 so the compiler can prove role branches warp-uniform and keep their
  // counters and descriptors in uniform registers.
  const int warp = __shfl_sync(0xffffffffu, (int)(threadIdx.x >> 5), 0);
  const int lane = threadIdx.x & 31;
  const int S = p.stages;
  const uint32_t sub_bytes = nvfp4_hid_sub_bytes(p.bn);
  const uint32_t stage_bytes = nvfp4_stage_bytes(p.bn);
  const uint32_t off_q = kRawK * sub_bytes;
  const uint32_t off_s = off_q + kRawCodeBytes;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)S * stage_bytes);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = smem_u32(bars + S);
  const uint32_t afull0 = smem_u32(bars + 2 * S);
  const uint32_t aempty0 = smem_u32(bars + 2 * S + kMaxSlots);
  const uint32_t tfull0 = smem_u32(bars + 2 * S + 2 * kMaxSlots);
  const uint32_t tempty0 = smem_u32(bars + 2 * S + 2 * kMaxSlots + 2);
  const uint32_t done_bar = smem_u32(bars + 2 * S + 2 * kMaxSlots + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 2 * kMaxSlots + 5);
  const int NA = p.slots;
  const uint32_t slot_col0 = kTmemCols - (uint32_t)NA * kSlotCols;  // weight slots at the top
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      // expect_tx arrive (+ 32 scale-copy arrivals when the scales come by async copies)
      mbar_init(full0 + 8 * s, p.scale_tma ? 1 : 1 + 32);
      // the dequantisers have read the codes and the MMAs have read the hidden rows
      mbar_init(empty0 + 8 * s, kDequantThreads + 1);
    }
    for (int a = 0; a < kMaxSlots; ++a) {
      mbar_init(afull0 + 8 * a, kDequantThreads);
      mbar_init(aempty0 + 8 * a, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull0 + 8 * a, 1);
      mbar_init(tempty0 + 8 * a, kEpilogueThreads);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_q);
    if (p.scale_tma) prefetch_tmap(&tmap_s);
    prefetch_tmap(&tmap_h);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  for (int c = threadIdx.x; c < 256; c += blockDim.x) scale_lut[c] = scale_bf16x2((uint32_t)c);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const int64_t scale_pitch = p.H / 16;
  const int my_tiles = sched_count(p.sched);
  const int n_raw = (p.num_kb + kRawK - 1) / kRawK;  // stages per tile

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    const uint64_t pol_w = l2_policy_weights();
    const uint64_t pol_h = l2_policy_evict_last();
    const uint32_t hid_tx = (uint32_t)p.hid_rows * kBK * 2;
    int gr = 0;  // stages issued so far
    int st = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int t = 0; ok && t < my_tiles; ++t) {
      const TileCoord tc = sched_tile(p.sched, p.V, t);
      for (int r = 0; r < n_raw; ++r, ++gr) {
        if (!wait_bounded(empty0 + 8 * st, ph ^ 1u, p.wait, abort_flag)) {
          fail(kRoleProducer, abort_flag);
          ok = false;
          break;
        }
        const int nk = p.num_kb - r * kRawK < kRawK ? p.num_kb - r * kRawK : kRawK;
        if (!p.wait.starve_loads) {
          const uint32_t full = full0 + 8 * st;
          const uint32_t sbase = smem_u32(smem + (size_t)st * stage_bytes);
          if (lane == 0) {
            mbar_arrive_expect_tx(full, kRawCodeBytes + (p.scale_tma ? kRawScaleBytes : 0u) +
                                            (uint32_t)nk * hid_tx);
            tma_load_2d(sbase + off_q, &tmap_q, full, tma_x(r * (kRawK * kBK / 2), 1),
                        (int32_t)tc.v0, pol_w);
            if (p.scale_tma)
              tma_load_2d(sbase + off_s, &tmap_s, full, tma_x(r * (kRawK * 4), 1),
                          (int32_t)tc.v0, pol_w);
            for (int j = 0; j < nk; ++j)
              tma_load_2d(sbase + (uint32_t)j * sub_bytes, &tmap_h, full,
                          tma_x((r * kRawK + j) * kBK * 2, 2), (int32_t)tc.r0, pol_h);
          }
          if (!p.scale_tma) {
            // 4 rows per lane, 4 K steps of 4 bytes each; rows past V and K steps past H copy
            // nothing (zero-filled).
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int row = lane * 4 + i;
              const bool in_row = tc.v0 + row < p.V;
#pragma unroll
              for (int j = 0; j < kRawK; ++j) {
                const bool in = in_row && j < nk;
                const uint8_t* src =
                    p.scales +
                    (in ? (tc.v0 + row) * scale_pitch + (int64_t)(r * kRawK + j) * 4 : 0);
                cp_async_4(sbase + off_s + (uint32_t)(row * 16 + j * 4), src, in ? 4u : 0u);
              }
            }
            cp_async_arrive_noinc(full);
          }
        }
        __syncwarp();
        if (++st == S) {
          st = 0;
          ph ^= 1u;
        }
      }
    }
    // Drain: wait for the loads of the last stages issued.
    if (!p.wait.starve_loads) {
      for (int i = 0; i < (gr < S ? gr : S); ++i) {
        if (--st < 0) {
          st = S - 1;
          ph ^= 1u;
        }
        if (!wait_bounded(full0 + 8 * st, ph, p.wait, nullptr)) {
          fail(kRoleDrain, abort_flag);
          break;
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    const uint32_t idesc = idesc_bf16_f32(kBM, p.bn);
    int gr = 0;
    int st = 0;
    uint32_t ph = 0;
    int sl = 0;  // weight slot of stage gr, and its phase
    uint32_t sph = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int t = 0; ok && t < my_tiles; ++t) {
      if (!wait_bounded(tempty0 + 8 * acc, acc_phase ^ 1u, p.wait, abort_flag)) {
        fail(kRoleMma, abort_flag);
        break;
      }
      tc_fence_after_sync();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * p.bn);
      for (int r = 0; r < n_raw; ++r, ++gr) {
        if (!wait_bounded(full0 + 8 * st, ph, p.wait, abort_flag) ||
            !wait_bounded(afull0 + 8 * sl, sph, p.wait, abort_flag)) {
          fail(kRoleMma, abort_flag);
          ok = false;
          break;
        }
        tc_fence_after_sync();
        {
          const int nk = p.num_kb - r * kRawK < kRawK ? p.num_kb - r * kRawK : kRawK;
          const uint32_t sb = smem_u32(smem + (size_t)st * stage_bytes);
          const uint64_t bdesc0 = sdesc_kmajor_sw128(sb);
          const uint32_t a0 = tmem_base + slot_col0 + (uint32_t)sl * kSlotCols;
          // descriptor start addresses are in 16-byte units
          if (nk == kRawK) {
            mma16_bf16_ts_elect(d_tmem, a0, bdesc0, sub_bytes >> 4, idesc, r != 0);
          } else {
            for (int j = 0; j < nk; ++j)
              mma4_bf16_ts_elect(d_tmem, a0 + (uint32_t)(j * (kBK / 2)),
                                 bdesc0 + (uint64_t)((j * sub_bytes) >> 4), idesc,
                                 (r | j) != 0);
          }
          mma_commit_elect(empty0 + 8 * st);
          mma_commit_elect(aempty0 + 8 * sl);
        }
        __syncwarp();
        if (++st == S) {
          st = 0;
          ph ^= 1u;
        }
        if (++sl == NA) {
          sl = 0;
          sph ^= 1u;
        }
      }
      if (!ok) break;
      mma_commit_elect(tfull0 + 8 * acc);
      __syncwarp();
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    mma_commit_elect(done_bar);
    __syncwarp();
    if (!wait_bounded(done_bar, 0, p.wait, nullptr)) fail(kRoleDrain, abort_flag);
  } else if (warp < kDequantWarp0) {
    // ---------------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int v_local = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = 0; t < my_tiles; ++t) {
      const TileCoord tc = sched_tile(p.sched, p.V, t);
      if (!wait_bounded(tfull0 + 8 * acc, acc_phase, p.wait, abort_flag, kSleepHintNs)) {
        fail(kRoleEpilogue, abort_flag);
        break;
      }
      tc_fence_after_sync();
      const int64_t v = tc.v0 + v_local;
      const int64_t r0 = tc.r0;
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * p.bn);
      const bool v_ok = v_local < tc.vrows;
      for (int c = 0; c < p.bn; c += 16) {
        if (r0 + c >= p.rows) break;
        uint32_t r[16];
        tmem_ld_32x32b_x16(taddr + (uint32_t)c, r);
        tmem_ld_wait();
        if (v_ok) {
          uint16_t* dst = p.out + (r0 + c) * p.V + v;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (r0 + c + j < p.rows) {
              const float a = __fmul_rn(__uint_as_float(r[j]), 128.0f);  // undo the 2^-7
              const float y = __fmul_rn(__fmul_rn(a, p.gscale), p.alpha);
              dst[(int64_t)j * p.V] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
            }
          }
        }
      }
      tc_fence_before_sync();
      mbar_arrive(tempty0 + 8 * acc);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  } else {
    // ---------------------------------------------------------------- dequantisers
    // Group g converts stages g, g + 2, ...; stage i goes to TMEM weight slot i mod slots. Each
    // thread converts one weight row, 64 elements per K step; the stores of a stage are waited
    // for once, at its end.
    const int group = (warp - kDequantWarp0) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t sw = (uint32_t)(row & 7);  // 128-byte swizzle of the codes box
    const uint32_t t_slots = tmem_base + ((uint32_t)(quarter * 32) << 16) + slot_col0;
    const int total_raw = my_tiles * n_raw;
    int st = group % S;             // stage and phase of stage index gr, advanced by the group
    uint32_t ph = (uint32_t)(group / S) & 1u;  // count each iteration (no divisions in the loop)
    int r = group % n_raw;          // stage within its tile
    int sl = group % NA;            // weight slot of stage gr, and its phase
    uint32_t sph = (uint32_t)(group / NA) & 1u;
    for (int gr = group; gr < total_raw; gr += kDequantGroups) {
      const int nk = p.num_kb - r * kRawK < kRawK ? p.num_kb - r * kRawK : kRawK;
      if (!wait_bounded(full0 + 8 * st, ph, p.wait, abort_flag) ||
          !wait_bounded(aempty0 + 8 * sl, sph ^ 1u, p.wait, abort_flag)) {
        fail(kRoleDequant, abort_flag);
        break;
      }
      tc_fence_after_sync();
      const uint8_t* sbase = smem + (size_t)st * stage_bytes;
      const uint8_t* crow = sbase + off_q + row * 128;
      const uint4 sc4 = *reinterpret_cast<const uint4*>(sbase + off_s + row * 16);
      const uint32_t scw[4] = {sc4.x, sc4.y, sc4.z, sc4.w};
      for (int j = 0; j < nk; ++j) {
        const uint4 c0 = *reinterpret_cast<const uint4*>(crow + (((2u * j) ^ sw) << 4));
        const uint4 c1 = *reinterpret_cast<const uint4*>(crow + (((2u * j + 1u) ^ sw) << 4));
        const uint32_t sc = scw[j];
        uint32_t w[32];
        const uint32_t s0 = scale_lut[sc & 0xFFu];
        dequant8(c0.x, s0, w + 0);
        dequant8(c0.y, s0, w + 4);
        const uint32_t s1 = scale_lut[(sc >> 8) & 0xFFu];
        dequant8(c0.z, s1, w + 8);
        dequant8(c0.w, s1, w + 12);
        const uint32_t s2 = scale_lut[(sc >> 16) & 0xFFu];
        dequant8(c1.x, s2, w + 16);
        dequant8(c1.y, s2, w + 20);
        const uint32_t s3 = scale_lut[sc >> 24];
        dequant8(c1.z, s3, w + 24);
        dequant8(c1.w, s3, w + 28);
        tmem_st_32x32b_x32(t_slots + (uint32_t)sl * kSlotCols + (uint32_t)j * (kBK / 2), w);
      }
      mbar_arrive(empty0 + 8 * st);  // this row's codes and scales are in registers
      tmem_st_wait();
      tc_fence_before_sync();
      mbar_arrive(afull0 + 8 * sl);
      sl += kDequantGroups;
      while (sl >= NA) {
        sl -= NA;
        sph ^= 1u;
      }
      st += kDequantGroups;
      if (st >= S) {
        st -= S;
        ph ^= 1u;
      }
      r += kDequantGroups;
      while (r >= n_raw) r -= n_raw;
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace lmh
