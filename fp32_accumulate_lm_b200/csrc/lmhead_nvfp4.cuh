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
// Conversion, two equivalent ways (identical bits; the host picks one per call, so a row's
// logits do not depend on which):
//   pair table  each byte of codes (two E2M1 values) indexes a 256-entry table of bf16x2 words
//               in shared memory, one copy per lane so a warp's 32 lookups never share a bank.
//               The table sits on a 64 KB boundary with entries 256 bytes apart, so one prmt
//               builds the lookup address from the code byte and the lane's base. Three
//               instructions per two weights (prmt, lds, one bf16x2 multiply by the scale).
//   spread      integer multiplies spread nibbles into bf16 bit positions (dequant8 below); no
//               table, used when the table leaves room for fewer than two stages (large row
//               tiles).
//
// Every hand-off covers 4 K steps (256 elements of K). The single-thread roles (TMA producers,
// MMA issuer) share their SM sub-partitions with busy dequantiser warps, so each of their
// instructions is slow; paying one wait and one commit per K step of 64 made them the
// bottleneck. A stage's two halves live in two shared-memory rings, because they are done with
// at different times:
//   codes stage  the packed codes [128 rows x 128 bytes] of 4 K steps in one box, and their
//                block scales [128 rows x 16 bytes]; free once the dequantisers have read them,
//                so this ring runs far ahead (up to 8 stages) and keeps the weight stream going.
//   hidden stage the hidden rows [BN x 64] x 4; free only once the MMAs that read them are done.
//                At 256 rows a hidden stage is 64 KB: when both halves shared one ring, only 2
//                stages fitted, and each new stage waited for the MMAs two stages back.
//   slot         (tensor memory) the dequantised weights of one stage, [128 x 256] bf16; a ring
//                of 3 slots (2 when the row tile is 128), so refilling a slot never waits for the
//                MMAs that were just issued.
// Roles (224 + 128 * kWarpsPerQuarter * kDequantGroups threads):
//   warp 0      codes producer: fills codes stages.
//   warp 1      TMEM allocator and MMA issuer: per stage waits for its weight slot and its
//               hidden stage, 16 x tcgen05.mma with A from TMEM, commits free the hidden stage
//               and the slot.
//   warps 2-5   epilogue.
//   warps 6-    dequantisers: two groups of 4 * kWarpsPerQuarter warps; group g takes stages
//               g, g + 2, ...; stage i goes to slot i mod slots. In a group, each TMEM lane
//               quarter has kWarpsPerQuarter warps, which split the stage's 4 K steps between
//               them; each thread converts one weight row of its K steps.
//   last warp   hidden producer: fills hidden stages.
#pragma once

#include "lmhead_common.cuh"

namespace lmh {

// Two dequantiser groups of four warps take stages in turn. The slot ring's phase waits assume
// no more groups than TMEM weight slots (a group is never two uses of a slot ahead).
#ifndef LMHEAD_NVFP4_WPQ
#define LMHEAD_NVFP4_WPQ 2
#endif
#ifndef LMHEAD_NVFP4_GROUPS
#define LMHEAD_NVFP4_GROUPS 2
#endif
constexpr int kDequantGroups = LMHEAD_NVFP4_GROUPS;  // groups taking stages in turn
constexpr int kDequantWarp0 = 6;
constexpr int kWarpsPerQuarter = LMHEAD_NVFP4_WPQ;       // warps per TMEM lane quarter and group
constexpr int kDequantThreads = 128 * kWarpsPerQuarter;  // threads of one group (one stage)
constexpr int kHidProducerWarp = kDequantWarp0 + kDequantThreads * kDequantGroups / 32;
constexpr int kNvfp4Threads = 32 * (kHidProducerWarp + 1);
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxSlots = 3;         // dequantised weight slots at the top of TMEM
static_assert(kDequantGroups <= 2, "the slot ring may have only 2 slots");
static_assert(kWarpsPerQuarter == 1 || kWarpsPerQuarter == 2 || kWarpsPerQuarter == 4,
              "the warps of a lane quarter split a stage's 4 K steps evenly");
constexpr int kBnMax = 128;          // row tile cap: two accumulators of <= 128 columns

constexpr int kRawK = 4;                                  // K steps per stage
constexpr uint32_t kRawCodeBytes = kBM * kRawK * kBK / 2;  // 16 KB
constexpr uint32_t kRawScaleBytes = kBM * kRawK * 4;       // 2 KB
constexpr uint32_t kSlotCols = kRawK * kBK / 2;            // TMEM columns of one weight slot

constexpr int kMaxCodeStages = 8;
constexpr int kMaxHidStages = 4;

// Suspend-time hint of the producer's, MMA issuer's and dequantisers' barrier waits (ns). Every
// SM sub-partition holds converting dequantiser warps next to warps that wait (the producer, the
// MMA issuer, the other group): a waiter that spins on try_wait takes issue slots from them.
#ifndef LMHEAD_NVFP4_WAIT_SLEEP_NS
#define LMHEAD_NVFP4_WAIT_SLEEP_NS 0
#endif
constexpr uint32_t kWaitSleepNs = LMHEAD_NVFP4_WAIT_SLEEP_NS;
constexpr uint32_t kBarrierBytes = 1024;   // barrier block at the start of dynamic smem
constexpr uint32_t kPairTableBytes = 65536;  // 256 entries x 256 bytes, on a 64 KB boundary
// Entry e of the pair table: bytes [0, 128) hold the 32 lanes' copies of the code-pair word e,
// bytes [128, 256) the 32 lanes' copies of E4M3 scale e as bf16x2 (value * 2^119).
constexpr uint32_t kScaleTableOffset = 128;

struct Nvfp4HeadParams {
  int64_t rows, H, V;
  uint16_t* out;          // bf16 logits
  const uint8_t* scales;  // [V, H/16] E4M3
  float alpha;
  float gscale;
  int32_t bn;
  int32_t hid_rows;       // hidden rows per K step in a stage: a multiple of 8, <= bn (MMA
                          // columns past the call's rows read neighbouring data, never stored)
  TileSched sched;
  int32_t num_kb;         // K steps of 64 per tile: ceil(H / 64)
  int32_t slots;          // TMEM weight slots (3, or 2 when forced)
  int32_t accs;           // TMEM accumulators: 2 when 2 * bn + 3 * 128 <= 512 (the epilogue of a
                          // tile overlaps the next tile's MMAs), else 1
  int32_t scale_mode;     // block scales: kScaleTma, kScaleAsync4 or kScalePlain (see below)
  int32_t half_tail;      // 1 when H % 64 == 32: the last K step holds 32 elements (2 MMAs)
  int32_t hid_2d;         // 1: hidden rows by one 2-D box per K step (needed when H % 64 != 0)
  WaitCfg wait;
};

// How the producer brings a stage's block scales into shared memory:
//   kScaleTma     one TMA box [128 rows x 16 bytes]; needs H % 256 == 0 and 16-byte aligned scales
//   kScaleAsync4  4-byte async copies, one per row and K step; needs H % 64 == 0 (whole words)
//   kScalePlain   2-byte loads and shared stores by the producer's lanes, for H % 64 == 32, where
//                 a scale row is not a whole number of words (its K steps' 4 bytes straddle rows)
constexpr int32_t kScaleAsync4 = 0;
constexpr int32_t kScaleTma = 1;
constexpr int32_t kScalePlain = 2;

// Shared-memory stages. Codes stage (4 K steps): [codes: 128 rows x 128 bytes, 128-byte
// swizzle][scales: 128 rows x 16 bytes] = 18 KB. Hidden stage: 4 sub-tiles of hid_rows x 64 bf16,
// 128-byte swizzle, from one 3-D box, plus room for the last sub-tile's MMA to read bn rows.
// Both are multiples of 1024 bytes.
constexpr uint32_t kCodeStageBytes = kRawCodeBytes + kRawScaleBytes;
__host__ __device__ constexpr uint32_t nvfp4_hid_stage_bytes(int bn, int hid_rows) {
  return (uint32_t)(((kRawK - 1) * hid_rows + bn) * kBK * 2);
}

// Where everything goes in dynamic shared memory [base, end) (shared-window addresses): the
// barrier block first; with the pair table, the table on the next 64 KB boundary, which splits
// the rest into two regions. Hidden stages are placed first, the larger region first: 4, 3 or 2
// of them, the most that still leaves room for 4 codes stages (else 2); then as many codes stages
// as fit, at most 8. Host and device use the same arithmetic, the host on the window layout it
// expects, the kernel on the real one.
struct Nvfp4Layout {
  uint32_t bars;   // barrier block (kBarrierBytes)
  uint32_t table;  // pair table, or 0
  int n_code, n_hid;
};
// Writes the stage addresses to code[kMaxCodeStages] and hid[kMaxHidStages] (the kernel passes
// its shared arrays, the host local ones).
__host__ __device__ inline Nvfp4Layout nvfp4_layout(uint32_t base, uint32_t end,
                                                    uint32_t hid_bytes, bool pair_table,
                                                    uint32_t* code, uint32_t* hid) {
  Nvfp4Layout L{};
  L.bars = (base + 1023u) & ~1023u;
  const uint32_t start = L.bars + kBarrierBytes;
  uint32_t lo0 = start, hi0, lo1 = start, hi1 = start;
  int nr = 1;
  if (pair_table) {
    L.table = (start + 0xFFFFu) & ~0xFFFFu;
    hi0 = L.table;
    lo1 = L.table + kPairTableBytes;
    hi1 = end > lo1 ? end : lo1;
    nr = 2;
  } else {
    L.table = 0;
    hi0 = end > start ? end : start;
  }
  const bool second_first = nr == 2 && hi1 - lo1 > hi0 - lo0;
  for (int want = kMaxHidStages; want >= 2; --want) {
    uint32_t cur0 = lo0, cur1 = lo1;
    int nh = 0, nc = 0;
    for (int pass = 0; pass < nr; ++pass) {
      const bool use1 = (pass == 0) == second_first;
      uint32_t& cur = use1 ? cur1 : cur0;
      const uint32_t top = use1 ? hi1 : hi0;
      while (nh < want && cur + hid_bytes <= top) {
        hid[nh++] = cur;
        cur += hid_bytes;
      }
    }
    while (nc < kMaxCodeStages && cur0 + kCodeStageBytes <= hi0) {
      code[nc++] = cur0;
      cur0 += kCodeStageBytes;
    }
    while (nr == 2 && nc < kMaxCodeStages && cur1 + kCodeStageBytes <= hi1) {
      code[nc++] = cur1;
      cur1 += kCodeStageBytes;
    }
    L.n_hid = nh;
    L.n_code = nc;
    if ((nh == want && nc >= 4) || want == 2) break;
  }
  return L;
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

// Half a K step (32 elements) with A from TMEM: two K = 16 MMAs; only the first may start a fresh
// accumulator. For the last K step of a head whose H is an odd multiple of 32.
__device__ __forceinline__ void mma2_bf16_ts_elect(uint32_t d_tmem, uint32_t a_tmem,
                                                   uint64_t b_desc, uint32_t idesc,
                                                   uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t.reg .b32 a1;\n\t.reg .b64 b1;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "add.s32 a1, %1, 8;\n\tadd.s64 b1, %2, 2;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], b1, %3, 1;\n\t}" ::"r"(d_tmem),
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

// Pair-table entry for code byte e (element 2j in the low nibble, 2j + 1 in the high one): the
// bf16x2 word dequant8's step 1 gives for those two nibbles, in natural order.
__host__ __device__ constexpr uint32_t pair_entry(uint32_t e) {
  return ((e & 7u) << 6) | ((e & 8u) << 12) | (((e >> 4) & 7u) << 22) | (((e >> 4) & 8u) << 28);
}

// dequant8 through the pair table. lane_base = table address (64 KB aligned) + 4 * lane, so its
// bits 8..15 are zero and prmt can drop code byte k there: entry address = table + 256 * byte +
// 4 * lane.
__device__ __forceinline__ void dequant8_table(uint32_t x, uint32_t s2, uint32_t lane_base,
                                               uint32_t* w) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t a = prmt(x, lane_base, 0x7604u | ((uint32_t)k << 4));
    uint32_t v;
    asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    w[k] = mul_bf16x2(v, s2);
  }
}

template <bool kTable>
__device__ __forceinline__ void dequant8_any(uint32_t x, uint32_t s2, uint32_t lane_base,
                                             uint32_t* w) {
  if (kTable)
    dequant8_table(x, s2, lane_base, w);
  else
    dequant8(x, s2, w);
}

// Block scale k (byte k of `sc`) as bf16x2. With the pair table: from this lane's own copy in
// the table's second half, so a warp's 32 lookups never share a bank (one prmt builds the
// address, as for the code pairs). Without it: from the one 256-word table `lut`.
template <bool kTable>
__device__ __forceinline__ uint32_t scale_of(uint32_t sc, int k, const uint32_t* lut,
                                             uint32_t lane_base) {
  if (kTable) {
    const uint32_t a = prmt(sc, lane_base + kScaleTableOffset, 0x7604u | ((uint32_t)k << 4));
    uint32_t v;
    asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
  }
  return lut[(sc >> (8 * k)) & 0xFFu];
}

// With the pair table, how many of a K step's eight 4-byte code words go through the table; the
// others are spread with integer arithmetic. The table costs one shared-memory wavefront per
// two weights of a warp, the spread none but five ALU instructions; shared-memory bandwidth is
// what bounds the kernel at decode sizes, so the best split leaves both pipes about equally
// busy. Both give identical bits.
#ifndef LMHEAD_NVFP4_TABLE_WORDS
#define LMHEAD_NVFP4_TABLE_WORDS 8
#endif
constexpr int kTableWords = LMHEAD_NVFP4_TABLE_WORDS;
static_assert(kTableWords >= 0 && kTableWords <= 8, "a K step has 8 code words");

// One K step of one weight row: 64 codes (two 16-byte words) and their four block scales (one
// byte each in `sc`, low byte first) to 32 bf16x2 words in K order.
template <bool kTable>
__device__ __forceinline__ void convert_kstep(const uint4& c0, const uint4& c1, uint32_t sc,
                                              const uint32_t* lut, uint32_t lane_base,
                                              uint32_t (&w)[32]) {
  const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {  // block scale q covers code words 2q, 2q + 1
    const uint32_t sq = scale_of<kTable>(sc, q, lut, lane_base);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = 2 * q + h;
      if (kTable && i < kTableWords)
        dequant8_table(words[i], sq, lane_base, w + 4 * i);
      else
        dequant8(words[i], sq, w + 4 * i);
    }
  }
}

template <bool kTable>
__global__ void __launch_bounds__(kNvfp4Threads, 1)
    lmhead_w4a16_nvfp4_kernel(const __grid_constant__ CUtensorMap tmap_q,
                              const __grid_constant__ CUtensorMap tmap_s,
                              const __grid_constant__ CUtensorMap tmap_h,
                              const Nvfp4HeadParams p) {
  extern __shared__ uint8_t smem_raw[];
  if (threadIdx.x == 0) pdl_trigger();
  __shared__ uint32_t scale_lut[256];  // E4M3 code -> bf16x2 of its value * 2^119 (no table)
  __shared__ uint32_t s_code[kMaxCodeStages];  // codes stage addresses (shared window)
  __shared__ uint32_t s_hid[kMaxHidStages];    // hidden stage addresses
  __shared__ uint32_t s_layout[4];             // barrier block, table, codes and hidden stages
  // Broadcast from lane 0 so the compiler can prove role branches warp-uniform and keep their
  // counters and descriptors in uniform registers.
  const int warp = __shfl_sync(0xffffffffu, (int)(threadIdx.x >> 5), 0);
  const int lane = threadIdx.x & 31;
  const uint32_t hsub = (uint32_t)p.hid_rows * kBK * 2;  // hidden sub-tile stride in a stage
  const uint32_t raw = smem_u32(smem_raw);
  if (threadIdx.x == 0) {
    uint32_t dyn_bytes;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn_bytes));
    const Nvfp4Layout L = nvfp4_layout(raw, raw + dyn_bytes,
                                       nvfp4_hid_stage_bytes(p.bn, p.hid_rows), kTable, s_code,
                                       s_hid);
    s_layout[0] = L.bars;
    s_layout[1] = L.table;
    s_layout[2] = (uint32_t)L.n_code;
    s_layout[3] = (uint32_t)L.n_hid;
  }
  __syncthreads();
  const int SC = (int)s_layout[2];
  const int SH = (int)s_layout[3];
  if (SC < 2 || SH < 2) {  // the host sizes calls so this cannot happen; never run a short ring
    if (threadIdx.x == 0) atomicCAS(&g_lmhead_status, 0u, kStatusNoRoom);
    return;
  }
  const uint32_t table_addr = s_layout[1];

  // Barrier block: codes full / empty [8], hidden full / empty [4], slot full / empty [3],
  // accumulator full / empty [2], done, then the TMEM address and the abort flag.
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw + (s_layout[0] - raw));
  const uint32_t cfull0 = smem_u32(bars);
  const uint32_t cempty0 = smem_u32(bars + kMaxCodeStages);
  const uint32_t hfull0 = smem_u32(bars + 2 * kMaxCodeStages);
  const uint32_t hempty0 = smem_u32(bars + 2 * kMaxCodeStages + kMaxHidStages);
  const uint32_t afull0 = smem_u32(bars + 2 * kMaxCodeStages + 2 * kMaxHidStages);
  const uint32_t aempty0 = afull0 + 8 * kMaxSlots;
  const uint32_t tfull0 = aempty0 + 8 * kMaxSlots;
  const uint32_t tempty0 = tfull0 + 16;
  const uint32_t done_bar = tempty0 + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(
      bars + 2 * kMaxCodeStages + 2 * kMaxHidStages + 2 * kMaxSlots + 5);
  const int NA = p.slots;
  const uint32_t slot_col0 = kTmemCols - (uint32_t)NA * kSlotCols;  // weight slots at the top
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < SC; ++s) {
      // expect_tx arrive (+ 32 producer-lane arrivals when the scales do not come by TMA)
      mbar_init(cfull0 + 8 * s, p.scale_mode == kScaleTma ? 1 : 1 + 32);
      mbar_init(cempty0 + 8 * s, kDequantThreads);  // the group has read the codes and scales
    }
    for (int s = 0; s < SH; ++s) {
      mbar_init(hfull0 + 8 * s, 1);
      mbar_init(hempty0 + 8 * s, 1);  // the stage's MMAs are done
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
    if (p.scale_mode == kScaleTma) prefetch_tmap(&tmap_s);
  }
  if (warp == kHidProducerWarp && lane == 0) prefetch_tmap(&tmap_h);
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  if (!kTable)
    for (int c = threadIdx.x; c < 256; c += blockDim.x) scale_lut[c] = scale_bf16x2((uint32_t)c);
  if (kTable) {
    // 256 entries x 32 lane copies: code pair e of lane l at table + 256 e + 4 l, scale e of
    // lane l at table + 256 e + 128 + 4 l.
    uint8_t* table = smem_raw + (table_addr - raw);
    for (int c = threadIdx.x; c < 256 * 32; c += blockDim.x) {
      uint8_t* e = table + (c >> 5) * 256 + (c & 31) * 4;
      *reinterpret_cast<uint32_t*>(e) = pair_entry((uint32_t)c >> 5);
      *reinterpret_cast<uint32_t*>(e + kScaleTableOffset) = scale_bf16x2((uint32_t)c >> 5);
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  pdl_wait();  // from here on global memory: earlier kernels of the stream are done
  const uint32_t tmem_base = *tmem_slot;
  const int64_t scale_pitch = p.H / 16;
  const int my_tiles = sched_count(p.sched);
  const int n_raw = (p.num_kb + kRawK - 1) / kRawK;  // stages per tile

  if (warp == 0) {
    // ---------------------------------------------------------------- codes producer
    const uint64_t pol_w = l2_policy_weights();
    int gr = 0;  // stages issued so far
    int st = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int t = 0; ok && t < my_tiles; ++t) {
      const TileCoord tc = sched_tile(p.sched, p.V, t);
      for (int r = 0; r < n_raw; ++r, ++gr) {
        if (!wait_bounded(cempty0 + 8 * st, ph ^ 1u, p.wait, abort_flag, kWaitSleepNs)) {
          fail(kRoleProducer, abort_flag);
          ok = false;
          break;
        }
        const int nk = p.num_kb - r * kRawK < kRawK ? p.num_kb - r * kRawK : kRawK;
        if (!p.wait.starve_loads) {
          const uint32_t full = cfull0 + 8 * st;
          const uint32_t cbase = s_code[st];
          const uint32_t sbase = cbase + kRawCodeBytes;  // this stage's scales
          if (lane == 0) {
            // Boxes are counted whole: K steps past H arrive zero-filled.
            mbar_arrive_expect_tx(
                full, kRawCodeBytes + (p.scale_mode == kScaleTma ? kRawScaleBytes : 0u));
            tma_load_2d(cbase, &tmap_q, full, tma_x(r * (kRawK * kBK / 2), 1), (int32_t)tc.v0,
                        pol_w);
            if (p.scale_mode == kScaleTma)
              tma_load_2d(sbase, &tmap_s, full, tma_x(r * (kRawK * 4), 1), (int32_t)tc.v0, pol_w);
          }
          if (p.scale_mode == kScaleAsync4) {
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
                cp_async_4(sbase + (uint32_t)(row * 16 + j * 4), src, in ? 4u : 0u);
              }
            }
            cp_async_arrive_noinc(full);
          } else if (p.scale_mode == kScalePlain) {
            // The scale row's pitch is 2 mod 4 bytes: read it in 2-byte pieces (every piece is
            // 2-byte aligned), zeros past H and past V, so the dequantisers' words are whole.
            uint32_t word[4][kRawK];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int row = lane * 4 + i;
              const bool in_row = tc.v0 + row < p.V;
              const uint16_t* srow = reinterpret_cast<const uint16_t*>(
                  p.scales + (in_row ? (tc.v0 + row) * scale_pitch : 0));
#pragma unroll
              for (int j = 0; j < kRawK; ++j) {
                const int64_t b0 = (int64_t)(r * kRawK + j) * 4;  // byte of the K step in a row
                const uint32_t lo = (in_row && b0 < scale_pitch) ? srow[b0 >> 1] : 0u;
                const uint32_t hi = (in_row && b0 + 2 < scale_pitch) ? srow[(b0 >> 1) + 1] : 0u;
                word[i][j] = lo | (hi << 16);
              }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
              for (int j = 0; j < kRawK; ++j)
                asm volatile("st.shared.u32 [%0], %1;" ::"r"(sbase +
                                                             (uint32_t)((lane * 4 + i) * 16 + j * 4)),
                             "r"(word[i][j])
                             : "memory");
            mbar_arrive(full);  // release: the stores above are seen by whoever waits on `full`
          }
        }
        __syncwarp();
        if (++st == SC) {
          st = 0;
          ph ^= 1u;
        }
      }
    }
    // Drain: wait for the loads of the last stages issued.
    if (!p.wait.starve_loads) {
      for (int i = 0; i < (gr < SC ? gr : SC); ++i) {
        if (--st < 0) {
          st = SC - 1;
          ph ^= 1u;
        }
        if (!wait_bounded(cfull0 + 8 * st, ph, p.wait, nullptr)) {
          fail(kRoleDrain, abort_flag);
          break;
        }
      }
    }
  } else if (warp == kHidProducerWarp) {
    // ---------------------------------------------------------------- hidden producer
    const uint64_t pol_h = l2_policy_evict_last();
    const uint32_t hid_tx = (uint32_t)kRawK * hsub;  // one box: 4 K steps of hid_rows rows
    int gr = 0;
    int st = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int t = 0; ok && t < my_tiles; ++t) {
      const TileCoord tc = sched_tile(p.sched, p.V, t);
      for (int r = 0; r < n_raw; ++r, ++gr) {
        if (!wait_bounded(hempty0 + 8 * st, ph ^ 1u, p.wait, abort_flag, kWaitSleepNs)) {
          fail(kRoleProducer, abort_flag);
          ok = false;
          break;
        }
        const int nk = p.num_kb - r * kRawK < kRawK ? p.num_kb - r * kRawK : kRawK;
        if (!p.wait.starve_loads && lane == 0) {
          const uint32_t full = hfull0 + 8 * st;
          const uint32_t hbase = s_hid[st];
          // With 2-D hidden boxes only the stage's nk K steps are loaded; the 3-D box is counted
          // whole (K steps past H arrive zero-filled).
          mbar_arrive_expect_tx(full, p.hid_2d ? (uint32_t)nk * hsub : hid_tx);
          if (p.hid_2d) {
            // [hid_rows x 64] boxes of a [rows, H] map: elements past H are zero-filled
            for (int j = 0; j < nk; ++j)
              tma_load_2d(hbase + (uint32_t)j * hsub, &tmap_h, full,
                          tma_x((int64_t)(r * kRawK + j) * kBK * 2, 2), (int32_t)tc.r0, pol_h);
          } else {
            tma_load_3d(hbase, &tmap_h, full, 0, (int32_t)tc.r0, r * kRawK, pol_h);
          }
        }
        __syncwarp();
        if (++st == SH) {
          st = 0;
          ph ^= 1u;
        }
      }
    }
    if (!p.wait.starve_loads) {
      for (int i = 0; i < (gr < SH ? gr : SH); ++i) {
        if (--st < 0) {
          st = SH - 1;
          ph ^= 1u;
        }
        if (!wait_bounded(hfull0 + 8 * st, ph, p.wait, nullptr)) {
          fail(kRoleDrain, abort_flag);
          break;
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    const uint32_t idesc = idesc_bf16_f32(kBM, p.bn);
    int hs = 0;  // hidden stage of stage gr, and its phase
    uint32_t hph = 0;
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
      for (int r = 0; r < n_raw; ++r) {
        if (!wait_bounded(afull0 + 8 * sl, sph, p.wait, abort_flag, kWaitSleepNs) ||
            !wait_bounded(hfull0 + 8 * hs, hph, p.wait, abort_flag, kWaitSleepNs)) {
          fail(kRoleMma, abort_flag);
          ok = false;
          break;
        }
        tc_fence_after_sync();
        {
          const int nk = p.num_kb - r * kRawK < kRawK ? p.num_kb - r * kRawK : kRawK;
          const uint64_t bdesc0 = sdesc_kmajor_sw128(s_hid[hs]);
          const uint32_t a0 = tmem_base + slot_col0 + (uint32_t)sl * kSlotCols;
          // The tile's last K step is half a step when H % 64 == 32: two MMAs, not four (the
          // zero codes past H are never multiplied).
          const bool half_last = p.half_tail && r == n_raw - 1;
          // descriptor start addresses are in 16-byte units
          if (nk == kRawK && !half_last) {
            mma16_bf16_ts_elect(d_tmem, a0, bdesc0, hsub >> 4, idesc, r != 0);
          } else {
            for (int j = 0; j < nk; ++j) {
              const uint32_t aj = a0 + (uint32_t)(j * (kBK / 2));
              const uint64_t bj = bdesc0 + (uint64_t)((j * hsub) >> 4);
              if (half_last && j == nk - 1)
                mma2_bf16_ts_elect(d_tmem, aj, bj, idesc, (r | j) != 0);
              else
                mma4_bf16_ts_elect(d_tmem, aj, bj, idesc, (r | j) != 0);
            }
          }
          mma_commit_elect(hempty0 + 8 * hs);
          mma_commit_elect(aempty0 + 8 * sl);
        }
        __syncwarp();
        if (++hs == SH) {
          hs = 0;
          hph ^= 1u;
        }
        if (++sl == NA) {
          sl = 0;
          sph ^= 1u;
        }
      }
      if (!ok) break;
      mma_commit_elect(tfull0 + 8 * acc);
      __syncwarp();
      if (++acc == p.accs) {
        acc = 0;
        acc_phase ^= 1u;
      }
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
      if (++acc == p.accs) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  } else {
    // ---------------------------------------------------------------- dequantisers
    // Group g converts stages g, g + 2, ...; stage i goes to TMEM weight slot i mod slots. In a
    // group, warp w serves lane quarter w mod 4 and K steps [part * kPer, (part + 1) * kPer) of
    // each stage, part = its index among the quarter's warps. Each thread converts one weight
    // row, 64 elements per K step; the stores of a stage are waited for once, at its end.
    constexpr int kPer = kRawK / kWarpsPerQuarter;  // K steps per warp and stage
    const int gw = warp - kDequantWarp0;
    const int group = gw / (4 * kWarpsPerQuarter);
    const int part = (gw % (4 * kWarpsPerQuarter)) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int j0 = part * kPer;
    const uint32_t sw = (uint32_t)(row & 7);  // 128-byte swizzle of the codes box
    const uint32_t t_slots = tmem_base + ((uint32_t)(quarter * 32) << 16) + slot_col0;
    const uint32_t lane_base = table_addr + (uint32_t)lane * 4u;  // pair table only
    const int total_raw = my_tiles * n_raw;
    int st = group % SC;            // codes stage and phase of stage index gr, advanced by the
    uint32_t ph = (uint32_t)(group / SC) & 1u;  // group each iteration (no divisions in the loop)
    int r = group % n_raw;          // stage within its tile
    int sl = group % NA;            // weight slot of stage gr, and its phase
    uint32_t sph = (uint32_t)(group / NA) & 1u;
    for (int gr = group; gr < total_raw; gr += kDequantGroups) {
      const int nk = p.num_kb - r * kRawK < kRawK ? p.num_kb - r * kRawK : kRawK;
      if (!wait_bounded(cfull0 + 8 * st, ph, p.wait, abort_flag, kWaitSleepNs) ||
          !wait_bounded(aempty0 + 8 * sl, sph ^ 1u, p.wait, abort_flag, kWaitSleepNs)) {
        fail(kRoleDequant, abort_flag);
        break;
      }
      tc_fence_after_sync();
      const uint8_t* sbase = smem_raw + (s_code[st] - raw);
      const uint8_t* crow = sbase + row * 128;
      const uint32_t* srow = reinterpret_cast<const uint32_t*>(sbase + kRawCodeBytes + row * 16);
      uint32_t scw[kPer];
#pragma unroll
      for (int j = 0; j < kPer; ++j) scw[j] = srow[j0 + j];
      const uint32_t t_dst = t_slots + (uint32_t)sl * kSlotCols;
      if (j0 + kPer <= nk) {
        // All of this warp's K steps: every 16-byte code read first, so their latency overlaps.
        uint4 c[2 * kPer];
#pragma unroll
        for (int h = 0; h < 2 * kPer; ++h)
          c[h] = *reinterpret_cast<const uint4*>(crow + (((uint32_t)(2 * j0 + h) ^ sw) << 4));
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
          uint32_t w[32];
          convert_kstep<kTable>(c[2 * j], c[2 * j + 1], scw[j], scale_lut, lane_base, w);
          tmem_st_32x32b_x32(t_dst + (uint32_t)(j0 + j) * (kBK / 2), w);
        }
      } else {
        for (int j = 0; j < kPer && j0 + j < nk; ++j) {
          const uint32_t h0 = 2u * (uint32_t)(j0 + j);
          const uint4 c0 = *reinterpret_cast<const uint4*>(crow + ((h0 ^ sw) << 4));
          const uint4 c1 = *reinterpret_cast<const uint4*>(crow + (((h0 + 1u) ^ sw) << 4));
          uint32_t w[32];
          convert_kstep<kTable>(c0, c1, scw[j], scale_lut, lane_base, w);
          tmem_st_32x32b_x32(t_dst + (uint32_t)(j0 + j) * (kBK / 2), w);
        }
      }
      mbar_arrive(cempty0 + 8 * st);  // this row's codes and scales are in registers
      tmem_st_wait();
      tc_fence_before_sync();
      mbar_arrive(afull0 + 8 * sl);
      sl += kDequantGroups;
      while (sl >= NA) {
        sl -= NA;
        sph ^= 1u;
      }
      st += kDequantGroups;
      if (st >= SC) {
        st -= SC;
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
