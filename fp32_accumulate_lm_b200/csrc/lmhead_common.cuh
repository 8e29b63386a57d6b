// Pieces shared by the LM-head kernels: tile constants, the bounded barrier wait, and the
// per-device status word that a timed-out wait writes.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sm100_ptx.cuh"

// Build-time tuning knobs (defaults are the measured best on B200; see the design notes):
//   LMHEAD_WEIGHT_L2_POLICY  L2 hint for weight loads: 0 none, 1 evict-first, 2 evict-normal
//   LMHEAD_TMA_WIDE          1: tensor maps see rows as 32-bit elements (same bytes, fewer
//                            elements per box); 0: their natural types (bf16 / bytes)
//   LMHEAD_HID_BOX_EXACT     1: a single row tile loads only the call's rows of hidden, not
//                            the padded tile height
#ifndef LMHEAD_WEIGHT_L2_POLICY
#define LMHEAD_WEIGHT_L2_POLICY 1
#endif
#ifndef LMHEAD_TMA_WIDE
#define LMHEAD_TMA_WIDE 1
#endif
#ifndef LMHEAD_HID_BOX_EXACT
#define LMHEAD_HID_BOX_EXACT 1
#endif
//   LMHEAD_HIDDEN_L2_POLICY  L2 hint for the fp32 head's hidden-row loads: 1 evict-first,
//                            2 evict-normal, 3 evict-last
#ifndef LMHEAD_HIDDEN_L2_POLICY
#define LMHEAD_HIDDEN_L2_POLICY 3
#endif

namespace lmh {

// TMA x coordinate of byte offset `bytes` within a row whose natural element is `esize` bytes.
__host__ __device__ constexpr int32_t tma_x(int64_t bytes, int esize) {
  return (int32_t)(LMHEAD_TMA_WIDE ? bytes / 4 : bytes / esize);
}

constexpr int kBM = 128;   // vocab rows per tile (MMA M)
constexpr int kBK = 64;    // K elements per pipeline stage (one 128-byte swizzle row of bf16)
constexpr int kUK = 16;    // K per tcgen05.mma of kind::f16
// Epilogue warps of the fp32 head (build-time knob): 4 (one per TMEM lane quarter) or 8 (two
// per lane quarter, each taking every other 16-column chunk of a tile).
#ifndef LMHEAD_EPI_WARPS
#define LMHEAD_EPI_WARPS 8
#endif
constexpr int kBf16EpiWarps = LMHEAD_EPI_WARPS;
constexpr int kHeadThreads = 64 + 32 * kBf16EpiWarps;
constexpr int kEpilogueThreads = 128;  // the NVFP4 head's epilogue

// Which role gave up waiting (bits 8..15 of the status word).
enum : unsigned {
  kRoleProducer = 1,
  kRoleMma = 2,
  kRoleEpilogue = 3,
  kRoleDrain = 4,
  kRoleDequant = 5,
};

constexpr unsigned kStatusTimeout = 6;  // == LMHEAD_ERR_TIMEOUT
constexpr unsigned kStatusNoRoom = 2;   // == LMHEAD_ERR_SHAPE: shared memory too small

// Waits that are expected to last (the epilogue waiting for a whole tile's MMAs) let the
// hardware suspend the thread up to this long per try instead of spinning on issue slots.
constexpr uint32_t kSleepHintNs = 2000;

struct WaitCfg {
  uint64_t limit_ns;     // wall-time limit of one barrier wait
  int32_t starve_loads;  // test-only: issue no loads, so consumers must time out
};

// First error recorded on this device since the last clear (0 = none).
static __device__ unsigned int g_lmhead_status;

__device__ __forceinline__ uint8_t* align_up_1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Spin on an mbarrier phase; false once `limit_ns` of wall time has passed or another role of
// this CTA has already given up. Every lane of the calling warp waits and the warp agrees on the
// result, so control flow stays warp-uniform.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, const WaitCfg& w,
                                             volatile int* abort_flag, uint32_t sleep_ns = 0) {
  bool ok = mbar_try_wait(bar, parity);
  if (!ok) {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t n = 1;; ++n) {
      if (sleep_ns ? mbar_try_wait_sleep(bar, parity, sleep_ns) : mbar_try_wait(bar, parity)) {
        ok = true;
        break;
      }
      if ((n & 63u) == 0) {
        if (abort_flag != nullptr && *abort_flag) break;
        if (globaltimer_ns() - t0 > w.limit_ns) break;
      }
    }
  }
  return __all_sync(0xffffffffu, ok);
}

// Which output tiles a CTA owns. A tile is 128 vocab rows by bn hidden rows, or, with `pair`
// set, 256 vocab rows by bn hidden rows computed by the two CTAs of a cluster (CTA rank k of the
// pair holds vocab rows [128 k, 128 k + 128) of it). Row tiles come in groups of `rgroup` (whose
// hidden rows fit comfortably in L2); tiles run group by group, and within a group v-major:
// t -> (v-tile, row-tile) = (local / rg, group * rgroup + local % rg), rg = the group's row
// tiles. Unit i of G (a CTA, or a CTA pair) takes t = i, i + G, i + 2G, ... At any moment the G
// units work on neighbouring v-tiles of one group: the weight stream stays on few DRAM pages,
// units share each weight tile through L2, and the group's hidden rows stay in L2 instead of
// being re-read for every v-tile (at 8192 x 4096 hidden rows, 64 MB, they did not survive the
// weight and logits streams). With rgroup >= the row tiles there is one group: plain v-major
// order. (Balanced per-CTA strips of W and splitting the last partial wave into 16-row pieces
// were both measured slower on B200.) Every tile runs the same MMA chain over K, so the
// schedule changes no output bit.
struct TileSched {
  int32_t n_rtiles;
  int32_t num_tiles;
  int32_t bn;
  int32_t n_vtiles;
  int32_t rgroup;
  int32_t pair;  // 1: units are CTA pairs (clusters of 2) and v-tiles 256 vocab rows
};

struct TileCoord {
  int64_t v0;     // first vocab row of this CTA's part
  int32_t vrows;  // vocab rows that belong to it (0..128; rows past V are zero-filled)
  int64_t r0;     // first hidden row
};

__device__ __forceinline__ int sched_count(const TileSched& s) {
  const int unit = (int)blockIdx.x >> s.pair;
  const int units = (int)gridDim.x >> s.pair;
  return unit < s.num_tiles ? (s.num_tiles - 1 - unit) / units + 1 : 0;
}

// The coordinates of tile t (this CTA's part of it, for a pair).
__device__ __forceinline__ TileCoord sched_tile_at(const TileSched& s, int64_t V, int t) {
  TileCoord c;
  const int per_group = s.n_vtiles * s.rgroup;
  const int g = t / per_group;
  const int local = t - g * per_group;
  const int left_rt = s.n_rtiles - g * s.rgroup;
  const int rg = left_rt < s.rgroup ? left_rt : s.rgroup;
  const int vt = local / rg;
  const int rt = g * s.rgroup + (local - vt * rg);
  c.v0 = ((int64_t)vt << s.pair) * kBM + (int64_t)((int)blockIdx.x & s.pair) * kBM;
  const int64_t left = V - c.v0;
  c.vrows = (int32_t)(left < 0 ? 0 : left < kBM ? left : kBM);
  c.r0 = (int64_t)rt * s.bn;
  return c;
}

// The coordinates of this unit's i-th tile under the static schedule.
__device__ __forceinline__ TileCoord sched_tile(const TileSched& s, int64_t V, int i) {
  return sched_tile_at(s, V, ((int)blockIdx.x >> s.pair) + i * ((int)gridDim.x >> s.pair));
}

__device__ __forceinline__ uint64_t l2_policy_weights() {
#if LMHEAD_WEIGHT_L2_POLICY == 1
  return l2_policy_evict_first();
#elif LMHEAD_WEIGHT_L2_POLICY == 2
  return l2_policy_evict_normal();
#else
  return 0;
#endif
}

__device__ __forceinline__ uint64_t l2_policy_hidden() {
#if LMHEAD_HIDDEN_L2_POLICY == 1
  return l2_policy_evict_first();
#elif LMHEAD_HIDDEN_L2_POLICY == 2
  return l2_policy_evict_normal();
#else
  return l2_policy_evict_last();
#endif
}

__device__ __forceinline__ void fail(unsigned role, volatile int* abort_flag) {
  atomicCAS(&g_lmhead_status, 0u, kStatusTimeout | (role << 8));
  *abort_flag = 1;
}

}  // namespace lmh
