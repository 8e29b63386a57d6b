// Pieces shared by the LM-head kernels: tile constants, the bounded barrier wait, and the
// per-device status word that a timed-out wait writes.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sm100_ptx.cuh"

namespace lmh {

constexpr int kBM = 128;   // vocab rows per tile (MMA M)
constexpr int kBK = 64;    // K elements per pipeline stage (one 128-byte swizzle row of bf16)
constexpr int kUK = 16;    // K per tcgen05.mma of kind::f16
constexpr int kHeadThreads = 192;
constexpr int kEpilogueThreads = 128;

// Which role gave up waiting (bits 8..15 of the status word).
enum : unsigned {
  kRoleProducer = 1,
  kRoleMma = 2,
  kRoleEpilogue = 3,
  kRoleDrain = 4,
  kRoleDequant = 5,
};

constexpr unsigned kStatusTimeout = 6;  // == LMHEAD_ERR_TIMEOUT

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
                                             volatile int* abort_flag) {
  bool ok = mbar_try_wait(bar, parity);
  if (!ok) {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t n = 1;; ++n) {
      if (mbar_try_wait(bar, parity)) {
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

__device__ __forceinline__ void fail(unsigned role, volatile int* abort_flag) {
  atomicCAS(&g_lmhead_status, 0u, kStatusTimeout | (role << 8));
  *abort_flag = 1;
}

}  // namespace lmh
