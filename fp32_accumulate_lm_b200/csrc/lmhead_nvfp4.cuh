// W4A16 NVFP4 LM head: bf16 logits from E2M1 weights with E4M3 block scales and bf16 hidden
// rows that are never quantised (lm_head_nvfp4_rows.rs, module doc: the declared W4A16 head on
// tensor-core row tiles, bf16 logits, a row's logits independent of the row count).
//
// The weight tile is dequantised in registers to bf16 and fed to the same tcgen05 bf16 MMA
// chain as the bf16 head. W[v, k] = e2m1 * e4m3 has at most 6 significant bits and lies in
// [2^-10, 2688], so it is exact in bf16 and every product with a bf16 hidden value is exact in
// the fp32 accumulator, as for the bf16 head. The per-tensor scale g and alpha are applied in
// the epilogue: logits = bf16_rn(fl32(fl32(acc * g) * alpha)).
//
// Roles (448 threads):
//   warp 0      producer: TMA of the packed codes [128 rows x 32 bytes] and the hidden tile
//               [BN x 64] per K step of 64, plus 4-byte async copies of the block scales
//               [128 rows x 4]; all land on full[s].
//   warp 1      TMEM allocator and MMA issuer (waits on full[s] and deq_full[s]).
//   warps 2-5   epilogue.
//   warps 6-13  dequantisers: codes + scales of stage s -> bf16 tile in the 128-byte swizzled
//               K-major layout the MMA reads, then deq_full[s].
#pragma once

#include "lmhead_common.cuh"

namespace lmh {

constexpr int kNvfp4Threads = 448;
constexpr int kDequantWarp0 = 6;
constexpr int kDequantThreads = 256;

struct Nvfp4HeadParams {
  int64_t rows, H, V;
  uint16_t* out;          // bf16 logits
  const uint8_t* scales;  // [V, H/16] E4M3
  float alpha;
  float gscale;
  int32_t bn;
  int32_t n_rtiles, n_vtiles, num_tiles;
  int32_t num_kb;
  int32_t stages;
  uint32_t tmem_cols;
  uint32_t raw_bytes;  // packed codes of one stage
  uint32_t a_bytes;    // bf16 weight tile
  uint32_t b_bytes;    // bf16 hidden tile
  WaitCfg wait;
};

// Stage layout: [A bf16 16 KB][B hidden BN*128][codes 4 KB][scales 512 B][pad 512 B]
__host__ __device__ constexpr uint32_t nvfp4_stage_bytes(int bn) {
  return (uint32_t)(kBM * kBK * 2 + bn * kBK * 2 + kBM * kBK / 2 + 1024);
}

__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}

__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// bf16x2 (s', s') with s' = e4m3(code) * 2^112, exact (at most 4 significant bits, exponent
// within bf16's range).
__device__ __forceinline__ uint32_t scale_bf16x2_shifted(uint32_t code) {
  const uint32_t both = code | (code << 8);
  uint32_t h2;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
      : "=r"(h2)
      : "r"(both));
  const float f = __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu))) * 0x1p112f;
  uint32_t out;
  asm("cvt.rn.bf16x2.f32 %0, %1, %1;" : "=r"(out) : "f"(f));
  return out;
}

// Two E2M1 codes (one byte: element 2j low nibble, 2j+1 high nibble) times the block scale,
// as bf16x2 (element 2j in the low half). All steps are exact:
//   h = f16x2 of the codes; (h >> 3) & 0x0FFF0FFF keeps each magnitude's exponent and mantissa
//   in bf16 position, which reads as |q| * 2^-112 (zero stays zero); one bf16x2 multiply by
//   s * 2^112 gives |q| * s; the codes' sign bits are put back with an XOR.
__device__ __forceinline__ uint32_t dequant_pair(uint32_t byte, uint32_t s2) {
  uint32_t h;
  asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
      : "=r"(h)
      : "r"(byte));
  const uint32_t mag = (h >> 3) & 0x0FFF0FFFu;
  uint32_t p;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(p) : "r"(mag), "r"(s2));
  return p ^ (h & 0x80008000u);
}

__global__ void __launch_bounds__(kNvfp4Threads, 1)
    lmhead_w4a16_nvfp4_kernel(const __grid_constant__ CUtensorMap tmap_q,
                              const __grid_constant__ CUtensorMap tmap_h,
                              const Nvfp4HeadParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_up_1024(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S = p.stages;
  const uint32_t stage_bytes = nvfp4_stage_bytes(p.bn);
  const uint32_t off_b = p.a_bytes;
  const uint32_t off_q = p.a_bytes + p.b_bytes;
  const uint32_t off_s = off_q + p.raw_bytes;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)S * stage_bytes);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t deq0 = smem_u32(bars + S);
  const uint32_t empty0 = smem_u32(bars + 2 * S);
  const uint32_t tfull0 = smem_u32(bars + 3 * S);
  const uint32_t tempty0 = smem_u32(bars + 3 * S + 2);
  const uint32_t done_bar = smem_u32(bars + 3 * S + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * S + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 1 + 32);  // expect_tx arrive + 32 scale-copy arrivals
      mbar_init(deq0 + 8 * s, kDequantThreads);
      mbar_init(empty0 + 8 * s, 1);
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
    prefetch_tmap(&tmap_h);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const int64_t scale_pitch = p.H / 16;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    const uint64_t pol_w = l2_policy_evict_first();
    const uint64_t pol_h = l2_policy_evict_last();
    const uint32_t tx_bytes = p.raw_bytes + p.b_bytes;
    int stage = 0;
    uint32_t phase = 0;
    int issued = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
      const int vt = tile / p.n_rtiles;
      const int rt = tile - vt * p.n_rtiles;
      for (int kb = 0; kb < p.num_kb; ++kb) {
        if (!wait_bounded(empty0 + 8 * stage, phase ^ 1u, p.wait, abort_flag)) {
          fail(kRoleProducer, abort_flag);
          ok = false;
          break;
        }
        if (!p.wait.starve_loads) {
          const uint32_t full = full0 + 8 * stage;
          const uint32_t sbase = smem_u32(smem + (size_t)stage * stage_bytes);
          if (lane == 0) {
            mbar_arrive_expect_tx(full, tx_bytes);
            tma_load_2d(sbase + off_q, &tmap_q, full, kb * (kBK / 2), vt * kBM, pol_w);
            tma_load_2d(sbase + off_b, &tmap_h, full, kb * kBK, rt * p.bn, pol_h);
          }
          // Block scales: 4 bytes (one K step) for each of the 128 rows, 4 rows per lane.
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int row = lane * 4 + i;
            const int64_t v = (int64_t)vt * kBM + row;
            const bool in = v < p.V;
            const uint8_t* src = p.scales + (in ? v : 0) * scale_pitch + (int64_t)kb * 4;
            cp_async_4(sbase + off_s + (uint32_t)row * 4, src, in ? 4u : 0u);
          }
          cp_async_arrive_noinc(full);
        }
        __syncwarp();
        ++issued;
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!p.wait.starve_loads) {
      const int outstanding = issued < S ? issued : S;
      for (int i = 0; i < outstanding; ++i) {
        if (--stage < 0) {
          stage = S - 1;
          phase ^= 1u;
        }
        if (!wait_bounded(full0 + 8 * stage, phase, p.wait, nullptr)) {
          fail(kRoleDrain, abort_flag);
          break;
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    const uint32_t idesc = idesc_bf16_f32(kBM, p.bn);
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
      if (!wait_bounded(tempty0 + 8 * acc, acc_phase ^ 1u, p.wait, abort_flag)) {
        fail(kRoleMma, abort_flag);
        break;
      }
      tc_fence_after_sync();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * p.bn);
      for (int kb = 0; kb < p.num_kb; ++kb) {
        if (!wait_bounded(full0 + 8 * stage, phase, p.wait, abort_flag) ||
            !wait_bounded(deq0 + 8 * stage, phase, p.wait, abort_flag)) {
          fail(kRoleMma, abort_flag);
          ok = false;
          break;
        }
        tc_fence_after_sync();
        if (lane == 0) {
          const uint32_t sa = smem_u32(smem + (size_t)stage * stage_bytes);
          const uint32_t sb = sa + off_b;
#pragma unroll
          for (int k = 0; k < kBK / kUK; ++k) {
            mma_bf16_ss(d_tmem, sdesc_kmajor_sw128(sa + k * kUK * 2),
                        sdesc_kmajor_sw128(sb + k * kUK * 2), idesc, (kb | k) != 0);
          }
          mma_commit(empty0 + 8 * stage);
        }
        __syncwarp();
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (lane == 0) mma_commit(tfull0 + 8 * acc);
      __syncwarp();
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (lane == 0) mma_commit(done_bar);
    __syncwarp();
    if (!wait_bounded(done_bar, 0, p.wait, nullptr)) fail(kRoleDrain, abort_flag);
  } else if (warp < kDequantWarp0) {
    // ---------------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int v_local = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
      const int vt = tile / p.n_rtiles;
      const int rt = tile - vt * p.n_rtiles;
      if (!wait_bounded(tfull0 + 8 * acc, acc_phase, p.wait, abort_flag)) {
        fail(kRoleEpilogue, abort_flag);
        break;
      }
      tc_fence_after_sync();
      const int64_t v = (int64_t)vt * kBM + v_local;
      const int64_t r0 = (int64_t)rt * p.bn;
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * p.bn);
      const bool v_ok = v < p.V;
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
              const float y = __fmul_rn(__fmul_rn(__uint_as_float(r[j]), p.gscale), p.alpha);
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
    // Thread -> (row, half): 16 rows per warp, two threads per row, each 32 elements (16 code
    // bytes, two scale blocks). A quarter-warp covers 128 contiguous code bytes (no bank
    // conflicts), and its 16-byte stores land in 8 distinct swizzled chunks.
    const int dw = warp - kDequantWarp0;
    const int row = dw * 16 + (lane >> 1);
    const int half = lane & 1;
    const uint32_t sw = (uint32_t)(row & 7);
    int stage = 0;
    uint32_t phase = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
      bool ok = true;
      for (int kb = 0; kb < p.num_kb; ++kb) {
        if (!wait_bounded(full0 + 8 * stage, phase, p.wait, abort_flag)) {
          fail(kRoleDequant, abort_flag);
          ok = false;
          break;
        }
        uint8_t* sbase = smem + (size_t)stage * stage_bytes;
        const uint4 codes = *reinterpret_cast<const uint4*>(sbase + off_q + row * 32 + half * 16);
        const uint32_t sc = *reinterpret_cast<const uint16_t*>(sbase + off_s + row * 4 + half * 2);
        const uint32_t s_lo = scale_bf16x2_shifted(sc & 0xFFu);
        const uint32_t s_hi = scale_bf16x2_shifted(sc >> 8);
        const uint32_t cw[4] = {codes.x, codes.y, codes.z, codes.w};
        uint8_t* arow = sbase + row * 128;
#pragma unroll
        for (int q = 0; q < 4; ++q) {  // 16-byte chunk = 8 elements = 4 code bytes
          const uint32_t s2 = q < 2 ? s_lo : s_hi;
          uint4 o;
          o.x = dequant_pair(cw[q] & 0xFFu, s2);
          o.y = dequant_pair((cw[q] >> 8) & 0xFFu, s2);
          o.z = dequant_pair((cw[q] >> 16) & 0xFFu, s2);
          o.w = dequant_pair(cw[q] >> 24, s2);
          const uint32_t chunk = (uint32_t)(half * 4 + q);
          *reinterpret_cast<uint4*>(arow + ((chunk ^ sw) << 4)) = o;
        }
        fence_proxy_async_smem();
        mbar_arrive(deq0 + 8 * stage);
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

}  // namespace lmh
