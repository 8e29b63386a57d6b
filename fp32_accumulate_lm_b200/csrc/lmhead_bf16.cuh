// fp32-accumulate LM head, bf16 or fp16 operands:
//   logits[r, v] = fl32(alpha * sum_k h[r, k] * W[v, k])                       (no bias)
//   logits[r, v] = fl32(alpha * fl32(sum_k h[r, k] * W[v, k] + bias[v]))      (with bias)
// ("[Model] Honor fp32 head_dtype in Inkling muP logits", "Purpose": the projection with its
// embedding bias, then the multiply by 1/mup; "FP32 LM head skip FP32 cast": fp16 or bf16
// hidden states of the weight's dtype, fp32 accumulation and output).
//
// One persistent, warp-specialised tcgen05 kernel serves every row count (decode, speculative
// verify and prefill alike), so a row's reduction order never depends on how many rows a call
// carries. lm_head_nvfp4_rows.rs (module doc) promises this for its NVFP4 head; it is applied
// here to the bf16 head as well.
//
// Orientation ("swap-AB"): W supplies the MMA's M = 128 side and the hidden rows the N side, so
// a handful of decode rows pads N (16..256 in steps of 16), never M, and each TMEM lane holds one
// vocab entry: the epilogue's 32 lanes of a warp write 32 consecutive logits of one row.
//
// Roles (64 + 32 * kBf16EpiWarps threads: 320 with the default 8 epilogue warps):
//   warp 0     TMA producer: per pipeline stage, NSUB sub-tiles of 64 K-elements each of W
//              [128 x 64] and of the hidden rows [BN x 64] (128-byte swizzle), landing on full[s].
//   warp 1     TMEM allocator and MMA issuer: 4 * NSUB tcgen05.mma (K = 16 each) per stage into
//              one of two TMEM accumulators; tcgen05.commit frees the stage (empty[s]) and, after
//              the last K step, hands the accumulator to the epilogue (tmem_full[a]).
//   warps 2-9  epilogue (two warps per TMEM lane quarter, warp w on quarter w % 4, each taking
//              every other 16-column chunk; with 4 epilogue warps, warps 2-5 take all chunks):
//              tcgen05.ld of the accumulator, the bias (one IEEE fp32 add) if any, one
//              IEEE fp32 multiply by alpha, store. In log-prob mode the logits are not stored:
//              each warp reduces its 32 vocab entries to (max, sum of exp(z - max)) per row
//              and writes that pair to the workspace, and the lane holding a row's target token
//              writes that logit; a combine kernel (lmhead_logprob_combine_kernel) finishes,
//              or, when W is one vocab slice of a larger head, writes the row's (max, sum,
//              target logit) for lmhead_logprob_merge_shards_kernel to fold across slices.
// Tile ownership: see TileSched.
#pragma once

#include "lmhead_common.cuh"

namespace lmh {

// Copies of the logits one call can write (the vocab-slice entry: one per GPU of the group).
constexpr int kMaxLogitCopies = 8;

struct Bf16HeadParams {
  int64_t rows, H, V;
  // logits row r, vocab entry v at out[d][r * ld_out + v] for every d < n_out (n_out >= 1)
  float* out[kMaxLogitCopies];
  int32_t n_out;
  int64_t ld_out;
  const uint16_t* bias;  // [V] in the operand type, or null
  float alpha;
  int32_t fp16;          // operands (and bias) are IEEE fp16, else bf16
  int32_t bn;        // rows per tile: multiple of 16 in [16, 256]
  int32_t hid_rows;  // rows of hidden one TMA box brings (<= bn; MMA columns past it unused)
  TileSched sched;
  int32_t clc;       // 1: units take their tiles after the first by cluster launch control
  int32_t num_ks;    // pipeline stages per tile: ceil(H / (64 * NSUB))
  int32_t stages;
  uint32_t tmem_cols;
  uint32_t stage_bytes;
  // log-prob mode (logprob != 0): no logits are written; see the epilogue
  int32_t logprob;
  int32_t n_chunks;         // 32-entry vocab chunks per row: 4 * ceil(V / 128)
  float2* partials;         // [n_chunks, rows] (max, sum of exp(z - max)) per chunk and row
  const int32_t* targets;   // [rows] token ids
  int64_t target_base;      // vocab id of W's first row (a vocab shard's offset; 0 otherwise)
  float* target_z;          // the target's logit, row r at target_z[r * tz_stride] (written by
  int32_t tz_stride;        // the chunk that holds it)
  WaitCfg wait;
};

// (m, s) pairs standing for the partial sums s * exp(m): the pair of their union, with no branch
// (lanes of a warp take different sides). Symmetric in its two arguments bit for bit; a pair
// with s = 0 (no entries) contributes nothing.
__device__ __forceinline__ void merge_max_sum(float m1, float s1, float m2, float s2, float& m,
                                              float& s) {
  const bool first = m1 >= m2;
  const float big = first ? s1 : s2;
  const float small = first ? s2 : s1;
  m = first ? m1 : m2;
  const float e = __expf(__fsub_rn(first ? m2 : m1, m));
  s = small > 0.0f ? __fadd_rn(big, __fmul_rn(small, e)) : big;
}

// Log-sum-exp of each row from its chunk pairs, then logprob = z[target] - lse. A block of 32
// warps serves 32 rows: lane i is row i; warp w folds chunk segment w in order (coalesced reads
// of the chunk-major pairs), then warp 0 folds the 32 segment pairs of its row in order. The
// result depends only on the row's logits and V.
//
// With `stats` set (one vocab shard of a larger head, whose first row is vocab id v_begin), the
// row's pair and target logit are written instead: stats[3 r .. 3 r + 2] = (max, sum of
// exp(z - max), z[target]), the last NaN when the shard does not hold the target. The main
// kernel left z[target] in stats[3 r + 2].
constexpr int kCombineRows = 32;
__global__ void __launch_bounds__(1024)
    lmhead_logprob_combine_kernel(const float2* __restrict__ partials, int32_t n_chunks,
                                  int64_t rows, int64_t V, const int32_t* __restrict__ targets,
                                  float* logprobs, float* lse_out, int64_t v_begin,
                                  float* stats) {
  __shared__ float2 seg[32][kCombineRows + 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kCombineRows + lane;
  const int per_seg = (n_chunks + 31) / 32;
  const int c0 = warp * per_seg;
  const int c1 = min(n_chunks, c0 + per_seg);
  float m = -INFINITY, s = 0.0f;
  if (row < rows) {
    for (int c = c0; c < c1; ++c) {
      const float2 q = partials[(int64_t)c * rows + row];
      merge_max_sum(m, s, q.x, q.y, m, s);
    }
  }
  seg[warp][lane] = make_float2(m, s);
  __syncthreads();
  if (warp == 0 && row < rows) {
    m = -INFINITY;
    s = 0.0f;
    for (int w = 0; w < 32; ++w) merge_max_sum(m, s, seg[w][lane].x, seg[w][lane].y, m, s);
    const int64_t t = (int64_t)targets[row] - v_begin;
    const bool held = t >= 0 && t < V;
    if (stats != nullptr) {
      stats[3 * row] = m;
      stats[3 * row + 1] = s;
      if (!held) stats[3 * row + 2] = __int_as_float(0x7fc00000);
      return;
    }
    const float l = __fadd_rn(m, logf(s));
    if (lse_out != nullptr) lse_out[row] = l;
    logprobs[row] = held ? __fsub_rn(logprobs[row], l) : __int_as_float(0x7fc00000);
  }
}

// The vocab-parallel finish: stats [shards][rows][3] holds each shard's (max, sum, target logit)
// of every row; fold the shards in order into the row's pair, then lse = max + log(sum) and
// logprob = z[target] - lse, taking z[target] from the first shard that holds it (NaN if none).
// One thread per row; the reads of a warp are 12-byte strided, a few KB per call.
constexpr int kMergeThreads = 256;
__global__ void __launch_bounds__(kMergeThreads)
    lmhead_logprob_merge_shards_kernel(const float* __restrict__ stats, int32_t shards,
                                       int64_t rows, float* logprobs, float* lse_out) {
  const int64_t row = (int64_t)blockIdx.x * kMergeThreads + threadIdx.x;
  if (row >= rows) return;
  float m = -INFINITY, s = 0.0f, zt = __int_as_float(0x7fc00000);
  bool found = false;
  for (int g = 0; g < shards; ++g) {
    const float* q = stats + 3 * ((int64_t)g * rows + row);
    merge_max_sum(m, s, q[0], q[1], m, s);
    const float z = q[2];
    if (!found && !isnan(z)) {
      zt = z;
      found = true;
    }
  }
  const float l = __fadd_rn(m, logf(s));
  if (lse_out != nullptr) lse_out[row] = l;
  logprobs[row] = __fsub_rn(zt, l);
}

// Tile streams. Every role walks the same tiles of its unit in the same order: under the static
// schedule tile j is unit + j * units while j < the unit's count; under cluster launch control
// (one unit launched per tile) tile 0 is the unit's own and tile j >= 1 comes from the j-th
// answer, which the leader's producer asks for when it starts tile j - 1. The answers live in a
// ring of kClcSlots 16-byte slots: full[k] counts the answer's 16 bytes, empty[k] the reads of
// every role that takes tile ids (the leader's MMA warp, both CTAs' producers and epilogue
// warps), so a slot is asked again only after all of them have read it.
constexpr int kClcSlots = 4;

struct ClcRing {
  uint32_t resp0, full0, empty0;
};

// Tile j (j >= 1) of this unit from the cluster launch control answers, or -1 when none is left
// (or the wait gave up; `ok` is then false). The whole warp reads the answer; lane 0 releases
// the slot on the pair leader's empty barrier.
template <bool kPair>
__device__ __forceinline__ int clc_take(const ClcRing& r, int j, const WaitCfg& w,
                                        volatile int* abort_flag, bool& ok) {
  const int slot = (j - 1) % kClcSlots;
  const uint32_t phase = (uint32_t)((j - 1) / kClcSlots) & 1u;
  if (!wait_bounded(r.full0 + 8 * slot, phase, w, abort_flag)) {
    ok = false;
    return -1;
  }
  const int x = clc_first_ctaid_x(r.resp0 + 16 * slot);
  __syncwarp();
  if ((threadIdx.x & 31) == 0) {
    if constexpr (kPair) {
      mbar_arrive_remote(r.empty0 + 8 * slot, 0);
    } else {
      mbar_arrive(r.empty0 + 8 * slot);
    }
  }
  return x < 0 ? -1 : (x >> (kPair ? 1 : 0));
}

// The leader's producer asks for tile j (j >= 1) of its unit. Both CTAs' full barriers are
// armed for the 16-byte answer before the request goes out.
template <bool kPair>
__device__ __forceinline__ bool clc_ask(const ClcRing& r, int j, const WaitCfg& w,
                                        volatile int* abort_flag) {
  const int slot = (j - 1) % kClcSlots;
  const uint32_t phase = ((uint32_t)((j - 1) / kClcSlots) & 1u) ^ 1u;
  if (!wait_bounded(r.empty0 + 8 * slot, phase, w, abort_flag)) return false;
  if ((threadIdx.x & 31) == 0) {
    mbar_arrive_expect_tx(r.full0 + 8 * slot, 16);
    if constexpr (kPair) {
      mbar_arrive_expect_tx_remote(r.full0 + 8 * slot, 1, 16);
      clc_try_cancel_all(r.resp0 + 16 * slot, r.full0 + 8 * slot);
    } else {
      clc_try_cancel(r.resp0 + 16 * slot, r.full0 + 8 * slot);
    }
  }
  __syncwarp();
  return true;
}

template <int NSUB, bool kPair>
__global__ void __launch_bounds__(kHeadThreads, 1)
    lmhead_bf16_f32_kernel(const __grid_constant__ CUtensorMap tmap_w,
                           const __grid_constant__ CUtensorMap tmap_h, const Bf16HeadParams p) {
  extern __shared__ uint8_t smem_raw[];
  if (threadIdx.x == 0) pdl_trigger();
  uint8_t* smem = align_up_1024(smem_raw);
  // Broadcast from lane 0 so the compiler can prove role branches warp-uniform and keep their
  // counters and descriptors in uniform registers.
  const int warp = __shfl_sync(0xffffffffu, (int)(threadIdx.x >> 5), 0);
  const int lane = threadIdx.x & 31;
  const int S = p.stages;
  // CTA pair: rank 0 (the leader) issues the MMAs and owns the full barriers; both CTAs load
  // their halves, and both run an epilogue over their own TMEM rows.
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;

  // stage s: [A sub-tile 0 .. NSUB-1, 16 KB each][B sub-tile 0 .. NSUB-1, b_sub bytes each]
  // (a CTA pair: this CTA's 128 W rows and its half of the bn hidden rows)
  constexpr uint32_t a_sub = kBM * kBK * 2;
  const uint32_t b_sub = (uint32_t)(kPair ? p.bn / 2 : p.bn) * kBK * 2;
  const uint32_t b_tx = (uint32_t)p.hid_rows * kBK * 2;
  uint8_t* stage_base = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)S * p.stage_bytes);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = smem_u32(bars + S);
  const uint32_t tfull0 = smem_u32(bars + 2 * S);
  const uint32_t tempty0 = smem_u32(bars + 2 * S + 2);
  const uint32_t done_bar = smem_u32(bars + 2 * S + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // cluster launch control: 4 answer slots (16-byte aligned), then their full and empty barriers
  const ClcRing clc{smem_u32(bars + 2 * S + 6), smem_u32(bars + 2 * S + 14),
                    smem_u32(bars + 2 * S + 18)};
  // readers of an answer: both CTAs' producers and epilogue warps, the leader's MMA warp
  constexpr uint32_t kClcReaders = (kPair ? 2u : 1u) * (1u + kBf16EpiWarps) + 1u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int k = 0; k < kClcSlots; ++k) {
      mbar_init(clc.full0 + 8 * k, 1);
      mbar_init(clc.empty0 + 8 * k, kClcReaders);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull0 + 8 * a, 1);
      // a pair's accumulator is free once both CTAs' epilogues have read their rows
      mbar_init(tempty0 + 8 * a, (kPair ? 2 : 1) * 32 * kBf16EpiWarps);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_w);
    prefetch_tmap(&tmap_h);
  }
  if (warp == 1) {
    if constexpr (kPair) {
      tmem_alloc_pair(smem_u32(tmem_slot), p.tmem_cols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), p.tmem_cols);
      tmem_relinquish();
    }
  }
  tc_fence_before_sync();
  if constexpr (kPair) {
    cluster_sync_all();  // both CTAs' barriers are initialised before either signals the other's
  } else {
    __syncthreads();
  }
  tc_fence_after_sync();
  pdl_wait();  // from here on global memory: earlier kernels of the stream are done
  const uint32_t tmem_base = *tmem_slot;
  const int my_tiles = sched_count(p.sched);
  const int unit = (int)blockIdx.x >> (kPair ? 1 : 0);
  const int units = (int)gridDim.x >> (kPair ? 1 : 0);
  // this unit's first tile; -1 when the static schedule gives it none
  const int first_tile = my_tiles > 0 ? unit : -1;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    const uint64_t pol_w = l2_policy_weights();
    const uint64_t pol_h = l2_policy_hidden();  // hidden rows are re-read per v-tile
    int stage = 0;
    uint32_t phase = 0;
    int issued = 0;
    bool ok = true;
    int asked = 0;  // cluster launch control requests issued (answers read: j below)
    int tile = first_tile;
    for (int j = 0; ok && tile >= 0; ++j) {
      // ask for the next tile as this one starts, so the answer is in before it is needed
      if (p.clc && leader) {
        if (!clc_ask<kPair>(clc, j + 1, p.wait, abort_flag)) {
          fail(kRoleProducer, abort_flag);
          break;
        }
        asked = j + 1;
      }
      const TileCoord tc = sched_tile_at(p.sched, p.V, tile);
      // a pair's full barrier (the leader's) counts both CTAs' bytes
      const uint32_t tx = (uint32_t)NSUB * (a_sub + b_tx) * (kPair ? 2u : 1u);
      const int32_t hid_y = (int32_t)(tc.r0 + (kPair ? (int64_t)rank * (p.bn / 2) : 0));
      for (int ks = 0; ks < p.num_ks; ++ks) {
        if (!wait_bounded(empty0 + 8 * stage, phase ^ 1u, p.wait, abort_flag)) {
          fail(kRoleProducer, abort_flag);
          ok = false;
          break;
        }
        if (lane == 0 && !p.wait.starve_loads) {
          const uint32_t full = full0 + 8 * stage;
          const uint32_t sa = smem_u32(stage_base + (size_t)stage * p.stage_bytes);
          const uint32_t sb = sa + NSUB * a_sub;
          if (leader) mbar_arrive_expect_tx(full, tx);
#pragma unroll
          for (int j = 0; j < NSUB; ++j) {
            const int32_t x = tma_x((ks * NSUB + j) * kBK * 2, 2);
            if constexpr (kPair) {
              tma_load_2d_pair(sa + j * a_sub, &tmap_w, full, x, (int32_t)tc.v0, pol_w);
              tma_load_2d_pair(sb + j * b_sub, &tmap_h, full, x, hid_y, pol_h);
            } else {
              tma_load_2d(sa + j * a_sub, &tmap_w, full, x, (int32_t)tc.v0, pol_w);
              tma_load_2d(sb + j * b_sub, &tmap_h, full, x, hid_y, pol_h);
            }
          }
        }
        __syncwarp();
        ++issued;
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (p.clc) {
        tile = clc_take<kPair>(clc, j + 1, p.wait, abort_flag, ok);
        if (!ok) fail(kRoleProducer, abort_flag);
      } else {
        tile = j + 1 < my_tiles ? unit + (j + 1) * units : -1;
      }
    }
    // An answer asked for but not read (an error path) must still land before the CTA exits.
    if (p.clc && leader && asked > 0) {
      const int slot = (asked - 1) % kClcSlots;
      const uint32_t ph = (uint32_t)((asked - 1) / kClcSlots) & 1u;
      if (!wait_bounded(clc.full0 + 8 * slot, ph, p.wait, nullptr)) fail(kRoleDrain, abort_flag);
    }
    // Drain: every load this CTA issued must land before the CTA may exit. A lone CTA sees that
    // on its full barriers. A pair's loads are counted on the leader's full barriers, so both
    // CTAs wait instead until the MMAs have released every stage they filled (which they do only
    // after the stage's bytes arrived).
    if (!p.wait.starve_loads) {
      const int outstanding = issued < S ? issued : S;
      for (int i = 0; i < outstanding; ++i) {
        if (--stage < 0) {
          stage = S - 1;
          phase ^= 1u;
        }
        // the fill's round parity: its completion on full, its release on empty
        if (!wait_bounded((kPair ? empty0 : full0) + 8 * stage, phase, p.wait, nullptr)) {
          fail(kRoleDrain, abort_flag);
          break;
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // (a CTA pair: the leader's warp issues for both CTAs; the other CTA's warp only holds the
    // pair's TMEM allocation)
    const uint32_t idesc = idesc_f16kind_f32(kPair ? 2 * kBM : kBM, p.bn, p.fp16 == 0);
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    int tile = leader ? first_tile : -1;
    for (int tj = 0; ok && tile >= 0; ++tj) {
      if (!wait_bounded(tempty0 + 8 * acc, acc_phase ^ 1u, p.wait, abort_flag)) {
        fail(kRoleMma, abort_flag);
        break;
      }
      tc_fence_after_sync();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * p.bn);
      for (int ks = 0; ks < p.num_ks; ++ks) {
        if (!wait_bounded(full0 + 8 * stage, phase, p.wait, abort_flag)) {
          fail(kRoleMma, abort_flag);
          ok = false;
          break;
        }
        tc_fence_after_sync();
        {
          const uint32_t sa = smem_u32(stage_base + (size_t)stage * p.stage_bytes);
          const uint64_t adesc0 = sdesc_kmajor_sw128(sa);
          const uint64_t bdesc0 = sdesc_kmajor_sw128(sa + NSUB * a_sub);
#pragma unroll
          for (int j = 0; j < NSUB; ++j) {
            // descriptor start addresses are in 16-byte units
            const uint64_t ad = adesc0 + (uint64_t)((j * a_sub) >> 4);
            const uint64_t bd = bdesc0 + (uint64_t)((j * b_sub) >> 4);
            if constexpr (kPair) {
              mma4_bf16_ss_pair_elect(d_tmem, ad, bd, idesc, (ks | j) != 0);
            } else {
              mma4_bf16_ss_elect(d_tmem, ad, bd, idesc, (ks | j) != 0);
            }
          }
          // frees the stage in both CTAs of a pair
          if constexpr (kPair) {
            mma_commit_pair_elect(empty0 + 8 * stage, 0x3);
          } else {
            mma_commit_elect(empty0 + 8 * stage);
          }
        }
        __syncwarp();
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if constexpr (kPair) {
        mma_commit_pair_elect(tfull0 + 8 * acc, 0x3);
      } else {
        mma_commit_elect(tfull0 + 8 * acc);
      }
      __syncwarp();
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
      if (p.clc) {
        tile = clc_take<kPair>(clc, tj + 1, p.wait, abort_flag, ok);
        if (!ok) fail(kRoleMma, abort_flag);
      } else {
        tile = tj + 1 < my_tiles ? unit + (tj + 1) * units : -1;
      }
    }
    // Every MMA this warp issued must finish before TMEM is released (a pair's other CTA
    // learns it at the closing cluster barrier).
    if (leader) {
      if constexpr (kPair) {
        mma_commit_pair_elect(done_bar, 0x1);
      } else {
        mma_commit_elect(done_bar);
      }
      __syncwarp();
      if (!wait_bounded(done_bar, 0, p.wait, nullptr)) fail(kRoleDrain, abort_flag);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    // with two warps per lane quarter, each takes every other 16-column chunk of the tile
    const int half = kBf16EpiWarps == 8 ? (warp - 2) >> 2 : 0;
    constexpr int kChunkStep = kBf16EpiWarps == 8 ? 32 : 16;
    const int v_local = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    int tile = first_tile;
    for (int tj = 0; ok && tile >= 0; ++tj) {
      const TileCoord tc = sched_tile_at(p.sched, p.V, tile);
      if (!wait_bounded(tfull0 + 8 * acc, acc_phase, p.wait, abort_flag, kSleepHintNs)) {
        fail(kRoleEpilogue, abort_flag);
        break;
      }
      tc_fence_after_sync();
      const int64_t v = tc.v0 + v_local;
      const int64_t r0 = tc.r0;
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * p.bn);
      const bool v_ok = v_local < tc.vrows;
      // This lane's vocab entry's bias, decoded exactly to fp32 (null: none, and no add).
      float b = 0.0f;
      if (p.bias != nullptr && v_ok) {
        const uint16_t bits = p.bias[v];
        b = p.fp16 ? __half2float(__ushort_as_half(bits)) : __uint_as_float((uint32_t)bits << 16);
      }
      // (a pair's odd CTA holds no vocab rows of the last v-tile when V % 256 <= 128)
      for (int c = 16 * half; tc.vrows > 0 && c < p.bn; c += kChunkStep) {
        if (r0 + c >= p.rows) break;  // warp-uniform
        uint32_t r[16];
        tmem_ld_32x32b_x16(taddr + (uint32_t)c, r);
        tmem_ld_wait();
        if (p.logprob) {
          // This warp's 32 vocab entries of rows r0 + c + j: the same fp32 logits the store
          // path writes, reduced per row to (max, sum of exp(z - max)) in two butterfly phases
          // over the lanes, so lanes 2i and 2i + 1 both hold row i's pair.
          const int32_t chunk = (int32_t)(tc.v0 / kBM) * 4 + quarter;
          const int64_t rl = r0 + c + lane;
          // The target as an index into this call's W (-1 when W does not hold it).
          int32_t tgt = -1;
          if (lane < 16 && rl < p.rows) {
            const int64_t tv = (int64_t)p.targets[rl] - p.target_base;
            tgt = (tv >= 0 && tv < p.V) ? (int32_t)tv : -1;
          }
          // Which of these 16 rows has its target among this warp's 32 entries (usually none).
          const int64_t wv0 = tc.v0 + quarter * 32;
          const uint32_t hits = __ballot_sync(0xffffffffu, tgt >= wv0 && tgt < wv0 + 32);
          float zz[16], pm[16], ps[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float a = __uint_as_float(r[j]);
            const float z = !v_ok ? -INFINITY
                            : p.bias == nullptr ? __fmul_rn(p.alpha, a)
                                                : __fmul_rn(p.alpha, __fadd_rn(a, b));
            if (hits & (1u << j)) {  // warp-uniform
              const int32_t tj = __shfl_sync(0xffffffffu, tgt, j);
              if (v_ok && v == (int64_t)tj) p.target_z[(r0 + c + j) * p.tz_stride] = z;
            }
            zz[j] = z;
            pm[j] = z;
          }
          // Phase 1, the maxima: butterfly over the lanes, each step keeping half the rows; lanes
          // 2i and 2i + 1 end with row i's max, which every lane then fetches.
#pragma unroll
          for (int w = 8, off = 16; w >= 1; w >>= 1, off >>= 1) {
            const bool upper = (lane & off) != 0;
#pragma unroll
            for (int j = 0; j < w; ++j) {
              const float keep = upper ? pm[j + w] : pm[j];
              const float send = upper ? pm[j] : pm[j + w];
              pm[j] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, off));
            }
          }
          pm[0] = fmaxf(pm[0], __shfl_xor_sync(0xffffffffu, pm[0], 1));
          // Phase 2, the sums of exp(z - max), the same butterfly with adds.
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float mj = __shfl_sync(0xffffffffu, pm[0], 2 * j);
            ps[j] = v_ok ? __expf(__fsub_rn(zz[j], mj)) : 0.0f;
          }
#pragma unroll
          for (int w = 8, off = 16; w >= 1; w >>= 1, off >>= 1) {
            const bool upper = (lane & off) != 0;
#pragma unroll
            for (int j = 0; j < w; ++j) {
              const float keep = upper ? ps[j + w] : ps[j];
              const float send = upper ? ps[j] : ps[j + w];
              const float got = __shfl_xor_sync(0xffffffffu, send, off);
              // the lower lane's half first, so partners add in the same order
              ps[j] = upper ? __fadd_rn(got, keep) : __fadd_rn(keep, got);
            }
          }
          {
            const float got = __shfl_xor_sync(0xffffffffu, ps[0], 1);
            ps[0] = (lane & 1) ? __fadd_rn(got, ps[0]) : __fadd_rn(ps[0], got);
          }
          const int64_t row = r0 + c + ((lane >> 1) & 15);
          // A streaming (evict-first) store, like the logits': with the default priority these
          // pairs (0.3 GB at the prefill shape) would outrank the evict-first weight tiles in L2
          // and push them out before the other row tiles of their group read them.
          if ((lane & 1) == 0 && row < p.rows)
            __stcs(p.partials + (int64_t)chunk * p.rows + row, make_float2(pm[0], ps[0]));
          continue;
        }
        if (v_ok) {
          float z[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            z[j] = p.bias == nullptr ? __fmul_rn(p.alpha, __uint_as_float(r[j]))
                                     : __fmul_rn(p.alpha, __fadd_rn(__uint_as_float(r[j]), b));
          const int64_t off = (r0 + c) * p.ld_out + v;
          if (p.n_out == 1) {  // warp-uniform
            float* dst = p.out[0] + off;
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (r0 + c + j < p.rows) __stcs(dst + (int64_t)j * p.ld_out, z[j]);
          } else {
            // every copy of the logits (a vocab slice's columns in each GPU's buffer); the
            // index into the parameter array stays a constant
#pragma unroll
            for (int d = 0; d < kMaxLogitCopies; ++d) {
              if (d < p.n_out) {  // warp-uniform
                float* dst = p.out[d] + off;
#pragma unroll
                for (int j = 0; j < 16; ++j)
                  if (r0 + c + j < p.rows) __stcs(dst + (int64_t)j * p.ld_out, z[j]);
              }
            }
          }
        }
      }
      tc_fence_before_sync();
      if constexpr (kPair) {
        mbar_arrive_remote(tempty0 + 8 * acc, 0);  // the leader's barrier, counting both CTAs
      } else {
        mbar_arrive(tempty0 + 8 * acc);
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
      if (p.clc) {
        tile = clc_take<kPair>(clc, tj + 1, p.wait, abort_flag, ok);
        if (!ok) fail(kRoleEpilogue, abort_flag);
      } else {
        tile = tj + 1 < my_tiles ? unit + (tj + 1) * units : -1;
      }
    }
  }

  tc_fence_before_sync();
  if constexpr (kPair) {
    // Neither CTA releases the pair's TMEM or exits while the other may still signal its
    // barriers or the leader's MMAs may still read its tiles.
    cluster_sync_all();
  } else {
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after_sync();
    if constexpr (kPair) {
      tmem_dealloc_pair(tmem_base, p.tmem_cols);
    } else {
      tmem_dealloc(tmem_base, p.tmem_cols);
    }
  }
}

}  // namespace lmh
