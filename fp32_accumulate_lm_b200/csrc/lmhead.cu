// C ABI of the LM-head library (declared in include/lmhead.h): argument validation, TMA
// descriptor set-up and the launches on the caller's stream (one kernel per head call; two for
// the log-probabilities and for the quantiser; one for the vocab-slice merge).
//
// The operation: logits = alpha * hidden @ W^T with bf16 inputs, fp32 accumulation and alpha in
// the epilogue ("[Model] Honor fp32 head_dtype in Inkling muP logits (target + MTP draft)",
// "muP is folded into the fp32 GEMM"; "FP32 LM head skip FP32 cast", implementation breakdown),
// and the W4A16 NVFP4 head with bf16 logits (lm_head_nvfp4_rows.rs, lm_head_nvfp4_rows_run).
// As on that page, a call that cannot run launches nothing and reports why.
//
// Built twice: liblmhead.so (the release library) and, with LMHEAD_TEST_HOOKS=1,
// liblmhead_test.so, which adds the two host-side test knobs (load starvation for the timeout
// path, a forced NVFP4 conversion). The kernels are the same in both.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <mutex>
#include <utility>

#include "lmhead.h"
#include "lmhead_bf16.cuh"
#include "lmhead_nvfp4.cuh"
#include "lmhead_quant.cuh"

#ifndef LMHEAD_TEST_HOOKS
#define LMHEAD_TEST_HOOKS 0
#endif

namespace {

constexpr int kVersion = 100;  // 0.1.0
constexpr int kMaxDevices = 64;
constexpr int kMaxStages = 16;
constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;  // 2 s per barrier wait

// L2 sector promotion of weight loads: 0 none, 1 64 B, 2 128 B, 3 256 B (build-time knob).
#ifndef LMHEAD_WEIGHT_L2_PROMOTION
#define LMHEAD_WEIGHT_L2_PROMOTION 3
#endif
// Force the bf16 head's K sub-tiles per stage (0 = choose by shared-memory room).
#ifndef LMHEAD_FORCE_NSUB
#define LMHEAD_FORCE_NSUB 0
#endif
// 256-row tiles of the bf16 head on CTA pairs (cta_group::2 MMAs): 1 on, 0 off (build-time knob).
#ifndef LMHEAD_PAIR
#define LMHEAD_PAIR 1
#endif
// Tiles after a unit's first taken by cluster launch control (one unit launched per tile, the
// running units cancel the launches of the rest in order): 1 on, 0 static (build-time knob).
#ifndef LMHEAD_CLC
#define LMHEAD_CLC 1
#endif
// CTA pairs in the log-prob modes too: 1 on, 0 off (build-time knob).
#ifndef LMHEAD_PAIR_LOGPROB
#define LMHEAD_PAIR_LOGPROB 0
#endif
// Hidden-row bytes of one row-tile group (build-time knob; see make_sched).
#ifndef LMHEAD_RGROUP_MB
#define LMHEAD_RGROUP_MB 32
#endif
constexpr CUtensorMapL2promotion kWeightPromo =
    (CUtensorMapL2promotion)(CU_TENSOR_MAP_L2_PROMOTION_NONE + LMHEAD_WEIGHT_L2_PROMOTION);

std::atomic<int> g_starve_loads{0};
std::atomic<int> g_nvfp4_path{0};  // 0: automatic, 1: pair table, 2: spread (test hook)
std::atomic<int> g_no_cta_pairs{0};  // 1: the bf16 head runs 256-row tiles on lone CTAs (test hook)
std::atomic<int> g_static_tiles{0};  // 1: the bf16 head's static schedule only (test hook)
std::atomic<uint64_t> g_wait_limit_ns{0};

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct DeviceInfo {
  bool probed = false;
  bool arch_ok = false;
  bool attrs_set = false;
  unsigned long long ctx_id = 0;  // the context the kernel attributes were set in
  int num_sms = 0;
  int smem_optin = 0;        // per-block shared-memory opt-in limit (static + dynamic)
  int nvfp4_static_smem[2] = {0, 0};  // static shared memory of the NVFP4 kernel <false>, <true>
  int smem_reserved = 0;      // shared memory the system reserves per block
  int pair_clusters = 0;      // CTA pairs of the bf16 head that fit the device at once (0: none)
};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// The unique ID of the calling thread's current context (0 if it cannot be had). Per-context
// set-up (kernel attributes, the scratch array's address) is redone when the ID changes, as it
// does after cudaDeviceReset: context IDs are never reused within a process.
unsigned long long current_context_id() {
  static std::once_flag once;
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(fn);
  });
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  return get_id(ctx, &id) == CUDA_SUCCESS ? id : 0;
}

// Let `kernel` use every byte of shared memory the device allows beside its static part.
template <typename K>
bool raise_smem_limit(K kernel, int optin, int* static_bytes) {
  cudaFuncAttributes a;
  if (cudaFuncGetAttributes(&a, kernel) != cudaSuccess) return false;
  if (static_bytes) *static_bytes = (int)a.sharedSizeBytes;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              optin - (int)a.sharedSizeBytes) == cudaSuccess;
}

std::mutex g_mu;
DeviceInfo g_devices[kMaxDevices];
EncodeTiledFn g_encode = nullptr;

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
  });
  return g_encode;
}

// Probe the current device once: architecture, SM count, shared-memory opt-in; raise the
// kernels' dynamic shared-memory limit.
int current_device(DeviceInfo* out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LMHEAD_ERR_LAUNCH;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_devices[dev];
  if (!d.probed) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&d.smem_reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) !=
            cudaSuccess) {
      return LMHEAD_ERR_LAUNCH;
    }
    d.arch_ok = (major == 10 && minor == 0);
    d.probed = true;
  }
  if (!d.arch_ok) return LMHEAD_ERR_ARCH;
  // Bind the device's primary context to this thread if nothing is bound yet (the runtime would
  // do so at the first launch anyway), so that its ID can key the per-context set-up.
  unsigned long long ctx = current_context_id();
  if (ctx == 0) {
    if (cudaSetDevice(dev) != cudaSuccess) return LMHEAD_ERR_LAUNCH;
    ctx = current_context_id();
    if (ctx == 0) return LMHEAD_ERR_LAUNCH;
  }
  if (d.ctx_id != ctx) {
    d.attrs_set = false;
    d.ctx_id = ctx;
  }
  if (!d.attrs_set) {
    if (!raise_smem_limit(lmh::lmhead_bf16_f32_kernel<1, false>, d.smem_optin, nullptr) ||
        !raise_smem_limit(lmh::lmhead_bf16_f32_kernel<2, false>, d.smem_optin, nullptr) ||
        !raise_smem_limit(lmh::lmhead_bf16_f32_kernel<4, false>, d.smem_optin, nullptr) ||
        !raise_smem_limit(lmh::lmhead_bf16_f32_kernel<1, true>, d.smem_optin, nullptr) ||
        !raise_smem_limit(lmh::lmhead_bf16_f32_kernel<2, true>, d.smem_optin, nullptr) ||
        !raise_smem_limit(lmh::lmhead_w4a16_nvfp4_kernel<true>, d.smem_optin,
                          &d.nvfp4_static_smem[1]) ||
        !raise_smem_limit(lmh::lmhead_w4a16_nvfp4_kernel<false>, d.smem_optin,
                          &d.nvfp4_static_smem[0])) {
      return LMHEAD_ERR_LAUNCH;
    }
    // How many CTA pairs fit at once with a whole SM's shared memory each: a pair must sit in
    // one GPC, so this can be below half the SM count.
    d.pair_clusters = 0;
    if (LMHEAD_PAIR) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)(d.num_sms & ~1));
      cfg.blockDim = dim3(lmh::kHeadThreads);
      cfg.dynamicSmemBytes = (size_t)d.smem_optin;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, lmh::lmhead_bf16_f32_kernel<2, true>, &cfg) ==
          cudaSuccess)
        d.pair_clusters = n;
      else
        (void)cudaGetLastError();
    }
    d.attrs_set = true;
  }
  *out = d;
  return LMHEAD_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

#ifndef LMHEAD_PDL
#define LMHEAD_PDL 1
#endif
// Launch a head kernel with programmatic stream serialisation (see pdl_trigger / pdl_wait): the
// kernel's set-up may overlap the tail of the previous kernel on the stream; its global-memory
// work still follows it. Returns an lmhead_status.
// `cluster` = 2 launches the grid as CTA pairs (clusters of two along x).
template <typename... KArgs, typename... Args>
int launch_head(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem,
                lmhead_stream_t stream, unsigned cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = (cudaStream_t)stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = LMHEAD_PDL;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cluster > 1 ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) == cudaSuccess
             ? LMHEAD_OK
             : LMHEAD_ERR_LAUNCH;
}

bool overlaps(const void* a, int64_t abytes, const void* b, int64_t bbytes) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + (uintptr_t)bbytes && b0 < a0 + (uintptr_t)abytes;
}

// Row-major [outer, inner] tensor, tile box [box_outer, box_inner], 128-byte swizzle unless
// `swizzle` says otherwise.
int encode_2d(CUtensorMap* map, CUtensorMapDataType dtype, int elem_bytes, const void* base,
              int64_t inner, int64_t outer, uint32_t box_inner, uint32_t box_outer,
              CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B,
              CUtensorMapL2promotion promo = CU_TENSOR_MAP_L2_PROMOTION_L2_256B) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return LMHEAD_ERR_LAUNCH;
  const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  const cuuint64_t strides[1] = {(cuuint64_t)(inner * elem_bytes)};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, promo,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LMHEAD_OK : LMHEAD_ERR_LAUNCH;
}

// Tensor map over a row-major [outer, inner_bytes / esize] matrix of esize-byte elements, box
// [box_outer rows x box_bytes bytes]. With LMHEAD_TMA_WIDE the rows are described as 32-bit
// elements (identical bytes in global and shared memory, a quarter or half as many elements).
int encode_rows(CUtensorMap* map, CUtensorMapDataType natural, int esize, const void* base,
                int64_t inner_bytes, int64_t outer, uint32_t box_bytes, uint32_t box_outer,
                CUtensorMapSwizzle swizzle, CUtensorMapL2promotion promo) {
  if (LMHEAD_TMA_WIDE)
    return encode_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, base, inner_bytes / 4, outer,
                     box_bytes / 4, box_outer, swizzle, promo);
  return encode_2d(map, natural, esize, base, inner_bytes / esize, outer, box_bytes / esize,
                   box_outer, swizzle, promo);
}

// Tensor map over hidden [rows, H] bf16 seen as [H/64 K steps][rows][64 elements]: one box
// brings `box_k` K steps of `box_rows` rows, each K step a 128-byte-swizzled [box_rows x 128 B]
// sub-tile, the sub-tiles back to back.
int encode_hidden_ksteps(CUtensorMap* map, const void* hidden, int64_t rows, int64_t H,
                         uint32_t box_rows, uint32_t box_k) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return LMHEAD_ERR_LAUNCH;
  const int esize = LMHEAD_TMA_WIDE ? 4 : 2;
  const cuuint64_t dims[3] = {(cuuint64_t)(lmh::kBK * 2 / esize), (cuuint64_t)rows,
                              (cuuint64_t)(H / lmh::kBK)};
  const cuuint64_t strides[2] = {(cuuint64_t)(H * 2), (cuuint64_t)(lmh::kBK * 2)};
  const cuuint32_t box[3] = {(cuuint32_t)(lmh::kBK * 2 / esize), box_rows, box_k};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r =
      enc(map, LMHEAD_TMA_WIDE ? CU_TENSOR_MAP_DATA_TYPE_UINT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
          3, const_cast<void*>(hidden), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LMHEAD_OK : LMHEAD_ERR_LAUNCH;
}

// Rows of hidden one TMA box brings: the call's rows when they fit one row tile (the MMA still
// spans bn columns; columns past the call's rows are never stored), else the tile height.
int32_t hid_box_rows(int64_t rows, int32_t bn) {
  return (LMHEAD_HID_BOX_EXACT && rows < bn) ? (int32_t)rows : bn;
}

lmh::WaitCfg wait_cfg() {
  lmh::WaitCfg w;
  const uint64_t lim = g_wait_limit_ns.load(std::memory_order_relaxed);
  w.limit_ns = lim ? lim : kDefaultWaitLimitNs;
  w.starve_loads = g_starve_loads.load(std::memory_order_relaxed);
  return w;
}

// Rows per tile: the padded row count up to 256, else 256. Every choice runs the same
// per-element MMA chain over K, so it affects speed only, never a row's bits.
int32_t pick_bn(int64_t rows) { return rows >= 256 ? 256 : (int32_t)((rows + 15) / 16 * 16); }

uint32_t tmem_cols_for(int32_t bn) {
  uint32_t need = 2u * (uint32_t)bn, c = 32;
  while (c < need) c <<= 1;
  return c;
}

constexpr int kInt32Max = 0x7fffffff;

// Tile ownership (see TileSched) and grid size: one persistent unit (a CTA, or with `pair` a
// CTA pair) per slot, `units` slots at most.
int make_sched(int64_t rows, int64_t V, int64_t H, int32_t bn, int pair, int units,
               lmh::TileSched* s, int* grid) {
  s->bn = bn;
  s->pair = pair;
  s->n_rtiles = (int32_t)((rows + bn - 1) / bn);
  const int64_t vt_rows = (int64_t)lmh::kBM << pair;
  const int64_t n_vtiles = (V + vt_rows - 1) / vt_rows;
  const int64_t tiles = (int64_t)s->n_rtiles * n_vtiles;
  if (tiles > kInt32Max) return LMHEAD_ERR_SHAPE;
  s->num_tiles = (int32_t)tiles;
  s->n_vtiles = (int32_t)n_vtiles;
  // Row tiles per group: their hidden rows within LMHEAD_RGROUP_MB (32 MB, a quarter of L2;
  // 16 MB read W twice as often at the prefill shape, 64 MB was slower on B200).
  const int64_t tile_hidden_bytes = (int64_t)bn * H * 2;
  const int64_t rg =
      ((int64_t)LMHEAD_RGROUP_MB << 20) / (tile_hidden_bytes > 0 ? tile_hidden_bytes : 1);
  s->rgroup = (int32_t)(rg < 1 ? 1 : (rg > s->n_rtiles ? s->n_rtiles : rg));
  *grid = (s->num_tiles < units ? s->num_tiles : units) << pair;
  return LMHEAD_OK;
}

// 64-wide K sub-tiles per pipeline stage of the bf16 head: the largest of 4, 2, 1 that still
// leaves room for 3 stages. Longer per-stage bursts along each weight row read HBM faster.
int pick_nsub(int32_t bn, int smem_budget) {
  if (LMHEAD_FORCE_NSUB) return LMHEAD_FORCE_NSUB;
  for (int nsub = 4; nsub > 1; nsub /= 2) {
    const int stage = nsub * (lmh::kBM * lmh::kBK * 2 + bn * lmh::kBK * 2);
    if (smem_budget / stage >= 3) return nsub;
  }
  return 1;
}

// ---- library-held scratch for lmhead_nvfp4_quantize_noalloc
// The absmax pass's per-CTA maxima, for callers that cannot hand the quantiser a workspace.
// 4 KB per GPU, held by every GPU that loads the library until the process exits.
static __device__ __align__(256) uint32_t g_quant_scratch[lmh::kQuantMaxPartials];

std::mutex g_scratch_mu;
struct ScratchAddr {
  unsigned long long ctx_id = 0;
  uint32_t* ptr = nullptr;
};
ScratchAddr g_scratch[kMaxDevices];

// The scratch array's device address in the current device's context. Host code may not use the
// array's name as a device address (it names a host-side stand-in), so the address is looked up
// with cudaGetSymbolAddress once per device, with that device current, and cached for as long as
// that context lives. The caller has already run current_device(), so a context is bound.
int quant_scratch(uint32_t** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LMHEAD_ERR_LAUNCH;
  const unsigned long long ctx = current_context_id();
  if (ctx == 0) return LMHEAD_ERR_LAUNCH;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  ScratchAddr& sa = g_scratch[dev];
  if (sa.ptr == nullptr || sa.ctx_id != ctx) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_quant_scratch) != cudaSuccess || ptr == nullptr) {
      (void)cudaGetLastError();  // leave no stale error for the next call's launch check
      return LMHEAD_ERR_LAUNCH;
    }
    sa.ptr = static_cast<uint32_t*>(ptr);
    sa.ctx_id = ctx;
  }
  *out = sa.ptr;
  return LMHEAD_OK;
}

// Every host-side check of the quantiser's arguments except the workspace's: shapes, NULLs,
// alignment and overlap of W and the three outputs. Touches no device state.
int check_quantize_args(const void* w, int64_t V, int64_t H, const uint8_t* w_packed,
                        const uint8_t* w_scales, const float* w_global_scale) {
  if (V <= 0 || H <= 0) return LMHEAD_ERR_SHAPE;
  if (H % 16 != 0) return LMHEAD_ERR_ALIGN;
  if (V > kInt32Max || H > kInt32Max) return LMHEAD_ERR_SHAPE;
  if (w == nullptr || w_packed == nullptr || w_scales == nullptr || w_global_scale == nullptr)
    return LMHEAD_ERR_NULL;
  if (!aligned(w, 16) || !aligned(w_packed, 8) || !aligned(w_global_scale, 4))
    return LMHEAD_ERR_ALIGN;
  const int64_t n = V * H;
  const struct { const void* p; int64_t bytes; } regions[4] = {
      {w, n * 2}, {w_packed, n / 2}, {w_scales, n / 16}, {w_global_scale, 4}};
  for (int i = 0; i < 4; ++i)
    for (int j = i + 1; j < 4; ++j)
      if (overlaps(regions[i].p, regions[i].bytes, regions[j].p, regions[j].bytes))
        return LMHEAD_ERR_ALIAS;
  return LMHEAD_OK;
}

// The two quantiser launches, after validation. `partial` holds at least `partial_words` words.
int launch_quantize(const DeviceInfo& dev, const void* w, int64_t V, int64_t H,
                    uint8_t* w_packed, uint8_t* w_scales, float* w_global_scale,
                    uint32_t* partial, size_t partial_words, lmhead_stream_t stream) {
  const int64_t n = V * H;
  // Pass 1 grid: a few CTAs per SM, one partial word each, never past the scratch.
  const int64_t n_chunks = n / 8;
  int64_t grid = (int64_t)dev.num_sms * 6;
  const int64_t by_work = (n_chunks + lmh::kQuantThreads - 1) / lmh::kQuantThreads;
  if (grid > by_work) grid = by_work;
  if (grid > lmh::kQuantMaxPartials) grid = lmh::kQuantMaxPartials;
  if ((size_t)grid > partial_words) return LMHEAD_ERR_SHAPE;
  const int64_t n_blocks = n / 16;
  int64_t grid2 = (int64_t)dev.num_sms * 8;
  const int64_t by_blocks = (n_blocks + lmh::kQuantThreads - 1) / lmh::kQuantThreads;
  if (grid2 > by_blocks) grid2 = by_blocks;
  lmh::nvfp4_absmax_kernel<<<(unsigned)grid, lmh::kQuantThreads, 0, (cudaStream_t)stream>>>(
      reinterpret_cast<const uint4*>(w), n_chunks, partial);
  lmh::nvfp4_encode_kernel<<<(unsigned)grid2, lmh::kQuantThreads, 0, (cudaStream_t)stream>>>(
      reinterpret_cast<const uint4*>(w), n_blocks, partial, (int)grid,
      reinterpret_cast<uint2*>(w_packed), w_scales, w_global_scale);
  return cudaGetLastError() == cudaSuccess ? LMHEAD_OK : LMHEAD_ERR_LAUNCH;
}

}  // namespace

extern "C" {

int lmhead_version(void) { return kVersion; }

const char* lmhead_status_string(int status) {
  switch (status) {
    case LMHEAD_OK: return "ok";
    case LMHEAD_ERR_NULL: return "a required pointer is NULL";
    case LMHEAD_ERR_SHAPE: return "unsupported or invalid size";
    case LMHEAD_ERR_ALIGN: return "pointer or row pitch misaligned";
    case LMHEAD_ERR_ARCH: return "current device is not an sm_100 GPU";
    case LMHEAD_ERR_LAUNCH: return "CUDA runtime refused a set-up call or the launch";
    case LMHEAD_ERR_TIMEOUT: return "a kernel timed out waiting on one of its barriers";
    case LMHEAD_ERR_ALIAS: return "output overlaps an input";
    default: return "unknown status";
  }
}

#if LMHEAD_TEST_HOOKS
void lmhead_debug_set_fault_injection(int starve_loads, uint64_t wait_limit_ns) {
  g_starve_loads.store(starve_loads ? 1 : 0);
  g_wait_limit_ns.store(wait_limit_ns);
}

void lmhead_debug_set_nvfp4_conversion(int path) {
  g_nvfp4_path.store(path == 1 || path == 2 ? path : 0);
}

void lmhead_debug_set_cta_pairs(int enabled) { g_no_cta_pairs.store(enabled ? 0 : 1); }

void lmhead_debug_set_dynamic_tiles(int enabled) { g_static_tiles.store(enabled ? 0 : 1); }
#endif

size_t lmhead_nvfp4_quantize_workspace_bytes(void) {
  return (size_t)lmh::kQuantMaxPartials * sizeof(uint32_t);
}

int lmhead_nvfp4_quantize(const void* w, int64_t V, int64_t H, uint8_t* w_packed,
                          uint8_t* w_scales, float* w_global_scale, void* workspace,
                          size_t workspace_bytes, lmhead_stream_t stream) {
  int st = check_quantize_args(w, V, H, w_packed, w_scales, w_global_scale);
  if (st != LMHEAD_OK) return st;
  if (workspace == nullptr) return LMHEAD_ERR_NULL;
  if (!aligned(workspace, 4)) return LMHEAD_ERR_ALIGN;
  const int64_t n = V * H;
  const struct { const void* p; int64_t bytes; } regions[4] = {
      {w, n * 2}, {w_packed, n / 2}, {w_scales, n / 16}, {w_global_scale, 4}};
  for (const auto& r : regions)
    if (overlaps(workspace, (int64_t)workspace_bytes, r.p, r.bytes)) return LMHEAD_ERR_ALIAS;
  DeviceInfo dev;
  st = current_device(&dev);
  if (st != LMHEAD_OK) return st;
  return launch_quantize(dev, w, V, H, w_packed, w_scales, w_global_scale,
                         reinterpret_cast<uint32_t*>(workspace), workspace_bytes / 4, stream);
}

int lmhead_nvfp4_quantize_noalloc(const void* w, int64_t V, int64_t H, uint8_t* w_packed,
                                  uint8_t* w_scales, float* w_global_scale,
                                  lmhead_stream_t stream) {
  // Every argument check first, so an invalid call touches no device state; then the device
  // check (ARCH before anything else), and only then the scratch lookup.
  int st = check_quantize_args(w, V, H, w_packed, w_scales, w_global_scale);
  if (st != LMHEAD_OK) return st;
  DeviceInfo dev;
  st = current_device(&dev);
  if (st != LMHEAD_OK) return st;
  uint32_t* scratch = nullptr;
  st = quant_scratch(&scratch);
  if (st != LMHEAD_OK) return st;
  // The absmax grid is capped at kQuantMaxPartials words, the array's size, so a valid call
  // always fits; launch_quantize still rejects one that would not (LMHEAD_ERR_SHAPE).
  return launch_quantize(dev, w, V, H, w_packed, w_scales, w_global_scale, scratch,
                         sizeof(g_quant_scratch) / sizeof(uint32_t), stream);
}

int lmhead_stream_status(lmhead_stream_t stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) {
    (void)cudaGetLastError();
    return LMHEAD_ERR_LAUNCH;
  }
  return lmhead_device_status(1);
}

int lmhead_device_status(int clear) {
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, lmh::g_lmhead_status, sizeof v) != cudaSuccess)
    return LMHEAD_ERR_LAUNCH;
  if (clear) {
    const unsigned int z = 0;
    if (cudaMemcpyToSymbol(lmh::g_lmhead_status, &z, sizeof z) != cudaSuccess)
      return LMHEAD_ERR_LAUNCH;
  }
  return (int)v;
}

int lmhead_logits_bf16_f32(const void* hidden, int64_t rows, int64_t H, const void* W, int64_t V,
                           float alpha, float* logits, lmhead_stream_t stream) {
  return lmhead_logits_f32(hidden, LMHEAD_DTYPE_BF16, rows, H, W, V, alpha, nullptr, logits,
                           stream);
}

}  // extern "C"

namespace {

// Everything after validation for the fp32 head: logits to `logits`, or, when lp is given,
// log-probabilities of its targets (no logits written).
struct LogprobArgs {
  const int32_t* targets;
  float* logprobs;
  float* lse;
  void* workspace;
  int64_t v_begin;  // vocab id of W's first row
  float* stats;     // vocab-shard mode: per-row (max, sum, target logit) instead of logprobs
};

// Where the logits of a vocab slice go: columns [v_begin, v_begin + V) of each of n row-major
// [rows, ld] buffers.
struct LogitCopies {
  float* const* bufs;
  int n;
  int64_t ld;
  int64_t v_begin;
};

int run_f32_head(const void* hidden, int dtype, int64_t rows, int64_t H, const void* W, int64_t V,
                 float alpha, const void* bias, float* logits, const LogprobArgs* lp,
                 lmhead_stream_t stream, const LogitCopies* copies = nullptr) {
  DeviceInfo dev;
  int st = current_device(&dev);
  if (st != LMHEAD_OK) return st;

  lmh::Bf16HeadParams p;
  p.rows = rows;
  p.H = H;
  p.V = V;
  for (int d = 0; d < lmh::kMaxLogitCopies; ++d) p.out[d] = nullptr;
  if (copies != nullptr) {
    for (int d = 0; d < copies->n; ++d) p.out[d] = copies->bufs[d] + copies->v_begin;
    p.n_out = copies->n;
    p.ld_out = copies->ld;
  } else {
    p.out[0] = logits;
    p.n_out = 1;
    p.ld_out = V;
  }
  p.logprob = lp != nullptr ? 1 : 0;
  p.n_chunks = (int32_t)(4 * ((V + lmh::kBM - 1) / lmh::kBM));
  p.partials = lp != nullptr ? reinterpret_cast<float2*>(lp->workspace) : nullptr;
  p.targets = lp != nullptr ? lp->targets : nullptr;
  p.target_base = lp != nullptr ? lp->v_begin : 0;
  // The target's logit is parked where the combine kernel reads it: the logprobs slot of the
  // row, or the third word of the row's shard stats.
  p.target_z = lp == nullptr ? nullptr : lp->stats != nullptr ? lp->stats + 2 : lp->logprobs;
  p.tz_stride = lp != nullptr && lp->stats != nullptr ? 3 : 1;
  p.bias = reinterpret_cast<const uint16_t*>(bias);
  p.alpha = alpha;
  p.fp16 = dtype == LMHEAD_DTYPE_F16 ? 1 : 0;
  p.bn = pick_bn(rows);
  // Full 256-row tiles of the logits run on CTA pairs: M = 256 vocab rows per MMA, so each CTA
  // loads its 128 W rows and half the hidden rows per K step (a third less shared-memory fill
  // per flop). The log-prob modes keep lone CTAs: with pairs they measured slower at 8192 rows,
  // moving twice the DRAM reads.
  const int pair = (LMHEAD_PAIR && p.bn == 256 && (lp == nullptr || LMHEAD_PAIR_LOGPROB) &&
                    dev.pair_clusters > 0 &&
                    !g_no_cta_pairs.load(std::memory_order_relaxed))
                       ? 1
                       : 0;
  const int32_t b_rows = p.bn >> pair;  // hidden rows in one CTA's tile
  int grid = 0;
  st = make_sched(rows, V, H, p.bn, pair, pair ? dev.pair_clusters : dev.num_sms, &p.sched,
                  &grid);
  if (st != LMHEAD_OK) return st;
  // every tile a unit of its own at launch (the static schedule when that grid would not fit)
  p.clc = LMHEAD_CLC && !g_static_tiles.load(std::memory_order_relaxed) &&
          ((int64_t)p.sched.num_tiles << pair) <= kInt32Max;
  if (p.clc) grid = p.sched.num_tiles << pair;
  const int reserve = 1024 + 512;  // alignment slack + barriers
  // (pairs: one K sub-tile per stage, six stages; two sub-tiles and three stages measured ~1 %
  // slower at 2048 and 8192 rows)
  int nsub = pair && !LMHEAD_FORCE_NSUB ? 1 : pick_nsub(b_rows, dev.smem_optin - reserve);
  if (pair && nsub > 2) nsub = 2;  // the pair kernel is built for one or two
  p.num_ks = (int32_t)((H + nsub * lmh::kBK - 1) / (nsub * lmh::kBK));
  p.stage_bytes = (uint32_t)(nsub * (lmh::kBM * lmh::kBK * 2 + b_rows * lmh::kBK * 2));
  int stages = (dev.smem_optin - reserve) / (int)p.stage_bytes;
  if (stages > kMaxStages) stages = kMaxStages;
  if (stages < 2) return LMHEAD_ERR_SHAPE;
  p.stages = stages;
  p.tmem_cols = tmem_cols_for(p.bn);
  p.wait = wait_cfg();

  CUtensorMap tmap_w, tmap_h;
  const CUtensorMapDataType tdt =
      p.fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  st = encode_rows(&tmap_w, tdt, 2, W, H * 2, V, lmh::kBK * 2,
                   lmh::kBM, CU_TENSOR_MAP_SWIZZLE_128B, kWeightPromo);
  if (st != LMHEAD_OK) return st;
  p.hid_rows = pair ? b_rows : hid_box_rows(rows, p.bn);
  st = encode_rows(&tmap_h, tdt, 2, hidden, H * 2, rows,
                   lmh::kBK * 2, (uint32_t)p.hid_rows, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
  if (st != LMHEAD_OK) return st;

  const size_t smem = (size_t)reserve + (size_t)stages * p.stage_bytes;
  auto kernel = pair ? (nsub == 2 ? lmh::lmhead_bf16_f32_kernel<2, true>
                                  : lmh::lmhead_bf16_f32_kernel<1, true>)
                : nsub == 4 ? lmh::lmhead_bf16_f32_kernel<4, false>
                : nsub == 2 ? lmh::lmhead_bf16_f32_kernel<2, false>
                            : lmh::lmhead_bf16_f32_kernel<1, false>;
  st = launch_head(kernel, (unsigned)grid, lmh::kHeadThreads, smem, stream, pair ? 2u : 1u,
                   tmap_w, tmap_h, p);
  if (st != LMHEAD_OK) {
    (void)cudaGetLastError();
    return st;
  }
  if (lp != nullptr) {
    const int64_t blocks = (rows + lmh::kCombineRows - 1) / lmh::kCombineRows;
    lmh::lmhead_logprob_combine_kernel<<<(unsigned)blocks, 1024, 0, (cudaStream_t)stream>>>(
        p.partials, p.n_chunks, rows, V, lp->targets, lp->logprobs, lp->lse, lp->v_begin,
        lp->stats);
  }
  return cudaGetLastError() == cudaSuccess ? LMHEAD_OK : LMHEAD_ERR_LAUNCH;
}


int check_f32_head_args(const void* hidden, int dtype, int64_t rows, int64_t H, const void* W,
                        int64_t V, const void* bias) {
  if (dtype != LMHEAD_DTYPE_BF16 && dtype != LMHEAD_DTYPE_F16) return LMHEAD_ERR_SHAPE;
  if (rows < 0 || H <= 0 || V <= 0) return LMHEAD_ERR_SHAPE;
  if (H % 8 != 0) return LMHEAD_ERR_ALIGN;
  if (rows > kInt32Max || H > kInt32Max || V > kInt32Max) return LMHEAD_ERR_SHAPE;
  if (rows == 0) return LMHEAD_OK;
  if (hidden == nullptr || W == nullptr) return LMHEAD_ERR_NULL;
  if (!aligned(hidden, 16) || !aligned(W, 16) || (bias != nullptr && !aligned(bias, 2)))
    return LMHEAD_ERR_ALIGN;
  return LMHEAD_OK;
}

}  // namespace

extern "C" {

int lmhead_logits_f32(const void* hidden, int dtype, int64_t rows, int64_t H, const void* W,
                      int64_t V, float alpha, const void* bias, float* logits,
                      lmhead_stream_t stream) {
  const int st = check_f32_head_args(hidden, dtype, rows, H, W, V, bias);
  if (st != LMHEAD_OK || rows == 0) return st;
  if (logits == nullptr) return LMHEAD_ERR_NULL;
  if (!aligned(logits, 4)) return LMHEAD_ERR_ALIGN;
  if (overlaps(logits, rows * V * 4, hidden, rows * H * 2) ||
      overlaps(logits, rows * V * 4, W, V * H * 2) ||
      (bias != nullptr && overlaps(logits, rows * V * 4, bias, V * 2))) {
    return LMHEAD_ERR_ALIAS;
  }
  return run_f32_head(hidden, dtype, rows, H, W, V, alpha, bias, logits, nullptr, stream);
}

int lmhead_logits_vocab_slice_f32(const void* hidden, int dtype, int64_t rows, int64_t H,
                                  const void* W_slice, int64_t V_slice, int64_t v_begin,
                                  float alpha, const void* bias_slice, float* const* logits,
                                  int n_logits, int64_t ld_logits, lmhead_stream_t stream) {
  int st = check_f32_head_args(hidden, dtype, rows, H, W_slice, V_slice, bias_slice);
  if (st != LMHEAD_OK) return st;
  if (n_logits < 1 || n_logits > lmh::kMaxLogitCopies) return LMHEAD_ERR_SHAPE;
  if (v_begin < 0 || ld_logits < 1 || V_slice > ld_logits - v_begin) return LMHEAD_ERR_SHAPE;
  // every buffer spans rows * ld_logits floats, which must fit an int64 byte count
  if (rows > 0 && ld_logits > (INT64_MAX / 4) / rows) return LMHEAD_ERR_SHAPE;
  if (rows == 0) return LMHEAD_OK;
  if (logits == nullptr) return LMHEAD_ERR_NULL;
  const int64_t span = ((rows - 1) * ld_logits + v_begin + V_slice) * 4;  // bytes touched
  const struct { const void* p; int64_t bytes; } in[3] = {
      {hidden, rows * H * 2}, {W_slice, V_slice * H * 2}, {bias_slice, bias_slice ? V_slice * 2 : 0}};
  for (int d = 0; d < n_logits; ++d) {
    if (logits[d] == nullptr) return LMHEAD_ERR_NULL;
    if (!aligned(logits[d], 4)) return LMHEAD_ERR_ALIGN;
    for (const auto& i : in)
      if (i.p != nullptr && overlaps(logits[d], span, i.p, i.bytes)) return LMHEAD_ERR_ALIAS;
    for (int e = 0; e < d; ++e)
      if (overlaps(logits[d], span, logits[e], span)) return LMHEAD_ERR_ALIAS;
  }
  const LogitCopies copies{logits, n_logits, ld_logits, v_begin};
  return run_f32_head(hidden, dtype, rows, H, W_slice, V_slice, alpha, bias_slice, nullptr,
                      nullptr, stream, &copies);
}

size_t lmhead_logprobs_workspace_bytes(int64_t rows, int64_t V) {
  if (rows <= 0 || V <= 0) return 0;
  return (size_t)rows * (size_t)(4 * ((V + lmh::kBM - 1) / lmh::kBM)) * 8u;
}

int lmhead_logprobs_f32(const void* hidden, int dtype, int64_t rows, int64_t H, const void* W,
                        int64_t V, float alpha, const void* bias, const int32_t* targets,
                        float* logprobs, float* lse, void* workspace, size_t workspace_bytes,
                        lmhead_stream_t stream) {
  const int st = check_f32_head_args(hidden, dtype, rows, H, W, V, bias);
  if (st != LMHEAD_OK || rows == 0) return st;
  if (targets == nullptr || logprobs == nullptr || workspace == nullptr) return LMHEAD_ERR_NULL;
  if (!aligned(targets, 4) || !aligned(logprobs, 4) || (lse != nullptr && !aligned(lse, 4)) ||
      !aligned(workspace, 8)) {
    return LMHEAD_ERR_ALIGN;
  }
  if (workspace_bytes < lmhead_logprobs_workspace_bytes(rows, V)) return LMHEAD_ERR_SHAPE;
  const struct { const void* p; int64_t bytes; } in[4] = {
      {hidden, rows * H * 2}, {W, V * H * 2}, {bias, bias ? V * 2 : 0}, {targets, rows * 4}};
  const struct { const void* p; int64_t bytes; } out[3] = {
      {logprobs, rows * 4}, {lse, lse ? rows * 4 : 0}, {workspace, (int64_t)workspace_bytes}};
  for (const auto& o : out) {
    if (o.p == nullptr) continue;
    for (const auto& i : in)
      if (i.p != nullptr && overlaps(o.p, o.bytes, i.p, i.bytes)) return LMHEAD_ERR_ALIAS;
    for (const auto& o2 : out)
      if (&o2 != &o && o2.p != nullptr && overlaps(o.p, o.bytes, o2.p, o2.bytes))
        return LMHEAD_ERR_ALIAS;
  }
  const LogprobArgs lp{targets, logprobs, lse, workspace, 0, nullptr};
  return run_f32_head(hidden, dtype, rows, H, W, V, alpha, bias, nullptr, &lp, stream);
}

int lmhead_logprobs_shard_stats_f32(const void* hidden, int dtype, int64_t rows, int64_t H,
                                    const void* W_shard, int64_t V_shard, int64_t v_begin,
                                    float alpha, const void* bias_shard, const int32_t* targets,
                                    float* stats, void* workspace, size_t workspace_bytes,
                                    lmhead_stream_t stream) {
  const int st = check_f32_head_args(hidden, dtype, rows, H, W_shard, V_shard, bias_shard);
  if (st != LMHEAD_OK) return st;
  // Token ids are int32: the shard must lie inside [0, 2^31).
  if (v_begin < 0 || v_begin > kInt32Max || V_shard > (int64_t)kInt32Max + 1 - v_begin)
    return LMHEAD_ERR_SHAPE;
  if (rows == 0) return LMHEAD_OK;
  if (targets == nullptr || stats == nullptr || workspace == nullptr) return LMHEAD_ERR_NULL;
  if (!aligned(targets, 4) || !aligned(stats, 4) || !aligned(workspace, 8))
    return LMHEAD_ERR_ALIGN;
  if (workspace_bytes < lmhead_logprobs_workspace_bytes(rows, V_shard)) return LMHEAD_ERR_SHAPE;
  const struct { const void* p; int64_t bytes; } in[4] = {
      {hidden, rows * H * 2},
      {W_shard, V_shard * H * 2},
      {bias_shard, bias_shard ? V_shard * 2 : 0},
      {targets, rows * 4}};
  const int64_t stats_bytes = rows * 12;
  for (const auto& i : in) {
    if (i.p == nullptr) continue;
    if (overlaps(stats, stats_bytes, i.p, i.bytes) ||
        overlaps(workspace, (int64_t)workspace_bytes, i.p, i.bytes))
      return LMHEAD_ERR_ALIAS;
  }
  if (overlaps(stats, stats_bytes, workspace, (int64_t)workspace_bytes)) return LMHEAD_ERR_ALIAS;
  const LogprobArgs lp{targets, nullptr, nullptr, workspace, v_begin, stats};
  return run_f32_head(hidden, dtype, rows, H, W_shard, V_shard, alpha, bias_shard, nullptr, &lp,
                      stream);
}

int lmhead_logprobs_merge_shards(const float* stats, int64_t shards, int64_t rows,
                                 float* logprobs, float* lse, lmhead_stream_t stream) {
  if (shards <= 0 || shards > kInt32Max || rows < 0) return LMHEAD_ERR_SHAPE;
  if (rows > kInt32Max) return LMHEAD_ERR_SHAPE;
  if (rows == 0) return LMHEAD_OK;
  if (stats == nullptr || logprobs == nullptr) return LMHEAD_ERR_NULL;
  if (!aligned(stats, 4) || !aligned(logprobs, 4) || (lse != nullptr && !aligned(lse, 4)))
    return LMHEAD_ERR_ALIGN;
  const int64_t stats_bytes = shards * rows * 12;
  if (overlaps(logprobs, rows * 4, stats, stats_bytes) ||
      (lse != nullptr && (overlaps(lse, rows * 4, stats, stats_bytes) ||
                          overlaps(lse, rows * 4, logprobs, rows * 4))))
    return LMHEAD_ERR_ALIAS;
  DeviceInfo dev;
  const int st = current_device(&dev);
  if (st != LMHEAD_OK) return st;
  const int64_t blocks = (rows + lmh::kMergeThreads - 1) / lmh::kMergeThreads;
  lmh::lmhead_logprob_merge_shards_kernel<<<(unsigned)blocks, lmh::kMergeThreads, 0,
                                            (cudaStream_t)stream>>>(stats, (int32_t)shards, rows,
                                                                    logprobs, lse);
  return cudaGetLastError() == cudaSuccess ? LMHEAD_OK : LMHEAD_ERR_LAUNCH;
}

int lmhead_logits_w4a16_nvfp4(const void* hidden, int64_t rows, int64_t H, const uint8_t* w_packed,
                              const uint8_t* w_scales, float w_global_scale, int64_t V,
                              float alpha, void* logits, lmhead_stream_t stream) {
  if (rows < 0 || H <= 0 || V <= 0) return LMHEAD_ERR_SHAPE;
  if (H % 32 != 0) return LMHEAD_ERR_ALIGN;
  if (rows > kInt32Max || H > kInt32Max || V > kInt32Max) return LMHEAD_ERR_SHAPE;
  if (rows == 0) return LMHEAD_OK;
  if (hidden == nullptr || w_packed == nullptr || w_scales == nullptr || logits == nullptr)
    return LMHEAD_ERR_NULL;
  if (!aligned(hidden, 16) || !aligned(w_packed, 16) || !aligned(w_scales, 4) ||
      !aligned(logits, 2)) {
    return LMHEAD_ERR_ALIGN;
  }
  const int64_t out_bytes = rows * V * 2;
  if (overlaps(logits, out_bytes, hidden, rows * H * 2) ||
      overlaps(logits, out_bytes, w_packed, V * H / 2) ||
      overlaps(logits, out_bytes, w_scales, V * H / 16)) {
    return LMHEAD_ERR_ALIAS;
  }
  DeviceInfo dev;
  int st = current_device(&dev);
  if (st != LMHEAD_OK) return st;

  lmh::Nvfp4HeadParams p;
  p.rows = rows;
  p.H = H;
  p.V = V;
  p.out = reinterpret_cast<uint16_t*>(logits);
  p.scales = w_scales;
  p.alpha = alpha;
  p.gscale = w_global_scale;
  p.bn = pick_bn(rows) < lmh::kBnMax ? pick_bn(rows) : lmh::kBnMax;
  int grid = 0;
  st = make_sched(rows, V, H, p.bn, 0, dev.num_sms, &p.sched, &grid);
  if (st != LMHEAD_OK) return st;
  p.num_kb = (int32_t)((H + lmh::kBK - 1) / lmh::kBK);
  p.half_tail = (H % lmh::kBK) != 0 ? 1 : 0;  // H % 64 == 32: the last K step is half a step
  p.hid_2d = p.half_tail;
  // Hidden sub-tiles start on 1024-byte swizzle atoms: rows per K step rounded up to 8.
  p.hid_rows = rows < p.bn ? (int32_t)((rows + 7) / 8 * 8) : p.bn;
  // Dynamic shared memory: all the opt-in room; the kernel lays its rings out in it. The window
  // holds the reserved block, then the kernel's static variables, then the dynamic block.
  const uint32_t hid_bytes = lmh::nvfp4_hid_stage_bytes(p.bn, p.hid_rows);
  auto layout = [&](bool table) {
    const int stat = dev.nvfp4_static_smem[table ? 1 : 0];
    const uint32_t win_base = (uint32_t)(dev.smem_reserved + stat);
    uint32_t code[lmh::kMaxCodeStages], hid[lmh::kMaxHidStages];
    return lmh::nvfp4_layout(win_base, win_base + (uint32_t)(dev.smem_optin - stat), hid_bytes,
                             table, code, hid);
  };
  auto viable = [](const lmh::Nvfp4Layout& L) { return L.n_code >= 2 && L.n_hid >= 2; };
  const lmh::Nvfp4Layout with_table = layout(true);
  const lmh::Nvfp4Layout spread = layout(false);
  const int path = g_nvfp4_path.load(std::memory_order_relaxed);
  // The pair table when it leaves room for 4 codes stages (both conversions give the same bits).
  const bool use_table = path == 1   ? viable(with_table)
                         : path == 2 ? false
                                     : viable(with_table) && with_table.n_code >= 4;
  if (!viable(use_table ? with_table : spread)) return LMHEAD_ERR_SHAPE;
  const int dyn_bytes = dev.smem_optin - dev.nvfp4_static_smem[use_table ? 1 : 0];
  // TMEM: three weight slots at the top and two accumulators below them when they fit (row
  // tiles <= 64), else two slots and two accumulators. (One accumulator and three slots for the
  // wider tiles was measured slower on B200: the epilogue then no longer overlaps the next tile's
  // MMAs, 153 -> 189 us at 256 rows; build-time knob LMHEAD_NVFP4_TWO_SLOTS=0.)
#ifndef LMHEAD_NVFP4_TWO_SLOTS
#define LMHEAD_NVFP4_TWO_SLOTS 1
#endif
  const bool two_acc = 2 * p.bn + 3 * (int)lmh::kSlotCols <= (int)lmh::kTmemCols;
  p.slots = (LMHEAD_NVFP4_TWO_SLOTS && !two_acc) ? 2 : 3;
  p.accs = (two_acc || p.slots == 2) ? 2 : 1;
  // Block scales come by TMA when each scale row is a whole number of 16-byte units, by 4-byte
  // async copies when it is a whole number of words, else by the producer's 2-byte loads.
  p.scale_mode = ((H / 16) % 16 == 0 && aligned(w_scales, 16)) ? lmh::kScaleTma
                 : (H / 16) % 4 == 0                             ? lmh::kScaleAsync4
                                                                 : lmh::kScalePlain;
  p.wait = wait_cfg();

  // Packed codes as a [V, H/2] byte matrix, boxes of [128 rows x 128 bytes] (4 K steps) with the
  // 128-byte swizzle; scales as a [V, H/16] byte matrix, boxes of [128 rows x 16 bytes].
  CUtensorMap tmap_q, tmap_s, tmap_h;
  st = encode_rows(&tmap_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w_packed, H / 2, V,
                   lmh::kRawK * lmh::kBK / 2, lmh::kBM, CU_TENSOR_MAP_SWIZZLE_128B, kWeightPromo);
  if (st != LMHEAD_OK) return st;
  if (p.scale_mode == lmh::kScaleTma) {
    st = encode_rows(&tmap_s, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w_scales, H / 16, V,
                     lmh::kRawK * 4, lmh::kBM, CU_TENSOR_MAP_SWIZZLE_NONE, kWeightPromo);
    if (st != LMHEAD_OK) return st;
  } else {
    tmap_s = tmap_q;  // unused
  }
  if (p.hid_2d)  // [rows, H] with [hid_rows x 64] boxes: K past H is zero-filled
    st = encode_rows(&tmap_h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, hidden, H * 2, rows,
                     lmh::kBK * 2, (uint32_t)p.hid_rows, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
  else
    st = encode_hidden_ksteps(&tmap_h, hidden, rows, H, (uint32_t)p.hid_rows, lmh::kRawK);
  if (st != LMHEAD_OK) return st;

  st = launch_head(use_table ? lmh::lmhead_w4a16_nvfp4_kernel<true>
                             : lmh::lmhead_w4a16_nvfp4_kernel<false>,
                   (unsigned)grid, lmh::kNvfp4Threads, (size_t)dyn_bytes, stream, 1u, tmap_q,
                   tmap_s, tmap_h, p);
  if (st != LMHEAD_OK) (void)cudaGetLastError();
  return st;
}

}  // extern "C"
