/*
 * lmhead -- LM-head logits projection for NVIDIA B200 (sm_100a), C ABI.
 *
 *   logits[rows, V] = alpha * (hidden[rows, H] @ W[V, H]^T)
 *
 * Entry 1 takes bf16 hidden and W, accumulates in fp32 and writes fp32 logits; no fp32 copy of
 * either operand is ever made. Its general form also takes fp16 operands and an embedding bias.
 * Entry 2 is the W4A16 NVFP4 head: E2M1 weights with per-16 E4M3 block scales and one fp32
 * per-tensor scale, bf16 activations that are never quantised, bf16 logits. Around them: the
 * log-probabilities of given tokens over the fp32 logits (whole vocabulary, or one vocab slice
 * per GPU plus a merge), and the NVFP4 quantiser.
 *
 * The operation comes from these pages:
 *  - "[Model] Honor fp32 head_dtype in Inkling muP logits (target + MTP draft)", "Purpose" and
 *    "muP is folded into the fp32 GEMM (not a bypass)": out = alpha * (hidden @ w.t()) with
 *    alpha = 1/mup, bf16 inputs accumulated into fp32 without materialising an fp32 weight copy,
 *    alpha applied in the GEMM epilogue, bit-identical to the projection followed by a separate
 *    fp32 multiply by alpha.
 *  - "FP32 LM head skip FP32 cast" (SGLang PR #32370 summary), implementation breakdown:
 *    torch.mm(hidden, W.T, out_dtype=float32) -- bf16 x bf16 -> fp32 with an fp32 accumulator,
 *    replacing a cast of both operands to fp32.
 *  - lm_head_nvfp4_rows.rs, module doc and lm_head_nvfp4_rows_run: the NVFP4 head kept at the
 *    W4A16 precision its checkpoint declares, bf16 logits[rows, vocab], row-major hidden and
 *    logits, launching nothing unless the head can run, and logits of a row that are the same
 *    whatever the number of rows in the call.
 *
 * Conventions for every entry point:
 *  - All array arguments are DEVICE pointers owned by the caller. The library keeps no reference
 *    after the call returns; buffers must stay alive until the work on `stream` has finished.
 *  - Matrices are row-major and contiguous: hidden [rows, H], W [V, H] (used transposed), logits
 *    [rows, V].
 *  - A call validates its arguments synchronously on the host and launches nothing on error; it
 *    then enqueues its kernel (two for the log-probabilities and for the quantiser) on `stream`
 *    and returns without waiting. Faults surface at the caller's next synchronisation. There is
 *    no fallback path of any kind.
 *  - rows == 0 is valid and launches nothing.
 *  - Determinism: the same inputs give the same bits on every run (no atomics, no split-K). Each
 *    output element is one fp32 accumulator chain over k in ascending 16-element steps, the same
 *    for every row count, row position and tile, so a row's logits are bit-identical whether it
 *    is computed alone or with any other rows.
 *  - Outputs must not overlap inputs (LMHEAD_ERR_ALIAS).
 *  - Functions are thread-safe; calls on different streams may run concurrently.
 */
#ifndef LMHEAD_H
#define LMHEAD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
/* The same type as cudaStream_t / CUstream. NULL is the legacy default stream. */
typedef struct CUstream_st* lmhead_stream_t;

typedef enum {
  LMHEAD_OK = 0,
  LMHEAD_ERR_NULL = 1,    /* a required pointer is NULL */
  LMHEAD_ERR_SHAPE = 2,   /* a size is negative, zero where it must not be, or unsupported */
  LMHEAD_ERR_ALIGN = 3,   /* a pointer or row pitch breaks the alignment rules below */
  LMHEAD_ERR_ARCH = 4,    /* the current device is not an sm_100 (B200-class) GPU */
  LMHEAD_ERR_LAUNCH = 5,  /* the CUDA runtime refused the launch or a setup call */
  LMHEAD_ERR_TIMEOUT = 6, /* a kernel gave up waiting on one of its own barriers (see below) */
  LMHEAD_ERR_ALIAS = 7    /* the output range overlaps an input range */
} lmhead_status;

/*
 * Entry 1: fp32 logits from bf16 operands.
 *   logits[r, v] = fl32(alpha * acc[r, v]),  acc[r, v] = sum_k hidden[r, k] * W[v, k] in fp32.
 * The multiply by alpha is one IEEE round-to-nearest fp32 multiply of the finished accumulator
 * (no FMA contraction, no flush to zero), so lmhead_logits_bf16_f32(alpha) equals
 * fl32(lmhead_logits_bf16_f32(1.0f) * alpha) bit for bit. alpha = 1.0f gives the plain head.
 *
 *   hidden  bf16 [rows, H], 16-byte aligned          rows >= 0
 *   W       bf16 [V, H],    16-byte aligned          H > 0, H % 8 == 0 (16-byte row pitch)
 *   logits  fp32 [rows, V], 4-byte aligned           V > 0
 * Returns an lmhead_status.
 */
int lmhead_logits_bf16_f32(const void* hidden, int64_t rows, int64_t H, const void* W, int64_t V,
                           float alpha, float* logits, lmhead_stream_t stream);

/* Operand types of lmhead_logits_f32. */
typedef enum { LMHEAD_DTYPE_BF16 = 0, LMHEAD_DTYPE_F16 = 1 } lmhead_dtype;

/*
 * Entry 1 in general form: fp32 logits from bf16 or IEEE fp16 operands, with an optional
 * embedding bias.
 *   no bias:   logits[r, v] = fl32(alpha * acc[r, v])                (exactly entry 1)
 *   bias:      logits[r, v] = fl32(alpha * fl32(acc[r, v] + bias[v]))
 *   acc[r, v]  = sum_k hidden[r, k] * W[v, k] in fp32 (every product exact).
 * "FP32 LM head skip FP32 cast" takes the fused fp32-accumulate path for fp16 as well as bf16
 * hidden states of the weight's dtype; the first page ("Purpose") applies 1/mup after the
 * projection with its embedding bias, so the bias joins the sum before alpha. The add and the
 * multiply are single IEEE round-to-nearest fp32 operations (no FMA contraction).
 *
 *   hidden  dtype [rows, H], 16-byte aligned         rows >= 0
 *   W       dtype [V, H],    16-byte aligned         H > 0, H % 8 == 0
 *   bias    dtype [V], 2-byte aligned, or NULL       read only, must not overlap logits
 *   logits  fp32 [rows, V], 4-byte aligned           V > 0
 * dtype is an lmhead_dtype (anything else: LMHEAD_ERR_SHAPE). Returns an lmhead_status.
 */
int lmhead_logits_f32(const void* hidden, int dtype, int64_t rows, int64_t H, const void* W,
                      int64_t V, float alpha, const void* bias, float* logits,
                      lmhead_stream_t stream);

/*
 * Log-probabilities of given tokens, without writing logits. With z[r, v] the fp32 logits that
 * lmhead_logits_f32 would write for the same arguments (same bits),
 *   lse[r]       = log sum_v exp(z[r, v])
 *   logprobs[r]  = z[r, targets[r]] - lse[r]      (NaN when targets[r] is outside [0, V))
 * The first page ("Purpose") wants fp32 logits for RL training-inference consistency and for
 * speculative decoding, whose rejection sampling consumes exactly these; at prefill sizes this
 * avoids writing rows * V * 4 bytes of logits (5 GB at 8192 x 151936).
 * The head's epilogue reduces every 32-entry vocab chunk of a row to (max, sum of exp(z - max))
 * in fp32 and stores that pair in `workspace` (chunk-major); a second kernel folds a row's pairs
 * in a fixed order. So a row's results are the same whatever other rows the call carries, and
 * they are reproducible.
 * Accuracy: lse and logprobs are fp32 sums of expf terms; against the exact values over the same
 * fp32 logits they are good to a few units in 1e-6 relative.
 *
 *   hidden, W, bias, dtype, alpha: as lmhead_logits_f32
 *   targets    int32 [rows], 4-byte aligned
 *   logprobs   fp32 [rows], 4-byte aligned (output)
 *   lse        fp32 [rows], 4-byte aligned (output), or NULL
 *   workspace  at least lmhead_logprobs_workspace_bytes(rows, V) bytes, 8-byte aligned, owned by
 *              the caller (rows * 4 * ceil(V / 128) * 8 bytes)
 * Outputs and workspace must not overlap each other or the inputs. Two kernels are enqueued.
 * Returns an lmhead_status (LMHEAD_ERR_SHAPE also when the workspace is too small).
 */
size_t lmhead_logprobs_workspace_bytes(int64_t rows, int64_t V);
int lmhead_logprobs_f32(const void* hidden, int dtype, int64_t rows, int64_t H, const void* W,
                        int64_t V, float alpha, const void* bias, const int32_t* targets,
                        float* logprobs, float* lse, void* workspace, size_t workspace_bytes,
                        lmhead_stream_t stream);

/*
 * Vocab-parallel log-probabilities, in two calls around one exchange. "FP32 LM head skip FP32
 * cast" (key source excerpt, `_compute_lm_head`) takes the head as a VocabParallelEmbedding: each
 * of g GPUs holds a contiguous slice of W's rows, and the log-softmax of a row needs all of them.
 * lm_head_nvfp4_rows.rs (its install guard) keeps its own head to one GPU (tp_world_size 1);
 * this pair is for the fp32 head.
 *
 * 1. lmhead_logprobs_shard_stats_f32: on the GPU holding W_shard = W[v_begin, v_begin + V_shard),
 *    for each row r, with z the fp32 logits lmhead_logits_f32 would write for that slice (same
 *    bits as the same columns of the whole head):
 *      stats[3 r]     = m = max_v z[r, v]
 *      stats[3 r + 1] = s = sum_v exp(z[r, v] - m)          (fp32, fixed order)
 *      stats[3 r + 2] = z[r, targets[r]] if v_begin <= targets[r] < v_begin + V_shard, else NaN
 *    targets are global token ids. bias_shard is the slice of the bias (or NULL). The workspace
 *    is as lmhead_logprobs_f32's for V_shard rows of W. Two kernels are enqueued.
 * 2. The caller gathers the g stats arrays into one [g][rows][3] array in shard order (an
 *    all-gather of rows * 12 bytes per GPU).
 * 3. lmhead_logprobs_merge_shards folds the shards of each row in order:
 *      (m, s) = union of the shards' pairs,  lse[r] = m + log s,
 *      logprobs[r] = z[r, targets[r]] - lse[r]   (from the first shard that holds the target;
 *                                                 NaN when none does)
 *    One kernel is enqueued.
 * Results are deterministic for a given split; against the exact values over the same fp32
 * logits they are as accurate as lmhead_logprobs_f32's (one more fold per shard).
 *
 *   v_begin    >= 0; v_begin + V_shard <= 2^31 (token ids are int32), else LMHEAD_ERR_SHAPE
 *   stats      fp32 [rows][3], 4-byte aligned (output of 1, input of 3)
 *   shards     g >= 1
 *   logprobs   fp32 [rows]; lse fp32 [rows] or NULL; 4-byte aligned (outputs of 3)
 * Outputs must not overlap the inputs, the workspace or each other. Each returns an
 * lmhead_status.
 */
int lmhead_logprobs_shard_stats_f32(const void* hidden, int dtype, int64_t rows, int64_t H,
                                    const void* W_shard, int64_t V_shard, int64_t v_begin,
                                    float alpha, const void* bias_shard, const int32_t* targets,
                                    float* stats, void* workspace, size_t workspace_bytes,
                                    lmhead_stream_t stream);
int lmhead_logprobs_merge_shards(const float* stats, int64_t shards, int64_t rows,
                                 float* logprobs, float* lse, lmhead_stream_t stream);

/*
 * Vocab-parallel fp32 logits, gathered by the head itself. With the head split as above (each
 * of g GPUs holds W_slice = W[v_begin, v_begin + V_slice)), the GPU's slice of the logits is
 * written straight into columns [v_begin, v_begin + V_slice) of every buffer in `logits`:
 *   logits[d][r * ld_logits + v_begin + v] = z[r, v]      for d < n_logits, v < V_slice,
 * z the fp32 logits lmhead_logits_f32 would write for the slice (the same bits as those columns
 * of the whole head's logits: no row's reduction order depends on the split). Nothing else of
 * a buffer is written. Given every GPU's [rows, V] buffer (this GPU's own, and its peers'
 * mapped for peer access: symmetric or IPC memory over NVLink), one call per GPU plus a barrier
 * across the GPUs after it (and before the next call reuses the buffers) is the head and its
 * all-gather in one pass: each element is stored once into each buffer, by the epilogue that
 * produced it. The pages gather the sliced logits after the projection ("FP32 LM head skip FP32
 * cast", `_compute_lm_head` with its VocabParallelEmbedding head); here no second pass exists.
 *
 *   hidden, W_slice, bias_slice, dtype, alpha: as lmhead_logits_f32 (V = V_slice)
 *   logits     host array of n_logits device pointers, 1 <= n_logits <= 8, each 4-byte aligned,
 *              to a row-major fp32 buffer of at least rows rows of ld_logits floats
 *   v_begin    >= 0, with v_begin + V_slice <= ld_logits
 * The buffers must not overlap each other or the inputs. One kernel is enqueued; the library
 * synchronises nothing across GPUs. Returns an lmhead_status.
 */
int lmhead_logits_vocab_slice_f32(const void* hidden, int dtype, int64_t rows, int64_t H,
                                  const void* W_slice, int64_t V_slice, int64_t v_begin,
                                  float alpha, const void* bias_slice, float* const* logits,
                                  int n_logits, int64_t ld_logits, lmhead_stream_t stream);

/*
 * Entry 2: bf16 logits from the W4A16 NVFP4 head.
 *   W[v, k]      = e2m1(code[v, k]) * e4m3(w_scales[v, k / 16])      (exact in bf16)
 *   logits[r, v] = bf16_rn( fl32( fl32(acc[r, v] * w_global_scale) * alpha ) ),
 *   acc[r, v]    = sum_k hidden[r, k] * W[v, k] in fp32.
 * Layouts: w_packed is [V, H/2] bytes, element 2j of a row in the LOW nibble of byte j and
 * element 2j+1 in the high nibble; each E2M1 code is sign (bit 3), exponent (bits 2..1, bias 1),
 * mantissa (bit 0). w_scales is a plain row-major [V, H/16] array of E4M3 (fn variant) bytes;
 * scale j of row v covers k in [16j, 16j + 16). NaN scales give unspecified logits.
 * w_global_scale is the decode multiplier (w = code * scale * w_global_scale).
 *
 *   hidden    bf16 [rows, H], 16-byte aligned        rows >= 0
 *   w_packed  u8 [V, H/2],    16-byte aligned        H > 0, H % 32 == 0 (16-byte code rows)
 *   w_scales  u8 [V, H/16],   4-byte aligned
 *   logits    bf16 [rows, V], 2-byte aligned         V > 0
 * The kernel works in K steps of 64; when H % 64 == 32 the last step is half a step (the codes
 * past H read as zero and are not multiplied), with the same bits for every row count.
 * Returns an lmhead_status.
 */
int lmhead_logits_w4a16_nvfp4(const void* hidden, int64_t rows, int64_t H, const uint8_t* w_packed,
                              const uint8_t* w_scales, float w_global_scale, int64_t V,
                              float alpha, void* logits, lmhead_stream_t stream);

/*
 * NVFP4 quantiser: bf16 W -> the three inputs of lmhead_logits_w4a16_nvfp4. The pages name a
 * two-kernel quantiser, an absmax pass then an encode pass (lm_head_nvfp4_rows.rs and
 * mtp_head/new_bf16_moe.rs: `quantize_to_nvfp4` is handed the weight, its shape, the device, the
 * two kernels and a stream), but print no rules. This library's rules take every decision as one IEEE binary32 operation:
 *   amax = max |w|;  g = amax / 2688 (= 6 * 448), or 1 when amax = 0
 *   w_scales[v, j]  = RN_e4m3(max_{k in block j} |w[v, k]| / (6 * g)), saturating at 448
 *   code[v, k]      = RN_e2m1(w[v, k] / d), d = e4m3(w_scales[v, k/16]) * g, saturating at
 *                     +-6, with no negative zero; 0 where d is 0 (a block whose scale code is
 *                     0, or a product that underflows); RN = nearest, ties to the even code
 * Packing as lmhead_logits_w4a16_nvfp4 reads it (element 2j in the low nibble of byte j).
 *
 *   w               bf16 [V, H], 16-byte aligned, finite    H > 0, H % 16 == 0, V > 0
 *   w_packed        u8 [V, H/2], 8-byte aligned (output)
 *   w_scales        u8 [V, H/16] (output)
 *   w_global_scale  one fp32 in DEVICE memory, 4-byte aligned (output: g)
 *   workspace       device scratch of at least lmhead_nvfp4_quantize_workspace_bytes() bytes,
 *                   4-byte aligned, owned by the caller; it carries the absmax pass's per-block
 *                   maxima to the encode pass and may be reused once the call's work is done
 * No region may overlap another. Two kernels are enqueued on `stream`: the absmax pass reads W
 * once, the encode pass reads it again and writes the outputs. Returns an lmhead_status
 * (LMHEAD_ERR_SHAPE also when the workspace is too small).
 */
size_t lmhead_nvfp4_quantize_workspace_bytes(void);
int lmhead_nvfp4_quantize(const void* w, int64_t V, int64_t H, uint8_t* w_packed,
                          uint8_t* w_scales, float* w_global_scale, void* workspace,
                          size_t workspace_bytes, lmhead_stream_t stream);

/*
 * lmhead_nvfp4_quantize without a workspace argument, for callers that cannot obtain device
 * memory of their own: code that is handed its weight and output buffers by another component
 * (a model loader or a serving engine's memory pool) and is not allowed to call cudaMalloc, which
 * can synchronise the whole device and bypasses the pool that owns the GPU's memory. The method's
 * published description has no counterpart to this entry point; it exists for those callers.
 *
 * Same arguments, rules and results as lmhead_nvfp4_quantize. The absmax pass's scratch is a 4 KB
 * array that the library keeps on every GPU it is loaded on, until the process exits; the call
 * allocates nothing. Every argument is checked before any device state is touched. The first
 * call on a device (and the first after that device's context was replaced, e.g. by
 * cudaDeviceReset) looks up the array's device address, a host-side set-up step done while that
 * device is current, so make that first call before any stream capture. All calls on a device
 * share the one array: calls whose work overlaps on the GPU (on different streams without
 * ordering between them) race and give undefined results, so order them. The array needs no
 * clearing: each call's absmax pass writes every word its encode pass reads, and the encode pass
 * reads no other word. A call that would need more than the 4 KB is rejected with
 * LMHEAD_ERR_SHAPE (the quantiser's grid is sized to stay within it). Returns an lmhead_status.
 */
int lmhead_nvfp4_quantize_noalloc(const void* w, int64_t V, int64_t H, uint8_t* w_packed,
                                  uint8_t* w_scales, float* w_global_scale,
                                  lmhead_stream_t stream);

/* A static English description of a status code. Never NULL. */
const char* lmhead_status_string(int status);

/*
 * Every wait inside the kernels is bounded. When one runs out (the default limit is 2 s of wall
 * time per wait) the kernel records LMHEAD_ERR_TIMEOUT, and where it gave up, in a per-device
 * status word, stops its work and exits cleanly, so the CUDA context stays usable; the outputs
 * of that call are then undefined. The call itself returned LMHEAD_OK before its kernels ran, so
 * a caller that must not consume such outputs checks after synchronising:
 *
 * lmhead_device_status: the recorded status of the CURRENT device (LMHEAD_OK if none) and, when
 * `clear` is non-zero, resets it. The low byte is the lmhead_status; bits 8..15 name the waiting
 * role. It does not synchronise; read it after the work of interest has finished.
 *
 * lmhead_stream_status: synchronises `stream`, then returns and clears the current device's
 * status word (LMHEAD_OK when no wait ran out; LMHEAD_ERR_LAUNCH when the synchronisation itself
 * reported a CUDA error). The word is per device, not per stream: a timeout of work on another
 * stream of the same device that finished before this call is reported here too.
 */
int lmhead_device_status(int clear);
int lmhead_stream_status(lmhead_stream_t stream);

/* Library version as 10000 * major + 100 * minor + patch. */
int lmhead_version(void);

#if defined(LMHEAD_TEST_HOOKS) && LMHEAD_TEST_HOOKS
/*
 * Test build only (liblmhead_test.so, compiled with LMHEAD_TEST_HOOKS=1; the release
 * liblmhead.so does not export these). Host-side, per process:
 *
 * lmhead_debug_set_fault_injection: when `starve_loads` is non-zero, subsequent launches issue
 * no weight/activation loads, so their consumers wait on barriers that never complete and must
 * time out after `wait_limit_ns` nanoseconds. wait_limit_ns == 0 restores the default limit.
 *
 * lmhead_debug_set_nvfp4_conversion: selects lmhead_logits_w4a16_nvfp4's way of turning codes
 * into bf16: 1 = the shared-memory pair table whenever it leaves room for two pipeline stages,
 * 2 = integer spreading only, anything else = automatic (the table when it leaves room for
 * three stages). Both give identical bits; the knob lets tests show that.
 *
 * lmhead_debug_set_cta_pairs: enabled != 0 (the default) lets the fp32 head run full 256-row
 * tiles on CTA pairs (cta_group::2 MMAs, 256 vocab rows per tile); 0 keeps every tile on one
 * CTA. Both give identical bits; the knob lets tests show that.
 *
 * lmhead_debug_set_dynamic_tiles: enabled != 0 (the default) lets the fp32 head's persistent
 * units take their tiles after the first by cluster launch control, in launch order; 0 keeps
 * the static round-robin schedule. Both give identical bits; the knob lets tests show that.
 */
void lmhead_debug_set_fault_injection(int starve_loads, uint64_t wait_limit_ns);
void lmhead_debug_set_nvfp4_conversion(int path);
void lmhead_debug_set_cta_pairs(int enabled);
void lmhead_debug_set_dynamic_tiles(int enabled);
#endif

#ifdef __cplusplus
}
#endif

#endif /* LMHEAD_H */
