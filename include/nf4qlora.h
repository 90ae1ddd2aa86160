/*
 * nf4qlora.h -- C ABI of the B200 (sm_100a) NF4 quantization and QLoRA
 * linear-layer library (libnf4qlora.so).
 *
 * What it computes (sources are the web pages on the subject):
 *   - NF4 quantization: qlora-rs README, "Honest capability matrix" (NF4
 *     pack/unpack + block absmax scales; simplified double quant) and
 *     "Quick Start" (quantize_nf4(&weights, 64)); "LoRA and QLoRA,
 *     mathematically", section "NF4: quantizing the frozen base" (sixteen
 *     levels at normal quantiles).  Storage follows the QuantizedTensor fields
 *     shown on the qlora-rs src/export.rs page (data, scales,
 *     scales_quantized, scales_scales, shape).
 *   - QLoRA linear: y = x W'^T + (alpha/r) (x A^T) B^T with W' the dequantized
 *     base in the compute dtype ("LoRA and QLoRA, mathematically", sections
 *     "Rank, alpha, and target modules" and "The merge math", equation 6.3.6;
 *     rust-ai-core QLoraConfig, scale() = alpha / r and "Compute Dtype").
 *   - Adapter backward of L = sum(dy * y) with W frozen:
 *     dB = s dy^T (x A^T), dA = s (dy B)^T x, dx = dy W' + s (dy B) A.
 *
 * Conventions shared by every entry point
 *   Memory     Every pointer argument is DEVICE memory owned by the caller,
 *              unless stated otherwise.  The library keeps no pointer after a
 *              call returns and allocates no device memory.
 *   Streams    `stream` is a cudaStream_t passed as void* (NULL = the legacy
 *              default stream).  All work is enqueued on it; buffers must stay
 *              alive until it completes.  Nothing synchronizes except
 *              nf4_read_status.  Several kernels (quantize, double quant,
 *              dequantize, decode, the forward GEMM) are launched with
 *              programmatic stream serialisation: each reads nothing that
 *              earlier work on the stream may still be writing (and writes
 *              nothing it may still be reading) before that work has
 *              completed, and some let the kernel after them launch early.  A kernel the
 *              caller launches after a call with that attribute must wait
 *              (griddepcontrol.wait / cudaGridDependencySynchronize) before it
 *              reads the call's outputs, as any such kernel must.
 *   Layouts    Row-major, densely packed.  W is [rows = N out, cols = K in].
 *              x is [M, K], A is [r, K], B is [N, r], y and dy are [M, N].
 *   Alignment  Device pointers must be 16-byte aligned unless the entry
 *              point states otherwise (NF4_ERR_ALIGNMENT).
 *   Errors     Arguments are validated, and every launch of a call is
 *              prepared (tensor maps encoded, grid sizes checked), on the
 *              host before the first launch: a call that returns any error
 *              other than NF4_ERR_CUDA has enqueued nothing.  NF4_ERR_CUDA
 *              means the CUDA runtime refused a launch or copy; launches of
 *              the same call that were enqueued before it may still run.
 *              Conditions only the GPU can see (non-finite input to quantize,
 *              an internal wait that exceeded its limit) are recorded in the
 *              status word at the head of `workspace` and returned by
 *              nf4_read_status.
 *   Workspace  Caller-allocated device scratch of at least
 *              nf4_workspace_bytes(...) bytes, zero-filled once before first
 *              use (the status word must start at 0).  Calls that share a
 *              workspace must be ordered on one stream.
 */
#ifndef NF4QLORA_H_
#define NF4QLORA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NF4_API __attribute__((visibility("default")))
#else
#define NF4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NF4_OK = 0,
  NF4_ERR_INVALID_ARG = 1,  /* NULL where a pointer is required, r out of range, ...   */
  NF4_ERR_SHAPE = 2,        /* sizes the operation does not accept                    */
  NF4_ERR_ALIGNMENT = 3,    /* a pointer that is not 16-byte aligned                  */
  NF4_ERR_UNSUPPORTED = 4,  /* a valid request this build does not implement          */
  NF4_ERR_WORKSPACE = 5,    /* workspace NULL or smaller than nf4_workspace_bytes     */
  NF4_ERR_CUDA = 6,         /* a CUDA runtime/driver call failed (launch error, ...)  */
  NF4_ERR_NONFINITE = 7,    /* device-detected: NaN or Inf in the quantize input      */
  NF4_ERR_TIMEOUT = 8       /* device-detected: an internal wait exceeded its limit   */
} nf4_status;

typedef enum { NF4_F32 = 0, NF4_BF16 = 1, NF4_F16 = 2 } nf4_dtype;

typedef enum {
  NF4_OP_QUANTIZE = 0,
  NF4_OP_DEQUANTIZE = 1,
  NF4_OP_LINEAR_FWD = 2,
  NF4_OP_LINEAR_BWD = 3,
  NF4_OP_MERGE = 4
} nf4_op;

/*
 * A quantized weight, mirroring the QuantizedTensor of the qlora-rs
 * src/export.rs page (data -> codes, scales -> absmax, scales_quantized ->
 * absmax_q, scales_scales -> absmax_scale, shape -> rows/cols).  Asymmetric
 * zero-points are not part of NF4 and are not represented.
 *   codes         ceil(rows*cols/2) bytes.  Element e of the row-major
 *                 flattened tensor has a 4-bit code in byte e/2: the HIGH
 *                 nibble for even e, the LOW nibble for odd e.  For an odd
 *                 element count the last byte's low nibble is 7 (level 0.0).
 *   absmax        fp32 per block (nblocks = ceil(rows*cols/block_size)), block
 *                 b covering elements [b*block_size, (b+1)*block_size); the
 *                 last block may be short and covers the elements that
 *                 remain.  Used when double_quant == 0.  May be NULL when
 *                 double_quant != 0.
 *   absmax_q      u8 per block, used when double_quant != 0.
 *   absmax_scale  one fp32 (the scale of the scales), used when
 *                 double_quant != 0.  Block b decodes with
 *                 scale_b = fp32((float)absmax_q[b] * absmax_scale[0]).
 */
typedef struct {
  const uint8_t* codes;
  const float* absmax;
  const uint8_t* absmax_q;
  const float* absmax_scale;
  int64_t rows;
  int64_t cols;
  int32_t block_size;
  int32_t double_quant;
} nf4_weight;

/* Human-readable name of a status code (static string, never NULL). */
NF4_API const char* nf4_status_string(int status);

/* Library ABI version (major * 100 + minor). */
NF4_API int nf4_version(void);

/*
 * Host copy of the device codebook.  levels[i] is the fp32 NF4 level of code
 * i (ascending, levels[0] = -1, levels[7] = 0, levels[15] = +1).
 * thresholds[i] is the largest fp32 value not above the exact midpoint of
 * levels[i] and levels[i+1]; the encoder's code for a normalised value v is
 * the number of thresholds strictly below v (nearest level, lower code on an
 * exact tie).  Either pointer may be NULL.  Host memory; needs no GPU.
 */
NF4_API void nf4_codebook(float* levels, float* thresholds);

/*
 * Number of kernel launches the library has made in this process (host-side
 * counter, incremented once per successful launch).  Needs no GPU.
 */
NF4_API int64_t nf4_launch_count(void);

/*
 * Per-kernel timing, for benchmarks.  nf4_profile_begin() turns recording on
 * (and clears earlier totals): every kernel the library launches is then
 * bracketed by two CUDA events on its launch stream.  nf4_profile_end()
 * waits for the recorded events, adds each bracket's elapsed time to its
 * kernel's total and turns recording off.  nf4_profile_get() returns the
 * number of timed launches and their summed milliseconds for a kernel id
 * (0 <= id < nf4_profile_kernel_count()); nf4_kernel_name() names it.
 * The events are created by the library (no device memory).  Returns
 * NF4_OK, NF4_ERR_INVALID_ARG for a bad id, NF4_ERR_CUDA on event failure.
 */
NF4_API nf4_status nf4_profile_begin(void);
NF4_API nf4_status nf4_profile_end(void);
NF4_API int nf4_profile_kernel_count(void);
NF4_API const char* nf4_kernel_name(int kernel_id);
NF4_API nf4_status nf4_profile_get(int kernel_id, int64_t* launches, double* total_ms);

/*
 * Bytes of workspace an operation needs (0 = none).  M, N, K, r are the
 * linear-layer sizes (N = W rows, K = W cols); for NF4_OP_QUANTIZE and
 * NF4_OP_DEQUANTIZE pass N = rows, K = cols and M = r = 0.  Needs no GPU.
 */
NF4_API size_t nf4_workspace_bytes(int op, int64_t M, int64_t N, int64_t K, int r, int block_size,
                           int double_quant);

/*
 * Synchronizes `stream`, returns the device status recorded in `workspace`
 * since the last call (NF4_OK if none), and resets it to NF4_OK.  A failing
 * CUDA call gives NF4_ERR_CUDA.
 */
NF4_API nf4_status nf4_read_status(void* workspace, void* stream);

/*
 * Blockwise NF4 quantization (qlora-rs quantize_nf4; capability matrix
 * "NF4 pack/unpack + block absmax scales" and "Double quant (simplified
 * global u8 scales)").
 *   w            fp32 [rows, cols], read only.
 *   block_size   positive and even.  Multiples of 8 up to 256 that are
 *                powers of two take the vectorized path; other even sizes a
 *                per-block path.  rows*cols need not be a multiple of it: the
 *                last block then holds the remaining elements, its absmax is
 *                the max over those alone, and a small extra kernel encodes
 *                it (the pages' quantize_nf4 takes tensors of any size).
 *   For each block: absmax = max |w|; v = w / absmax (IEEE fp32 division);
 *   code = index of the nearest NF4 level (lower code on an exact tie);
 *   absmax == 0 gives code 7 for the whole block.
 *   codes        u8 [ceil(rows*cols/2)], written (packing as in nf4_weight).
 *   absmax       fp32 [nblocks]; written when non-NULL.  Required when
 *                double_quant == 0.
 *   double_quant 0 or 1.  When 1: G = max absmax, absmax_scale[0] =
 *                fp32(G / 255) and absmax_q[b] = clamp(rint(absmax_b /
 *                absmax_scale), 0, 255) with ties to even; G == 0 gives 0
 *                and 0.  absmax_q (u8 [nblocks]) and absmax_scale (fp32[1])
 *                are then required.  The codes do not depend on
 *                double_quant.
 *   workspace    >= nf4_workspace_bytes(NF4_OP_QUANTIZE, ...).
 * NaN/Inf in w is outside the contract: the kernels flag NF4_ERR_NONFINITE
 * in the workspace status word (the outputs are then unspecified).
 */
NF4_API nf4_status nf4_quantize(const float* w, int64_t rows, int64_t cols, int block_size,
                        int double_quant, uint8_t* codes, float* absmax, uint8_t* absmax_q,
                        float* absmax_scale, void* workspace, size_t ws_bytes, void* stream);

/*
 * nf4_quantize without a workspace, for callers that cannot allocate device
 * memory at all: an engine plugin handed fixed buffers and no scratch
 * allocator, an application whose own pool owns all device memory, a serving
 * path that must not allocate after start-up.  The pages describe no such
 * entry point; it exists for those callers.
 * Arguments and results are those of nf4_quantize (same kernels, bit-identical
 * output); the scratch that nf4_quantize keeps in `workspace` lives instead in
 * a fixed device array inside the library, 4 MiB + 8 KiB + 256 B, which every
 * GPU that loads the library holds until the process exits.  With double_quant
 * and absmax == NULL the block scales are kept there, so rows*cols/block_size
 * may not exceed 1048576 (NF4_ERR_WORKSPACE otherwise); with a caller absmax
 * buffer there is no size limit.  Calls no allocator (no cudaMalloc or
 * cudaFree).  Every call looks up the array's device address on the current
 * device (cudaGetSymbolAddress); the first call on a device is the one that
 * may load the library's device code there, so it should come before any
 * stream capture.  All calls share the array and it keeps the last call's
 * contents (each call writes every value it reads from it, so nothing needs
 * clearing); calls whose GPU work overlaps race.  Launches are counted in nf4_launch_count.
 * Non-finite input is not reported (there is no status word to read).
 */
NF4_API nf4_status nf4_quantize_noalloc(const float* w, int64_t rows, int64_t cols,
                                        int block_size, int double_quant, uint8_t* codes,
                                        float* absmax, uint8_t* absmax_q, float* absmax_scale,
                                        void* stream);

/*
 * nf4_quantize for a weight held in another element type: in_dtype NF4_F32
 * (identical to nf4_quantize), NF4_BF16 or NF4_F16.  Each element is widened
 * to fp32 exactly and quantized as nf4_quantize would quantize that fp32
 * value (the pages' quantize_nf4 takes any tensor; a bf16 model's weights
 * are quantized without an fp32 copy).  w is rows*cols elements of in_dtype,
 * 16-byte aligned; every other argument, result and error as nf4_quantize.
 * NF4_ERR_INVALID_ARG for any other in_dtype.
 */
NF4_API nf4_status nf4_quantize_typed(const void* w, int in_dtype, int64_t rows, int64_t cols,
                                      int block_size, int double_quant, uint8_t* codes,
                                      float* absmax, uint8_t* absmax_q, float* absmax_scale,
                                      void* workspace, size_t ws_bytes, void* stream);

/*
 * The two halves of the simplified double quant, for a tensor whose rows are
 * quantized on several ranks (data parallel): each rank quantizes its shard
 * with double_quant = 0 and keeps its fp32 block scales, takes their max with
 * nf4_absmax_max, the ranks all-reduce that float with MAX (the one exchange;
 * NCCL over NVLink), and each rank then encodes its scales against the global
 * max with nf4_double_quant.  With shards that start on block boundaries the
 * result is bit for bit the rows of a single-device nf4_quantize with
 * double_quant = 1 (qlora-rs README, "Double quantization (simplified)": one
 * scale of scales for the whole tensor).
 *
 * nf4_absmax_max: gmax[0] = max over absmax[0 .. n_blocks) (all >= 0; 0 for
 *   n_blocks == 0).  absmax fp32 [n_blocks] and gmax fp32 [1] are device
 *   memory, 4-byte aligned; gmax is overwritten.  Enqueued on `stream`.
 */
NF4_API nf4_status nf4_absmax_max(const float* absmax, int64_t n_blocks, float* gmax, void* stream);

/*
 * nf4_double_quant: with G = gmax[0] (device, >= 0, normally the global max
 *   of the block scales), absmax_scale[0] = fp32(G / 255) and absmax_q[b] =
 *   clamp(rint(absmax[b] / absmax_scale[0]), 0, 255), ties to even; G == 0
 *   gives 0 and 0 -- exactly the double-quant stage of nf4_quantize.
 *   absmax fp32 [n_blocks] and absmax_q u8 [n_blocks] 16-byte aligned;
 *   absmax_scale fp32 [1] and gmax 4-byte aligned.  Enqueued on `stream`.
 */
NF4_API nf4_status nf4_double_quant(const float* absmax, int64_t n_blocks, const float* gmax,
                                    uint8_t* absmax_q, float* absmax_scale, void* stream);

/*
 * Self-check of the bounded-wait path (no counterpart on the pages).  Every
 * mbarrier wait in the library's kernels gives up after a time limit, records
 * NF4_ERR_TIMEOUT in the workspace status word and raises its CTA's abort
 * flag, on which the CTA's other roles unwind; a lost arrival therefore ends
 * in an error status, never in a hung GPU.  This call runs that path on
 * purpose: two CTAs each wait on an mbarrier that nothing arrives on, with a
 * limit of limit_us microseconds (1 .. 1000000), while a second warp per CTA
 * waits with a 100x longer limit and must be released by the abort flag.
 * Synchronizes `stream`; returns the status word the kernel left (NF4_ERR_TIMEOUT
 * when the path works), clears it, and stores in *released the number of CTAs
 * whose second warp was released by the abort (2 when the path works).
 *   workspace  >= 256 bytes, 16-byte aligned.
 */
NF4_API nf4_status nf4_check_wait_timeout(void* workspace, size_t ws_bytes, uint32_t limit_us,
                                          uint32_t* released, void* stream);

/*
 * Dequantization (qlora-rs dequantize_nf4; "Honor compute_dtype
 * (BF16/F16/F32) in forward dequant").  out[e] = fp32(L[code_e] * scale_b)
 * as one fp32 product; NF4_BF16 / NF4_F16 store its round-to-nearest-even.
 *   w->block_size must be positive and even (multiples of 8 take the
 *   vectorized path); rows*cols need not be a multiple of it (a short last
 *   block decodes with its own scale).  out has rows*cols elements of
 *   out_dtype.
 */
NF4_API nf4_status nf4_dequantize(const nf4_weight* w, int out_dtype, void* out, void* stream);

/*
 * QLoRA linear forward (QuantizedLinear::forward of the qlora-rs README;
 * equation 6.3.6 of "LoRA and QLoRA, mathematically" read as a layer):
 *   y = x W'^T + s (x A^T) B^T (+ bias),  s = alpha / r,
 * W' the dequantized base rounded to compute_dtype, operands in
 * compute_dtype, fp32 accumulation, y rounded to compute_dtype.
 *   w              N = w->rows (out), K = w->cols (in); block_size a power
 *                  of two from 64 to 4096 (others: NF4_ERR_UNSUPPORTED);
 *                  K % 64 == 0, N % 8 == 0.  Blocks run over the flattened
 *                  weight, so K need not be a multiple of the block size.
 *   x              [M, K] compute_dtype; M >= 1.
 *   A, B           [r, K] and [N, r] compute_dtype; 8 <= r <= 256, r % 8 == 0.
 *   compute_dtype  NF4_BF16, NF4_F16 or NF4_F32.  NF4_F32 is the pages'
 *                  debugging mode (rust-ai-core QLoraConfig, "Compute
 *                  Dtype"): x, A, B, bias, y, T (and dy, dx) fp32, W' the
 *                  fp32 dequant itself (not rounded further), every product
 *                  and sum an IEEE fp32 operation on the CUDA cores (no tf32
 *                  rounding of the operands), s applied as one fp32 multiply.
 *                  It is a reference mode: about 33x slower than BF16 on an
 *                  11008 x 4096 layer with 4096 tokens.
 *   bias           [N] compute_dtype, or NULL.
 *   y              [M, N] compute_dtype, written.
 *   t_out          [M, r] compute_dtype, or NULL: when given, receives
 *                  T = s (x A^T) -- the adapter activation already scaled
 *                  by s and rounded to compute_dtype (2-byte elements for
 *                  BF16 / F16, not an fp32 x A^T) -- which qlora_linear_bwd
 *                  accepts as `t`.
 *   workspace      >= nf4_workspace_bytes(NF4_OP_LINEAR_FWD, M, N, K, r, 64, dq)
 *                  (the same size serves every compute dtype).
 * BF16 / F16: M <= 32 uses the weight-streaming decode path, larger M the
 * fused dequantize + tensor-core GEMM; both compute the same function.
 */
NF4_API nf4_status qlora_linear_fwd(const nf4_weight* w, const void* x, int64_t M, const void* A,
                            const void* B, int r, float alpha, int compute_dtype,
                            const void* bias, void* y, void* t_out, void* workspace,
                            size_t ws_bytes, void* stream);

/*
 * QLoRA linear adapter backward for L = sum(dy * y), the base W frozen
 * (qlora-rs capability matrix: adapters train on a frozen NF4 base):
 *   U  = s (dy B)                                [M, r]
 *   dB = s dy^T (x A^T)  = dy^T T                 fp32 [N, r], overwritten
 *   dA = s (dy B)^T x    = U^T x                  fp32 [r, K], overwritten
 *   dx = dy W' + s (dy B) A = dy W' + U A         [M, K] compute_dtype, or NULL
 * Arguments as for qlora_linear_fwd; dy is [M, N] compute_dtype; `t` is the
 * T written by the forward's t_out, or NULL to recompute it.
 *   workspace      >= nf4_workspace_bytes(NF4_OP_LINEAR_BWD, M, N, K, r, 64, dq).
 * Streams: with BF16 / F16 and dx given, dx runs on a high-priority stream the
 * library keeps per device and calling stream (made on the first such call;
 * up to 8 calling streams per device have their own, more share them), forked
 * from `stream` after U and joined back with events before the call returns,
 * so work the caller enqueues on `stream` afterwards sees every output;
 * `stream` must belong to the current device.  Calls from several host
 * threads serialise on a lock while they enqueue.  The fork and join are
 * ordinary event dependencies, so a backward call enqueued while `stream` is
 * being captured into a CUDA graph becomes part of the graph, side branch
 * included (the side stream is made on the first call, so make one call
 * before capturing).
 */
NF4_API nf4_status qlora_linear_bwd(const nf4_weight* w, const void* x, int64_t M, const void* A,
                            const void* B, int r, float alpha, int compute_dtype,
                            const void* dy, const void* t, float* dA, float* dB, void* dx,
                            void* workspace, size_t ws_bytes, void* stream);

/*
 * Merge of the quantized base with its trained adapter into one dense weight
 * (qlora-rs src/export.rs, merge_and_export_gguf: W_merged = W_base +
 * (B @ A) * scale; "LoRA and QLoRA, mathematically", "The merge math",
 * equation 6.3.6 -- the merged weight stays in BF16, it is not requantized):
 *   out[n, k] = w'[n, k] + s (B A)[n, k],  s = alpha / r,
 * w' = fp32(L[code] * scale) the fp32 dequant, B A accumulated in fp32, the sum
 * rounded once to fp32 (one FMA) and then, for NF4_BF16 or NF4_F16, to that
 * type (nearest, ties to even; beyond the f16 range, +-inf).
 *   w          block_size a power of two from 64 to 4096; cols % 64 == 0,
 *              rows % 8 == 0.
 *   A, B       [r, K] and [N, r] bf16; 8 <= r <= 256, r % 8 == 0.
 *   out_dtype  NF4_BF16, NF4_F16 or NF4_F32; out has rows * cols elements,
 *              written.
 *   workspace  >= nf4_workspace_bytes(NF4_OP_MERGE, 0, N, K, r, 64, dq): the
 *              status word only.
 * Same validation, ownership and error rules as the linear entry points.
 */
NF4_API nf4_status nf4_merge(const nf4_weight* w, const void* A, const void* B, int r, float alpha,
                             int out_dtype, void* out, void* workspace, size_t ws_bytes,
                             void* stream);

#ifdef __cplusplus
}
#endif

#endif /* NF4QLORA_H_ */
