// Internal launchers (host side).  Each returns the CUDA error of its launch
// and increments *launches once per kernel it launched successfully.
#pragma once

#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/nf4qlora.h"

namespace nf4 {

// One-time setup per device (a kernel's shared-memory opt-in applies to the
// current device only): one bit per device index, set atomically, so that
// several host threads or several devices in one process are safe.  Two
// threads may both run the setup once; it is idempotent.
struct PerDeviceOnce {
  std::atomic<uint64_t> bits{0};
  static int current() {
    int dev = -1;
    return cudaGetDevice(&dev) == cudaSuccess ? dev : -1;
  }
  bool done(int dev) const {
    return dev >= 0 && dev < 64 && ((bits.load(std::memory_order_acquire) >> dev) & 1u) != 0;
  }
  void mark(int dev) {
    if (dev >= 0 && dev < 64) bits.fetch_or(uint64_t(1) << dev, std::memory_order_acq_rel);
  }
};

// Adds to the library's launch counter (nf4_launch_count), for entry points
// outside api.cu.
void add_launches(int n);

// w holds numel elements of in_dtype (NF4_F32, NF4_BF16 or NF4_F16).  With
// max_slots, every CTA writes the max |w| it saw to one slot; *n_slots
// receives how many were written (at most kMaxSlots).
cudaError_t launch_quantize(const void* w, int in_dtype, int64_t numel, int bs, uint8_t* codes,
                            float* absmax_out, uint32_t* status, float* max_slots, int* n_slots,
                            int sms, cudaStream_t stream, int* launches);

// Double quant with G = max over max_slots[0 .. n_slots).
cudaError_t launch_double_quant(const float* absmax, int64_t n_blocks, const float* max_slots,
                                int n_slots, uint8_t* absmax_q, float* absmax_scale, int sms,
                                cudaStream_t stream, int* launches);
// Max of n non-negative fp32 scales into *gmax (bits), zeroing it first.
cudaError_t launch_absmax_max(const float* absmax, int64_t n, uint32_t* gmax, int sms,
                              cudaStream_t stream, int* launches);

cudaError_t launch_dequantize(const nf4_weight& w, int out_dtype, void* out, int sms,
                              cudaStream_t stream, int* launches);

// ---- QLoRA linear (qlora_gemm.cu) ----

struct LinearArgs {
  const nf4_weight* w;
  int64_t M, N, K;
  int r;
  float s;                 // alpha / r
  int f16;                 // compute type f16 (else bf16): x, A, B, bias, dy, y, dx, T, U
  int f32;                 // compute type fp32 (the CUDA-core path); f16 is then 0
  const void* x;           // [M, K] bf16 / f16
  const void* A;           // [r, K] bf16
  const void* B;           // [N, r] bf16
  const void* bias;        // [N] bf16 or null
  const void* dy;          // [M, N] bf16 (backward)
  const void* t_in;        // [M, r] bf16 T = s x A^T (backward, may be null)
  void* y;                 // [M, N] bf16
  void* t_out;             // [M, r] bf16 (forward, may be null)
  float* dA;               // [r, K] fp32
  float* dB;               // [N, r] fp32
  void* dx;                // [M, K] bf16 or null
  uint8_t* ws;             // workspace base
  size_t ws_bytes;
  uint32_t* status;
};

size_t linear_workspace_bytes(bool backward, int64_t M, int64_t N, int64_t K, int r);

// log2 of a block size the GEMM paths take (a power of two, 64 .. 4096), else -1.
inline int log2_block(int64_t bs) {
  for (int s = 6; s <= 12; ++s)
    if (bs == (int64_t(1) << s)) return s;
  return -1;
}

// 2-D TMA map over a row-major matrix (`inner` elements per row, `outer`
// rows; bf16 or u8), optional 128-byte swizzle.  False if it cannot be encoded.
bool make_map_2d(CUtensorMap* map, const void* base, bool bf16, uint64_t inner, uint64_t outer,
                 uint32_t box_inner, uint32_t box_outer, bool swizzle128);
// The same for fp32 and bf16 elements with any swizzle mode.
bool make_map_2d_f32(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                     uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle);
bool make_map_2d_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                      uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle);

// 3-D map (bf16 or u8 elements): dims innermost first, strides of dims 1 and
// 2 in bytes, box per dim, optional 128-byte swizzle.
bool make_map_3d(CUtensorMap* map, const void* base, bool bf16, uint64_t d0, uint64_t d1,
                 uint64_t d2, uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0,
                 uint32_t box1, uint32_t box2, bool swizzle128);

// Decode-shape forward (gemv.cu): one kernel for M <= 32 tokens.
bool decode_supported(int64_t M, int64_t N, int64_t K, int r);
// t_given: T = s x A^T [M, r] written by the kernel just before on the stream
// (then the decode kernel is its programmatic dependent and holds no A tiles),
// or null to compute it inside.  dry_run: check that the launch would go
// ahead (cudaErrorNotSupported if the shape does not fit), launch nothing.
cudaError_t launch_decode_fwd(const LinearArgs& a, int sms, cudaStream_t stream, int* launches,
                              const void* t_given = nullptr, bool dry_run = false);
// T = s x A^T [M, r] in the compute type for a decode call (M <= 32), the
// T the decode kernel takes finished; pdl: launch as a programmatic dependent.
cudaError_t launch_decode_t(const LinearArgs& a, void* T, cudaStream_t stream, int* launches, bool pdl);
cudaError_t launch_linear_fwd(const LinearArgs& a, int sms, cudaStream_t stream, int* launches);
cudaError_t launch_linear_bwd(const LinearArgs& a, int sms, cudaStream_t stream, int* launches);
// The F32 compute dtype (f32_gemm.cu): fp32 operands and outputs, CUDA-core fp32 FMAs.
cudaError_t launch_linear_fwd_f32(const LinearArgs& a, cudaStream_t stream, int* launches);
cudaError_t launch_linear_bwd_f32(const LinearArgs& a, cudaStream_t stream, int* launches);

// Bounded-wait self-check (selfcheck.cu): waits that nothing completes give
// up after limit_ns, record NF4_ERR_TIMEOUT in *status and raise the abort
// flag, which the second role counts into *seen_abort (one per CTA).
cudaError_t launch_wait_timeout_check(uint32_t* status, uint64_t limit_ns, uint32_t* seen_abort,
                                      cudaStream_t st, int* launches);

// Dense merge W' + s B A (merge.cu).
// Output types of the merge.
constexpr int kMergeBf16 = 0;
constexpr int kMergeF32 = 1;
constexpr int kMergeF16 = 2;
cudaError_t launch_merge(const nf4_weight& w, const void* A, const void* B, int r, float alpha,
                         int out_kind, void* out, uint32_t* status, cudaStream_t st, int* launches);

}  // namespace nf4

// ---- per-kernel event profiling (api.cu) ----
namespace nf4 {

enum KernelId {
  kKQuantize = 0,
  kKDoubleQuant,
  kKDequantize,
  kKAdapterT,        // adapter_gemm computing T = s x A^T
  kKFusedFwd,
  kKFusedDx,
  kKGemv,
  kKMerge,
  kKGemmF32,
  kKAbsmaxMax,
  kKAdapterU,        // adapter_gemm computing U = s dy B
  kKAdapterDB,       // adapter_gemm computing dB = dy^T T
  kKAdapterDA,       // adapter_gemm computing dA^T = x^T U
  kNumKernelIds
};

// When profiling is on, record an event on `stream` before / after a launch.
void prof_mark(cudaStream_t stream, int kernel_id, bool after);
// Whether per-kernel event profiling is on.  A launch that would otherwise
// overlap the kernel before it (programmatic dependent launch) runs fully
// serialised then, so each bracket times one kernel alone.
bool prof_on();

}  // namespace nf4

#define NF4_PROF_BEGIN(st, id) ::nf4::prof_mark((st), (id), false)
#define NF4_PROF_END(st, id) ::nf4::prof_mark((st), (id), true)
