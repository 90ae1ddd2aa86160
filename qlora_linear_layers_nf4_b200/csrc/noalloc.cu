// nf4_quantize_noalloc: NF4 quantization for callers that cannot allocate
// device memory, not even a workspace.
//
// Who needs this: code that runs where cudaMalloc is off limits -- an engine
// plugin invoked with fixed buffers and no scratch allocator, a host
// application that has handed all device memory to its own pool, or a serving
// path that must not allocate after start-up.  nf4_quantize needs a caller
// workspace for the double-quant path (the fp32 block scales and the global
// max live there between its two kernels); this variant keeps that scratch in
// a fixed device array inside the library instead.
//
// The scratch array is a file-scope __device__ variable: every GPU that loads
// the library holds it (kNoAllocScratchBytes) until the process exits.  Its
// host-side name is only a stand-in for the symbol, never a device address;
// every call looks the address up with cudaGetSymbolAddress on the current
// device (cheap once the module is loaded, and never stale after the context
// was reset) and hands it to the kernels.  All calls on a device share the
// array and it keeps the last call's contents: every call writes the per-CTA
// maxima it reads, so nothing needs clearing; calls whose GPU work overlaps
// (different streams, no ordering) race on it.
#include "kernels.h"
#include "nf4_common.cuh"
#include "nvtx_range.h"

namespace nf4 {
namespace {

// Header (unused) + the quantize grid's per-CTA maxima + fp32 block scales
// for up to 2^20 blocks (64 Mi elements at block size 64).
constexpr int64_t kNoAllocMaxBlocks = int64_t(1) << 20;
constexpr size_t kNoAllocScratchBytes =
    kWsHeader + kWsMaxSlotsBytes + size_t(kNoAllocMaxBlocks) * sizeof(float);

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array on the current device.  Looked up on
// every call: a cached pointer would dangle once the context it came from is
// destroyed (cudaDeviceReset) and the module is loaded again.
cudaError_t scratch_address(uint8_t** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  *out = static_cast<uint8_t*>(p);
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace
}  // namespace nf4

extern "C" nf4_status nf4_quantize_noalloc(const float* w, int64_t rows, int64_t cols,
                                           int block_size, int double_quant, uint8_t* codes,
                                           float* absmax, uint8_t* absmax_q, float* absmax_scale,
                                           void* stream) {
  NF4_API_RANGE("nf4_quantize_noalloc");
  using namespace nf4;
  if (rows < 0 || cols < 0) return NF4_ERR_SHAPE;
  if (block_size <= 0 || (block_size % 2) != 0) return NF4_ERR_SHAPE;
  if (double_quant != 0 && double_quant != 1) return NF4_ERR_INVALID_ARG;
  if (rows != 0 && cols > INT64_MAX / rows) return NF4_ERR_SHAPE;
  const int64_t numel = rows * cols;
  const int64_t n_blocks = (numel + block_size - 1) / block_size;  // the last may be short
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (numel == 0) {  // empty tensor: nothing to encode; the scale of no scales is 0
    if (double_quant && absmax_scale != nullptr) {
      if (!aligned4(absmax_scale)) return NF4_ERR_ALIGNMENT;
      if (cudaMemsetAsync(absmax_scale, 0, sizeof(float), st) != cudaSuccess) return NF4_ERR_CUDA;
    }
    return NF4_OK;
  }
  if (w == nullptr || codes == nullptr) return NF4_ERR_INVALID_ARG;
  if (!double_quant && absmax == nullptr) return NF4_ERR_INVALID_ARG;
  if (double_quant && (absmax_q == nullptr || absmax_scale == nullptr)) return NF4_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(codes) || (absmax && !aligned16(absmax)) ||
      (absmax_q && !aligned16(absmax_q)) || (absmax_scale && !aligned4(absmax_scale)))
    return NF4_ERR_ALIGNMENT;
  // The fixed array only has to hold the block scales when the caller gives
  // no absmax buffer of its own.
  if (double_quant && absmax == nullptr && n_blocks > kNoAllocMaxBlocks) return NF4_ERR_WORKSPACE;

  uint8_t* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return NF4_ERR_CUDA;
  float* max_slots = reinterpret_cast<float*>(scratch + kWsHeader);
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
      sms = n;
  }
  int launches = 0;
  float* amax = absmax;
  if (double_quant && amax == nullptr)
    amax = reinterpret_cast<float*>(scratch + kWsHeader + kWsMaxSlotsBytes);
  int n_slots = 0;
  cudaError_t e = launch_quantize(w, NF4_F32, numel, block_size, codes, amax, /*status=*/nullptr,
                                  double_quant ? max_slots : nullptr, &n_slots, sms, st, &launches);
  if (e == cudaSuccess && double_quant)
    e = launch_double_quant(amax, n_blocks, max_slots, n_slots, absmax_q, absmax_scale, sms, st,
                            &launches);
  add_launches(launches);
  return e == cudaSuccess ? NF4_OK : NF4_ERR_CUDA;
}
