// C-ABI entry points: argument validation on the host, then launches.
// Every check happens before anything is enqueued, so an error return means
// the stream was left untouched (the "refuse before writing anything" rule).
#include <atomic>
#include <cstring>
#include <mutex>
#include <vector>

#include "nf4_common.cuh"
#include "kernels.h"
#include "nvtx_range.h"

namespace {

std::atomic<int64_t> g_launches{0};

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

nf4_status finish(cudaError_t e, int launches) {
  g_launches += launches;
  return e == cudaSuccess ? NF4_OK : NF4_ERR_CUDA;
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Quantize workspace: the header; with double quant also the per-CTA maxima of
// the quantize grid and room for the fp32 block scales.
size_t quantize_ws(int64_t numel, int bs, int dq) {
  size_t bytes = nf4::kWsHeader;
  if (dq && bs > 0 && numel > 0)
    bytes += nf4::kWsMaxSlotsBytes + round_up(size_t((numel + bs - 1) / bs) * sizeof(float), 256);
  return bytes;
}

// Checks shared by the two linear entry points.
nf4_status check_linear(const nf4_weight* w, const void* x, int64_t M, const void* A,
                        const void* B, int r, float alpha, int compute_dtype) {
  if (w == nullptr || x == nullptr || A == nullptr || B == nullptr || w->codes == nullptr)
    return NF4_ERR_INVALID_ARG;
  if (w->double_quant) {
    if (w->absmax_q == nullptr || w->absmax_scale == nullptr) return NF4_ERR_INVALID_ARG;
  } else if (w->absmax == nullptr) {
    return NF4_ERR_INVALID_ARG;
  }
  if (!(alpha == alpha) || r < 8 || r > 256 || (r % 8) != 0) return NF4_ERR_INVALID_ARG;
  if (compute_dtype != NF4_BF16 && compute_dtype != NF4_F16 && compute_dtype != NF4_F32)
    return NF4_ERR_INVALID_ARG;
  if (M < 1 || w->rows < 1 || w->cols < 1) return NF4_ERR_SHAPE;
  if (w->block_size < 1) return NF4_ERR_SHAPE;
  if (nf4::log2_block(w->block_size) < 0) return NF4_ERR_UNSUPPORTED;   // 64, 128, ..., 4096
  if (w->cols % 64 != 0 || w->rows % 8 != 0) return NF4_ERR_SHAPE;
  if (M > (int64_t(1) << 31) || w->rows > (int64_t(1) << 31) || w->cols > (int64_t(1) << 31))
    return NF4_ERR_SHAPE;
  if (!aligned16(w->codes) || !aligned16(x) || !aligned16(A) || !aligned16(B))
    return NF4_ERR_ALIGNMENT;
  if (w->double_quant ? (!aligned16(w->absmax_q) || !aligned4(w->absmax_scale))
                      : !aligned16(w->absmax))
    return NF4_ERR_ALIGNMENT;
  return NF4_OK;
}

// Event brackets recorded while profiling is on.
struct ProfRecord {
  cudaEvent_t start;
  cudaEvent_t stop;
  int id;
};

std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRecord> g_prof_pending;
std::vector<cudaEvent_t> g_prof_free;
ProfRecord g_prof_open{nullptr, nullptr, -1};
int64_t g_prof_count[nf4::kNumKernelIds];
double g_prof_ms[nf4::kNumKernelIds];

const char* const kKernelNames[nf4::kNumKernelIds] = {
    "nf4_quantize", "nf4_double_quant", "nf4_dequantize", "adapter_gemm_T",
    "fused_nf4_gemm_fwd", "fused_nf4_gemm_dx", "nf4_gemv", "nf4_merge", "gemm_f32", "nf4_absmax_max",
    "adapter_gemm_U", "adapter_gemm_dB", "adapter_gemm_dA"};

cudaEvent_t prof_event() {
  if (!g_prof_free.empty()) {
    cudaEvent_t e = g_prof_free.back();
    g_prof_free.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

}  // namespace

namespace nf4 {
void add_launches(int n) { g_launches += n; }

bool prof_on() {
  std::lock_guard<std::mutex> lock(g_prof_mu);
  return g_prof_on;
}

void prof_mark(cudaStream_t stream, int kernel_id, bool after) {
  std::lock_guard<std::mutex> lock(g_prof_mu);
  if (!g_prof_on) return;
  if (!after) {
    g_prof_open.start = prof_event();
    g_prof_open.id = kernel_id;
    if (g_prof_open.start) cudaEventRecord(g_prof_open.start, stream);
  } else if (g_prof_open.start != nullptr && g_prof_open.id == kernel_id) {
    g_prof_open.stop = prof_event();
    if (g_prof_open.stop) {
      cudaEventRecord(g_prof_open.stop, stream);
      g_prof_pending.push_back(g_prof_open);
    }
    g_prof_open = ProfRecord{nullptr, nullptr, -1};
  }
}
}  // namespace nf4

extern "C" {

nf4_status nf4_profile_begin(void) {
  std::lock_guard<std::mutex> lock(g_prof_mu);
  for (int i = 0; i < nf4::kNumKernelIds; ++i) {
    g_prof_count[i] = 0;
    g_prof_ms[i] = 0.0;
  }
  g_prof_on = true;
  return NF4_OK;
}

nf4_status nf4_profile_end(void) {
  std::lock_guard<std::mutex> lock(g_prof_mu);
  g_prof_on = false;
  nf4_status st = NF4_OK;
  for (const ProfRecord& r : g_prof_pending) {
    float ms = 0.0f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess ||
        cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess) {
      st = NF4_ERR_CUDA;
    } else {
      g_prof_count[r.id] += 1;
      g_prof_ms[r.id] += ms;
    }
    g_prof_free.push_back(r.start);
    g_prof_free.push_back(r.stop);
  }
  g_prof_pending.clear();
  return st;
}

int nf4_profile_kernel_count(void) { return nf4::kNumKernelIds; }

const char* nf4_kernel_name(int kernel_id) {
  if (kernel_id < 0 || kernel_id >= nf4::kNumKernelIds) return "unknown";
  return kKernelNames[kernel_id];
}

nf4_status nf4_profile_get(int kernel_id, int64_t* launches, double* total_ms) {
  if (kernel_id < 0 || kernel_id >= nf4::kNumKernelIds) return NF4_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_prof_mu);
  if (launches) *launches = g_prof_count[kernel_id];
  if (total_ms) *total_ms = g_prof_ms[kernel_id];
  return NF4_OK;
}

const char* nf4_status_string(int status) {
  switch (status) {
    case NF4_OK: return "NF4_OK";
    case NF4_ERR_INVALID_ARG: return "NF4_ERR_INVALID_ARG: invalid argument";
    case NF4_ERR_SHAPE: return "NF4_ERR_SHAPE: unsupported shape";
    case NF4_ERR_ALIGNMENT: return "NF4_ERR_ALIGNMENT: pointer not 16-byte aligned";
    case NF4_ERR_UNSUPPORTED: return "NF4_ERR_UNSUPPORTED: not implemented in this build";
    case NF4_ERR_WORKSPACE: return "NF4_ERR_WORKSPACE: workspace missing or too small";
    case NF4_ERR_CUDA: return "NF4_ERR_CUDA: CUDA call failed";
    case NF4_ERR_NONFINITE: return "NF4_ERR_NONFINITE: NaN or Inf in quantize input";
    case NF4_ERR_TIMEOUT: return "NF4_ERR_TIMEOUT: device wait exceeded its limit";
    default: return "unknown nf4 status";
  }
}

int nf4_version(void) { return 100; }

void nf4_codebook(float* levels, float* thresholds) {
  if (levels != nullptr)
    for (int i = 0; i < 16; ++i) std::memcpy(&levels[i], &nf4::kLevelBits[i], 4);
  if (thresholds != nullptr)
    for (int i = 0; i < 15; ++i) std::memcpy(&thresholds[i], &nf4::kThresholdBits[i], 4);
}

int64_t nf4_launch_count(void) { return g_launches.load(); }

size_t nf4_workspace_bytes(int op, int64_t M, int64_t N, int64_t K, int r, int block_size,
                           int double_quant) {
  switch (op) {
    case NF4_OP_QUANTIZE: return quantize_ws(N * K, block_size, double_quant);
    case NF4_OP_DEQUANTIZE: return 0;
    case NF4_OP_LINEAR_FWD: return nf4::kWsHeader + nf4::linear_workspace_bytes(false, M, N, K, r);
    case NF4_OP_LINEAR_BWD: return nf4::kWsHeader + nf4::linear_workspace_bytes(true, M, N, K, r);
    case NF4_OP_MERGE: return nf4::kWsHeader;
    default: return 0;
  }
}

nf4_status nf4_read_status(void* workspace, void* stream) {
  if (workspace == nullptr) return NF4_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t host = 0;
  uint32_t* dev = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + nf4::kWsStatus);
  if (cudaMemcpyAsync(&host, dev, sizeof(host), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return NF4_ERR_CUDA;
  if (cudaMemsetAsync(dev, 0, sizeof(uint32_t), st) != cudaSuccess) return NF4_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return NF4_ERR_CUDA;
  return static_cast<nf4_status>(host);
}

}  // extern "C"

namespace {

nf4_status quantize_impl(const void* w, int in_dtype, int64_t rows, int64_t cols, int block_size,
                         int double_quant, uint8_t* codes, float* absmax, uint8_t* absmax_q,
                         float* absmax_scale, void* workspace, size_t ws_bytes, void* stream) {
  if (rows < 0 || cols < 0) return NF4_ERR_SHAPE;
  if (block_size <= 0 || (block_size % 2) != 0) return NF4_ERR_SHAPE;
  if (double_quant != 0 && double_quant != 1) return NF4_ERR_INVALID_ARG;
  if (rows != 0 && cols > INT64_MAX / rows) return NF4_ERR_SHAPE;
  const int64_t numel = rows * cols;  // a short last block is allowed
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
  if (workspace == nullptr || !aligned16(workspace)) return NF4_ERR_WORKSPACE;
  if (ws_bytes < quantize_ws(numel, block_size, double_quant)) return NF4_ERR_WORKSPACE;

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + nf4::kWsStatus);
  float* max_slots = reinterpret_cast<float*>(ws + nf4::kWsHeader);
  const int sms = sm_count();
  int launches = 0;
  float* amax = absmax;
  if (double_quant && amax == nullptr)
    amax = reinterpret_cast<float*>(ws + nf4::kWsHeader + nf4::kWsMaxSlotsBytes);
  int n_slots = 0;
  cudaError_t e = nf4::launch_quantize(w, in_dtype, numel, block_size, codes, amax, status,
                                       double_quant ? max_slots : nullptr, &n_slots, sms, st, &launches);
  if (e == cudaSuccess && double_quant)
    e = nf4::launch_double_quant(amax, (numel + block_size - 1) / block_size, max_slots, n_slots,
                                 absmax_q, absmax_scale, sms, st, &launches);
  return finish(e, launches);
}

}  // namespace

extern "C" {

nf4_status nf4_quantize(const float* w, int64_t rows, int64_t cols, int block_size,
                        int double_quant, uint8_t* codes, float* absmax, uint8_t* absmax_q,
                        float* absmax_scale, void* workspace, size_t ws_bytes, void* stream) {
  NF4_API_RANGE("nf4_quantize");
  return quantize_impl(w, NF4_F32, rows, cols, block_size, double_quant, codes, absmax, absmax_q,
                       absmax_scale, workspace, ws_bytes, stream);
}

nf4_status nf4_quantize_typed(const void* w, int in_dtype, int64_t rows, int64_t cols,
                              int block_size, int double_quant, uint8_t* codes, float* absmax,
                              uint8_t* absmax_q, float* absmax_scale, void* workspace,
                              size_t ws_bytes, void* stream) {
  NF4_API_RANGE("nf4_quantize_typed");
  if (in_dtype != NF4_F32 && in_dtype != NF4_BF16 && in_dtype != NF4_F16) return NF4_ERR_INVALID_ARG;
  return quantize_impl(w, in_dtype, rows, cols, block_size, double_quant, codes, absmax, absmax_q,
                       absmax_scale, workspace, ws_bytes, stream);
}

nf4_status nf4_absmax_max(const float* absmax, int64_t n_blocks, float* gmax, void* stream) {
  NF4_API_RANGE("nf4_absmax_max");
  if (n_blocks < 0) return NF4_ERR_SHAPE;
  if (gmax == nullptr || (n_blocks > 0 && absmax == nullptr)) return NF4_ERR_INVALID_ARG;
  if (!aligned4(gmax) || (absmax && !aligned4(absmax))) return NF4_ERR_ALIGNMENT;
  int launches = 0;
  cudaError_t e = nf4::launch_absmax_max(absmax, n_blocks, reinterpret_cast<uint32_t*>(gmax),
                                         sm_count(), static_cast<cudaStream_t>(stream), &launches);
  return finish(e, launches);
}

nf4_status nf4_double_quant(const float* absmax, int64_t n_blocks, const float* gmax,
                            uint8_t* absmax_q, float* absmax_scale, void* stream) {
  NF4_API_RANGE("nf4_double_quant");
  if (n_blocks < 0) return NF4_ERR_SHAPE;
  if (gmax == nullptr || absmax_scale == nullptr) return NF4_ERR_INVALID_ARG;
  if (n_blocks > 0 && (absmax == nullptr || absmax_q == nullptr)) return NF4_ERR_INVALID_ARG;
  if (!aligned4(gmax) || !aligned4(absmax_scale) || (absmax && !aligned16(absmax)) ||
      (absmax_q && !aligned16(absmax_q)))
    return NF4_ERR_ALIGNMENT;
  int launches = 0;
  cudaError_t e = nf4::launch_double_quant(absmax, n_blocks, gmax, 1, absmax_q, absmax_scale, sm_count(),
                                           static_cast<cudaStream_t>(stream), &launches);
  return finish(e, launches);
}

nf4_status nf4_dequantize(const nf4_weight* w, int out_dtype, void* out, void* stream) {
  NF4_API_RANGE("nf4_dequantize");
  if (w == nullptr || out == nullptr || w->codes == nullptr) return NF4_ERR_INVALID_ARG;
  if (out_dtype != NF4_F32 && out_dtype != NF4_BF16 && out_dtype != NF4_F16)
    return NF4_ERR_INVALID_ARG;
  if (w->rows < 0 || w->cols < 0) return NF4_ERR_SHAPE;
  if (w->block_size <= 0 || (w->block_size % 2) != 0) return NF4_ERR_SHAPE;
  if (w->rows != 0 && w->cols > INT64_MAX / w->rows) return NF4_ERR_SHAPE;
  const int64_t numel = w->rows * w->cols;  // a short last block is allowed
  if (w->double_quant) {
    if (w->absmax_q == nullptr || w->absmax_scale == nullptr) return NF4_ERR_INVALID_ARG;
    if (!aligned16(w->absmax_q) || !aligned4(w->absmax_scale)) return NF4_ERR_ALIGNMENT;
  } else {
    if (w->absmax == nullptr) return NF4_ERR_INVALID_ARG;
    if (!aligned16(w->absmax)) return NF4_ERR_ALIGNMENT;
  }
  if (!aligned16(w->codes) || !aligned16(out)) return NF4_ERR_ALIGNMENT;
  if (numel == 0) return NF4_OK;
  int launches = 0;
  cudaError_t e = nf4::launch_dequantize(*w, out_dtype, out, sm_count(),
                                         static_cast<cudaStream_t>(stream), &launches);
  return finish(e, launches);
}

nf4_status qlora_linear_fwd(const nf4_weight* w, const void* x, int64_t M, const void* A,
                            const void* B, int r, float alpha, int compute_dtype,
                            const void* bias, void* y, void* t_out, void* workspace,
                            size_t ws_bytes, void* stream) {
  NF4_API_RANGE("qlora_linear_fwd");
  nf4_status s = check_linear(w, x, M, A, B, r, alpha, compute_dtype);
  if (s != NF4_OK) return s;
  if (y == nullptr) return NF4_ERR_INVALID_ARG;
  if (!aligned16(y) || (bias && !aligned16(bias)) || (t_out && !aligned16(t_out)))
    return NF4_ERR_ALIGNMENT;
  if (workspace == nullptr || !aligned16(workspace)) return NF4_ERR_WORKSPACE;
  if (ws_bytes < nf4_workspace_bytes(NF4_OP_LINEAR_FWD, M, w->rows, w->cols, r, 64,
                                     w->double_quant))
    return NF4_ERR_WORKSPACE;
  nf4::LinearArgs a{};
  a.w = w;
  a.M = M;
  a.N = w->rows;
  a.K = w->cols;
  a.r = r;
  a.s = alpha / float(r);
  a.f16 = compute_dtype == NF4_F16 ? 1 : 0;
  a.f32 = compute_dtype == NF4_F32 ? 1 : 0;
  a.x = x;
  a.A = A;
  a.B = B;
  a.bias = bias;
  a.y = y;
  a.t_out = t_out;
  a.ws = static_cast<uint8_t*>(workspace);
  a.ws_bytes = ws_bytes;
  a.status = reinterpret_cast<uint32_t*>(a.ws + nf4::kWsStatus);
  int launches = 0;
  cudaError_t e = a.f32 ? nf4::launch_linear_fwd_f32(a, static_cast<cudaStream_t>(stream), &launches)
                        : nf4::launch_linear_fwd(a, sm_count(), static_cast<cudaStream_t>(stream),
                                                 &launches);
  if (e == cudaErrorNotSupported) { g_launches += launches; return NF4_ERR_UNSUPPORTED; }
  return finish(e, launches);
}

nf4_status qlora_linear_bwd(const nf4_weight* w, const void* x, int64_t M, const void* A,
                            const void* B, int r, float alpha, int compute_dtype,
                            const void* dy, const void* t, float* dA, float* dB, void* dx,
                            void* workspace, size_t ws_bytes, void* stream) {
  NF4_API_RANGE("qlora_linear_bwd");
  nf4_status s = check_linear(w, x, M, A, B, r, alpha, compute_dtype);
  if (s != NF4_OK) return s;
  if (dy == nullptr || dA == nullptr || dB == nullptr) return NF4_ERR_INVALID_ARG;
  if (!aligned16(dy) || !aligned16(dA) || !aligned16(dB) || (dx && !aligned16(dx)) ||
      (t && !aligned16(t)))
    return NF4_ERR_ALIGNMENT;
  if (workspace == nullptr || !aligned16(workspace)) return NF4_ERR_WORKSPACE;
  if (ws_bytes < nf4_workspace_bytes(NF4_OP_LINEAR_BWD, M, w->rows, w->cols, r, 64,
                                     w->double_quant))
    return NF4_ERR_WORKSPACE;
  nf4::LinearArgs a{};
  a.w = w;
  a.M = M;
  a.N = w->rows;
  a.K = w->cols;
  a.r = r;
  a.s = alpha / float(r);
  a.f16 = compute_dtype == NF4_F16 ? 1 : 0;
  a.f32 = compute_dtype == NF4_F32 ? 1 : 0;
  a.x = x;
  a.A = A;
  a.B = B;
  a.dy = dy;
  a.t_in = t;
  a.dA = dA;
  a.dB = dB;
  a.dx = dx;
  a.ws = static_cast<uint8_t*>(workspace);
  a.ws_bytes = ws_bytes;
  a.status = reinterpret_cast<uint32_t*>(a.ws + nf4::kWsStatus);
  int launches = 0;
  cudaError_t e = a.f32 ? nf4::launch_linear_bwd_f32(a, static_cast<cudaStream_t>(stream), &launches)
                        : nf4::launch_linear_bwd(a, sm_count(), static_cast<cudaStream_t>(stream),
                                                 &launches);
  if (e == cudaErrorNotSupported) { g_launches += launches; return NF4_ERR_UNSUPPORTED; }
  return finish(e, launches);
}

nf4_status nf4_check_wait_timeout(void* workspace, size_t ws_bytes, uint32_t limit_us,
                                  uint32_t* released, void* stream) {
  NF4_API_RANGE("nf4_check_wait_timeout");
  if (workspace == nullptr || !aligned16(workspace) || ws_bytes < nf4::kWsHeader) return NF4_ERR_WORKSPACE;
  if (released == nullptr || limit_us < 1 || limit_us > 1000000) return NF4_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + nf4::kWsStatus);
  uint32_t* seen = reinterpret_cast<uint32_t*>(ws + nf4::kWsHeader - 4);   // last header word
  if (cudaMemsetAsync(seen, 0, sizeof(uint32_t), st) != cudaSuccess) return NF4_ERR_CUDA;
  int launches = 0;
  if (nf4::launch_wait_timeout_check(status, uint64_t(limit_us) * 1000u, seen, st, &launches) != cudaSuccess)
    return NF4_ERR_CUDA;
  g_launches += launches;
  uint32_t host[2] = {0, 0};
  if (cudaMemcpyAsync(&host[0], status, sizeof(uint32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemcpyAsync(&host[1], seen, sizeof(uint32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemsetAsync(status, 0, sizeof(uint32_t), st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return NF4_ERR_CUDA;
  *released = host[1];
  return static_cast<nf4_status>(host[0]);
}

nf4_status nf4_merge(const nf4_weight* w, const void* A, const void* B, int r, float alpha,
                     int out_dtype, void* out, void* workspace, size_t ws_bytes, void* stream) {
  NF4_API_RANGE("nf4_merge");
  // the linear checks with a stand-in x (the merge has no activations)
  nf4_status s = check_linear(w, A, 1, A, B, r, alpha, NF4_BF16);
  if (s != NF4_OK) return s;
  if (out_dtype != NF4_BF16 && out_dtype != NF4_F32 && out_dtype != NF4_F16) return NF4_ERR_INVALID_ARG;
  if (out == nullptr) return NF4_ERR_INVALID_ARG;
  if (!aligned16(out)) return NF4_ERR_ALIGNMENT;
  if (workspace == nullptr || !aligned16(workspace)) return NF4_ERR_WORKSPACE;
  if (ws_bytes < nf4_workspace_bytes(NF4_OP_MERGE, 0, w->rows, w->cols, r, 64, w->double_quant))
    return NF4_ERR_WORKSPACE;
  uint32_t* status = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + nf4::kWsStatus);
  int launches = 0;
  const int kind = out_dtype == NF4_F32 ? nf4::kMergeF32 : (out_dtype == NF4_F16 ? nf4::kMergeF16 : nf4::kMergeBf16);
  const cudaError_t e = nf4::launch_merge(*w, A, B, r, alpha, kind, out,
                                          status, static_cast<cudaStream_t>(stream), &launches);
  return finish(e, launches);
}

}  // extern "C"
