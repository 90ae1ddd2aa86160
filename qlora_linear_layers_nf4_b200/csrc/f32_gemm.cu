// The QLoRA linear layer in the F32 compute dtype: every product and sum in
// IEEE fp32 on the CUDA cores.
//
// The pages list BF16, F16 and F32 as the compute dtypes the forward dequant
// honours (qlora-rs README, "Honest capability matrix") and call F32 the
// debugging mode (rust-ai-core QLoraConfig, "Compute Dtype").  A debugging
// mode is there to give the reference answer of the 16-bit modes, so this
// path keeps fp32 throughout: the base is w' itself (one fp32 product
// L[code] * scale, the dequant of "NF4: quantizing the frozen base"), the
// operands are fp32 and the tensor cores are not used (their fp32-input
// kind rounds the operands to tf32).
//
// One kernel does every product of the layer.  C[rows, cols] = alpha * (sum
// over up to two reduction segments of A_s(i, kk) * B_s(j, kk)) (+ bias[j]),
// where each operand is either a dense fp32 matrix read in either major
// order or the NF4 weight decoded on load.  A 128 x 128 output tile per CTA,
// 256 threads with an 8 x 8 register tile each, the reduction in slices of 8
// staged through double-buffered shared memory with the next slice's global
// loads in flight while the current one is multiplied.
#include <algorithm>

#include <cuda_runtime.h>

#include "kernels.h"
#include "nf4_common.cuh"

namespace nf4 {
namespace {

constexpr int kFT = 128;          // output tile edge
constexpr int kFK = 8;            // reduction slice
constexpr int kFThreads = 256;
constexpr int kFPad = 4;          // row padding of the shared tiles (floats)
constexpr int kFRow = kFT + kFPad;

// One operand: element (i, kk), i an output index, kk the reduction index.
struct F32Operand {
  const float* p;          // dense fp32 matrix (nf4 == 0)
  int64_t ld;              // elements between consecutive stored rows
  int kmajor;              // 1: (i, kk) at p[i * ld + kk]; 0: at p[kk * ld + i]
  int nf4;                 // 1: the NF4 weight W [*, wcols], decoded to w'
  int64_t extent;          // number of valid i
  const uint8_t* codes;
  const float* absmax;
  const uint8_t* absmax_q;
  const float* absmax_scale;
  int dq;
  int bs_shift;            // log2 of the NF4 block size (6 .. 12)
  int64_t wcols;           // W's row length; kmajor: (i, kk) = W[i, kk], else W[kk, i]
};

struct F32Segment {
  F32Operand a, b;
  int64_t kdim;
};

struct F32GemmParams {
  F32Segment seg[2];
  int nseg;
  int64_t rows, cols;      // C [rows, cols], row-major with leading dimension ldc
  float* c;
  int64_t ldc;
  float alpha;
  const float* bias;       // [cols] or null
  int64_t col_tiles;
};

// Four consecutive-i or consecutive-kk elements of an operand for one thread
// of the slice load.  kmajor operands: thread t takes i = i0 + t / 2 and
// kk = k0 + 4 (t % 2) .. +3; the others: kk = k0 + t / 32 and
// i = i0 + 4 (t % 32) .. +3 (coalesced along the stored rows either way).
__device__ __forceinline__ void load_slice(const F32Operand& o, int64_t i0, int64_t k0,
                                           int64_t kdim, const float* lut, float (&v)[4]) {
  const int t = threadIdx.x;
  int64_t i, kk;
  if (o.kmajor) {
    i = i0 + (t >> 1);
    kk = k0 + 4 * (t & 1);
  } else {
    kk = k0 + (t >> 5);
    i = i0 + 4 * (t & 31);
  }
  v[0] = v[1] = v[2] = v[3] = 0.0f;
  if (o.nf4) {
    // four consecutive elements along a row of W: two code bytes, one scale
    // block (the row length and the column are multiples of 4, the block a
    // power of two of at least 64 elements)
    bool ok;
    int64_t e;
    if (o.kmajor) {
      ok = i < o.extent && kk < kdim;
      e = i * o.wcols + kk;
    } else {
      ok = kk < kdim && i < o.extent;
      e = kk * o.wcols + i;
    }
    if (!ok) return;
    const uint16_t two = *reinterpret_cast<const uint16_t*>(o.codes + (e >> 1));
    const int64_t blk = e >> o.bs_shift;
    const float scale =
        o.dq ? __fmul_rn(float(o.absmax_q[blk]), *o.absmax_scale) : o.absmax[blk];
    const uint32_t b0 = two & 0xffu, b1 = two >> 8;
    v[0] = __fmul_rn(lut[b0 >> 4], scale);
    v[1] = __fmul_rn(lut[b0 & 15u], scale);
    v[2] = __fmul_rn(lut[b1 >> 4], scale);
    v[3] = __fmul_rn(lut[b1 & 15u], scale);
    return;
  }
  if (o.kmajor) {
    if (i >= o.extent) return;
    const float* q = o.p + i * o.ld + kk;
    if (kk + 3 < kdim) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(q));
      v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
    } else {
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = (kk + u < kdim) ? __ldg(q + u) : 0.0f;
    }
  } else {
    if (kk >= kdim) return;
    const float* q = o.p + kk * o.ld + i;
    if (i + 3 < o.extent) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(q));
      v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
    } else {
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = (i + u < o.extent) ? __ldg(q + u) : 0.0f;
    }
  }
}

// Store a thread's four values into the [kk][i] shared tile.
__device__ __forceinline__ void store_slice(const F32Operand& o, float* s, const float (&v)[4]) {
  const int t = threadIdx.x;
  if (o.kmajor) {
    const int i = t >> 1, kk = 4 * (t & 1);
#pragma unroll
    for (int u = 0; u < 4; ++u) s[(kk + u) * kFRow + i] = v[u];
  } else {
    const int kk = t >> 5, i = 4 * (t & 31);
    *reinterpret_cast<float4*>(s + kk * kFRow + i) = make_float4(v[0], v[1], v[2], v[3]);
  }
}

__global__ void __launch_bounds__(kFThreads, 2) f32_gemm_kernel(const F32GemmParams p) {
  __shared__ __align__(16) float sa[2][kFK * kFRow];
  __shared__ __align__(16) float sb[2][kFK * kFRow];
  __shared__ float lut[16];
  if (threadIdx.x < 16) lut[threadIdx.x] = level(threadIdx.x);

  const int64_t tile = blockIdx.x;
  const int64_t i0 = (tile / p.col_tiles) * kFT;   // C rows
  const int64_t j0 = (tile % p.col_tiles) * kFT;   // C columns
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;

  // slices of both segments, in order
  const int64_t n0 = (p.seg[0].kdim + kFK - 1) / kFK;
  const int64_t n1 = p.nseg > 1 ? (p.seg[1].kdim + kFK - 1) / kFK : 0;
  const int64_t nslices = n0 + n1;

  float acc[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[a][b] = 0.0f;

  float va[4], vb[4];
  __syncthreads();   // lut
  auto fetch = [&](int64_t s) {
    const int g = s < n0 ? 0 : 1;
    const int64_t k0 = (s < n0 ? s : s - n0) * kFK;
    const F32Segment& sg = p.seg[g];
    load_slice(sg.a, i0, k0, sg.kdim, lut, va);
    load_slice(sg.b, j0, k0, sg.kdim, lut, vb);
    return g;
  };
  if (nslices > 0) {
    const int g = fetch(0);
    store_slice(p.seg[g].a, sa[0], va);
    store_slice(p.seg[g].b, sb[0], vb);
  }
  __syncthreads();
  for (int64_t s = 0; s < nslices; ++s) {
    const int cur = int(s & 1);
    int g_next = 0;
    if (s + 1 < nslices) g_next = fetch(s + 1);
    const float* A = sa[cur];
    const float* B = sb[cur];
#pragma unroll
    for (int kk = 0; kk < kFK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(A + kk * kFRow + 4 * ty);
      const float4 a1 = *reinterpret_cast<const float4*>(A + kk * kFRow + 64 + 4 * ty);
      const float4 b0 = *reinterpret_cast<const float4*>(B + kk * kFRow + 4 * tx);
      const float4 b1 = *reinterpret_cast<const float4*>(B + kk * kFRow + 64 + 4 * tx);
      const float ar[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float br[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(ar[a], br[b], acc[a][b]);
    }
    if (s + 1 < nslices) {
      store_slice(p.seg[g_next].a, sa[cur ^ 1], va);
      store_slice(p.seg[g_next].b, sb[cur ^ 1], vb);
    }
    __syncthreads();
  }

  // epilogue: rows 4ty..+3 and 64+4ty..+3, columns 4tx..+3 and 64+4tx..+3
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int64_t i = i0 + (a < 4 ? 4 * ty + a : 64 + 4 * ty + (a - 4));
    if (i >= p.rows) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t j = j0 + 64 * h + 4 * tx;
      float o[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        o[u] = __fmul_rn(p.alpha, acc[a][4 * h + u]);
        if (p.bias != nullptr && j + u < p.cols) o[u] = __fadd_rn(o[u], p.bias[j + u]);
      }
      float* dst = p.c + i * p.ldc + j;
      if (j + 3 < p.cols) {
        *reinterpret_cast<float4*>(dst) = make_float4(o[0], o[1], o[2], o[3]);
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (j + u < p.cols) dst[u] = o[u];
      }
    }
  }
}

F32Operand dense(const void* p, int64_t ld, bool kmajor, int64_t extent) {
  F32Operand o{};
  o.p = static_cast<const float*>(p);
  o.ld = ld;
  o.kmajor = kmajor ? 1 : 0;
  o.extent = extent;
  return o;
}

F32Operand nf4_weight_operand(const nf4_weight* w, bool kmajor, int64_t extent) {
  F32Operand o{};
  o.nf4 = 1;
  o.kmajor = kmajor ? 1 : 0;
  o.extent = extent;
  o.codes = w->codes;
  o.absmax = w->absmax;
  o.absmax_q = w->absmax_q;
  o.absmax_scale = w->absmax_scale;
  o.dq = w->double_quant ? 1 : 0;
  o.bs_shift = log2_block(w->block_size);
  o.wcols = w->cols;
  return o;
}

cudaError_t run_gemm(F32GemmParams& p, cudaStream_t st, int* launches) {
  const int64_t rt = (p.rows + kFT - 1) / kFT;
  p.col_tiles = (p.cols + kFT - 1) / kFT;
  const int64_t tiles = rt * p.col_tiles;
  if (tiles <= 0) return cudaSuccess;
  if (tiles > int64_t(0x7fffffff)) return cudaErrorInvalidValue;
  NF4_PROF_BEGIN(st, kKGemmF32);
  f32_gemm_kernel<<<unsigned(tiles), kFThreads, 0, st>>>(p);
  NF4_PROF_END(st, kKGemmF32);
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) ++*launches;
  return e;
}

size_t mr_f32_bytes(int64_t M, int r) {
  return (size_t(M) * size_t(r) * sizeof(float) + 255) / 256 * 256;
}

// T = s x A^T  [M, r]
cudaError_t gemm_T(const LinearArgs& a, float* T, cudaStream_t st, int* launches) {
  F32GemmParams p{};
  p.nseg = 1;
  p.seg[0].a = dense(a.x, a.K, true, a.M);
  p.seg[0].b = dense(a.A, a.K, true, a.r);
  p.seg[0].kdim = a.K;
  p.rows = a.M;
  p.cols = a.r;
  p.c = T;
  p.ldc = a.r;
  p.alpha = a.s;
  return run_gemm(p, st, launches);
}

// Every product of the layer fits one launch's grid (checked before the first
// launch, so a refused call enqueues nothing): the largest is M x max(N, K).
bool grids_fit(const LinearArgs& a) {
  const int64_t big = std::max(std::max(a.N, a.K), int64_t(a.r));
  return ((a.M + kFT - 1) / kFT) * ((big + kFT - 1) / kFT) <= int64_t(0x7fffffff) &&
         ((a.N + kFT - 1) / kFT) * ((a.r + kFT - 1) / kFT) <= int64_t(0x7fffffff) &&
         ((a.K + kFT - 1) / kFT) * ((a.r + kFT - 1) / kFT) <= int64_t(0x7fffffff);
}

}  // namespace

cudaError_t launch_linear_fwd_f32(const LinearArgs& a, cudaStream_t st, int* launches) {
  if (!grids_fit(a)) return cudaErrorInvalidValue;
  float* T = a.t_out ? static_cast<float*>(a.t_out) : reinterpret_cast<float*>(a.ws + kWsHeader);
  cudaError_t e = gemm_T(a, T, st, launches);
  if (e != cudaSuccess) return e;
  // y = x W'^T + T B^T (+ bias)
  F32GemmParams p{};
  p.nseg = 2;
  p.seg[0].a = dense(a.x, a.K, true, a.M);
  p.seg[0].b = nf4_weight_operand(a.w, true, a.N);
  p.seg[0].kdim = a.K;
  p.seg[1].a = dense(T, a.r, true, a.M);
  p.seg[1].b = dense(a.B, a.r, true, a.N);
  p.seg[1].kdim = a.r;
  p.rows = a.M;
  p.cols = a.N;
  p.c = static_cast<float*>(a.y);
  p.ldc = a.N;
  p.alpha = 1.0f;
  p.bias = static_cast<const float*>(a.bias);
  return run_gemm(p, st, launches);
}

cudaError_t launch_linear_bwd_f32(const LinearArgs& a, cudaStream_t st, int* launches) {
  if (!grids_fit(a)) return cudaErrorInvalidValue;
  uint8_t* ws = a.ws + kWsHeader;
  const float* T = static_cast<const float*>(a.t_in);
  cudaError_t e = cudaSuccess;
  if (T == nullptr) {
    float* Tw = reinterpret_cast<float*>(ws);
    e = gemm_T(a, Tw, st, launches);
    if (e != cudaSuccess) return e;
    T = Tw;
  }
  float* U = reinterpret_cast<float*>(ws + mr_f32_bytes(a.M, a.r));
  {  // U = s dy B  [M, r]: (i = m, kk = n) of dy, (j, kk = n) = B[n, j]
    F32GemmParams p{};
    p.nseg = 1;
    p.seg[0].a = dense(a.dy, a.N, true, a.M);
    p.seg[0].b = dense(a.B, a.r, false, a.r);
    p.seg[0].kdim = a.N;
    p.rows = a.M;
    p.cols = a.r;
    p.c = U;
    p.ldc = a.r;
    p.alpha = a.s;
    e = run_gemm(p, st, launches);
    if (e != cudaSuccess) return e;
  }
  {  // dB = dy^T T  [N, r]: (i = n, kk = m) = dy[m, n], (j, kk = m) = T[m, j]
    F32GemmParams p{};
    p.nseg = 1;
    p.seg[0].a = dense(a.dy, a.N, false, a.N);
    p.seg[0].b = dense(T, a.r, false, a.r);
    p.seg[0].kdim = a.M;
    p.rows = a.N;
    p.cols = a.r;
    p.c = a.dB;
    p.ldc = a.r;
    p.alpha = 1.0f;
    e = run_gemm(p, st, launches);
    if (e != cudaSuccess) return e;
  }
  {  // dA = U^T x  [r, K]: (i = j, kk = m) = U[m, j], (k, kk = m) = x[m, k]
    F32GemmParams p{};
    p.nseg = 1;
    p.seg[0].a = dense(U, a.r, false, a.r);
    p.seg[0].b = dense(a.x, a.K, false, a.K);
    p.seg[0].kdim = a.M;
    p.rows = a.r;
    p.cols = a.K;
    p.c = a.dA;
    p.ldc = a.K;
    p.alpha = 1.0f;
    e = run_gemm(p, st, launches);
    if (e != cudaSuccess) return e;
  }
  if (a.dx != nullptr) {  // dx = dy W' + U A  [M, K]
    F32GemmParams p{};
    p.nseg = 2;
    p.seg[0].a = dense(a.dy, a.N, true, a.M);
    p.seg[0].b = nf4_weight_operand(a.w, false, a.K);   // (k, kk = n) = W[n, k]
    p.seg[0].kdim = a.N;
    p.seg[1].a = dense(U, a.r, true, a.M);
    p.seg[1].b = dense(a.A, a.K, false, a.K);           // (k, kk = j) = A[j, k]
    p.seg[1].kdim = a.r;
    p.rows = a.M;
    p.cols = a.K;
    p.c = static_cast<float*>(a.dx);
    p.ldc = a.K;
    p.alpha = 1.0f;
    e = run_gemm(p, st, launches);
  }
  return e;
}

}  // namespace nf4
