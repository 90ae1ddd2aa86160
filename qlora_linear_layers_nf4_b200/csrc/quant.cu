// NF4 quantize / double-quant / dequantize kernels (memory-bound).
//
// Quantize follows the qlora-rs README ("Honest capability matrix": NF4
// pack/unpack + block absmax scales; "Double quantization (simplified)") and
// the level construction of "LoRA and QLoRA, mathematically" ("NF4: quantizing
// the frozen base").  Each thread owns 8 consecutive elements (32 bytes in,
// one u32 of packed codes out); the absmax of a block of bs elements is a
// shuffle-xor reduction over the bs/8 lanes that hold it.
#include <algorithm>
#include <mutex>
#include <utility>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "nf4_common.cuh"
#include "kernels.h"

namespace nf4 {

namespace {

// Max of |x| over 8 values as the integer max of their magnitude bits: for
// non-negative floats integer order is float order, and an Inf (0x7f800000)
// or NaN (above it) is the largest, so one compare of the block max finds
// every non-finite input.
__device__ __forceinline__ uint32_t max_abs_bits8(const float4& a, const float4& b) {
  const uint32_t m = 0x7fffffffu;
  uint32_t r = max(max(__float_as_uint(a.x) & m, __float_as_uint(a.y) & m),
                   max(__float_as_uint(a.z) & m, __float_as_uint(a.w) & m));
  return max(r, max(max(__float_as_uint(b.x) & m, __float_as_uint(b.y) & m),
                    max(__float_as_uint(b.z) & m, __float_as_uint(b.w) & m)));
}

// Fast encode.  v = RN(w / a) is formed without a division: y = RN(1/a) once
// per block (CUDA's correctly rounded reciprocal), q = RN(w y), then one
// FMA-based correction q' = q + (w - a q) y.  That is Markstein's correction
// step; with a correctly rounded reciprocal it yields the correctly rounded
// quotient when the remainder w - a q is representable.  Its lowest bit is
// ulp(a) ulp(q) = 2^(ea + eq - 46), so it must satisfy ea + eq >= -103 not to
// fall below the smallest subnormal.  Only quotients of magnitude >= 2^-5
// can decide an NF4 code (every decision threshold is >= 0.0398 from zero)
// and >= 2^-2 a double-quant code, so the step is taken for 2^-98 <= a <
// 2^120 and other blocks take the division.  A host test runs the three
// steps in C over that range against the IEEE quotient.
//
// The nearest level then comes from two small tables.  One FFMA rounds
// 32 v + 32 to an integer i in 0..64 (v is in [-1, 1]): bucket i covers
// [(i - 32.5) / 32, (i - 31.5) / 32).  base[i] is the number of decision
// thresholds below the bucket's lower edge, so the only threshold that can lie
// inside it is thr[base[i]] and code = base[i] + (v > thr[base[i]]).  No
// threshold lies within 2e-4 of a bucket edge, far beyond the index rounding,
// so a v next to an edge gets the same code from either bucket.  base has 128
// entries (every value of the low 7 bits, so a NaN, which the absmax pass
// flags, still indexes inside the table) and thr ends with +inf.  A 128-byte
// u8 table and a 64-byte fp32 table each occupy distinct banks, so no lookup
// conflicts whatever the 32 lanes ask for.
struct EncodeTables {
  uint8_t base[128];
  float thr[16];
};

__device__ __forceinline__ void init_tables(EncodeTables& t) {
  for (int i = threadIdx.x; i < 128; i += blockDim.x) {
    const float lo = (float(i) - 32.5f) * (1.0f / 32.0f);   // exact
    uint32_t base = 0;
#pragma unroll
    for (int j = 0; j < 15; ++j) base += (__uint_as_float(threshold_bits(j)) < lo) ? 1u : 0u;
    t.base[i] = uint8_t(i <= 64 ? base : 15u);
  }
#pragma unroll
  for (int j = 0; j < 15; ++j)
    if (threadIdx.x == j) t.thr[j] = __uint_as_float(threshold_bits(j));
  if (threadIdx.x == 15) t.thr[15] = __int_as_float(0x7f800000);   // +inf
}

__device__ __forceinline__ uint32_t encode_fast(float v, const EncodeTables& t) {
  // 12582944 = 1.5 * 2^23 + 32: the sum's ulp is 1, so the FFMA rounds 32 v to
  // an integer, and the low 7 bits hold 32 + round(32 v)
  const uint32_t i = __float_as_uint(fmaf(v, 32.0f, 12582944.0f)) & 0x7fu;
  const uint32_t b = t.base[i];
  return b + (v > t.thr[b] ? 1u : 0u);
}

__device__ __forceinline__ float div_corrected(float w, float a, float y) {
  const float q = __fmul_rn(w, y);
  return fmaf(fmaf(-a, q, w), y, q);
}

__device__ __forceinline__ bool fast_scale(float a) {
  return a >= 0x1p-98f && a < 0x1p120f;
}

// Codes of two elements packed as one byte, even element in the high nibble.
__device__ __forceinline__ uint32_t pair_byte_fast(float w0, float w1, float a, float y,
                                                   const EncodeTables& t) {
  return (encode_fast(div_corrected(w0, a, y), t) << 4) | encode_fast(div_corrected(w1, a, y), t);
}

// Codes of two elements packed as one byte, even element in the high nibble.
__device__ __forceinline__ uint32_t pair_byte(float w0, float w1, float amax) {
  if (amax == 0.0f) return 0x77u;
  const uint32_t c0 = encode(__fdiv_rn(w0, amax));
  const uint32_t c1 = encode(__fdiv_rn(w1, amax));
  return (c0 << 4) | c1;
}

// Block-wide max of a non-negative float into this CTA's slot: the double
// quant reduces the slots itself, so no word has to be zeroed before a call
// and none keeps a value from an earlier one.
__device__ __forceinline__ void cta_max_to_slot(float v, float* slot) {
  __shared__ float red[32];
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < int(blockDim.x >> 5) ? red[lane] : 0.0f;
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) *slot = v;
  }
}

// Block-wide max of a non-negative float, then one atomicMax per CTA on its
// bit pattern (non-negative floats order like their unsigned bits).
__device__ __forceinline__ void cta_global_max(float v, uint32_t* gmax) {
  __shared__ float red[32];
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < int(blockDim.x >> 5) ? red[lane] : 0.0f;
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0 && v > 0.0f) atomicMax(gmax, __float_as_uint(v));
  }
}

// Input element types: fp32, or bf16 / f16 widened exactly to fp32.
constexpr int kInF32 = 0;
constexpr int kInBF16 = 1;
constexpr int kInF16 = 2;

__device__ __forceinline__ float2 widen2(int in, uint32_t v) {
  if (in == kInBF16) return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v));
  return __half22float2(*reinterpret_cast<const __half2*>(&v));
}

// Elements 8i .. 8i+7 of the input as two float4 (streaming loads).
template <int IN>
__device__ __forceinline__ void load8(const void* w, int64_t i, float4& a, float4& b) {
  if (IN == kInF32) {
    const float4* p = static_cast<const float4*>(w) + 2 * i;
    a = __ldcs(p);
    b = __ldcs(p + 1);
  } else {
    const uint4 u = __ldcs(static_cast<const uint4*>(w) + i);
    const float2 e0 = widen2(IN, u.x), e1 = widen2(IN, u.y), e2 = widen2(IN, u.z), e3 = widen2(IN, u.w);
    a = make_float4(e0.x, e0.y, e1.x, e1.y);
    b = make_float4(e2.x, e2.y, e3.x, e3.y);
  }
}

// One element of the input as fp32.
template <int IN>
__device__ __forceinline__ float load1(const void* w, int64_t e) {
  if (IN == kInF32) return static_cast<const float*>(w)[e];
  if (IN == kInBF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(w)[e]);
  return __half2float(static_cast<const __half*>(w)[e]);
}

// G = block_size / 8 lanes per block (1, 2, 4, 8, 16 or 32); IN the input type.
// Launched as exactly one resident wave; each thread walks the words a grid
// stride apart, two words per step, and issues the next step's two loads
// before encoding the current two, so 64 bytes per thread are always in
// flight.
template <int G, int IN, typename Idx>
__global__ void __launch_bounds__(256) quantize_vec_kernel(
    const void* __restrict__ w, Idx n_words, uint32_t* __restrict__ codes,
    float* __restrict__ absmax, uint32_t* __restrict__ status, float* __restrict__ max_slots) {
  __shared__ EncodeTables tab;
  init_tables(tab);
  __syncthreads();
  // Launched as a programmatic dependent: the tables above read no input;
  // every read of w and every write comes after the previous kernel on the
  // stream has completed.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  uint32_t cta_max = 0;
  const Idx stride = Idx(gridDim.x) * blockDim.x;
  // Encode one word (8 elements) whose block max over the G lanes is known
  // (finite: a non-finite block was flagged and is left to the fallback).
  auto encode_word = [&](Idx i, bool valid, const float4& a, const float4& b, float m) {
    if (!valid) return;
    uint32_t word;
    if (fast_scale(m)) {
      const float y = __frcp_rn(m);
      word = pair_byte_fast(a.x, a.y, m, y, tab) | (pair_byte_fast(a.z, a.w, m, y, tab) << 8) |
             (pair_byte_fast(b.x, b.y, m, y, tab) << 16) | (pair_byte_fast(b.z, b.w, m, y, tab) << 24);
    } else {
      word = pair_byte(a.x, a.y, m) | (pair_byte(a.z, a.w, m) << 8) |
             (pair_byte(b.x, b.y, m) << 16) | (pair_byte(b.z, b.w, m) << 24);
    }
    __stcs(codes + i, word);
    if ((threadIdx.x & (G - 1)) == 0 && absmax != nullptr) absmax[i / G] = m;
  };
  const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
  Idx base = Idx(blockIdx.x) * blockDim.x;
  float4 a0 = z4, b0 = z4, a1 = z4, b1 = z4;
  {
    const Idx i0 = base + threadIdx.x, i1 = i0 + stride;
    if (i0 < n_words) load8<IN>(w, int64_t(i0), a0, b0);
    if (i1 < n_words) load8<IN>(w, int64_t(i1), a1, b1);
  }
  // The loop runs in whole warps so every lane takes part in the shuffles.
  for (; base < n_words; base += 2 * stride) {
    const Idx i0 = base + threadIdx.x, i1 = i0 + stride;
    const Idx n0 = i0 + 2 * stride, n1 = n0 + stride;
    float4 c0 = z4, d0 = z4, c1 = z4, d1 = z4;
    if (n0 < n_words) load8<IN>(w, int64_t(n0), c0, d0);
    if (n1 < n_words) load8<IN>(w, int64_t(n1), c1, d1);
    const bool v0 = i0 < n_words, v1 = i1 < n_words;
    uint32_t m0 = max_abs_bits8(a0, b0), m1 = max_abs_bits8(a1, b1);
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) {
      m0 = max(m0, __shfl_xor_sync(0xffffffffu, m0, o));
      m1 = max(m1, __shfl_xor_sync(0xffffffffu, m1, o));
    }
    encode_word(i0, v0, a0, b0, __uint_as_float(m0));
    encode_word(i1, v1, a1, b1, __uint_as_float(m1));
    cta_max = max(cta_max, max(v0 ? m0 : 0u, v1 ? m1 : 0u));
    a0 = c0;
    b0 = d0;
    a1 = c1;
    b1 = d1;
  }
  // a NaN or Inf anywhere makes its block's max bits >= 0x7f800000
  if (cta_max >= 0x7f800000u) report(status, NF4_ERR_NONFINITE);
  if (max_slots != nullptr) cta_max_to_slot(__uint_as_float(cta_max), max_slots + blockIdx.x);
  // let a programmatic dependent (the double-quant kernel) launch: only now,
  // so that its waiting CTAs never hold SM slots this grid still needs
  asm volatile("griddepcontrol.launch_dependents;");
}

// Any even block size: one thread per block, two passes over its elements.
template <int IN>
__global__ void __launch_bounds__(256) quantize_generic_kernel(
    const void* __restrict__ w, int64_t n_blocks, int bs, uint8_t* __restrict__ codes,
    float* __restrict__ absmax, uint32_t* __restrict__ status, float* __restrict__ max_slots) {
  float cta_max = 0.0f;
  bool bad = false;
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  for (int64_t base = int64_t(blockIdx.x) * blockDim.x; base < n_blocks; base += stride) {
    const int64_t blk = base + threadIdx.x;
    float m = 0.0f;
    if (blk < n_blocks) {
      const int64_t e0 = blk * bs;
      for (int e = 0; e < bs; ++e) {
        const float v = load1<IN>(w, e0 + e);
        bad |= !isfinite(v);
        m = fmaxf(m, fabsf(v));
      }
      uint8_t* c = codes + blk * (bs / 2);
      for (int e = 0; e < bs; e += 2)
        c[e / 2] = uint8_t(pair_byte(load1<IN>(w, e0 + e), load1<IN>(w, e0 + e + 1), m));
      if (absmax != nullptr) absmax[blk] = m;
    }
    cta_max = fmaxf(cta_max, m);
  }
  if (bad) report(status, NF4_ERR_NONFINITE);
  if (max_slots != nullptr) cta_max_to_slot(cta_max, max_slots + blockIdx.x);
  asm volatile("griddepcontrol.launch_dependents;");
}

// The short last block of a tensor whose size is not a multiple of the block
// size: t (1 <= t < bs) elements starting at element e0 (a multiple of bs, so
// at byte e0 / 2 of the codes).  One CTA: block max over the t elements, then
// one byte per pair; an odd t leaves the last byte's low nibble as code 7
// (level 0.0), which is what encoding a zero gives.
template <int IN>
__global__ void __launch_bounds__(256) quantize_tail_kernel(
    const void* __restrict__ w, int64_t e0, int t, uint8_t* __restrict__ codes,
    float* __restrict__ absmax, int64_t blk, uint32_t* __restrict__ status,
    float* __restrict__ max_slot) {
  __shared__ float red[8];
  float m = 0.0f;
  bool bad = false;
  for (int i = threadIdx.x; i < t; i += blockDim.x) {
    const float v = load1<IN>(w, e0 + i);
    bad |= !isfinite(v);
    m = fmaxf(m, fabsf(v));
  }
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  m = red[0];
  for (int k = 1; k < int(blockDim.x >> 5); ++k) m = fmaxf(m, red[k]);
  if (bad) report(status, NF4_ERR_NONFINITE);
  uint8_t* c = codes + e0 / 2;
  for (int p = threadIdx.x; 2 * p < t; p += blockDim.x) {
    const float w0 = load1<IN>(w, e0 + 2 * p);
    if (2 * p + 1 < t) {
      c[p] = uint8_t(pair_byte(w0, load1<IN>(w, e0 + 2 * p + 1), m));
    } else {
      c[p] = uint8_t((pair_byte(w0, 0.0f, m) & 0xf0u) | 0x7u);
    }
  }
  if (threadIdx.x == 0) {
    if (absmax != nullptr) absmax[blk] = m;
    if (max_slot != nullptr) *max_slot = m;
  }
}

// Simplified double quant of the block scales: one global scale G / 255 and a
// u8 per block, rint(absmax / s_g) with ties to even.
// Launched as a programmatic dependent of the quantize kernel: it starts
// early and waits (griddepcontrol.wait) until the quantize grid has finished
// and its writes are visible.
// Four scales per thread (one 16-byte load, one 4-byte store), the loads
// issued before the global maximum is read; the grid covers every group of
// four once, and the first threads take the n_blocks % 4 tail.
__device__ __forceinline__ uint32_t dq_code(float a, float g, float s_g, bool fast, float y) {
  if (!(g > 0.0f)) return 0u;
  const float ratio = fast ? div_corrected(a, s_g, y) : __fdiv_rn(a, s_g);
  return uint32_t(min(max(__float2int_rn(ratio), 0), 255));
}

// G = the max over n_slots values (the quantize grid's per-CTA maxima, or one
// global max from the caller), reduced by every CTA for itself.
__global__ void __launch_bounds__(256) double_quant_kernel(
    const float* __restrict__ absmax, int64_t n_blocks, const float* __restrict__ max_slots,
    int n_slots, uint8_t* __restrict__ absmax_q, float* __restrict__ absmax_scale) {
  // a programmatic dependent of this kernel (the next quantize on the stream)
  // may launch now: it waits for this grid before it touches memory
  asm volatile("griddepcontrol.launch_dependents;");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t n4 = n_blocks / 4;
  const int64_t i4 = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  float4 a4 = make_float4(0.f, 0.f, 0.f, 0.f);
  if (i4 < n4) a4 = reinterpret_cast<const float4*>(absmax)[i4];
  const int64_t tail = n4 * 4 + i4;
  const float at = (tail < n_blocks) ? absmax[tail] : 0.0f;
  __shared__ float red[8];
  float gm = 0.0f;
  for (int i = threadIdx.x; i < n_slots; i += blockDim.x) gm = fmaxf(gm, __ldg(max_slots + i));
  for (int o = 16; o > 0; o >>= 1) gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = gm;
  __syncthreads();
  float g = red[0];
  for (int k = 1; k < int(blockDim.x >> 5); ++k) g = fmaxf(g, red[k]);
  const float s_g = __fdiv_rn(g, 255.0f);
  if (blockIdx.x == 0 && threadIdx.x == 0) *absmax_scale = s_g;
  const bool fast = fast_scale(s_g);
  const float y = fast ? __frcp_rn(s_g) : 0.0f;
  if (i4 < n4) {
    const uint32_t q = dq_code(a4.x, g, s_g, fast, y) | (dq_code(a4.y, g, s_g, fast, y) << 8) |
                       (dq_code(a4.z, g, s_g, fast, y) << 16) | (dq_code(a4.w, g, s_g, fast, y) << 24);
    reinterpret_cast<uint32_t*>(absmax_q)[i4] = q;
  }
  if (tail < n_blocks) absmax_q[tail] = uint8_t(dq_code(at, g, s_g, fast, y));
}

// Max of n non-negative fp32 block scales into *gmax (bits; zeroed by the
// caller): the global max of the simplified double quant when the scales of
// one tensor are spread over several ranks.
__global__ void __launch_bounds__(256) absmax_max_kernel(const float* __restrict__ absmax,
                                                         int64_t n, uint32_t* __restrict__ gmax) {
  float m = 0.0f;
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride)
    m = fmaxf(m, __ldg(absmax + i));
  cta_global_max(m, gmax);
}

// ------------------------------------------------------------------ dequant

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}



// EPL elements per lane per step, so that every lane stores one 16-byte vector
// and a warp's store covers 512 contiguous bytes: 4 for fp32 output (two code
// bytes in), 8 for bf16 / f16 (four code bytes in).
template <typename OutT>
struct DqUnit;
template <>
struct DqUnit<float> {
  static constexpr int kElems = 4;
  using Code = uint16_t;
};
template <>
struct DqUnit<__nv_bfloat16> {
  static constexpr int kElems = 8;
  using Code = uint32_t;
};
template <>
struct DqUnit<__half> {
  static constexpr int kElems = 8;
  using Code = uint32_t;
};

template <typename OutT>
__device__ __forceinline__ void store_unit(OutT* out, int64_t unit, const float (&v)[8]);
template <>
__device__ __forceinline__ void store_unit<float>(float* out, int64_t unit, const float (&v)[8]) {
  __stcs(reinterpret_cast<float4*>(out) + unit, make_float4(v[0], v[1], v[2], v[3]));
}
template <>
__device__ __forceinline__ void store_unit<__nv_bfloat16>(__nv_bfloat16* out, int64_t unit, const float (&v)[8]) {
  __stcs(reinterpret_cast<uint4*>(out) + unit,
         make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                    pack_bf16x2(v[6], v[7])));
}
template <>
__device__ __forceinline__ void store_unit<__half>(__half* out, int64_t unit, const float (&v)[8]) {
  __stcs(reinterpret_cast<uint4*>(out) + unit,
         make_uint4(pack_f16x2(v[0], v[1]), pack_f16x2(v[2], v[3]), pack_f16x2(v[4], v[5]),
                    pack_f16x2(v[6], v[7])));
}

// Whole units of whole blocks (bs a multiple of 8).  Launched as one resident
// wave; each thread handles kDqSteps units a grid stride apart per iteration,
// all of their code and scale loads issued before the first is decoded.
constexpr int kDqSteps = 4;
template <typename OutT, bool kDouble>
__global__ void __launch_bounds__(256) dequant_vec_kernel(
    const uint8_t* __restrict__ codes, int64_t n_units, int unit_shift, int units_per_block,
    const float* __restrict__ absmax, const uint8_t* __restrict__ absmax_q,
    const float* __restrict__ absmax_scale, OutT* __restrict__ out) {
  using Code = typename DqUnit<OutT>::Code;
  constexpr int E = DqUnit<OutT>::kElems;
  __shared__ float lut[16];   // 16 words in 16 banks: conflict-free for any codes
  if (threadIdx.x < 16) lut[threadIdx.x] = level(threadIdx.x);
  __syncthreads();
  // Launched as a programmatic dependent, and lets the next one launch now:
  // nothing above reads an input, and nothing below reads or writes memory
  // before the previous kernel on the stream has completed.
  asm volatile("griddepcontrol.launch_dependents;");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const float s_g = kDouble ? *absmax_scale : 0.0f;
  const Code* c = reinterpret_cast<const Code*>(codes);
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  for (int64_t base = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; base < n_units;
       base += kDqSteps * stride) {
    uint32_t word[kDqSteps];
    float scale[kDqSteps];
#pragma unroll
    for (int u = 0; u < kDqSteps; ++u) {
      const int64_t i = base + u * stride;
      const bool ok = i < n_units;
      word[u] = ok ? uint32_t(__ldcs(c + i)) : 0u;
      const int64_t blk = unit_shift >= 0 ? (i >> unit_shift) : (i / units_per_block);
      scale[u] = ok ? (kDouble ? __fmul_rn(float(__ldg(absmax_q + blk)), s_g) : __ldg(absmax + blk)) : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < kDqSteps; ++u) {
      const int64_t i = base + u * stride;
      if (i >= n_units) break;
      float v[8];
#pragma unroll
      for (int j = 0; j < E / 2; ++j) {
        const uint32_t byte = (word[u] >> (8 * j)) & 0xffu;
        v[2 * j] = __fmul_rn(lut[byte >> 4], scale[u]);
        v[2 * j + 1] = __fmul_rn(lut[byte & 15u], scale[u]);
      }
      store_unit<OutT>(out, i, v);
    }
  }
}

// One fp32 value as the output type, rounded to nearest even.
template <typename OutT>
__device__ __forceinline__ OutT round_out(float v);
template <>
__device__ __forceinline__ float round_out<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 round_out<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }
template <>
__device__ __forceinline__ __half round_out<__half>(float v) { return __float2half_rn(v); }

// Any even block size, and the short last block: one code byte (two
// elements; bs is even, so both lie in one block) per thread, bytes
// [byte0, byte1).  numel is the tensor's element count; a last byte that holds
// one element writes only that one.
template <typename OutT, bool kDouble>
__global__ void __launch_bounds__(256) dequant_bytes_kernel(
    const uint8_t* __restrict__ codes, int64_t byte0, int64_t byte1, int64_t numel, int bs,
    const float* __restrict__ absmax, const uint8_t* __restrict__ absmax_q,
    const float* __restrict__ absmax_scale, OutT* __restrict__ out) {
  const float s_g = kDouble ? *absmax_scale : 0.0f;
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  for (int64_t i = byte0 + int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < byte1; i += stride) {
    const uint32_t byte = codes[i];
    const int64_t e = 2 * i;
    const int64_t blk = e / bs;
    const float scale = kDouble ? __fmul_rn(float(absmax_q[blk]), s_g) : absmax[blk];
    out[e] = round_out<OutT>(__fmul_rn(level(byte >> 4), scale));
    if (e + 1 < numel) out[e + 1] = round_out<OutT>(__fmul_rn(level(byte & 15u), scale));
  }
}

// A one-dimensional launch with programmatic stream serialisation: the kernel
// may start while the previous kernel on the stream finishes, and must touch
// no input or output before its griddepcontrol.wait.
template <typename... P, typename... A>
cudaError_t launch_dependent(void (*kernel)(P...), int grid, int threads, cudaStream_t stream,
                             A&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(grid), 1, 1);
  cfg.blockDim = dim3(unsigned(threads), 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}

// CTAs of `kernel` (threads per CTA, no dynamic shared memory) resident on one
// SM, from the occupancy calculator, cached per kernel and device.
int resident_ctas(const void* kernel, int threads) {
  struct Entry {
    const void* fn;
    int dev, n;
  };
  static std::mutex mu;
  static Entry cache[64];
  static int used = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (cache[i].fn == kernel && cache[i].dev == dev) return cache[i].n;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, 0) != cudaSuccess || n < 1) n = 1;
  if (used < 64) cache[used++] = Entry{kernel, dev, n};
  return n;
}

int grid_for(int64_t work_items, int threads, int sms, int per_sm) {
  int64_t g = (work_items + threads - 1) / threads;
  const int64_t cap = int64_t(sms) * per_sm;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return int(g);
}

int log2_exact(int v) {
  if (v <= 0 || (v & (v - 1))) return -1;
  int s = 0;
  while ((1 << s) < v) ++s;
  return s;
}

}  // namespace

template <int IN>
void launch_quantize_typed(const void* w, int64_t numel, int bs, uint8_t* codes, float* absmax_out,
                           uint32_t* status, float* max_slots, int* n_slots, int sms,
                           cudaStream_t stream, int* launches) {
  *n_slots = 0;
  const int threads = 256;
  const int64_t n_full = numel / bs;          // whole blocks
  const int tail = int(numel - n_full * bs);  // elements of the short last block
  const bool vec = (bs % 8 == 0) && bs <= 256 && log2_exact(bs) >= 0;
  if (n_full > 0 && vec) {
    const int64_t n_words = n_full * bs / 8;
    uint32_t* c32 = reinterpret_cast<uint32_t*>(codes);
    cudaError_t launch_error = cudaSuccess;
    auto run = [&](auto kernel, auto n) {
      // one resident wave: every CTA stays for the whole pass
      const int grid = std::min(kMaxSlots - 1, grid_for(n_words, threads, sms,
                                                         resident_ctas(reinterpret_cast<const void*>(kernel), threads)));
      launch_error = launch_dependent(kernel, grid, threads, stream, w, n, c32, absmax_out, status, max_slots);
      *n_slots = grid;
    };
    // 32-bit word indices while every index the loop forms (up to n_words plus
    // four grid strides) fits
    const bool small = n_words < (int64_t(1) << 30);
    const uint32_t n32 = uint32_t(n_words);
    switch (bs / 8) {
      case 1: if (small) run(quantize_vec_kernel<1, IN, uint32_t>, n32); else run(quantize_vec_kernel<1, IN, int64_t>, n_words); break;
      case 2: if (small) run(quantize_vec_kernel<2, IN, uint32_t>, n32); else run(quantize_vec_kernel<2, IN, int64_t>, n_words); break;
      case 4: if (small) run(quantize_vec_kernel<4, IN, uint32_t>, n32); else run(quantize_vec_kernel<4, IN, int64_t>, n_words); break;
      case 8: if (small) run(quantize_vec_kernel<8, IN, uint32_t>, n32); else run(quantize_vec_kernel<8, IN, int64_t>, n_words); break;
      case 16: if (small) run(quantize_vec_kernel<16, IN, uint32_t>, n32); else run(quantize_vec_kernel<16, IN, int64_t>, n_words); break;
      default: if (small) run(quantize_vec_kernel<32, IN, uint32_t>, n32); else run(quantize_vec_kernel<32, IN, int64_t>, n_words); break;
    }
    if (launch_error != cudaSuccess) return;   // the caller reads it back from cudaGetLastError
    ++*launches;
  } else if (n_full > 0) {
    const int grid = std::min(kMaxSlots - 1, grid_for(n_full, threads, sms, 8));
    quantize_generic_kernel<IN><<<grid, threads, 0, stream>>>(w, n_full, bs, codes, absmax_out,
                                                              status, max_slots);
    *n_slots = grid;
    ++*launches;
  }
  if (tail > 0) {
    // an ordinary launch: it starts once the full-block kernel has finished
    quantize_tail_kernel<IN><<<1, threads, 0, stream>>>(w, n_full * bs, tail, codes, absmax_out,
                                                        n_full, status,
                                                        max_slots ? max_slots + *n_slots : nullptr);
    *n_slots += 1;
    ++*launches;
  }
}

cudaError_t launch_quantize(const void* w, int in_dtype, int64_t numel, int bs, uint8_t* codes,
                            float* absmax_out, uint32_t* status, float* max_slots, int* n_slots,
                            int sms, cudaStream_t stream, int* launches) {
  int n = 0;
  NF4_PROF_BEGIN(stream, kKQuantize);
  if (in_dtype == NF4_BF16)
    launch_quantize_typed<kInBF16>(w, numel, bs, codes, absmax_out, status, max_slots, n_slots, sms, stream, &n);
  else if (in_dtype == NF4_F16)
    launch_quantize_typed<kInF16>(w, numel, bs, codes, absmax_out, status, max_slots, n_slots, sms, stream, &n);
  else
    launch_quantize_typed<kInF32>(w, numel, bs, codes, absmax_out, status, max_slots, n_slots, sms, stream, &n);
  NF4_PROF_END(stream, kKQuantize);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) *launches += n;
  return e;
}

cudaError_t launch_double_quant(const float* absmax, int64_t n_blocks, const float* max_slots,
                                int n_slots, uint8_t* absmax_q, float* absmax_scale, int sms,
                                cudaStream_t stream, int* launches) {
  const int threads = 256;
  (void)sms;
  // one thread per four scales, at least one thread for the tail
  const int64_t groups = std::max<int64_t>(n_blocks / 4, 1);
  const int grid = int((groups + threads - 1) / threads);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(grid), 1, 1);
  cfg.blockDim = dim3(unsigned(threads), 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  NF4_PROF_BEGIN(stream, kKDoubleQuant);
  cudaError_t e = cudaLaunchKernelEx(&cfg, double_quant_kernel, absmax, n_blocks, max_slots, n_slots,
                                     absmax_q, absmax_scale);
  NF4_PROF_END(stream, kKDoubleQuant);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e == cudaSuccess) ++*launches;
  return e;
}

cudaError_t launch_absmax_max(const float* absmax, int64_t n, uint32_t* gmax, int sms,
                              cudaStream_t stream, int* launches) {
  cudaError_t e = cudaMemsetAsync(gmax, 0, sizeof(uint32_t), stream);
  if (e != cudaSuccess) return e;
  if (n <= 0) return cudaSuccess;
  const int grid = grid_for(n, 256, sms, 2);
  NF4_PROF_BEGIN(stream, kKAbsmaxMax);
  absmax_max_kernel<<<grid, 256, 0, stream>>>(absmax, n, gmax);
  NF4_PROF_END(stream, kKAbsmaxMax);
  e = cudaGetLastError();
  if (e == cudaSuccess) ++*launches;
  return e;
}

cudaError_t launch_dequantize(const nf4_weight& w, int out_dtype, void* out, int sms,
                              cudaStream_t stream, int* launches) {
  const int64_t numel = w.rows * w.cols;
  const int bs = w.block_size;
  const int threads = 256;
  const bool dq = w.double_quant != 0;
  // Whole 8-element words of whole blocks go through the word kernel when the
  // block size is a multiple of 8; every other code byte (a block size that is
  // not, or the short last block) through the byte kernel.
  const int64_t n_words = (bs % 8 == 0) ? (numel / bs) * bs / 8 : 0;
  const int64_t byte0 = n_words * 4, byte1 = (numel + 1) / 2;
  int n = 0;
  cudaError_t launch_error = cudaSuccess;
  NF4_PROF_BEGIN(stream, kKDequantize);
  if (n_words > 0) {
    // units of E elements: 4 for fp32 output, 8 for bf16 / f16
    const int E = out_dtype == NF4_F32 ? 4 : 8;
    const int64_t n_units = n_words * 8 / E;
    const int units_per_block = bs / E;
    const int shift = log2_exact(units_per_block);
    auto run = [&](auto kernel, auto* o) {
      const int grid = grid_for((n_units + kDqSteps - 1) / kDqSteps, threads, sms,
                                resident_ctas(reinterpret_cast<const void*>(kernel), threads));
      launch_error = launch_dependent(kernel, grid, threads, stream, w.codes, n_units, shift, units_per_block,
                                      w.absmax, w.absmax_q, w.absmax_scale, o);
    };
    if (out_dtype == NF4_F32) {
      float* o = reinterpret_cast<float*>(out);
      if (dq) run(dequant_vec_kernel<float, true>, o); else run(dequant_vec_kernel<float, false>, o);
    } else if (out_dtype == NF4_BF16) {
      __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out);
      if (dq) run(dequant_vec_kernel<__nv_bfloat16, true>, o); else run(dequant_vec_kernel<__nv_bfloat16, false>, o);
    } else {
      __half* o = reinterpret_cast<__half*>(out);
      if (dq) run(dequant_vec_kernel<__half, true>, o); else run(dequant_vec_kernel<__half, false>, o);
    }
    ++n;
  }
  if (byte1 > byte0 && launch_error == cudaSuccess) {
    const int grid = grid_for(byte1 - byte0, threads, sms, 8);
#define NF4_DQB_LAUNCH(T, D)                                                               \
  dequant_bytes_kernel<T, D><<<grid, threads, 0, stream>>>(w.codes, byte0, byte1, numel, bs, \
                                                           w.absmax, w.absmax_q,            \
                                                           w.absmax_scale,                  \
                                                           reinterpret_cast<T*>(out))
    if (out_dtype == NF4_F32) {
      if (dq) NF4_DQB_LAUNCH(float, true); else NF4_DQB_LAUNCH(float, false);
    } else if (out_dtype == NF4_BF16) {
      if (dq) NF4_DQB_LAUNCH(__nv_bfloat16, true); else NF4_DQB_LAUNCH(__nv_bfloat16, false);
    } else {
      if (dq) NF4_DQB_LAUNCH(__half, true); else NF4_DQB_LAUNCH(__half, false);
    }
#undef NF4_DQB_LAUNCH
    ++n;
  }
  NF4_PROF_END(stream, kKDequantize);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = launch_error;
  if (e == cudaSuccess) *launches += n;
  return e;
}

}  // namespace nf4
