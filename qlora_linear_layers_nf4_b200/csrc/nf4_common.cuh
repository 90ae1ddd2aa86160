// Shared device-side definitions: the NF4 codebook, the decision thresholds,
// device status reporting and a few bit helpers.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "../../include/nf4qlora.h"

namespace nf4 {

// NF4 levels, code 0..15 ascending, as fp32 bit patterns.  Sixteen normal
// quantiles with an exact zero, scaled to [-1, 1] ("LoRA and QLoRA,
// mathematically", section "NF4: quantizing the frozen base"; three-decimal
// values printed in the qlora-rs README, section "NF4 Quantization").
#define NF4_LEVEL_BITS                                                                  \
  {0xbf800000u, 0xbf3239b1u, 0xbf066b2eu, 0xbeca329eu, 0xbe91a24bu, 0xbe3d353du,         \
   0xbdba7869u, 0x00000000u, 0x3da2fb01u, 0x3e24cadfu, 0x3e7c04dau, 0x3ead0336u,         \
   0x3ee1a4b5u, 0x3f1007a9u, 0x3f3913b0u, 0x3f800000u}
constexpr uint32_t kLevelBits[16] = NF4_LEVEL_BITS;        // host copy
static __constant__ uint32_t kLevelBitsDev[16] = NF4_LEVEL_BITS;

// Level i as a compile-time constant (i must be a literal after inlining).
__host__ __device__ constexpr uint32_t level_bits(int i) {
  constexpr uint32_t t[16] = NF4_LEVEL_BITS;
  return t[i];
}

// Decision thresholds: kThresholdBits[i] is the largest fp32 value not above
// the exact midpoint of levels i and i+1.  For an fp32 value v, v > t_i holds
// exactly when v is strictly nearer to level i+1 than to level i, so
// code(v) = #{i : v > t_i} is the nearest level with ties to the lower code.
#define NF4_THRESHOLD_BITS                                                        \
  {0xbf591cd9u, 0xbf1c5270u, 0xbeeb847du, 0xbeadea75u, 0xbe703ceau,                \
   0xbe0d38b9u, 0xbd3a7869u, 0x3d22fb01u, 0x3df6485fu, 0x3e5067dcu,                \
   0x3e9582d1u, 0x3ec753f5u, 0x3f006d01u, 0x3f248dacu, 0x3f5c89d8u}
constexpr uint32_t kThresholdBits[15] = NF4_THRESHOLD_BITS;  // host copy

// Threshold i as a compile-time constant (i must be a literal after inlining).
__host__ __device__ constexpr uint32_t threshold_bits(int i) {
  constexpr uint32_t t[15] = NF4_THRESHOLD_BITS;
  return t[i];
}

// Layout of the head of every workspace (bytes).
constexpr size_t kWsStatus = 0;        // u32 sticky device status (first error wins)
constexpr size_t kWsHeader = 256;      // op-specific scratch starts here
// Quantize with double quant: per-CTA maxima of the quantize grid (its size
// is capped below this), then the fp32 block scales when the caller keeps none.
constexpr int kMaxSlots = 2048;
constexpr size_t kWsMaxSlotsBytes = size_t(kMaxSlots) * 4;

__device__ __forceinline__ float level(int c) {
  return __uint_as_float(kLevelBitsDev[c]);
}

// Block index of the 64-element chunk `chunk` (along the row) of W row `row`:
// blocks run over the row-major flattened tensor and hold 2^bs_shift >= 64
// elements, so a 64-aligned chunk never straddles two blocks.
__host__ __device__ __forceinline__ int64_t chunk_block(int64_t row, int64_t cols, int64_t chunk,
                                                        int bs_shift) {
  return (row * cols + chunk * 64) >> bs_shift;
}

__device__ __forceinline__ void report(uint32_t* status, uint32_t code) {
  if (status != nullptr) atomicCAS(status, 0u, code);
}

// Nearest-level code of a normalised value, by a four-level binary decision
// over the thresholds (all compile-time immediates).
__device__ __forceinline__ uint32_t encode(float v) {
#define NF4_T(i) __uint_as_float(threshold_bits(i))
  const bool b3 = v > NF4_T(7);
  const float t2 = b3 ? NF4_T(11) : NF4_T(3);
  const bool b2 = v > t2;
  const float t1 = b3 ? (b2 ? NF4_T(13) : NF4_T(9)) : (b2 ? NF4_T(5) : NF4_T(1));
  const bool b1 = v > t1;
  float t0;
  if (b3) {
    t0 = b2 ? (b1 ? NF4_T(14) : NF4_T(12)) : (b1 ? NF4_T(10) : NF4_T(8));
  } else {
    t0 = b2 ? (b1 ? NF4_T(6) : NF4_T(4)) : (b1 ? NF4_T(2) : NF4_T(0));
  }
  const bool b0 = v > t0;
#undef NF4_T
  return (uint32_t(b3) << 3) | (uint32_t(b2) << 2) | (uint32_t(b1) << 1) | uint32_t(b0);
}

}  // namespace nf4
