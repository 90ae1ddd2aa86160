// QLoRA linear forward and adapter backward on the sm_100a tensor cores.
//
// The layer (qlora-rs README, QuantizedLinear::forward; "LoRA and QLoRA,
// mathematically", equation 6.3.6 read as a layer) is
//     y  = x W'^T + T B^T,          T = s x A^T,  s = alpha / r
// and its backward for L = sum(dy * y) with W frozen is
//     U  = s dy B,  dB = dy^T T,  dA = U^T x,  dx = dy W' + U A.
// W' = bf16(L[code] * scale) (f16 in the F16 compute dtype) is never
// written to HBM: the fused kernel dequantizes each NF4 tile into shared
// memory, in the swizzled layout the tensor core reads, right before the MMA
// that consumes it.  The adapter product rides in the same TMEM accumulator
// as extra K steps ([x | T] [W' | B]^T forward, [dy | U] [W' ; A] backward).
//
// Kernels (each fused kernel in bf16 and f16 instantiations)
//   fused_nf4_gemm_pair<kFwd>  y[M,N]  = x W'^T + T B^T (+ bias), M > 256:
//                              a 2-CTA cluster, tcgen05 cta_group::2, 512 x 256 tiles
//   fused_nf4_gemm_pair<kDx>   dx[M,K] = dy W' + U A (MN-major W' tiles)
//   fused_nf4_gemm<kFwd/kDx>   the same on one CTA, 256 x 256 tiles, 32 < M <= 256
//   adapter_gemm               the rank-r products T, U, dB, dA^T, split along
//                              the reduction over a thread-block cluster whose
//                              CTAs sum their fp32 partials through
//                              distributed shared memory
#include <algorithm>
#include <mutex>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kernels.h"
#include "nf4_common.cuh"
#include "tc_common.cuh"

namespace nf4 {
namespace {

using namespace tc;

// ------------------------------------------------------------------ dequant

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t f16x2_rn(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
// Two values rounded (nearest, ties to even) to the compute type: f16 or bf16.
__device__ __forceinline__ uint32_t pack2(bool f16, float lo, float hi) {
  return f16 ? f16x2_rn(lo, hi) : bf16x2_rn(lo, hi);
}
__device__ __forceinline__ float2 unpack2(bool f16, uint32_t w) {
  return f16 ? __half22float2(*reinterpret_cast<const __half2*>(&w))
             : __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w));
}

// The sixteen dequantized values of one block, bf16(L[c] * scale) (or f16)
// with the fp32 product rounded to nearest even, split into byte planes so a
// lookup is a register byte-permute: lo[q] holds the low bytes of entries
// 4q..4q+3, hi[q] their high bytes.
struct BlockTable {
  uint32_t lo[4];
  uint32_t hi[4];
};

__device__ __forceinline__ BlockTable make_table(float scale, bool f16) {
  uint32_t p[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    p[j] = pack2(f16, __fmul_rn(__uint_as_float(level_bits(2 * j)), scale),
                 __fmul_rn(__uint_as_float(level_bits(2 * j + 1)), scale));
  }
  BlockTable t;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    t.lo[q] = prmt(p[2 * q], p[2 * q + 1], 0x6420u);
    t.hi[q] = prmt(p[2 * q], p[2 * q + 1], 0x7531u);
  }
  return t;
}

// Four codes (the low 16 bits of `w`: two packed bytes, even element in the
// high nibble) -> four bf16 values as two bf16x2 words in element order.
__device__ __forceinline__ uint2 decode4(uint32_t w, const BlockTable& t) {
  const uint32_t sel = w & 0x7777u;                          // code & 7 per nibble
  const uint32_t pick = ((w >> 1) & 0x4444u) | 0x3210u;      // code >= 8 -> upper plane
  const uint32_t lo = prmt(prmt(t.lo[0], t.lo[1], sel), prmt(t.lo[2], t.lo[3], sel), pick);
  const uint32_t hi = prmt(prmt(t.hi[0], t.hi[1], sel), prmt(t.hi[2], t.hi[3], sel), pick);
  // lo/hi bytes are in nibble order (odd element first within a byte).
  return make_uint2(prmt(lo, hi, 0x4051u), prmt(lo, hi, 0x6273u));
}

// Dequantize one 64-element block (32 code bytes at `codes`, smem) into row
// `row` of a 128-byte-swizzled bf16 tile at `tile` (smem).
__device__ __forceinline__ void dequant_row(const uint8_t* codes, float scale, uint8_t* tile,
                                            uint32_t row, bool f16) {
  const uint4 c0 = *reinterpret_cast<const uint4*>(codes);
  const uint4 c1 = *reinterpret_cast<const uint4*>(codes + 16);
  const BlockTable t = make_table(scale, f16);
  const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint2 a = decode4(words[k], t);
    const uint2 b = decode4(words[k] >> 16, t);
    *reinterpret_cast<uint4*>(tile + sw128_offset(row, k)) = make_uint4(a.x, a.y, b.x, b.y);
  }
}

// Half a block (32 elements, 16 code bytes at `codes`, smem) into 16-byte
// chunks 4*half .. 4*half+3 of row `row` of a 128-byte-swizzled bf16 tile.
__device__ __forceinline__ void dequant_half_row(const uint8_t* codes, float scale, uint8_t* tile,
                                                 uint32_t row, uint32_t half, bool f16) {
  const uint4 c = *reinterpret_cast<const uint4*>(codes);
  const BlockTable t = make_table(scale, f16);
  const uint32_t words[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint2 a = decode4(words[k], t);
    const uint2 b = decode4(words[k] >> 16, t);
    *reinterpret_cast<uint4*>(tile + sw128_offset(row, 4 * half + k)) = make_uint4(a.x, a.y, b.x, b.y);
  }
}

__device__ __forceinline__ float load_scale(const uint8_t* absmax_q, const float* absmax,
                                            float s_g, bool dq, int64_t idx) {
  return dq ? __fmul_rn(float(__ldg(absmax_q + idx)), s_g) : __ldg(absmax + idx);
}

// ------------------------------------------------------------------ fused GEMM

constexpr int kFwd = 0;
constexpr int kDx = 1;

constexpr int kTileM = 256;     // two UMMA M=128 halves
constexpr int kTileN = 256;
constexpr int kTileK = 64;      // one 128-byte swizzle row of bf16
constexpr int kStages = 3;
constexpr int kDeqWarps = 8;
constexpr int kFusedThreads = 64 + kDeqWarps * 32;  // TMA warp, MMA warp, 8 dequant/epilogue
constexpr uint32_t kHalfABytes = 128 * 128;         // 128 rows x 128 B
constexpr uint32_t kABytes = 2 * kHalfABytes;
constexpr uint32_t kBBytes = kTileN * 128;
constexpr uint32_t kCBytes = kTileN * 32;           // 256 blocks x 32 code bytes
constexpr uint32_t kStageBytes = kABytes + kBBytes + kCBytes;
constexpr size_t kFusedSmem = size_t(kStages) * kStageBytes + 1024 + 256;

struct FusedParams {
  int M;             // rows of x / dy
  int N;             // W rows (out features)
  int K;             // W cols (in features)
  int r;
  int main_steps;    // fwd: K / 64; dx: ceil(N / 64)
  int adapter_steps; // ceil(r / 64)
  int out_cols;      // N (fwd) or K (dx)
  int kb_per_row;    // K / 64: 64-element chunks per W row
  int bs_shift;      // log2 of the NF4 block size (6 .. 12)
  int double_quant;
  int f16;           // operands and outputs in f16 (else bf16)
  const uint8_t* absmax_q;
  const float* absmax;
  const float* absmax_scale;
  const __nv_bfloat16* bias;   // 2-byte elements of the compute type
  __nv_bfloat16* out;
  uint32_t* status;
};

struct FusedShared {
  uint64_t full[kStages];    // TMA bytes landed (A + codes, or A2 + B2)
  uint64_t bready[kStages];  // dequantized B tile written (8 warp arrivals)
  uint64_t empty[kStages];   // MMAs reading the stage finished (umma_commit)
  uint64_t accum;            // all MMAs finished
  uint32_t tmem_base;
  uint32_t abort_flag;
};

template <int MODE, bool F16>
__global__ void __launch_bounds__(kFusedThreads, 1)
    fused_nf4_gemm(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_a2,
                   const __grid_constant__ CUtensorMap tm_b2,
                   const __grid_constant__ CUtensorMap tm_codes,
                   const __grid_constant__ CUtensorMap tm_out, const FusedParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  FusedShared* sh = reinterpret_cast<FusedShared*>(smem + kStages * kStageBytes);
  auto stage_a = [&](int s) { return smem + s * kStageBytes; };
  auto stage_b = [&](int s) { return smem + s * kStageBytes + kABytes; };
  auto stage_c = [&](int s) { return smem + s * kStageBytes + kABytes + kBBytes; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tile_n0 = blockIdx.x * kTileN;   // fwd: W rows; dx: W cols (output cols)
  const int m0 = blockIdx.y * kTileM;
  const int total_steps = p.main_steps + p.adapter_steps;
  volatile uint32_t* abort_flag = &sh->abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh->full[s], 1);
      mbar_init(&sh->bready[s], kDeqWarps);
      mbar_init(&sh->empty[s], 1);
    }
    mbar_init(&sh->accum, 1);
    sh->abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
    tma_prefetch(&tm_a);
    tma_prefetch(&tm_a2);
    tma_prefetch(&tm_b2);
    tma_prefetch(&tm_codes);
  }
  if (warp == 1) {
    tmem_alloc(&sh->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < total_steps; ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (!mbar_wait(&sh->empty[s], ph ^ 1, abort_flag, p.status)) break;
        uint8_t* a = stage_a(s);
        if (it < p.main_steps) {
          mbar_arrive_expect_tx(&sh->full[s], kABytes + kCBytes);
          const int k0 = it * kTileK;  // fwd: K index; dx: N index (the reduction)
          tma_load_2d(a, &tm_a, &sh->full[s], k0, m0);     // 256 rows: both halves
          if (MODE == kFwd) {
            tma_load_2d(stage_c(s), &tm_codes, &sh->full[s], k0 / 2, tile_n0);
          } else {
#pragma unroll
            for (int g = 0; g < 4; ++g)
              tma_load_2d(stage_c(s) + g * 2048, &tm_codes, &sh->full[s], (tile_n0 + 64 * g) / 2, k0);
          }
        } else {
          if (it == p.main_steps) grid_dep_wait();
          const int r0 = (it - p.main_steps) * kTileK;
          mbar_arrive_expect_tx(&sh->full[s], kABytes + kBBytes);
          tma_load_2d(a, &tm_a2, &sh->full[s], r0, m0);
          if (MODE == kFwd) {
            tma_load_2d(stage_b(s), &tm_b2, &sh->full[s], r0, tile_n0);
          } else {
#pragma unroll
            for (int g = 0; g < 4; ++g)
              tma_load_2d(stage_b(s) + g * 8192, &tm_b2, &sh->full[s], tile_n0 + 64 * g, r0);
          }
        }
        ++issued;
      }
      // Unwind after an abort: wait (bounded) for the copies still in flight.
      if (*abort_flag) {
        for (int it = issued - 1; it >= 0 && it >= issued - kStages; --it) {
          uint32_t dummy_abort = 0;
          mbar_wait(&sh->full[it % kStages], (it / kStages) & 1, &dummy_abort, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_f32acc(128, kTileN, false, MODE == kDx, F16);
      bool ok = true;
      int issued = 0;
      for (int it = 0; it < total_steps && ok; ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        const bool adapter = it >= p.main_steps;
        ok = mbar_wait(&sh->full[s], ph, abort_flag, p.status);
        if (ok && !adapter) ok = mbar_wait(&sh->bready[s], ph, abort_flag, p.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(stage_a(s));
        const uint32_t b_base = smem_u32(stage_b(s));
        int ksub = 4;
        if (adapter) {
          const int left = p.r - (it - p.main_steps) * kTileK;
          ksub = left >= 64 ? 4 : (left + 15) / 16;
        }
        for (int kk = 0; kk < ksub; ++kk) {
          const uint64_t bdesc = (MODE == kFwd) ? smem_desc_sw128(b_base + kk * 32, 16, 1024)
                                                : smem_desc_sw128(b_base + kk * 2048, 8192, 1024);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint64_t adesc = smem_desc_sw128(a_base + h * kHalfABytes + kk * 32, 16, 1024);
            umma_f16(tmem + h * kTileN, adesc, bdesc, idesc, (it > 0 || kk > 0) ? 1u : 0u);
          }
        }
        // The last step's commit goes to accum (nobody waits on its stage);
        // MMAs finish in order, so it covers the whole accumulation.
        umma_commit(it + 1 < total_steps ? &sh->empty[s] : &sh->accum);
        ++issued;
      }
      if (!ok) drain_issued(sh->empty, issued, kStages);
    }
  } else {
    // ---------------- dequant warps (one NF4 block = one tile row per thread)
    const int t = threadIdx.x - 64;                  // 0..255 = tile row
    const bool dq = p.double_quant != 0;
    const float s_g = dq ? __ldg(p.absmax_scale) : 0.0f;
    // Row of W and block column for main step `it`.
    int64_t w_row;
    int block_col0;
    int row_step;
    if (MODE == kFwd) {
      w_row = int64_t(tile_n0) + t;                  // fixed W row, block column = it
      block_col0 = 0;
      row_step = 0;
    } else {
      w_row = t & 63;                                // W row = it * 64 + (t & 63)
      block_col0 = tile_n0 / 64 + (t >> 6);          // fixed block column
      row_step = 64;
    }
    auto scale_at = [&](int it) -> float {
      const int64_t row = w_row + int64_t(row_step) * it;
      if (row >= p.N) return 0.0f;
      const int bcol = (MODE == kFwd) ? it : block_col0;
      if (MODE == kDx && bcol >= p.kb_per_row) return 0.0f;
      return load_scale(p.absmax_q, p.absmax, s_g, dq, chunk_block(row, p.K, bcol, p.bs_shift));
    };
    float next_scale = p.main_steps > 0 ? scale_at(0) : 0.0f;
    for (int it = 0; it < p.main_steps; ++it) {
      const int s = it % kStages;
      const uint32_t ph = (it / kStages) & 1;
      const float scale = next_scale;
      if (it + 1 < p.main_steps) next_scale = scale_at(it + 1);
      if (!__all_sync(0xffffffffu, mbar_wait(&sh->full[s], ph, abort_flag, p.status))) break;
      dequant_row(stage_c(s) + t * 32, scale, stage_b(s), uint32_t(t), F16);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->bready[s]);
    }

    // ---------------- epilogue: TMEM -> registers -> bf16 / f16 -> shared
    // staging -> TMA store.  Each warp owns 32 rows (its TMEM lanes) of one
    // accumulator and writes 32 x 32 pieces through two 2 KB buffers over
    // the idle stage ring, so the output leaves as whole lines.
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&sh->accum, 0, abort_flag, p.status));
    tc_fence_after();
    if (ok) {
      const int quad = warp & 3;                     // TMEM lanes 32*quad .. +31
      const int half = (warp - 2) >> 2;              // accumulator half
      const int row0 = m0 + half * 128 + quad * 32;  // this warp's first row
      uint8_t* stage = smem + (warp - 2) * 4096;
      constexpr bool f16 = F16;
#pragma unroll 1
      for (int c = 0; c < kTileN / 32; ++c) {
        const int col0 = tile_n0 + c * 32;
        // Stop at the first piece that lies wholly past the output (warp-uniform):
        // every piece staged below is then stored, so waiting for all but the
        // last store group frees the buffer the piece two back used.
        if (col0 >= p.out_cols || row0 >= p.M) break;
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + (uint32_t(quad * 32) << 16) + half * kTileN + c * 32, v);
        tmem_ld_wait();
        uint32_t packed[16];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[8 * g + e]);
          const int col = col0 + 8 * g;
          if (MODE == kFwd && p.bias != nullptr && col < p.out_cols) {
            const uint4 bb = __ldg(reinterpret_cast<const uint4*>(p.bias + col));
            const uint32_t bw[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 bf = unpack2(f16, bw[e]);
              f[2 * e] += bf.x;
              f[2 * e + 1] += bf.y;
            }
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) packed[4 * g + e] = pack2(f16, f[2 * e], f[2 * e + 1]);
        }
        uint8_t* buf = stage + (c & 1) * 2048;
        if (lane == 0 && c >= 2) bulk_wait_group_read<1>();
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 4; ++j)   // 64-byte rows, 64-byte swizzle: chunk j at j ^ ((row >> 1) & 3)
          *reinterpret_cast<uint4*>(buf + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) =
              make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tm_out, buf, col0, row0);   // rows past M, columns past the end: clipped
          bulk_commit_group();
        }
      }
      if (lane == 0) bulk_wait_group_all();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ pair-CTA fused GEMM
//
// The same product on a cluster of two CTAs issuing tcgen05 cta_group::2
// MMAs (M = 256 rows per MMA, half from each CTA).  A pair tile is 512 x 256:
// two M = 256 accumulators of 256 columns fill each CTA's TMEM, and each CTA
// dequantizes only its 128-row half of the W' tile per K step, so every
// dequantized element feeds twice the MMA work of the single-CTA kernel and
// each CTA reads half the B operand from shared memory.
//   rank r of the pair: A rows m0 + 256 r .. + 255 (one 256-row TMA box per
//   K step; its 128-row halves h = 0, 1 are the A operands of the two
//   accumulators, so accumulator h of rank r holds rows m0 + 256 r + 128 h)
//   and W' half n0 + 128 r; the leader (rank 0) issues the MMAs, both CTAs'
//   A loads complete on the leader's barrier, the leader's commits multicast
//   to both.

constexpr int kP2Stages = 4;
constexpr int kP2DeqWarps = 8;                          // 2 threads per W' row
constexpr int kP2CodeWarp = 2 + kP2DeqWarps;            // code-tile TMA producer
// The A tile of a step is split over this many producer warps (warp 0 and
// warps kP2CodeWarp + 1 ..): one warp keeps only about one TMA box in
// flight per few hundred ns, so several warps shorten the A-tile latency.
#ifndef NF4_P2_A_WARPS
#define NF4_P2_A_WARPS 2
#endif
constexpr int kP2AWarps = NF4_P2_A_WARPS;
#ifndef NF4_P2_ROT_MUL
#define NF4_P2_ROT_MUL 13
#endif
constexpr int kP2ARows = 256 / kP2AWarps;               // A rows per producer box
constexpr int kP2Threads = 64 + kP2DeqWarps * 32 + 32 * kP2AWarps;
constexpr uint32_t kP2ABytes = 2 * kHalfABytes;        // 256 A rows (two 128-row blocks)
constexpr uint32_t kP2BBytes = 128 * 128;              // this CTA's 128 W' rows
constexpr uint32_t kP2StageBytes = kP2ABytes + kP2BBytes;
// NF4 codes arrive in their own ring, four K steps per TMA box: forward,
// 128 W rows x 128 code bytes (128-byte swizzle); dx, 256 W rows x 64 code
// bytes (64-byte swizzle).  Either way 16 KB per box and a conflict-free
// 16-byte read per thread.
constexpr int kP2CodeSteps = 4;
constexpr int kP2CodeSlots = 2;
constexpr uint32_t kP2CodeBytes = 128 * 128;
constexpr size_t kP2Smem =
    size_t(kP2Stages) * kP2StageBytes + size_t(kP2CodeSlots) * kP2CodeBytes + 1024 + 256;
constexpr int kP2TileM = 512;

struct PairShared {
  uint64_t afull[kP2Stages];     // leader: A (+ adapter B) bytes of both CTAs landed
  uint64_t bready[kP2Stages];    // leader: both CTAs' W' halves written (16 warp arrivals)
  uint64_t empty[kP2Stages];     // each CTA: the MMAs reading the stage finished
  uint64_t cfull[kP2CodeSlots];  // each CTA: a code box landed
  uint64_t cempty[kP2CodeSlots]; // each CTA: its 8 dequant warps finished a code box
  uint64_t accum;
  uint32_t tmem_base;
  uint32_t abort_flag;
};

// Byte offset in a code slot of the 16 code bytes that thread (row, half)
// dequantizes at step j (0..3) of the slot's four: 128-byte swizzle of
// 128-byte rows (forward) or 64-byte swizzle of 64-byte rows (dx, where tile
// row `row` is W row j * 64 + (row & 63) and code column group row >> 6).
template <int MODE>
__device__ __forceinline__ uint32_t code_offset(uint32_t row, uint32_t half, uint32_t j) {
  if (MODE == kFwd) return row * 128u + ((((2u * j + half) ^ (row & 7u))) << 4);
  const uint32_t R = j * 64u + (row & 63u);
  const uint32_t c = 2u * (row >> 6) + half;
  return R * 64u + ((c ^ ((R >> 1) & 3u)) << 4);
}

template <int MODE, bool F16>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kP2Threads, 1)
    fused_nf4_gemm_pair(const __grid_constant__ CUtensorMap tm_a,
                        const __grid_constant__ CUtensorMap tm_a2,
                        const __grid_constant__ CUtensorMap tm_b2,
                        const __grid_constant__ CUtensorMap tm_codes,
                        const __grid_constant__ CUtensorMap tm_out, const FusedParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* code_base = smem + kP2Stages * kP2StageBytes;
  PairShared* sh = reinterpret_cast<PairShared*>(code_base + kP2CodeSlots * kP2CodeBytes);
  auto stage_a = [&](int s) { return smem + s * kP2StageBytes; };
  auto stage_b = [&](int s) { return smem + s * kP2StageBytes + kP2ABytes; };
  auto code_slot = [&](int c) { return code_base + c * kP2CodeBytes; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int tile_n0 = (blockIdx.x >> 1) * kTileN;     // fwd: W rows; dx: output cols
  const int my_n0 = tile_n0 + 128 * int(rank);        // this CTA's half of the tile
  const int m0 = blockIdx.y * kP2TileM;
  const int total_steps = p.main_steps + p.adapter_steps;
  volatile uint32_t* abort_flag = &sh->abort_flag;
  // The pairs of one M tile run at the same time and read the same A rows;
  // each starts its reduction at a different whole code box (rotation by
  // kstep_rot steps), so they do not all request the same lines at once.
  const int code_groups = p.main_steps / kP2CodeSteps;
  const int kstep_rot = (p.main_steps % kP2CodeSteps == 0 && NF4_P2_ROT_MUL > 0)
                            ? kP2CodeSteps * int(((blockIdx.x >> 1) * NF4_P2_ROT_MUL) % code_groups)
                            : 0;
  auto kstep = [&](int it) { return it + kstep_rot < p.main_steps ? it + kstep_rot : it + kstep_rot - p.main_steps; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kP2Stages; ++s) {
      mbar_init(&sh->afull[s], 1);
      // leader: its own 8 dequant warps + one forwarded arrival from the peer
      mbar_init(&sh->bready[s], rank == 0 ? kP2DeqWarps + 1 : kP2DeqWarps);
      mbar_init(&sh->empty[s], 1);
    }
    for (int c = 0; c < kP2CodeSlots; ++c) {
      mbar_init(&sh->cfull[c], 1);
      mbar_init(&sh->cempty[c], kP2DeqWarps);
    }
    mbar_init(&sh->accum, 1);
    sh->abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
    tma_prefetch(&tm_a);
    tma_prefetch(&tm_a2);
    tma_prefetch(&tm_b2);
    tma_prefetch(&tm_codes);
  }
  if (warp == 1) {
    tmem_alloc_pair(&sh->tmem_base, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;

  const int a_part = warp == 0 ? 0 : (warp > kP2CodeWarp ? warp - kP2CodeWarp : -1);
  if (a_part >= 0) {
    // ---------------- A (and adapter B) TMA producers (both CTAs): producer
    // a_part loads A rows a_part * kP2ARows .. + kP2ARows - 1 of this CTA's 256
    if (lane == 0) {
      const int arow = a_part * kP2ARows;
      for (int it = 0; it < total_steps; ++it) {
        const int s = it % kP2Stages;
        const uint32_t ph = (it / kP2Stages) & 1;
        if (!mbar_wait(&sh->empty[s], ph ^ 1, abort_flag, p.status)) break;
        const uint32_t afull_leader = mapa_shared(smem_u32(&sh->afull[s]), 0);
        uint8_t* a = stage_a(s) + arow * 128;
        if (it < p.main_steps) {
          if (rank == 0 && a_part == 0) mbar_arrive_expect_tx(&sh->afull[s], 2 * kP2ABytes);
          tma_load_2d_pair(a, &tm_a, afull_leader, kstep(it) * kTileK, m0 + 256 * int(rank) + arow);
        } else {
          if (it == p.main_steps) grid_dep_wait();
          const int r0 = (it - p.main_steps) * kTileK;
          if (rank == 0 && a_part == 0) mbar_arrive_expect_tx(&sh->afull[s], 2 * (kP2ABytes + kP2BBytes));
          tma_load_2d_pair(a, &tm_a2, afull_leader, r0, m0 + 256 * int(rank) + arow);
          if (a_part != 0) continue;
          if (MODE == kFwd) {
            tma_load_2d_pair(stage_b(s), &tm_b2, afull_leader, r0, my_n0);
          } else {
#pragma unroll
            for (int g = 0; g < 2; ++g)
              tma_load_2d_pair(stage_b(s) + g * 8192, &tm_b2, afull_leader, my_n0 + 64 * g, r0);
          }
        }
      }
    }
  } else if (warp == kP2CodeWarp) {
    // ---------------- code producer: one box per four K steps into a two-slot ring
    if (lane == 0) {
      const int groups = int((p.main_steps + kP2CodeSteps - 1) / kP2CodeSteps);
      int issued = 0;
      for (int g = 0; g < groups; ++g) {
        const int c = g % kP2CodeSlots;
        const uint32_t ph = (g / kP2CodeSlots) & 1;
        if (!mbar_wait(&sh->cempty[c], ph ^ 1, abort_flag, p.status)) break;
        mbar_arrive_expect_tx(&sh->cfull[c], kP2CodeBytes);
        const int kg = kstep(g * kP2CodeSteps) / kP2CodeSteps;   // code box of this group
        if (MODE == kFwd)   // code bytes kg*128 .. +127 of W rows my_n0 .. +127
          tma_load_2d(code_slot(c), &tm_codes, &sh->cfull[c], kg * 128, my_n0);
        else                // code bytes my_n0/2 .. +63 of W rows kg*256 .. +255
          tma_load_2d(code_slot(c), &tm_codes, &sh->cfull[c], my_n0 / 2, kg * 256);
        ++issued;
      }
      if (*abort_flag) {
        // Unwind: wait (bounded) for the code copies still in flight.
        for (int g = issued - 1; g >= 0 && g >= issued - kP2CodeSlots; --g) {
          uint32_t dummy_abort = 0;
          mbar_wait(&sh->cfull[g % kP2CodeSlots], (g / kP2CodeSlots) & 1, &dummy_abort, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- peer CTA: forward "W' half written" to the leader, one
    // cluster-scope arrival per step (the dequant warps arrive locally).
    if (lane == 0 && rank == 1) {
      const uint32_t leader_bready0 = mapa_shared(smem_u32(&sh->bready[0]), 0);
      for (int it = 0; it < p.main_steps; ++it) {
        const int s = it % kP2Stages;
        const uint32_t ph = (it / kP2Stages) & 1;
        if (!mbar_wait(&sh->bready[s], ph, abort_flag, p.status)) break;
        mbar_arrive_cluster(leader_bready0 + uint32_t(s) * uint32_t(sizeof(uint64_t)));
      }
    }
    // ---------------- MMA issuer (leader CTA only)
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = idesc_f32acc(256, kTileN, false, MODE == kDx, F16);
      bool ok = true;
      int issued = 0;
      for (int it = 0; it < total_steps && ok; ++it) {
        const int s = it % kP2Stages;
        const uint32_t ph = (it / kP2Stages) & 1;
        const bool adapter = it >= p.main_steps;
        // afull completes by TMA transactions (and empty / accum by
        // tcgen05.commit): a CTA-scope acquire is enough there.  bready is
        // arrived by the peer's thread, so its wait acquires at cluster scope.
        ok = mbar_wait(&sh->afull[s], ph, abort_flag, p.status);
        if (ok && !adapter) ok = mbar_wait_cluster(&sh->bready[s], ph, abort_flag, p.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(stage_a(s));
        const uint32_t b_base = smem_u32(stage_b(s));
        int ksub = 4;
        if (adapter) {
          const int left = p.r - (it - p.main_steps) * kTileK;
          ksub = left >= 64 ? 4 : (left + 15) / 16;
        }
        for (int kk = 0; kk < ksub; ++kk) {
          const uint64_t bdesc = (MODE == kFwd) ? smem_desc_sw128(b_base + kk * 32, 16, 1024)
                                                : smem_desc_sw128(b_base + kk * 2048, 8192, 1024);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint64_t adesc = smem_desc_sw128(a_base + h * kHalfABytes + kk * 32, 16, 1024);
            umma_f16_pair(tmem + h * kTileN, adesc, bdesc, idesc, (it > 0 || kk > 0) ? 1u : 0u);
          }
        }
        // One commit per step, multicast to both CTAs.  The last step's
        // commit goes to accum instead (nobody waits on its stage); MMAs
        // finish in order, so it covers the whole accumulation.  (A second
        // commit issued right behind the first was seen to arrive before the
        // MMAs had finished reading their operands.)
        umma_commit_pair_mc(it + 1 < total_steps ? &sh->empty[s] : &sh->accum, 0x3);
        ++issued;
      }
      if (!ok) drain_issued(sh->empty, issued, kP2Stages);
    }
  } else {
    // ---------------- dequant warps: thread pair per W' row (one NF4 block);
    // a warp covers 16 rows, lanes 0-15 the first half of each block and
    // lanes 16-31 the second, so each quarter-warp touches 8 consecutive rows.
    const int row = (warp - 2) * 16 + (lane & 15);    // 0..127 tile row
    const uint32_t half = uint32_t(lane >> 4);
    const bool dq = p.double_quant != 0;
    const float s_g = dq ? __ldg(p.absmax_scale) : 0.0f;
    int64_t w_row;
    int block_col0, row_step;
    if (MODE == kFwd) {
      w_row = int64_t(my_n0) + row;
      block_col0 = 0;
      row_step = 0;
    } else {
      w_row = row & 63;
      block_col0 = my_n0 / 64 + (row >> 6);
      row_step = 64;
    }
    auto scale_at = [&](int it) -> float {
      const int ks = kstep(it);
      const int64_t wr = w_row + int64_t(row_step) * ks;
      if (wr >= p.N) return 0.0f;
      const int bcol = (MODE == kFwd) ? ks : block_col0;
      if (MODE == kDx && bcol >= p.kb_per_row) return 0.0f;
      return load_scale(p.absmax_q, p.absmax, s_g, dq, chunk_block(wr, p.K, bcol, p.bs_shift));
    };
    // scales of the next four steps in flight (a small register ring)
    float sc[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) sc[j] = j < p.main_steps ? scale_at(j) : 0.0f;
    for (int it = 0; it < p.main_steps; ++it) {
      const int s = it % kP2Stages;
      const uint32_t ph = (it / kP2Stages) & 1;
      const float scale = sc[0];
      sc[0] = sc[1];
      sc[1] = sc[2];
      sc[2] = sc[3];
      sc[3] = (it + 4 < p.main_steps) ? scale_at(it + 4) : 0.0f;
      const int g = it / kP2CodeSteps;
      const int j = it % kP2CodeSteps;
      const int c = g % kP2CodeSlots;
      // the W' half of stage s is free once the MMAs of step it - kP2Stages
      // finished (the first round passes at once), and the codes of group g landed
      bool ok = mbar_wait(&sh->empty[s], ph ^ 1, abort_flag, p.status);
      if (ok && j == 0) ok = mbar_wait(&sh->cfull[c], (g / kP2CodeSlots) & 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      dequant_half_row(code_slot(c) + code_offset<MODE>(uint32_t(row), half, uint32_t(j)), scale,
                       stage_b(s), uint32_t(row), half, F16);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sh->bready[s]);
        if (j == kP2CodeSteps - 1 || it == p.main_steps - 1) mbar_arrive(&sh->cempty[c]);
      }
    }

    // ---------------- epilogue: this CTA's 128 rows of both accumulators.
    // Each warp owns 32 rows (its TMEM lanes) of one accumulator; every 32
    // columns it converts, stages the 32 x 32 piece in swizzled shared memory
    // (two 2 KB buffers over the now idle A ring) and writes it with a TMA
    // tensor store, so the output leaves as whole lines.
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&sh->accum, 0, abort_flag, p.status));
    tc_fence_after();
    if (ok) {
      const int quad = warp & 3;
      const int h = (warp - 2) >> 2;
      const int row0 = m0 + 256 * int(rank) + 128 * h + quad * 32;   // this warp's first row
      uint8_t* stage = smem + (warp - 2) * 4096;
      constexpr bool f16 = F16;
#pragma unroll 1
      for (int c = 0; c < kTileN / 32; ++c) {
        const int col0 = tile_n0 + c * 32;
        if (col0 >= p.out_cols || row0 >= p.M) break;   // see the single-CTA epilogue
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + (uint32_t(quad * 32) << 16) + h * kTileN + c * 32, v);
        tmem_ld_wait();
        uint32_t packed[16];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[8 * g + e]);
          const int col = col0 + 8 * g;
          if (MODE == kFwd && p.bias != nullptr && col < p.out_cols) {
            const uint4 bb = __ldg(reinterpret_cast<const uint4*>(p.bias + col));
            const uint32_t bw[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 bf = unpack2(f16, bw[e]);
              f[2 * e] += bf.x;
              f[2 * e + 1] += bf.y;
            }
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) packed[4 * g + e] = pack2(f16, f[2 * e], f[2 * e + 1]);
        }
        // buffer c & 1 is free once the store issued two pieces ago has read it
        uint8_t* buf = stage + (c & 1) * 2048;
        if (lane == 0 && c >= 2) bulk_wait_group_read<1>();
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 4; ++j)   // 64-byte rows, 64-byte swizzle: chunk j at j ^ ((row >> 1) & 3)
          *reinterpret_cast<uint4*>(buf + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) =
              make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tm_out, buf, col0, row0);   // rows past M, columns past the end: clipped
          bulk_commit_group();
        }
      }
      if (lane == 0) bulk_wait_group_all();
    }
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// ------------------------------------------------------------------ adapter GEMM
//
// D[Mo, NP] = sum over a reduction range of A[Mo, red] * B[NP, red], one
// 128-row tile per CTA and one slice of the reduction per blockIdx.y; fp32
// the slices of a tile form one thread-block cluster and are summed through
// distributed shared memory.  Operands come by TMA in 64-deep
// steps, each either K-major (rows of the reduction) or MN-major.

constexpr int kAdStages = 4;
constexpr int kAdThreads = 192;    // TMA warp, MMA warp, 4 epilogue warps
constexpr uint32_t kAdABytes = 128 * 128;

struct AdapterParams {
  int Mo;            // output rows
  int NP;            // output cols (r rounded up to 64)
  int r;             // output cols kept
  int red_steps;     // ceil(reduction / 64)
  int steps_per_slice;
  int slices;
  int a_mn;          // A operand MN-major
  int b_mn;          // B operand MN-major
  int kind;          // 0: bf16/f16(scale * D) [Mo][r]; 1: fp32 D [Mo][r]; 2: fp32 D^T [r][Mo]
  int f16;           // operands and the kind-0 output in f16 (else bf16)
  float scale;
  __nv_bfloat16* out_bf16;
  float* out_f32;
  uint32_t* status;
};

// Write 4 consecutive output columns (col .. col+3 < r) of one row.
__device__ __forceinline__ void adapter_store4(const AdapterParams& p, int row, int col, float4 v) {
  if (p.kind == 0) {
    const uint2 o = make_uint2(pack2(p.f16 != 0, v.x * p.scale, v.y * p.scale),
                               pack2(p.f16 != 0, v.z * p.scale, v.w * p.scale));
    *reinterpret_cast<uint2*>(p.out_bf16 + int64_t(row) * p.r + col) = o;
  } else if (p.kind == 1) {
    *reinterpret_cast<float4*>(p.out_f32 + int64_t(row) * p.r + col) = v;
  } else {
    float* o = p.out_f32 + int64_t(col) * p.Mo + row;
    o[0] = v.x;
    o[int64_t(p.Mo)] = v.y;
    o[2 * int64_t(p.Mo)] = v.z;
    o[3 * int64_t(p.Mo)] = v.w;
  }
}

struct AdapterShared {
  uint64_t full[kAdStages];
  uint64_t empty[kAdStages];
  uint64_t accum;
  uint32_t tmem_base;
  uint32_t abort_flag;
};

__global__ void __launch_bounds__(kAdThreads, 1)
    adapter_gemm(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                 const AdapterParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t b_bytes = uint32_t(p.NP) * 128u;
  const uint32_t stage_bytes = kAdABytes + b_bytes;
  AdapterShared* sh = reinterpret_cast<AdapterShared*>(smem + kAdStages * stage_bytes);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int mo0 = blockIdx.x * 128;
  const int step0 = blockIdx.y * p.steps_per_slice;
  const int step1 = min(step0 + p.steps_per_slice, p.red_steps);
  const int nsteps = max(step1 - step0, 0);
  volatile uint32_t* abort_flag = &sh->abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kAdStages; ++s) {
      mbar_init(&sh->full[s], 2);     // the A copies' issuer and the B copies' issuer
      mbar_init(&sh->empty[s], 1);
    }
    mbar_init(&sh->accum, 1);
    sh->abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
    tma_prefetch(&tm_a);
    tma_prefetch(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(&sh->tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  // A kernel launched as this one's programmatic dependent (the forward GEMM
  // after T) may start on the SMs this grid leaves free; it waits for this
  // grid's completion before it reads the result.
  grid_dep_launch();

  // TMA copies: the A tile from warp 0 and the B tile from warp 2 (one warp
  // keeps only a few TMA copies going per microsecond); each arrives on the
  // stage's full barrier with its own byte count.
  const bool a_issuer = warp == 0 && lane == 0;
  const bool b_issuer = warp == 2 && lane == 0;
  if (a_issuer || b_issuer) {
    int issued = 0;
    for (int i = 0; i < nsteps; ++i) {
      const int s = i % kAdStages;
      const uint32_t ph = (i / kAdStages) & 1;
      if (!mbar_wait(&sh->empty[s], ph ^ 1, abort_flag, p.status)) break;
      uint8_t* a = smem + s * stage_bytes;
      uint8_t* b = a + kAdABytes;
      const int red0 = (step0 + i) * 64;
      if (a_issuer) {
        mbar_arrive_expect_tx(&sh->full[s], kAdABytes);
        if (p.a_mn) {
          tma_load_2d(a, &tm_a, &sh->full[s], mo0, red0);
          tma_load_2d(a + 8192, &tm_a, &sh->full[s], mo0 + 64, red0);
        } else {
          tma_load_2d(a, &tm_a, &sh->full[s], red0, mo0);
        }
      } else {
        mbar_arrive_expect_tx(&sh->full[s], b_bytes);
        if (p.b_mn) {
          for (int g = 0; g < p.NP / 64; ++g) tma_load_2d(b + g * 8192, &tm_b, &sh->full[s], 64 * g, red0);
        } else {
          tma_load_2d(b, &tm_b, &sh->full[s], red0, 0);
        }
      }
      ++issued;
    }
    if (*abort_flag) {
      // Unwind: wait (bounded) for this issuer's copies still in flight.
      for (int i = issued - 1; i >= 0 && i >= issued - kAdStages; --i) {
        uint32_t dummy_abort = 0;
        mbar_wait(&sh->full[i % kAdStages], (i / kAdStages) & 1, &dummy_abort, nullptr);
      }
    }
  }
  if (warp == 0) {
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_f32acc(128, p.NP, p.a_mn != 0, p.b_mn != 0, p.f16 != 0);
      bool ok = true;
      int issued = 0;
      for (int i = 0; i < nsteps; ++i) {
        const int s = i % kAdStages;
        const uint32_t ph = (i / kAdStages) & 1;
        ok = mbar_wait(&sh->full[s], ph, abort_flag, p.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(smem + s * stage_bytes);
        const uint32_t b_base = a_base + kAdABytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t adesc = p.a_mn ? smem_desc_sw128(a_base + kk * 2048, 8192, 1024)
                                        : smem_desc_sw128(a_base + kk * 32, 16, 1024);
          const uint64_t bdesc = p.b_mn ? smem_desc_sw128(b_base + kk * 2048, 8192, 1024)
                                        : smem_desc_sw128(b_base + kk * 32, 16, 1024);
          umma_f16(tmem, adesc, bdesc, idesc, (i > 0 || kk > 0) ? 1u : 0u);
        }
        // the last step's commit goes to accum (nobody waits on its stage)
        umma_commit(i + 1 < nsteps ? &sh->empty[s] : &sh->accum);
        ++issued;
      }
      if (!ok) {
        drain_issued(sh->empty, issued, kAdStages);
      } else if (nsteps == 0) {
        mbar_arrive(&sh->accum);   // an empty slice: no MMAs to wait for
      }
    }
  } else {
    // epilogue warps 2..5 -> TMEM lane quadrants 2, 3, 0, 1: with one slice
    // the result goes straight out, otherwise this slice's fp32 partial.
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&sh->accum, 0, abort_flag, p.status));
    tc_fence_after();
    const int quad = warp & 3;
    const int row = mo0 + quad * 32 + lane;
    // partial tile [128][NP] fp32 over the (now idle) stage buffers; the
    // 16-byte chunk v of row R sits at chunk v ^ (R & 7), so the eight rows a
    // quarter-warp writes at once land in eight different bank groups
    const int prow = quad * 32 + lane;
    float* dst = reinterpret_cast<float*>(smem) + prow * p.NP;
    for (int c = 0; c < p.NP / 32; ++c) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem + (uint32_t(quad * 32) << 16) + c * 32, v);
      tmem_ld_wait();
      if (row < p.Mo) {
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
          if (ok && nsteps > 0)
            f = make_float4(__uint_as_float(v[4 * g]), __uint_as_float(v[4 * g + 1]),
                            __uint_as_float(v[4 * g + 2]), __uint_as_float(v[4 * g + 3]));
          const int col = c * 32 + 4 * g;
          if (p.slices == 1) {
            if (col < p.r) adapter_store4(p, row, col, f);
          } else {
            reinterpret_cast<float4*>(dst + 4 * ((col >> 2) ^ (prow & 7)))[0] = f;
          }
        }
      } else if (p.slices > 1) {
#pragma unroll
        for (int g = 0; g < 8; ++g)
          reinterpret_cast<float4*>(dst + 4 * ((c * 8 + g) ^ (prow & 7)))[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (p.slices > 1) {
    // The slices of this tile are the CTAs of one cluster (along y).  After
    // all partials are in shared memory, CTA q sums rows [q*128/S, (q+1)*128/S)
    // over the cluster's partials in slice order (deterministic) and writes
    // them out; a second cluster barrier keeps every partial alive until read.
    cluster_sync();
    const uint32_t q = cluster_ctarank();
    const int rows_per = 128 / p.slices;
    const int vec_per_row = p.r / 4;
    const int total = rows_per * vec_per_row;
    const uint32_t base = smem_u32(smem);
    for (int i = threadIdx.x; i < total; i += blockDim.x) {
      int rr, cv;
      if (p.kind == 2) {            // consecutive threads -> consecutive rows (coalesced D^T)
        cv = i / rows_per;
        rr = i % rows_per;
      } else {
        rr = i / vec_per_row;
        cv = i % vec_per_row;
      }
      const int trow = int(q) * rows_per + rr;
      const uint32_t off = uint32_t((trow * p.NP + 4 * (cv ^ (trow & 7))) * 4);   // the parking swizzle
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int sl = 0; sl < p.slices; ++sl) {
        const float4 v = ld_shared_cluster_f4(mapa_shared(base + off, uint32_t(sl)));
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      const int row = mo0 + trow;
      if (row < p.Mo) adapter_store4(p, row, 4 * cv, acc);
    }
    cluster_sync();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ------------------------------------------------------------------ host side

// High-priority side streams with their fork and join events, per device and
// per calling stream (up to kSideSlots calling streams each; more share the
// slots round robin, which only serialises their side work).  Created on
// first use, re-created if the context that owned them is gone.  Callers hold
// g_side_mu from the fork to the join.
struct SideStream {
  cudaStream_t owner = nullptr;   // the calling stream this slot serves
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr;
  cudaEvent_t join = nullptr;
};
constexpr int kSideSlots = 8;
std::mutex g_side_mu;
SideStream g_side[64][kSideSlots];
int g_side_next[64];

cudaError_t side_stream(cudaStream_t caller, SideStream** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  SideStream* slots = g_side[dev];
  int pick = -1;
  for (int i = 0; i < kSideSlots && pick < 0; ++i)
    if (slots[i].stream != nullptr && slots[i].owner == caller) pick = i;
  for (int i = 0; i < kSideSlots && pick < 0; ++i)
    if (slots[i].stream == nullptr) pick = i;
  if (pick < 0) pick = g_side_next[dev]++ % kSideSlots;
  SideStream& ss = slots[pick];
  ss.owner = caller;
  int prio = 0;
  if (ss.stream != nullptr && cudaStreamGetPriority(ss.stream, &prio) != cudaSuccess) {
    (void)cudaGetLastError();
    ss = SideStream{};
    ss.owner = caller;
  }
  if (ss.stream == nullptr) {
    int least = 0, greatest = 0;
    e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
    if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&ss.stream, cudaStreamNonBlocking, greatest);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming);
    if (e != cudaSuccess) {   // release whatever was made; the next call tries again
      if (ss.join != nullptr) (void)cudaEventDestroy(ss.join);
      if (ss.fork != nullptr) (void)cudaEventDestroy(ss.fork);
      if (ss.stream != nullptr) (void)cudaStreamDestroy(ss.stream);
      ss = SideStream{};
      return e;
    }
  }
  *out = &ss;
  return cudaSuccess;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 2-D map over a row-major matrix: `inner` elements per row, `outer` rows.
bool make_map(CUtensorMap* map, const void* base, bool bf16, uint64_t inner, uint64_t outer,
              uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const uint32_t esize = bf16 ? 2 : 1;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * esize};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult res = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                    const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS;
}

bool make_map(CUtensorMap* map, const void* base, bool bf16, uint64_t inner, uint64_t outer,
              uint32_t box_inner, uint32_t box_outer, bool swizzle128) {
  return make_map(map, base, bf16, inner, outer, box_inner, box_outer,
                  swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE);
}

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Split of a reduction of `red_steps` 64-deep steps over Mo/128 tiles so that
// about two CTAs per SM of a 148-SM part run; independent of the device so
// the workspace size is a pure function of the shapes.
struct SplitPlan {
  int tiles, slices, per;
};
SplitPlan plan_split(int64_t Mo, int64_t red) {
  SplitPlan sp;
  sp.tiles = int(cdiv(Mo, 128));
  const int steps = int(std::max<int64_t>(cdiv(red, 64), 1));
  // one wave of 2 CTAs per SM; the slices of a tile form one cluster (<= 8)
  const int cap = std::max(1, std::min(std::min(296 / sp.tiles, 8), std::max(1, steps / 4)));
  int sl = 1;
  while (sl * 2 <= cap) sl *= 2;
  sp.slices = sl;
  sp.per = int(cdiv(steps, sl));
  return sp;
}

int round_np(int r) { return int(cdiv(r, 64) * 64); }



PerDeviceOnce g_attr_done;

cudaError_t set_attrs() {
  const int dev = PerDeviceOnce::current();
  if (g_attr_done.done(dev)) return cudaSuccess;
  const void* single[4] = {(const void*)fused_nf4_gemm<kFwd, false>, (const void*)fused_nf4_gemm<kDx, false>,
                           (const void*)fused_nf4_gemm<kFwd, true>, (const void*)fused_nf4_gemm<kDx, true>};
  const void* pair[4] = {(const void*)fused_nf4_gemm_pair<kFwd, false>, (const void*)fused_nf4_gemm_pair<kDx, false>,
                         (const void*)fused_nf4_gemm_pair<kFwd, true>, (const void*)fused_nf4_gemm_pair<kDx, true>};
  cudaError_t e = cudaSuccess;
  for (int i = 0; i < 4 && e == cudaSuccess; ++i)
    e = cudaFuncSetAttribute(single[i], cudaFuncAttributeMaxDynamicSharedMemorySize, int(kFusedSmem));
  for (int i = 0; i < 4 && e == cudaSuccess; ++i)
    e = cudaFuncSetAttribute(pair[i], cudaFuncAttributeMaxDynamicSharedMemorySize, int(kP2Smem));
  const size_t ad_smem = kAdStages * (kAdABytes + 256 * 128) + 1024 + 256;
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(adapter_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, int(ad_smem));
  if (e == cudaSuccess) g_attr_done.mark(dev);
  return e;
}

// One rank-r product through adapter_gemm.
//   a_mn/b_mn: operand majorness; a_base/b_base: matrices as [outer][inner].
struct AdapterJob {
  const void* a; uint64_t a_inner, a_outer; bool a_mn;
  const void* b; uint64_t b_inner, b_outer; bool b_mn;
  int64_t Mo, red;
  int r;
  int kind;          // see AdapterParams::kind
  int f16;           // operands (and the kind-0 output) in f16
  float scale;
  __nv_bfloat16* out_bf16;
  float* out_f32;
  int prof_id;       // profiler kernel id of this product
};

// A launch fully prepared on the host (tensor maps encoded, parameters set),
// so that a call can build every launch before it enqueues the first one.
struct AdapterLaunch {
  CUtensorMap ma, mb;
  AdapterParams p;
  dim3 grid;
  size_t smem;
  int prof_id;
};

bool prepare_adapter(const AdapterJob& j, uint32_t* status, AdapterLaunch* L) {
  const int NP = round_np(j.r);
  bool ok = j.a_mn ? make_map(&L->ma, j.a, true, j.a_inner, j.a_outer, 64, 64, true)
                   : make_map(&L->ma, j.a, true, j.a_inner, j.a_outer, 64, 128, true);
  ok = ok && (j.b_mn ? make_map(&L->mb, j.b, true, j.b_inner, j.b_outer, 64, 64, true)
                     : make_map(&L->mb, j.b, true, j.b_inner, j.b_outer, 64, uint32_t(NP), true));
  if (!ok) return false;
  const SplitPlan sp = plan_split(j.Mo, j.red);
  AdapterParams& p = L->p;
  p.Mo = int(j.Mo);
  p.NP = NP;
  p.r = j.r;
  p.red_steps = int(std::max<int64_t>(cdiv(j.red, 64), 1));
  p.steps_per_slice = sp.per;
  p.slices = sp.slices;
  p.a_mn = j.a_mn;
  p.b_mn = j.b_mn;
  p.kind = j.kind;
  p.f16 = j.f16;
  p.scale = j.scale;
  p.out_bf16 = j.out_bf16;
  p.out_f32 = j.out_f32;
  p.status = status;
  L->grid = dim3(unsigned(sp.tiles), unsigned(sp.slices), 1);
  L->smem = kAdStages * (kAdABytes + size_t(NP) * 128) + 1024 + 256;
  L->prof_id = j.prof_id;
  return true;
}

cudaError_t launch_adapter(const AdapterLaunch& L, cudaStream_t st, int* launches) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = L.grid;
  cfg.blockDim = dim3(kAdThreads, 1, 1);
  cfg.dynamicSmemBytes = L.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = L.grid.y;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  NF4_PROF_BEGIN(st, L.prof_id);
  cudaError_t e = cudaLaunchKernelEx(&cfg, adapter_gemm, L.ma, L.mb, L.p);
  NF4_PROF_END(st, L.prof_id);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e == cudaSuccess) ++*launches;
  return e;
}

// Pair-CTA tiles (512 rows) once M fills them; single-CTA 256-row tiles below.
bool use_pair(int64_t M) { return M > 256; }

FusedParams fused_params(const LinearArgs& a, int mode) {
  FusedParams p;
  p.M = int(a.M);
  p.N = int(a.N);
  p.K = int(a.K);
  p.r = a.r;
  p.main_steps = mode == kFwd ? int(a.K / 64) : int(cdiv(a.N, 64));
  p.adapter_steps = int(cdiv(a.r, 64));
  p.out_cols = mode == kFwd ? int(a.N) : int(a.K);
  p.kb_per_row = int(a.K / 64);
  p.bs_shift = log2_block(a.w->block_size);
  p.double_quant = a.w->double_quant;
  p.f16 = a.f16;
  p.absmax_q = a.w->absmax_q;
  p.absmax = a.w->absmax;
  p.absmax_scale = a.w->absmax_scale;
  p.bias = static_cast<const __nv_bfloat16*>(mode == kFwd ? a.bias : nullptr);
  p.out = static_cast<__nv_bfloat16*>(mode == kFwd ? a.y : a.dx);
  p.status = a.status;
  return p;
}

// Workspace regions after the header (256-byte aligned):
//   fwd: [T bf16 M x r (when t_out is null)]
//   bwd: [T bf16 M x r (when t is null)] [U bf16 M x r]
// One [M, r] scratch matrix (T or U), sized for 4-byte elements so that the
// same workspace serves every compute dtype (the F32 path keeps them in fp32).
size_t mr_bytes(int64_t M, int r) { return align256(size_t(M) * size_t(r) * 4); }

AdapterJob job_T(const LinearArgs& a, __nv_bfloat16* T) {
  AdapterJob j{};
  j.a = a.x; j.a_inner = a.K; j.a_outer = a.M; j.a_mn = false;
  j.b = a.A; j.b_inner = a.K; j.b_outer = a.r; j.b_mn = false;
  j.Mo = a.M; j.red = a.K; j.r = a.r; j.kind = 0; j.scale = a.s; j.out_bf16 = T; j.f16 = a.f16;
  j.prof_id = kKAdapterT;
  return j;
}

// One fused dequant + tensor-core GEMM launch, prepared on the host.
struct FusedLaunch {
  CUtensorMap ta, ta2, tb2, tc, to;
  FusedParams p;
  bool pair;
  int mode;
  bool f16;
  dim3 grid;
};

// Forward: A = x, A2 = T, B2 = B_lora, out = y.  dx: A = dy, A2 = U, B2 = A_lora, out = dx.
bool prepare_fused(const LinearArgs& a, int mode, const __nv_bfloat16* a2, FusedLaunch* L) {
  L->pair = use_pair(a.M);
  L->mode = mode;
  L->f16 = a.f16 != 0;
  const bool pair = L->pair;
  const uint32_t arows = pair ? uint32_t(kP2ARows) : 256u;   // A rows per TMA box
  const int64_t m_tiles = cdiv(a.M, pair ? kP2TileM : kTileM);
  if (m_tiles > 65535) return false;                         // grid.y
  bool ok;
  if (mode == kFwd) {
    const uint32_t brows = pair ? 128 : 256;     // W' rows per CTA
    ok = make_map(&L->ta, a.x, true, a.K, a.M, 64, arows, true);
    ok = ok && make_map(&L->ta2, a2, true, a.r, a.M, 64, arows, true);
    ok = ok && make_map(&L->tb2, a.B, true, a.r, a.N, 64, brows, true);
    ok = ok && (pair ? make_map(&L->tc, a.w->codes, false, a.K / 2, a.N, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B)
                     : make_map(&L->tc, a.w->codes, false, a.K / 2, a.N, 32, brows, false));
    // y [M, N]: 32 x 32 boxes in the epilogues' staging layout
    ok = ok && make_map_2d_bf16(&L->to, a.y, uint64_t(a.N), uint64_t(a.M), 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
    L->grid = pair ? dim3(unsigned(2 * cdiv(a.N, kTileN)), unsigned(m_tiles))
                   : dim3(unsigned(cdiv(a.N, kTileN)), unsigned(m_tiles));
  } else {
    ok = make_map(&L->ta, a.dy, true, a.N, a.M, 64, arows, true);
    ok = ok && make_map(&L->ta2, a2, true, a.r, a.M, 64, arows, true);
    ok = ok && make_map(&L->tb2, a.A, true, a.K, a.r, 64, 64, true);
    ok = ok && (pair ? make_map(&L->tc, a.w->codes, false, a.K / 2, a.N, 64, 256, CU_TENSOR_MAP_SWIZZLE_64B)
                     : make_map(&L->tc, a.w->codes, false, a.K / 2, a.N, 32, 64, false));
    // dx [M, K]: 32 x 32 boxes in the epilogues' staging layout
    ok = ok && make_map_2d_bf16(&L->to, a.dx, uint64_t(a.K), uint64_t(a.M), 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
    L->grid = pair ? dim3(unsigned(2 * cdiv(a.K, kTileN)), unsigned(m_tiles))
                   : dim3(unsigned(cdiv(a.K, kTileN)), unsigned(m_tiles));
  }
  if (!ok) return false;
  L->p = fused_params(a, mode);
  return true;
}

// pdl: launch as a programmatic dependent of the kernel before it on the
// stream (which must be the producer of A2 and call grid_dep_launch); the
// kernel reads A2 only after grid_dep_wait.
template <typename K>
cudaError_t launch_fused_kernel(K kernel, const FusedLaunch& L, unsigned threads, size_t smem,
                                cudaStream_t st, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = L.grid;
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, L.ta, L.ta2, L.tb2, L.tc, L.to, L.p);
}

cudaError_t launch_fused(const FusedLaunch& L, cudaStream_t st, int* launches, bool pdl = false) {
  const int id = L.mode == kFwd ? kKFusedFwd : kKFusedDx;
  NF4_PROF_BEGIN(st, id);
  cudaError_t e;
  if (L.pair) {
    const unsigned t = kP2Threads;
    if (L.mode == kFwd)
      e = L.f16 ? launch_fused_kernel(fused_nf4_gemm_pair<kFwd, true>, L, t, kP2Smem, st, pdl)
                : launch_fused_kernel(fused_nf4_gemm_pair<kFwd, false>, L, t, kP2Smem, st, pdl);
    else
      e = L.f16 ? launch_fused_kernel(fused_nf4_gemm_pair<kDx, true>, L, t, kP2Smem, st, pdl)
                : launch_fused_kernel(fused_nf4_gemm_pair<kDx, false>, L, t, kP2Smem, st, pdl);
  } else {
    const unsigned t = kFusedThreads;
    if (L.mode == kFwd)
      e = L.f16 ? launch_fused_kernel(fused_nf4_gemm<kFwd, true>, L, t, kFusedSmem, st, pdl)
                : launch_fused_kernel(fused_nf4_gemm<kFwd, false>, L, t, kFusedSmem, st, pdl);
    else
      e = L.f16 ? launch_fused_kernel(fused_nf4_gemm<kDx, true>, L, t, kFusedSmem, st, pdl)
                : launch_fused_kernel(fused_nf4_gemm<kDx, false>, L, t, kFusedSmem, st, pdl);
  }
  NF4_PROF_END(st, id);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e == cudaSuccess) ++*launches;
  return e;
}

}  // namespace

bool make_map_2d(CUtensorMap* map, const void* base, bool bf16, uint64_t inner, uint64_t outer,
                 uint32_t box_inner, uint32_t box_outer, bool swizzle128) {
  return make_map(map, base, bf16, inner, outer, box_inner, box_outer, swizzle128);
}

bool make_map_2d_f32(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                     uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 4};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_2d_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                      uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  return make_map(map, base, true, inner, outer, box_inner, box_outer, swizzle);
}

bool make_map_3d(CUtensorMap* map, const void* base, bool bf16, uint64_t d0, uint64_t d1,
                 uint64_t d2, uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0,
                 uint32_t box1, uint32_t box2, bool swizzle128) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  cuuint32_t box[3] = {box0, box1, box2};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
            const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t linear_workspace_bytes(bool backward, int64_t M, int64_t N, int64_t K, int r) {
  (void)N;
  (void)K;
  return (backward ? 2 : 1) * mr_bytes(M, r);
}

// Every launch of a call is prepared (its tensor maps encoded) before the
// first is enqueued, so a call that fails on the host enqueues nothing.
cudaError_t launch_linear_fwd(const LinearArgs& a, int sms, cudaStream_t st, int* launches) {
  (void)sms;
  cudaError_t e = cudaSuccess;
  uint8_t* ws = a.ws + kWsHeader;
  __nv_bfloat16* T = a.t_out ? static_cast<__nv_bfloat16*>(a.t_out) : reinterpret_cast<__nv_bfloat16*>(ws);
  if (decode_supported(a.M, a.N, a.K, a.r)) {
    // With r > 32 the A tiles of a K slice would crowd the weight tiles out of
    // shared memory: T comes from the adapter kernel first, and the decode
    // kernel (its programmatic dependent) reads it.
    const bool t_first = a.r > 32;
    e = launch_decode_fwd(a, sms, st, launches, t_first ? T : nullptr, /*dry_run=*/true);
    if (e == cudaSuccess) {
      if (t_first) {
        // a programmatic dependent of the kernel before (a previous decode
        // call's tail overlaps its start), unless the per-kernel brackets are on
        e = launch_decode_t(a, T, st, launches, /*pdl=*/!prof_on());
        if (e != cudaSuccess) return e;
      }
      return launch_decode_fwd(a, sms, st, launches, t_first ? T : nullptr, false);
    }
    if (e != cudaErrorNotSupported) return e;
  }
  e = set_attrs();
  if (e != cudaSuccess) return e;
  AdapterLaunch lt;
  FusedLaunch lf;
  if (!prepare_adapter(job_T(a, T), a.status, &lt) || !prepare_fused(a, kFwd, T, &lf))
    return cudaErrorInvalidValue;
  e = launch_adapter(lt, st, launches);
  if (e != cudaSuccess) return e;
  return launch_fused(lf, st, launches, /*pdl=*/!prof_on());
}

cudaError_t launch_linear_bwd(const LinearArgs& a, int sms, cudaStream_t st, int* launches) {
  (void)sms;
  cudaError_t e = set_attrs();
  if (e != cudaSuccess) return e;
  uint8_t* ws = a.ws + kWsHeader;
  __nv_bfloat16* T_ws = reinterpret_cast<__nv_bfloat16*>(ws);
  __nv_bfloat16* U = reinterpret_cast<__nv_bfloat16*>(ws + mr_bytes(a.M, a.r));
  const bool recompute_t = a.t_in == nullptr;
  const __nv_bfloat16* T = recompute_t ? T_ws : static_cast<const __nv_bfloat16*>(a.t_in);

  AdapterLaunch lt, lu, ldb, lda;
  FusedLaunch ldx;
  bool ok = !recompute_t || prepare_adapter(job_T(a, T_ws), a.status, &lt);
  {  // U = s dy B   (A: dy K-major over n; B: B_lora [N, r] MN-major over n)
    AdapterJob j{};
    j.a = a.dy; j.a_inner = a.N; j.a_outer = a.M; j.a_mn = false;
    j.b = a.B; j.b_inner = a.r; j.b_outer = a.N; j.b_mn = true;
    j.Mo = a.M; j.red = a.N; j.r = a.r; j.kind = 0; j.scale = a.s; j.out_bf16 = U; j.f16 = a.f16;
    j.prof_id = kKAdapterU;
    ok = ok && prepare_adapter(j, a.status, &lu);
  }
  {  // dB = dy^T T   (A: dy^T MN-major over m; B: T [M, r] MN-major over m)
    AdapterJob j{};
    j.a = a.dy; j.a_inner = a.N; j.a_outer = a.M; j.a_mn = true;
    j.b = T; j.b_inner = a.r; j.b_outer = a.M; j.b_mn = true;
    j.Mo = a.N; j.red = a.M; j.r = a.r; j.kind = 1; j.scale = 1.0f; j.out_f32 = a.dB; j.f16 = a.f16;
    j.prof_id = kKAdapterDB;
    ok = ok && prepare_adapter(j, a.status, &ldb);
  }
  {  // dA^T = x^T U  (A: x^T MN-major over m; B: U [M, r] MN-major over m), stored as dA [r, K]
    AdapterJob j{};
    j.a = a.x; j.a_inner = a.K; j.a_outer = a.M; j.a_mn = true;
    j.b = U; j.b_inner = a.r; j.b_outer = a.M; j.b_mn = true;
    j.Mo = a.K; j.red = a.M; j.r = a.r; j.kind = 2; j.scale = 1.0f; j.out_f32 = a.dA; j.f16 = a.f16;
    j.prof_id = kKAdapterDA;
    ok = ok && prepare_adapter(j, a.status, &lda);
  }
  // dx = dy W' + U A
  ok = ok && (a.dx == nullptr || prepare_fused(a, kDx, U, &ldx));
  if (!ok) return cudaErrorInvalidValue;

  if (recompute_t) {
    e = launch_adapter(lt, st, launches);
    if (e != cudaSuccess) return e;
  }
  e = launch_adapter(lu, st, launches);
  if (e != cudaSuccess) return e;
  if (a.dx == nullptr) {
    e = launch_adapter(ldb, st, launches);
    if (e == cudaSuccess) e = launch_adapter(lda, st, launches);
    return e;
  }
  // dx on a high-priority side stream forked after U, dB and dA^T on the
  // caller's stream: the block scheduler gives dx every SM it can use, and the
  // two rank-r products (which dx does not need) run on the SMs its last,
  // partial wave leaves idle.  The caller's stream then waits for dx.
  SideStream* side = nullptr;
  std::unique_lock<std::mutex> lock(g_side_mu);
  if (side_stream(st, &side) != cudaSuccess) {
    lock.unlock();
    e = launch_adapter(ldb, st, launches);
    if (e == cudaSuccess) e = launch_adapter(lda, st, launches);
    if (e == cudaSuccess) e = launch_fused(ldx, st, launches);
    return e;
  }
  e = cudaEventRecord(side->fork, st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(side->stream, side->fork, 0);
  if (e != cudaSuccess) return e;
  const cudaError_t ex = launch_fused(ldx, side->stream, launches);
  e = launch_adapter(ldb, st, launches);
  if (e == cudaSuccess) e = launch_adapter(lda, st, launches);
  // join even after a failed launch, so the caller's stream never runs ahead
  // of work already on the side stream
  cudaError_t ej = cudaEventRecord(side->join, side->stream);
  if (ej == cudaSuccess) ej = cudaStreamWaitEvent(st, side->join, 0);
  if (e == cudaSuccess) e = ex;
  if (e == cudaSuccess) e = ej;
  return e;
}

}  // namespace nf4
