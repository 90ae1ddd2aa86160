// Decode-shape QLoRA forward (M <= 32 tokens): one kernel that streams the
// 4-bit weight once.
//
//   y[m, n] = sum_k W'[n, k] x[m, k] + s sum_j (x A^T)[m, j] B[n, j] (+ bias[n])
//
// (qlora-rs README, QuantizedLinear::forward; "LoRA and QLoRA,
// mathematically", equation 6.3.6 read as a layer.)  With a handful of tokens
// the weight bytes are the whole cost, so the design is about getting every
// byte in flight at once and spending few instructions per element:
//   - a CTA owns 128 W rows and one K slice; all of its code tiles are
//     requested by TMA before anything else happens;
//   - a 4-bit pair becomes two bf16 levels with one shared-memory lookup in a
//     256-entry table replicated per lane (conflict-free); the block scale is
//     applied to each 64-wide block's fp32 partial, not to every element;
//   - the dequantized values never leave registers: they are the A fragments
//     of mma.sync m16n8k16 with x as B (the K order inside each block is
//     permuted identically for both so a thread's fragments are contiguous
//     bytes); x A^T rides along as extra rows from the same x fragments;
//   - the S K-slices of a row tile are one thread-block cluster; partials are
//     summed through distributed shared memory in slice order, and the adapter
//     term, bias and bf16 rounding are applied in that reduction.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kernels.h"
#include "nf4_common.cuh"
#include "tc_common.cuh"

namespace nf4 {
namespace {

using namespace tc;

constexpr int kGvWWarps = 16;                       // 2 per 16-row group (alternate K blocks)
constexpr int kGvAWarps = 4;                        // up to 64 adapter rows of x A^T
constexpr int kGvThreads = (kGvWWarps + kGvAWarps) * 32;
constexpr int kGvRows = 128;                        // W rows per CTA
constexpr int kGvMaxBlocks = 16;                    // 64-wide K blocks per CTA
static_assert(kGvWWarps + kGvAWarps > kGvMaxBlocks, "one issuing warp per K block plus one for B");
constexpr int kGvMaxR = 16 * kGvAWarps;
constexpr int kGvLutBytes = 0;                      // the table is a static array

struct GemvParams {
  int M, N, K, r;
  int kb_per_row;       // K / 64
  int blocks_per_slice;
  int slices;
  int r_pad;            // r rounded up to 16 (rows of the A tiles)
  float s;              // alpha / r
  int double_quant;
  const uint8_t* absmax_q;
  const float* absmax;
  const float* absmax_scale;
  const __nv_bfloat16* B;
  const __nv_bfloat16* bias;
  __nv_bfloat16* y;
  __nv_bfloat16* t_out;
  uint32_t* status;
};

// Shared memory (after 1024-byte alignment), every region 1024-byte aligned:
//   lut    256 entries x 32 lanes x 4 B                  32 KB
//   codes  [block][128 W rows][32 B]                      4 KB per block
//   xs     [block][NP token rows][128 B], 128-byte swizzle
//   as     [block][r_pad adapter rows][128 B], 128-byte swizzle
//   bs     [128 W rows][r] bf16 (this tile's rows of B)
//   scales [128 rows][kGvMaxBlocks] fp32                 8 KB
//   part   [128][NP] fp32, tpart [64][NP] fp32, barriers
struct GemvLayout {
  size_t codes, xs, as, bs, scales, part, tpart, bar, total;
};

__host__ __device__ constexpr size_t align1k(size_t v) { return (v + 1023) & ~size_t(1023); }

__host__ __device__ inline GemvLayout gemv_layout(int bps, int np, int r_pad, int r) {
  GemvLayout L{};
  L.codes = kGvLutBytes;
  L.xs = align1k(L.codes + size_t(bps) * 4096);
  L.as = align1k(L.xs + size_t(bps) * np * 128);
  L.bs = align1k(L.as + size_t(bps) * r_pad * 128);
  L.scales = align1k(L.bs + size_t(kGvRows) * r * 2);
  L.part = L.scales + size_t(kGvRows) * kGvMaxBlocks * 4;
  L.tpart = L.part + size_t(kGvRows) * np * 4;
  L.bar = L.tpart + size_t(kGvMaxR) * np * 4;
  L.total = 1024 + L.bar + 8 * (kGvMaxBlocks + 1);
  return L;
}

template <bool F16>
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  if (F16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

// One 2-byte element of the compute type (f16 or bf16) to and from fp32.
template <bool F16>
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) {
  if (F16) return __half2float(*reinterpret_cast<const __half*>(&v));
  return __bfloat162float(v);
}
template <bool F16>
__device__ __forceinline__ __nv_bfloat16 from_f32(float v) {
  if (F16) {
    const __half h = __float2half_rn(v);
    return *reinterpret_cast<const __nv_bfloat16*>(&h);
  }
  return __float2bfloat16_rn(v);
}

__device__ __forceinline__ float ld_shared_cluster_f32(uint32_t cluster_addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(cluster_addr) : "memory");
  return v;
}

// Byte offset of lane `lane`'s copy of table entry `byte j of word`, for a
// table laid out [256 entries][32 lanes] x 4 B: (byte << 7) | (lane << 2).
__device__ __forceinline__ uint32_t lut_off(uint32_t word, int j, uint32_t lane_off) {
  const uint32_t shifted = j == 0 ? (word << 7) : (word >> (8 * j - 7));
  return (shifted & 0x7f80u) | lane_off;
}

// Elements 16q .. 16q+15 of row `row` of a 128-byte-swizzled [rows][64 bf16]
// tile: 16-byte chunks 2q and 2q+1.
__device__ __forceinline__ void load_row16(const uint8_t* tile, int row, int q, uint4& lo,
                                           uint4& hi) {
  lo = *reinterpret_cast<const uint4*>(tile + sw128_offset(uint32_t(row), uint32_t(2 * q)));
  hi = *reinterpret_cast<const uint4*>(tile + sw128_offset(uint32_t(row), uint32_t(2 * q + 1)));
}

// Fragments of MMA i (0..3) from 16 consecutive values: elements (4i, 4i+1)
// and (4i+2, 4i+3).
__device__ __forceinline__ void frag_pair(const uint4& lo, const uint4& hi, int i, uint32_t& f0,
                                          uint32_t& f1) {
  const uint4& v = i < 2 ? lo : hi;
  if ((i & 1) == 0) {
    f0 = v.x;
    f1 = v.y;
  } else {
    f0 = v.z;
    f1 = v.w;
  }
}

template <int NT8, bool F16>
__global__ void __launch_bounds__(kGvThreads, 1)
    nf4_gemv(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_x,
             const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
             const GemvParams p) {
  constexpr int NP = 8 * NT8;                  // token rows (M padded)
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(1024) uint32_t lut[256 * 32];      // [entry][lane] copies
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const GemvLayout L = gemv_layout(p.blocks_per_slice, NP, p.r_pad, p.r);
  uint8_t* codes = smem + L.codes;
  uint8_t* xs = smem + L.xs;
  uint8_t* as = smem + L.as;
  const __nv_bfloat16* bs = reinterpret_cast<const __nv_bfloat16*>(smem + L.bs);
  float* scales = reinterpret_cast<float*>(smem + L.scales);
  float* part = reinterpret_cast<float*>(smem + L.part);
  float* tpart = reinterpret_cast<float*>(smem + L.tpart);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L.bar);   // [block], then B rows
  __shared__ uint32_t abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;
  const int q = lane & 3;
  const int n0 = blockIdx.x * kGvRows;
  const int slice = blockIdx.y;                // = rank in the (1, S, 1) cluster
  const int kb0 = slice * p.blocks_per_slice;
  const int nblk = max(0, min(p.blocks_per_slice, p.kb_per_row - kb0));
  const uint32_t xbytes = uint32_t(NP) * 128u;
  const uint32_t abytes = uint32_t(p.r_pad) * 128u;

  // Every byte this CTA reads is requested before anything else, one barrier
  // per 64-wide K block so compute starts on the first block to land.  Warp b
  // issues block b's copies (and warp kGvMaxBlocks the B tile): one warp keeps
  // only a few TMA copies going per microsecond, so the issue is spread.
  if (threadIdx.x == 0) abort_flag = 0;
  if (lane == 0 && warp <= kGvMaxBlocks) {
    mbar_init(&bar[warp], 1);
    fence_barrier_init();
    fence_proxy_async_smem();
    if (warp == kGvMaxBlocks) {
      mbar_arrive_expect_tx(&bar[kGvMaxBlocks], uint32_t(kGvRows) * uint32_t(p.r) * 2u);
      tma_load_2d(smem + L.bs, &tm_b, &bar[kGvMaxBlocks], 0, n0);
    } else if (warp < nblk) {
      const int b = warp, kb = kb0 + b;
      mbar_arrive_expect_tx(&bar[b], 4096u + xbytes + abytes);
      tma_load_2d(codes + b * 4096, &tm_codes, &bar[b], kb * 32, n0);
      tma_load_2d(xs + b * xbytes, &tm_x, &bar[b], kb * 64, 0);
      tma_load_2d(as + b * abytes, &tm_a, &bar[b], kb * 64, 0);
    }
  }
  // Block scales: independent loads issued up front (row = t & 127).
  const bool dq = p.double_quant != 0;
  constexpr int kScaleSteps = kGvThreads / kGvRows;          // threads per row
  float sc_reg[(kGvMaxBlocks + kScaleSteps - 1) / kScaleSteps];
  {
    const float s_g = dq ? __ldg(p.absmax_scale) : 0.0f;
    const int row = threadIdx.x & (kGvRows - 1);
    const int64_t wr = int64_t(n0) + row;
#pragma unroll
    for (int j = 0; j < (kGvMaxBlocks + kScaleSteps - 1) / kScaleSteps; ++j) {
      const int b = (threadIdx.x >> 7) + kScaleSteps * j;
      float v = 0.0f;
      if (b < nblk && wr < p.N) {
        const int64_t idx = wr * p.kb_per_row + kb0 + b;
        v = dq ? __fmul_rn(float(__ldg(p.absmax_q + idx)), s_g) : __ldg(p.absmax + idx);
      }
      sc_reg[j] = v;
    }
  }
  // Lookup table: byte (even element in the high nibble) -> bf16x2 of the two
  // unscaled levels, one copy per lane so 32 lanes never share a bank.
  for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) {
    const int e = i >> 5;
    if (F16) {
      const __half2 h = __floats2half2_rn(level(e >> 4), level(e & 15));
      lut[i] = *reinterpret_cast<const uint32_t*>(&h);
    } else {
      const __nv_bfloat162 h = __floats2bfloat162_rn(level(e >> 4), level(e & 15));
      lut[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
  }
  {
    const int row = threadIdx.x & (kGvRows - 1);
#pragma unroll
    for (int j = 0; j < (kGvMaxBlocks + kScaleSteps - 1) / kScaleSteps; ++j) {
      const int b = (threadIdx.x >> 7) + kScaleSteps * j;
      if (b < kGvMaxBlocks) scales[row * kGvMaxBlocks + b] = sc_reg[j];
    }
  }
  __syncthreads();

  float acc[NT8][4];
#pragma unroll
  for (int t = 0; t < NT8; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.0f;
  bool ok = true;

  if (warp < kGvWWarps) {
    // ---- W rows r0 and r0 + 8 of a 16-row group; the two warps of a group
    // take alternate K blocks.
    const int r0 = (warp & 7) * 16 + g;
    const int half = warp >> 3;
    const uint32_t lane_off = uint32_t(lane) << 2;
    const uint8_t* lut_bytes = reinterpret_cast<const uint8_t*>(lut);
    for (int b = half; b < nblk; b += 2) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bar[b], 0, &abort_flag, p.status));
      if (!ok) break;
      const uint8_t* cb = codes + b * 4096;
      const uint2 w0 = *reinterpret_cast<const uint2*>(cb + r0 * 32 + 8 * q);
      const uint2 w1 = *reinterpret_cast<const uint2*>(cb + (r0 + 8) * 32 + 8 * q);
      uint32_t afr[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t wa = i < 2 ? w0.x : w0.y, wb = i < 2 ? w1.x : w1.y;
        const int j = (2 * i) & 3;
        afr[i][0] = *reinterpret_cast<const uint32_t*>(lut_bytes + lut_off(wa, j, lane_off));
        afr[i][1] = *reinterpret_cast<const uint32_t*>(lut_bytes + lut_off(wb, j, lane_off));
        afr[i][2] = *reinterpret_cast<const uint32_t*>(lut_bytes + lut_off(wa, j + 1, lane_off));
        afr[i][3] = *reinterpret_cast<const uint32_t*>(lut_bytes + lut_off(wb, j + 1, lane_off));
      }
      const float s0 = scales[r0 * kGvMaxBlocks + b];
      const float s8 = scales[(r0 + 8) * kGvMaxBlocks + b];
      const uint8_t* xt = xs + b * xbytes;
#pragma unroll
      for (int t = 0; t < NT8; ++t) {
        uint4 xl, xh;
        load_row16(xt, 8 * t + g, q, xl, xh);
        float blk[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint32_t b0, b1;
          frag_pair(xl, xh, i, b0, b1);
          mma_16816<F16>(blk, afr[i], b0, b1);
        }
        acc[t][0] = fmaf(s0, blk[0], acc[t][0]);
        acc[t][1] = fmaf(s0, blk[1], acc[t][1]);
        acc[t][2] = fmaf(s8, blk[2], acc[t][2]);
        acc[t][3] = fmaf(s8, blk[3], acc[t][3]);
      }
    }
  } else {
    // ---- adapter rows j0 + g and j0 + g + 8 of x A^T over this K slice
    const int j0 = (warp - kGvWWarps) * 16;
    if (j0 < p.r) {
      for (int b = 0; b < nblk; ++b) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bar[b], 0, &abort_flag, p.status));
        if (!ok) break;
        const uint8_t* at = as + b * abytes;
        const uint8_t* xt = xs + b * xbytes;
        uint4 al, ah, bl, bh;
        load_row16(at, j0 + g, q, al, ah);
        load_row16(at, j0 + g + 8, q, bl, bh);
        uint32_t afr[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          frag_pair(al, ah, i, afr[i][0], afr[i][2]);
          frag_pair(bl, bh, i, afr[i][1], afr[i][3]);
        }
#pragma unroll
        for (int t = 0; t < NT8; ++t) {
          uint4 xl, xh;
          load_row16(xt, 8 * t + g, q, xl, xh);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t b0, b1;
            frag_pair(xl, xh, i, b0, b1);
            mma_16816<F16>(acc[t], afr[i], b0, b1);
          }
        }
      }
#pragma unroll
      for (int t = 0; t < NT8; ++t) {
        tpart[(j0 + g) * NP + 8 * t + 2 * q] = acc[t][0];
        tpart[(j0 + g) * NP + 8 * t + 2 * q + 1] = acc[t][1];
        tpart[(j0 + g + 8) * NP + 8 * t + 2 * q] = acc[t][2];
        tpart[(j0 + g + 8) * NP + 8 * t + 2 * q + 1] = acc[t][3];
      }
    }
  }
  __syncthreads();

  // The odd-block half of each row group hands its sums to the even half.
  if (warp >= 8 && warp < kGvWWarps) {
    const int r0 = (warp & 7) * 16 + g;
#pragma unroll
    for (int t = 0; t < NT8; ++t) {
      part[r0 * NP + 8 * t + 2 * q] = acc[t][0];
      part[r0 * NP + 8 * t + 2 * q + 1] = acc[t][1];
      part[(r0 + 8) * NP + 8 * t + 2 * q] = acc[t][2];
      part[(r0 + 8) * NP + 8 * t + 2 * q + 1] = acc[t][3];
    }
  }
  __syncthreads();
  if (warp < 8) {
    // This slice's share of the adapter term, s (x A^T)_slice B^T, on the
    // W-row accumulators; then the partial tile goes to shared memory.
    const int r0 = warp * 16 + g;
#pragma unroll
    for (int t = 0; t < NT8; ++t) {
      acc[t][0] += part[r0 * NP + 8 * t + 2 * q];
      acc[t][1] += part[r0 * NP + 8 * t + 2 * q + 1];
      acc[t][2] += part[(r0 + 8) * NP + 8 * t + 2 * q];
      acc[t][3] += part[(r0 + 8) * NP + 8 * t + 2 * q + 1];
    }
    ok = __all_sync(0xffffffffu, mbar_wait(&bar[kGvMaxBlocks], 0, &abort_flag, p.status));
    if (ok) {
      const __nv_bfloat16* b0row = bs + r0 * p.r;
      const __nv_bfloat16* b8row = bs + (r0 + 8) * p.r;
      for (int j = 0; j < p.r; ++j) {
        const float bv0 = p.s * to_f32<F16>(b0row[j]);
        const float bv8 = p.s * to_f32<F16>(b8row[j]);
#pragma unroll
        for (int t = 0; t < NT8; ++t) {
          const float t0 = tpart[j * NP + 8 * t + 2 * q];
          const float t1 = tpart[j * NP + 8 * t + 2 * q + 1];
          acc[t][0] = fmaf(bv0, t0, acc[t][0]);
          acc[t][1] = fmaf(bv0, t1, acc[t][1]);
          acc[t][2] = fmaf(bv8, t0, acc[t][2]);
          acc[t][3] = fmaf(bv8, t1, acc[t][3]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < NT8; ++t) {
      part[r0 * NP + 8 * t + 2 * q] = acc[t][0];
      part[r0 * NP + 8 * t + 2 * q + 1] = acc[t][1];
      part[(r0 + 8) * NP + 8 * t + 2 * q] = acc[t][2];
      part[(r0 + 8) * NP + 8 * t + 2 * q + 1] = acc[t][3];
    }
  }

  cluster_sync();

  if (p.t_out != nullptr && blockIdx.x == 0 && slice == 0) {
    // T = s x A^T for the caller: the slices' adapter partials summed.
    const uint32_t tbase = smem_u32(tpart);
    for (int i = threadIdx.x; i < p.M * p.r; i += blockDim.x) {
      const int m = i / p.r, j = i % p.r;
      const uint32_t off = uint32_t((j * NP + m) * 4);
      float v = 0.0f;
      for (int sl = 0; sl < p.slices; ++sl) v += ld_shared_cluster_f32(mapa_shared(tbase + off, uint32_t(sl)));
      p.t_out[i] = from_f32<F16>(p.s * v);
    }
  }

  // This CTA's band of the 128 rows: the slices' partials summed in slice
  // order, plus bias, rounded to bf16.  Thread = (row, 4 tokens); consecutive
  // threads on consecutive rows so the y stores coalesce.
  const int rows_per = kGvRows / p.slices;
  const uint32_t pbase = smem_u32(part);
  for (int i = threadIdx.x; i < rows_per * (NP / 4); i += blockDim.x) {
    const int rr = i % rows_per, mq = i / rows_per;
    const int trow = slice * rows_per + rr;
    const int n = n0 + trow;
    if (n >= p.N || 4 * mq >= p.M) continue;
    const uint32_t off = uint32_t((trow * NP + 4 * mq) * 4);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int sl = 0; sl < p.slices; ++sl) {
      const float4 w = ld_shared_cluster_f4(mapa_shared(pbase + off, uint32_t(sl)));
      v.x += w.x;
      v.y += w.y;
      v.z += w.z;
      v.w += w.w;
    }
    const float bias = p.bias != nullptr ? to_f32<F16>(p.bias[n]) : 0.0f;
    const float vals[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int m = 4 * mq + e;
      if (m < p.M) p.y[int64_t(m) * p.N + n] = from_f32<F16>(vals[e] + bias);
    }
  }
  cluster_sync();
}

}  // namespace

bool decode_supported(int64_t M, int64_t N, int64_t K, int r) {
  (void)N;
  (void)K;
  return M >= 1 && M <= 32 && r <= kGvMaxR;
}

cudaError_t launch_decode_fwd(const LinearArgs& a, int sms, cudaStream_t st, int* launches) {
  (void)sms;
  const int kb = int(a.K / 64);
  const int tiles = int((a.N + kGvRows - 1) / kGvRows);
  const int nt8 = a.M <= 8 ? 1 : (a.M <= 16 ? 2 : 4);
  const int np = 8 * nt8;
  const int r_pad = (a.r + 15) / 16 * 16;
  // K slices: one wave of one CTA per SM where possible, and everything a CTA
  // reads fits in its shared memory at once.
  int slices = 1;
  while (slices < 8 && tiles * slices * 2 <= 148 && slices * 2 <= kb) slices *= 2;
  int bps = (kb + slices - 1) / slices;
  while ((bps > kGvMaxBlocks || gemv_layout(bps, np, r_pad, a.r).total > 190u * 1024u) && slices < 8) {
    slices *= 2;
    bps = (kb + slices - 1) / slices;
  }
  if (bps > kGvMaxBlocks || gemv_layout(bps, np, r_pad, a.r).total > 190u * 1024u)
    return cudaErrorNotSupported;
  CUtensorMap tc, tx, ta, tb;
  bool ok = make_map_2d(&tc, a.w->codes, false, uint64_t(a.K / 2), uint64_t(a.N), 32, kGvRows, false);
  ok = ok && make_map_2d(&tx, a.x, true, uint64_t(a.K), uint64_t(a.M), 64, uint32_t(np), true);
  ok = ok && make_map_2d(&ta, a.A, true, uint64_t(a.K), uint64_t(a.r), 64, uint32_t(r_pad), true);
  ok = ok && make_map_2d(&tb, a.B, true, uint64_t(a.r), uint64_t(a.N), uint32_t(a.r), kGvRows, false);
  if (!ok) return cudaErrorInvalidValue;
  GemvParams p;
  p.M = int(a.M);
  p.N = int(a.N);
  p.K = int(a.K);
  p.r = a.r;
  p.kb_per_row = kb;
  p.blocks_per_slice = bps;
  p.slices = slices;
  p.r_pad = r_pad;
  p.s = a.s;
  p.double_quant = a.w->double_quant;
  p.absmax_q = a.w->absmax_q;
  p.absmax = a.w->absmax;
  p.absmax_scale = a.w->absmax_scale;
  p.B = static_cast<const __nv_bfloat16*>(a.B);
  p.bias = static_cast<const __nv_bfloat16*>(a.bias);
  p.y = static_cast<__nv_bfloat16*>(a.y);
  p.t_out = static_cast<__nv_bfloat16*>(a.t_out);
  p.status = a.status;

  const size_t smem = gemv_layout(bps, np, r_pad, a.r).total;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(tiles), unsigned(slices), 1);
  cfg.blockDim = dim3(kGvThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = unsigned(slices);
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // The shared-memory opt-in is set once per instantiation (the maximum the
  // decode path can ask for), not on every call.
  auto kernel_for = [](int n8, bool f16) {
    if (f16) return n8 == 1 ? nf4_gemv<1, true> : (n8 == 2 ? nf4_gemv<2, true> : nf4_gemv<4, true>);
    return n8 == 1 ? nf4_gemv<1, false> : (n8 == 2 ? nf4_gemv<2, false> : nf4_gemv<4, false>);
  };
  static PerDeviceOnce attr_done[6];
  const int slot = (nt8 == 1 ? 0 : (nt8 == 2 ? 1 : 2)) + (a.f16 ? 3 : 0);
  auto* kernel = kernel_for(nt8, a.f16 != 0);
  cudaError_t e = cudaSuccess;
  const int dev = PerDeviceOnce::current();
  if (!attr_done[slot].done(dev)) {
    const int max_smem = 190 * 1024;   // + the 32 KB static lookup table
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
    if (e != cudaSuccess) return e;
    attr_done[slot].mark(dev);
  }
  NF4_PROF_BEGIN(st, kKGemv);
  e = cudaLaunchKernelEx(&cfg, kernel, tc, tx, ta, tb, p);
  NF4_PROF_END(st, kKGemv);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e == cudaSuccess) ++*launches;
  return e;
}

}  // namespace nf4
