// Decode-shape QLoRA forward (M <= 32 tokens): one kernel that streams the
// 4-bit weight once.
//
//   y[m, n] = sum_k W'[n, k] x[m, k] + s sum_j (x A^T)[m, j] B[n, j] (+ bias[n])
//
// (qlora-rs README, QuantizedLinear::forward; "LoRA and QLoRA,
// mathematically", equation 6.3.6 read as a layer.)  With a handful of tokens
// the weight bytes are the whole cost, so the design is about keeping every
// byte in flight and the SM busy while they land:
//   - a CTA owns 128 W rows and one K slice.  Its block scales are requested
//     first (plain loads, so they are not queued behind the weight bytes),
//     then every code tile, x tile and A tile of the slice by TMA, one
//     mbarrier per group of four 64-wide K blocks (one 128-byte code box), so
//     compute starts on the first group to land.  The scales sit in shared
//     memory block-major, so the eight rows a warp reads at once use eight
//     banks;
//   - a 4-bit pair becomes two bf16 levels with one shared-memory lookup in a
//     256-entry table replicated per lane (conflict-free); the block scale is
//     applied to each 64-wide block's fp32 partial, not to every element;
//   - the dequantized values never leave registers: they are the A fragments
//     of mma.sync m16n8k16 with x as B (the K order inside each block is
//     permuted identically for both so a thread's fragments are contiguous
//     bytes).  With up to 16 tokens a warp takes one K block at a time for
//     two 16-row groups, so each x fragment it loads serves both;
//   - x A^T (the slice's share of the adapter activation) is computed by four
//     more warps from the same x tiles, split by K block when r is small; its
//     product with the tile's B rows is one more short MMA chain on the W-row
//     accumulators (or T comes finished from a small kernel before, r > 32);
//   - the S K-slices of a row tile are one thread-block cluster.  CTA q owns
//     rows [q 128/S, (q+1) 128/S) of the tile: every CTA pushes its partial
//     for those rows into CTA q's shared memory and arrives on CTA q's
//     mbarrier; CTA q sums the S partials in slice order (deterministic), adds
//     the bias and rounds once.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kernels.h"
#include "nf4_common.cuh"
#include "tc_common.cuh"

namespace nf4 {
namespace {

using namespace tc;

constexpr int kGvWWarps = 16;                       // W-row warps
constexpr int kGvAWarps = 4;                        // up to 64 adapter rows of x A^T
constexpr int kGvWarps = kGvWWarps + kGvAWarps;
constexpr int kGvThreads = kGvWarps * 32;
constexpr int kGvRows = 128;                        // W rows per CTA
constexpr int kGvMaxBlocks = 16;                    // 64-wide K blocks per CTA
constexpr int kGvGroup = 4;                         // K blocks per TMA box: 128 code bytes a row
constexpr int kGvMaxGroups = kGvMaxBlocks / kGvGroup;
static_assert(3 * kGvMaxGroups + 1 <= kGvWarps, "one issuing warp per box");
constexpr int kGvMaxR = 16 * kGvAWarps;
constexpr int kGvMaxSlices = 8;
// 227 KB per CTA at most, less the 32 KB static lookup table (and a little).
constexpr size_t kGvMaxDynSmem = 194u * 1024u;

struct GemvParams {
  int M, N, K, r;
  int kb_per_row;       // K / 64: 64-element chunks per W row
  int bs_shift;         // log2 of the NF4 block size (6 .. 12)
  int blocks_per_slice;
  int vec_scales;       // 16-byte aligned scale rows: vector loads
  int slices;
  int r_pad;            // r rounded up to 16 (rows of the A tiles)
  float s;              // alpha / r
  int double_quant;
  const uint8_t* absmax_q;
  const float* absmax;
  const float* absmax_scale;
  const __nv_bfloat16* bias;
  __nv_bfloat16* y;
  __nv_bfloat16* t_out;
  const __nv_bfloat16* t_in;   // TP == 0: T = s x A^T [M, r] from the kernel before
  uint32_t* status;
};

// Shared memory (after 1024-byte alignment), every region 1024-byte aligned;
// G = ceil(blocks per slice / 4) TMA groups of four K blocks:
//   codes  [G][128 W rows][128 B], 128-byte swizzle (the codes of 4 blocks)
//   xs     [4 G blocks][NP token rows][128 B], 128-byte swizzle
//   as     [4 G blocks][r_pad adapter rows][128 B], 128-byte swizzle
//   bs     [128 W rows][r] bf16 (this tile's rows of B)
//   scales [kGvMaxBlocks][128 rows] fp32                 8 KB (block-major:
//          the eight rows a warp's lanes read at once sit in eight banks)
//   recv   [slice][128 / S rows][NP] fp32: partials pushed by the cluster
//   tpart  [t_parts][r_pad][NP] fp32: this slice's x A^T, in t_parts partial
//          sums over interleaved K blocks
//   red    [block phase - 1][128][NP] fp32: in-CTA partials (over codes and
//          xs once they are consumed, when they are large enough)
//   bars   [G] TMA groups, B tile, recv
struct GemvLayout {
  size_t codes, xs, as, bs, scales, recv, tpart, red, bar, total;
};

__host__ __device__ constexpr size_t align1k(size_t v) { return (v + 1023) & ~size_t(1023); }

__host__ __device__ inline GemvLayout gemv_layout(int bps, int np, int r_pad, int r, int phases,
                                                  int t_parts) {
  const int groups = (bps + kGvGroup - 1) / kGvGroup;
  const int blocks = groups * kGvGroup;
  GemvLayout L{};
  L.codes = 0;
  L.xs = align1k(L.codes + size_t(groups) * kGvRows * 128);
  L.as = align1k(L.xs + size_t(blocks) * np * 128);
  L.bs = align1k(L.as + size_t(blocks) * r_pad * 128);
  L.scales = align1k(L.bs + size_t(kGvRows) * r * 2);
  L.recv = align1k(L.scales + size_t(kGvRows) * kGvMaxBlocks * 4);
  L.tpart = L.recv + size_t(kGvRows) * np * 4;
  size_t end = align1k(L.tpart + size_t(t_parts) * r_pad * np * 4);
  const size_t red_bytes = size_t(phases - 1) * kGvRows * np * 4;
  if (red_bytes <= L.as - L.codes) {
    L.red = L.codes;
  } else {
    L.red = end;
    end = align1k(end + red_bytes);
  }
  L.bar = end;
  L.total = 1024 + L.bar + 8 * (kGvMaxGroups + 2);
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
template <bool F16>
__device__ __forceinline__ uint32_t pack2_rn(float lo, float hi) {
  if (F16) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
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

// The 8 code bytes of K block j (0..3 of its group) that lane quarter q owns,
// in row `row` of a group's [128 rows][128 B] 128-byte-swizzled code box.
__device__ __forceinline__ uint2 load_codes8(const uint8_t* box, uint32_t row, uint32_t j, uint32_t q) {
  const uint32_t chunk = 2u * j + (q >> 1);
  return *reinterpret_cast<const uint2*>(box + row * 128u + ((chunk ^ (row & 7u)) << 4) + ((q & 1u) << 3));
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

// NT8: token columns in groups of 8 (M <= 8 NT8).  RG: 16-row groups per W
// warp (each x fragment a warp loads serves RG groups).
//
// Row mapping: MMA row g (0..7) of a 16-row group is W row 2g of the group and
// MMA row g + 8 is W row 2g + 1.  In a half-warp the four rows a code load
// touches then differ in bits 1..2 of the row, which the 128-byte swizzle
// turns into four different 32-byte bank groups: the loads are conflict-free.
// TP: the x A^T of a slice as TP partial sums over interleaved K blocks (1, 2
// or 4); TP == 0: T = s x A^T comes finished from the kernel before (larger
// r, whose A tiles would not fit beside the weight tiles), read after the
// dependency wait, and slice 0 adds the whole T B^T.
template <int NT8, int RG, bool F16, int TP>
__global__ void __launch_bounds__(kGvThreads, 1)
    nf4_gemv(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_x,
             const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
             const GemvParams p) {
  constexpr int NP = 8 * NT8;                  // token rows (M padded)
  constexpr int kSets = 8 / RG;                // row-group sets = W warps per block phase
  constexpr int kPhases = kGvWWarps / kSets;   // W warps that share one row-group set
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(1024) uint32_t lut[256 * 32];      // [entry][lane] copies
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr bool kTGiven = TP == 0;
  const GemvLayout L = gemv_layout(p.blocks_per_slice, NP, kTGiven ? 0 : p.r_pad, p.r, kPhases, TP);
  uint8_t* codes = smem + L.codes;
  uint8_t* xs = smem + L.xs;
  uint8_t* as = smem + L.as;
  const __nv_bfloat16* bs = reinterpret_cast<const __nv_bfloat16*>(smem + L.bs);
  float* scales = reinterpret_cast<float*>(smem + L.scales);
  float* recv = reinterpret_cast<float*>(smem + L.recv);
  float* tpart = reinterpret_cast<float*>(smem + L.tpart);
  // x A^T partial sums: r_pad / 16 row groups times t_parts K-block parts
  // over the four adapter warps (r_pad / 16 * t_parts <= 4)
  constexpr int t_parts = TP;
  const int t_stride = p.r_pad * NP;
  auto t_sum = [&](int i) {   // the parts of entry i, summed in part order
    float v = tpart[i];
    for (int k = 1; k < t_parts; ++k) v += tpart[k * t_stride + i];
    return v;
  };
  float* red = reinterpret_cast<float*>(smem + L.red);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L.bar);   // [group], B rows, recv
  uint64_t* bar_b = &bar[kGvMaxGroups];
  uint64_t* bar_recv = &bar[kGvMaxGroups + 1];
  __shared__ uint32_t abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;
  const int q = lane & 3;
  const int n0 = blockIdx.x * kGvRows;
  const int slice = blockIdx.y;                // = rank in the (1, S, 1) cluster
  const int S = p.slices;
  const int kb0 = slice * p.blocks_per_slice;
  const int nblk = max(0, min(p.blocks_per_slice, p.kb_per_row - kb0));
  const int groups = (nblk + kGvGroup - 1) / kGvGroup;
  const uint32_t xbytes = uint32_t(NP) * 128u;
  const uint32_t abytes = uint32_t(p.r_pad) * 128u;
  const int band = kGvRows / S;                // rows of the tile this CTA finishes
  const bool pull_t = !kTGiven && p.t_out != nullptr && blockIdx.x == 0;   // uniform over the cluster

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int c = 0; c < kGvMaxGroups; ++c) mbar_init(&bar[c], 3);   // codes, x and A issuers
    mbar_init(bar_b, 1);
    mbar_init(bar_recv, 1);
    fence_barrier_init();
    // every slice pushes its partial of this CTA's band: S x band x NP fp32
    mbar_arrive_expect_tx(bar_recv, uint32_t(kGvRows) * NP * 4u);
    fence_proxy_async_smem();
  } else if (threadIdx.x == 32) {
    tma_prefetch(&tm_codes);
    tma_prefetch(&tm_x);
    tma_prefetch(&tm_a);
    tma_prefetch(&tm_b);
  }
  // Lookup table: byte (even element in the high nibble) -> the two unscaled
  // levels in the compute type, one copy per lane so 32 lanes never share a
  // bank.  A warp writes the 32 copies of one entry at a time; lane c holds
  // level c (mod 16) and the entry's two levels come by shuffle.  It reads no
  // input, so it runs before the wait on the previous kernel.
  {
    uint32_t my = 0;
#pragma unroll
    for (int c = 0; c < 16; ++c) my = (lane & 15) == c ? level_bits(c) : my;
    const float lv = __uint_as_float(my);
    for (int e = warp; e < 256; e += kGvWarps) {
      const float hi = __shfl_sync(0xffffffffu, lv, e >> 4);
      const float lo = __shfl_sync(0xffffffffu, lv, e & 15);
      lut[e * 32 + lane] = pack2_rn<F16>(hi, lo);
    }
  }
  __syncthreads();
  // This CTA's barriers are initialized: the cluster may push to it once every
  // CTA has arrived here (the matching wait comes before the first push).
  cluster_arrive();
  // Programmatic dependent launch: the next kernel on the stream may start its
  // own set-up now; this one reads no input and writes no output before the
  // previous kernel has completed and its writes are visible.
  asm volatile("griddepcontrol.launch_dependents;");
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // Block scales: raw loads, converted after the TMA copies are out.  A row's
  // 16 u8 scales (or 16 fp32) are one or four 16-byte loads when aligned.
  const bool dq = p.double_quant != 0;
  const float s_g = dq ? __ldg(p.absmax_scale) : 0.0f;
  const int srow = threadIdx.x & (kGvRows - 1);
  const int64_t swr = int64_t(n0) + srow;
  const int64_t sidx0 = swr * p.kb_per_row + kb0;
  const bool svec = nblk == kGvMaxBlocks && swr < p.N && p.vec_scales;
  uint4 sv = make_uint4(0u, 0u, 0u, 0u);
  if (svec && dq) {
    if (threadIdx.x < kGvRows) sv = __ldg(reinterpret_cast<const uint4*>(p.absmax_q + sidx0));
  } else if (svec) {
    if (threadIdx.x < 4 * kGvRows)
      sv = __ldg(reinterpret_cast<const uint4*>(p.absmax + sidx0) + (threadIdx.x >> 7));
  }
  constexpr int kScaleSteps = kGvThreads / kGvRows;          // threads per row
  constexpr int kScaleRegs = (kGvMaxBlocks + kScaleSteps - 1) / kScaleSteps;
  uint32_t sc_raw[kScaleRegs];
  if (!svec) {
#pragma unroll
    for (int j = 0; j < kScaleRegs; ++j) {
      const int b = (threadIdx.x >> 7) + kScaleSteps * j;
      uint32_t v = 0;
      if (b < nblk && swr < p.N) {
        const int64_t si = chunk_block(swr, p.K, kb0 + b, p.bs_shift);
        v = dq ? uint32_t(__ldg(p.absmax_q + si)) : __float_as_uint(__ldg(p.absmax + si));
      }
      sc_raw[j] = v;
    }
  }

  // Every byte this CTA reads is requested now: per group of four K blocks one
  // code box (128 rows x 128 B), one x box and one A box, each issued by its
  // own warp (one warp keeps only a few TMA copies going per microsecond), all
  // three completing on the group's barrier; the last warp loads the B rows.
  if (lane == 0) {
    if (warp < 3 * groups) {
      const int grp = warp / 3, part = warp % 3, b = grp * kGvGroup, kb = kb0 + b;
      if (part == 0) {
        mbar_arrive_expect_tx(&bar[grp], uint32_t(kGvRows) * 128u);
        tma_load_2d(codes + grp * (kGvRows * 128), &tm_codes, &bar[grp], kb * 32, n0);
      } else if (part == 1) {
        mbar_arrive_expect_tx(&bar[grp], xbytes * kGvGroup);
        tma_load_3d(xs + b * xbytes, &tm_x, &bar[grp], 0, 0, kb);
      } else if (kTGiven) {
        mbar_arrive(&bar[grp]);   // no A tiles: T comes finished
      } else {
        mbar_arrive_expect_tx(&bar[grp], abytes * kGvGroup);
        tma_load_3d(as + b * abytes, &tm_a, &bar[grp], 0, 0, kb);
      }
    } else if (warp == kGvWarps - 1) {
      mbar_arrive_expect_tx(bar_b, uint32_t(kGvRows) * uint32_t(p.r) * 2u);
      tma_load_2d(smem + L.bs, &tm_b, bar_b, 0, n0);
    }
  }

  {
    float* srow_dst = scales + srow;   // block b of this row at srow_dst[b * kGvRows]
    if (svec && dq) {
      if (threadIdx.x < kGvRows) {
        const uint32_t w[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
        for (int b = 0; b < 16; ++b)
          srow_dst[b * kGvRows] = __fmul_rn(float((w[b >> 2] >> (8 * (b & 3))) & 0xffu), s_g);
      }
    } else if (svec) {
      if (threadIdx.x < 4 * kGvRows) {
        const int b0 = 4 * (threadIdx.x >> 7);
        srow_dst[(b0 + 0) * kGvRows] = __uint_as_float(sv.x);
        srow_dst[(b0 + 1) * kGvRows] = __uint_as_float(sv.y);
        srow_dst[(b0 + 2) * kGvRows] = __uint_as_float(sv.z);
        srow_dst[(b0 + 3) * kGvRows] = __uint_as_float(sv.w);
      }
    } else {
#pragma unroll
      for (int j = 0; j < kScaleRegs; ++j) {
        const int b = (threadIdx.x >> 7) + kScaleSteps * j;
        const float v = dq ? __fmul_rn(float(sc_raw[j]), s_g) : __uint_as_float(sc_raw[j]);
        if (b < kGvMaxBlocks) srow_dst[b * kGvRows] = v;
      }
    }
  }
  __syncthreads();

  float acc[RG][NT8][4];
#pragma unroll
  for (int i = 0; i < RG; ++i)
#pragma unroll
    for (int t = 0; t < NT8; ++t) acc[i][t][0] = acc[i][t][1] = acc[i][t][2] = acc[i][t][3] = 0.0f;
  bool ok = true;
  const int set = warp % kSets;                // W warps: row groups set*RG .. +RG-1
  const int phase = warp / kSets;              //          K blocks phase, phase + kPhases, ...

  if (warp < kGvWWarps) {
    const uint32_t lane_off = uint32_t(lane) << 2;
    const uint8_t* lut_bytes = reinterpret_cast<const uint8_t*>(lut);
    for (int b = phase; b < nblk; b += kPhases) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bar[b / kGvGroup], 0, &abort_flag, p.status));
      if (!ok) break;
      const uint8_t* cb = codes + (b / kGvGroup) * (kGvRows * 128);
      const uint8_t* xt = xs + b * xbytes;
      uint4 xl[NT8], xh[NT8];
#pragma unroll
      for (int t = 0; t < NT8; ++t) load_row16(xt, 8 * t + g, q, xl[t], xh[t]);
#pragma unroll
      for (int i = 0; i < RG; ++i) {
        const int wr0 = (set * RG + i) * 16 + 2 * g;      // W rows wr0 (MMA row g), wr0 + 1 (g + 8)
        const uint2 w0 = load_codes8(cb, uint32_t(wr0), uint32_t(b % kGvGroup), uint32_t(q));
        const uint2 w1 = load_codes8(cb, uint32_t(wr0 + 1), uint32_t(b % kGvGroup), uint32_t(q));
        uint32_t afr[4][4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t wa = k < 2 ? w0.x : w0.y, wb = k < 2 ? w1.x : w1.y;
          const int j = (2 * k) & 3;
          afr[k][0] = *reinterpret_cast<const uint32_t*>(lut_bytes + lut_off(wa, j, lane_off));
          afr[k][1] = *reinterpret_cast<const uint32_t*>(lut_bytes + lut_off(wb, j, lane_off));
          afr[k][2] = *reinterpret_cast<const uint32_t*>(lut_bytes + lut_off(wa, j + 1, lane_off));
          afr[k][3] = *reinterpret_cast<const uint32_t*>(lut_bytes + lut_off(wb, j + 1, lane_off));
        }
        const float s0 = scales[b * kGvRows + wr0];
        const float s1 = scales[b * kGvRows + wr0 + 1];
#pragma unroll
        for (int t = 0; t < NT8; ++t) {
          float blk[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint32_t b0, b1;
            frag_pair(xl[t], xh[t], k, b0, b1);
            mma_16816<F16>(blk, afr[k], b0, b1);
          }
          acc[i][t][0] = fmaf(s0, blk[0], acc[i][t][0]);
          acc[i][t][1] = fmaf(s0, blk[1], acc[i][t][1]);
          acc[i][t][2] = fmaf(s1, blk[2], acc[i][t][2]);
          acc[i][t][3] = fmaf(s1, blk[3], acc[i][t][3]);
        }
      }
    }
  } else {
    // ---- adapter rows j0 + g and j0 + g + 8 of x A^T over the K blocks
    // part, part + parts, ... of this slice: the four adapter warps split the
    // r_pad / 16 row groups and, when there are fewer than four, the K
    // blocks, so no single warp walks every block alone.
    const int aw = warp - kGvWWarps;
    const int j0 = kTGiven ? p.r_pad : (aw / (kTGiven ? 1 : t_parts)) * 16;
    const int part = aw % (kTGiven ? 1 : t_parts);
    if (!kTGiven && j0 < p.r_pad) {
      float ta[NT8][4];
#pragma unroll
      for (int t = 0; t < NT8; ++t) ta[t][0] = ta[t][1] = ta[t][2] = ta[t][3] = 0.0f;
      for (int b = part; b < nblk; b += t_parts) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bar[b / kGvGroup], 0, &abort_flag, p.status));
        if (!ok) break;
        const uint8_t* at = as + b * abytes;
        const uint8_t* xt = xs + b * xbytes;
        uint4 al, ah, bl, bh;
        load_row16(at, j0 + g, q, al, ah);
        load_row16(at, j0 + g + 8, q, bl, bh);
        uint32_t afr[4][4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          frag_pair(al, ah, k, afr[k][0], afr[k][2]);
          frag_pair(bl, bh, k, afr[k][1], afr[k][3]);
        }
#pragma unroll
        for (int t = 0; t < NT8; ++t) {
          uint4 xl, xh;
          load_row16(xt, 8 * t + g, q, xl, xh);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint32_t b0, b1;
            frag_pair(xl, xh, k, b0, b1);
            mma_16816<F16>(ta[t], afr[k], b0, b1);
          }
        }
      }
      float* tp = tpart + part * t_stride;
#pragma unroll
      for (int t = 0; t < NT8; ++t) {
        tp[(j0 + g) * NP + 8 * t + 2 * q] = ta[t][0];
        tp[(j0 + g) * NP + 8 * t + 2 * q + 1] = ta[t][1];
        tp[(j0 + g + 8) * NP + 8 * t + 2 * q] = ta[t][2];
        tp[(j0 + g + 8) * NP + 8 * t + 2 * q + 1] = ta[t][3];
      }
    }
  }
  __syncthreads();    // every K block consumed; tpart complete

  // The block phases of each row-group set meet in phase 0.
  if (warp < kGvWWarps && phase > 0) {
    float* dst = red + size_t(phase - 1) * kGvRows * NP;
#pragma unroll
    for (int i = 0; i < RG; ++i) {
      const int wr0 = (set * RG + i) * 16 + 2 * g;
#pragma unroll
      for (int t = 0; t < NT8; ++t) {
        *reinterpret_cast<float2*>(dst + wr0 * NP + 8 * t + 2 * q) = make_float2(acc[i][t][0], acc[i][t][1]);
        *reinterpret_cast<float2*>(dst + (wr0 + 1) * NP + 8 * t + 2 * q) = make_float2(acc[i][t][2], acc[i][t][3]);
      }
    }
  }
  __syncthreads();
  cluster_wait();     // every CTA of the cluster has initialized its barriers

  if (warp < kGvWWarps && phase == 0) {
#pragma unroll
    for (int ph = 1; ph < kPhases; ++ph) {
      const float* src = red + size_t(ph - 1) * kGvRows * NP;
#pragma unroll
      for (int i = 0; i < RG; ++i) {
        const int wr0 = (set * RG + i) * 16 + 2 * g;
#pragma unroll
        for (int t = 0; t < NT8; ++t) {
          const float2 u = *reinterpret_cast<const float2*>(src + wr0 * NP + 8 * t + 2 * q);
          const float2 v = *reinterpret_cast<const float2*>(src + (wr0 + 1) * NP + 8 * t + 2 * q);
          acc[i][t][0] += u.x;
          acc[i][t][1] += u.y;
          acc[i][t][2] += v.x;
          acc[i][t][3] += v.y;
        }
      }
    }
    // This slice's share of the adapter term, (s T_slice) B^T, as MMAs with
    // the tile's B rows (bf16 in shared memory) as A and s T_slice rounded to
    // the compute type as B.
    ok = __all_sync(0xffffffffu, ok && mbar_wait(bar_b, 0, &abort_flag, p.status));
    if (ok && (!kTGiven || slice == 0)) {
      for (int j0 = 0; j0 < p.r_pad; j0 += 16) {
        uint32_t tfr[NT8][2];
#pragma unroll
        for (int t = 0; t < NT8; ++t) {
          const int m = 8 * t + g;
          const int ja = j0 + 2 * q, jb = j0 + 2 * q + 8;
          if (kTGiven) {
            // two consecutive adapter columns of token m (r is a multiple of 8)
            const uint32_t* trow = reinterpret_cast<const uint32_t*>(p.t_in + int64_t(m) * p.r);
            tfr[t][0] = (m < p.M && ja < p.r) ? __ldg(trow + (ja >> 1)) : 0u;
            tfr[t][1] = (m < p.M && jb < p.r) ? __ldg(trow + (jb >> 1)) : 0u;
          } else {
            tfr[t][0] = pack2_rn<F16>(p.s * t_sum(ja * NP + m), p.s * t_sum((ja + 1) * NP + m));
            tfr[t][1] = pack2_rn<F16>(p.s * t_sum(jb * NP + m), p.s * t_sum((jb + 1) * NP + m));
          }
        }
        // B columns j >= r hold no adapter: masked to 0 (tpart rows r .. r_pad-1
        // are 0 too, from the zero-filled A rows)
        const bool lo_ok = j0 + 2 * q < p.r, hi_ok = j0 + 2 * q + 8 < p.r;
#pragma unroll
        for (int i = 0; i < RG; ++i) {
          const int wr0 = (set * RG + i) * 16 + 2 * g;
          const uint32_t* b0row = reinterpret_cast<const uint32_t*>(bs + wr0 * p.r);
          const uint32_t* b1row = reinterpret_cast<const uint32_t*>(bs + (wr0 + 1) * p.r);
          uint32_t afr[4];
          afr[0] = lo_ok ? b0row[(j0 >> 1) + q] : 0u;
          afr[1] = lo_ok ? b1row[(j0 >> 1) + q] : 0u;
          afr[2] = hi_ok ? b0row[(j0 >> 1) + q + 4] : 0u;
          afr[3] = hi_ok ? b1row[(j0 >> 1) + q + 4] : 0u;
#pragma unroll
          for (int t = 0; t < NT8; ++t) mma_16816<F16>(acc[i][t], afr, tfr[t][0], tfr[t][1]);
        }
      }
    }
    // Push each row's partial to the CTA that owns its band of the tile; the
    // bytes complete on that CTA's receive barrier.
#pragma unroll
    for (int i = 0; i < RG; ++i) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = (set * RG + i) * 16 + 2 * g + h;
        const int owner = row / band;
        const uint32_t dst = mapa_shared(
            smem_u32(recv + (size_t(slice) * band + (row - owner * band)) * NP), uint32_t(owner));
        const uint32_t obar = mapa_shared(smem_u32(bar_recv), uint32_t(owner));
#pragma unroll
        for (int t = 0; t < NT8; ++t)
          st_async_f2(dst + uint32_t(8 * t + 2 * q) * 4u, acc[i][t][2 * h], acc[i][t][2 * h + 1], obar);
      }
    }
  }

  // This CTA's band: the slices' partials summed in slice order, plus bias,
  // rounded once.  Thread = (row, token); consecutive threads on consecutive
  // rows so the y stores coalesce.
  const bool got = mbar_wait_cluster(bar_recv, 0, &abort_flag, p.status);
  if (got) {
    for (int i = threadIdx.x; i < band * p.M; i += blockDim.x) {
      const int rr = i % band, m = i / band;
      const int n = n0 + slice * band + rr;
      if (n >= p.N) continue;
      float v = 0.0f;
      for (int sl = 0; sl < S; ++sl) v += recv[(size_t(sl) * band + rr) * NP + m];
      if (p.bias != nullptr) v += to_f32<F16>(p.bias[n]);
      p.y[int64_t(m) * p.N + n] = from_f32<F16>(v);
    }
  }
  if (pull_t) {
    // T = s x A^T for the caller: the slices' adapter partials summed in slice
    // order by slice 0, between two cluster barriers (the first publishes every
    // CTA's tpart, the second keeps it alive until it has been read).
    cluster_sync();
    if (slice == 0) {
      const uint32_t tbase = smem_u32(tpart);
      for (int i = threadIdx.x; i < p.M * p.r; i += blockDim.x) {
        const int m = i / p.r, j = i % p.r;
        const uint32_t off = uint32_t((j * NP + m) * 4);
        float v = 0.0f;
        for (int sl = 0; sl < S; ++sl) {
          float vs = ld_shared_cluster_f32(mapa_shared(tbase + off, uint32_t(sl)));
          for (int k = 1; k < t_parts; ++k)
            vs += ld_shared_cluster_f32(mapa_shared(tbase + off + uint32_t(k * t_stride * 4), uint32_t(sl)));
          v += vs;
        }
        p.t_out[i] = from_f32<F16>(p.s * v);
      }
    }
    cluster_sync();
  }
}

// T = s x A^T for a decode call (M <= 32 tokens, r <= 64) when the decode
// kernel takes T finished: one CTA per adapter row j and group of up to 8
// tokens, each thread a strided share of the K range for every token, fp32
// products and sums (fixed order: the thread's own K share, then a shuffle
// tree, then the warps in order), rounded once to the compute type.
// Launched as a programmatic dependent: x may be the previous kernel's output.
constexpr int kDtThreads = 256;
constexpr int kDtTokens = 8;
template <bool F16>
__global__ void __launch_bounds__(kDtThreads) decode_t_kernel(
    const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ A, int M, int K, int r,
    float s, __nv_bfloat16* __restrict__ T) {
  constexpr int MT = kDtTokens;
  asm volatile("griddepcontrol.launch_dependents;");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int j = blockIdx.x;
  const int m0 = blockIdx.y * MT;
  x += int64_t(m0) * K;
  T += int64_t(m0) * r;
  M = min(MT, M - m0);
  float acc[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
  const uint4* arow = reinterpret_cast<const uint4*>(A + int64_t(j) * K);
  for (int k8 = threadIdx.x; k8 < K / 8; k8 += kDtThreads) {
    const uint4 av = __ldg(arow + k8);
    const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
    float af[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&aw[e]);
      af[2 * e] = to_f32<F16>(h[0]);
      af[2 * e + 1] = to_f32<F16>(h[1]);
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m >= M) break;
      const uint4 xv = __ldg(reinterpret_cast<const uint4*>(x + int64_t(m) * K) + k8);
      const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&xw[e]);
        acc[m] = fmaf(to_f32<F16>(h[0]), af[2 * e], acc[m]);
        acc[m] = fmaf(to_f32<F16>(h[1]), af[2 * e + 1], acc[m]);
      }
    }
  }
  __shared__ float part[kDtThreads / 32][MT];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    if (m >= M) break;
    float v = acc[m];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) part[warp][m] = v;
  }
  __syncthreads();
  if (threadIdx.x < M) {
    float v = 0.0f;
#pragma unroll
    for (int w = 0; w < kDtThreads / 32; ++w) v += part[w][threadIdx.x];
    T[int64_t(threadIdx.x) * r + j] = from_f32<F16>(s * v);
  }
}

}  // namespace

bool decode_supported(int64_t M, int64_t N, int64_t K, int r) {
  (void)N;
  (void)K;
  return M >= 1 && M <= 32 && r <= kGvMaxR;
}

cudaError_t launch_decode_t(const LinearArgs& a, void* T, cudaStream_t st, int* launches, bool pdl) {
  if (a.M < 1 || a.M > 32 || a.r < 1 || a.K % 8 != 0) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(a.r), unsigned((a.M + kDtTokens - 1) / kDtTokens), 1);
  cfg.blockDim = dim3(kDtThreads, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  const auto* x = static_cast<const __nv_bfloat16*>(a.x);
  const auto* A = static_cast<const __nv_bfloat16*>(a.A);
  auto* t = static_cast<__nv_bfloat16*>(T);
  const int M = int(a.M), K = int(a.K), r = a.r;
  NF4_PROF_BEGIN(st, kKAdapterT);
  cudaError_t e;
  e = a.f16 ? cudaLaunchKernelEx(&cfg, decode_t_kernel<true>, x, A, M, K, r, a.s, t)
            : cudaLaunchKernelEx(&cfg, decode_t_kernel<false>, x, A, M, K, r, a.s, t);
  NF4_PROF_END(st, kKAdapterT);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e == cudaSuccess) ++*launches;
  return e;
}

cudaError_t launch_decode_fwd(const LinearArgs& a, int sms, cudaStream_t st, int* launches,
                              const void* t_given, bool dry_run) {
  (void)sms;
  const int kb = int(a.K / 64);
  const int tiles = int((a.N + kGvRows - 1) / kGvRows);
  const int nt8 = a.M <= 8 ? 1 : (a.M <= 16 ? 2 : 4);
  const int rg = nt8 == 4 ? 1 : 2;             // 16-row groups per W warp
  const int phases = kGvWWarps / (8 / rg);
  const int np = 8 * nt8;
  const int r_pad = (a.r + 15) / 16 * 16;
  // With one or two adapter row groups, the x A^T of a slice is split over the
  // four adapter warps by K block as well, so it finishes with the weight rows
  // (with 17..32 tokens into two parts only: four would not leave room for the
  // weight tiles).
  const int t_groups = r_pad / 16;
  const int t_parts = t_given != nullptr ? 0
                      : (t_groups > 2 ? 1 : (nt8 <= 2 ? 4 / t_groups : (t_groups == 1 ? 2 : 1)));
  const int lay_r = t_given != nullptr ? 0 : r_pad;   // A tile rows held in shared memory
  // K slices: one wave of one CTA per SM where possible, and everything a CTA
  // reads fits in its shared memory at once.
  int slices = 1;
  while (slices < kGvMaxSlices && tiles * slices * 2 <= 148 && slices * 2 <= kb) slices *= 2;
  int bps = (kb + slices - 1) / slices;
  auto fits = [&](int b) {
    return b <= kGvMaxBlocks && gemv_layout(b, np, lay_r, a.r, phases, t_parts).total <= kGvMaxDynSmem;
  };
  while (!fits(bps) && slices < kGvMaxSlices) {
    slices *= 2;
    bps = (kb + slices - 1) / slices;
  }
  if (!fits(bps)) return cudaErrorNotSupported;
  CUtensorMap tc, tx, ta, tb;
  // codes: 128 W rows x 128 code bytes (four K blocks) per box, 128-byte swizzle;
  // x and A: [64 elements][rows][K blocks] boxes of four K blocks
  bool ok = make_map_2d(&tc, a.w->codes, false, uint64_t(a.K / 2), uint64_t(a.N), 128, kGvRows, true);
  ok = ok && make_map_3d(&tx, a.x, true, 64, uint64_t(a.M), uint64_t(kb), uint64_t(a.K) * 2, 128, 64,
                         uint32_t(np), kGvGroup, true);
  ok = ok && make_map_3d(&ta, a.A, true, 64, uint64_t(a.r), uint64_t(kb), uint64_t(a.K) * 2, 128, 64,
                         uint32_t(r_pad), kGvGroup, true);
  ok = ok && make_map_2d(&tb, a.B, true, uint64_t(a.r), uint64_t(a.N), uint32_t(a.r), kGvRows, false);
  if (!ok) return cudaErrorInvalidValue;
  GemvParams p;
  p.M = int(a.M);
  p.N = int(a.N);
  p.K = int(a.K);
  p.r = a.r;
  p.kb_per_row = kb;
  p.bs_shift = log2_block(a.w->block_size);
  p.blocks_per_slice = bps;
  // a row's 16 scales of a slice start on a 16-byte boundary (u8) or a
  // 16-byte boundary of fp32 (four vectors) for every row and slice
  p.vec_scales = bps == kGvMaxBlocks && a.w->block_size == 64 &&
                 (a.w->double_quant ? (kb % 16 == 0 && (reinterpret_cast<uintptr_t>(a.w->absmax_q) & 15u) == 0)
                                    : (kb % 4 == 0 && (reinterpret_cast<uintptr_t>(a.w->absmax) & 15u) == 0));
  p.slices = slices;
  p.r_pad = r_pad;
  p.s = a.s;
  p.double_quant = a.w->double_quant;
  p.absmax_q = a.w->absmax_q;
  p.absmax = a.w->absmax;
  p.absmax_scale = a.w->absmax_scale;
  p.bias = static_cast<const __nv_bfloat16*>(a.bias);
  p.y = static_cast<__nv_bfloat16*>(a.y);
  p.t_out = static_cast<__nv_bfloat16*>(a.t_out);
  p.t_in = static_cast<const __nv_bfloat16*>(t_given);
  p.status = a.status;

  const size_t smem = gemv_layout(bps, np, lay_r, a.r, phases, t_parts).total;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(tiles), unsigned(slices), 1);
  cfg.blockDim = dim3(kGvThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = unsigned(slices);
  attr[0].val.clusterDim.z = 1;
  // The kernel reads its inputs only after griddepcontrol.wait, so it may be
  // launched while the previous kernel on the stream is still running.
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  // The shared-memory opt-in is set once per instantiation (the maximum the
  // decode path can ask for), not on every call.
  auto kernel_for = [](int n8, bool f16, int tp) {
    if (f16) {
      if (n8 == 1)
        return tp == 4 ? nf4_gemv<1, 2, true, 4>
                       : (tp == 2 ? nf4_gemv<1, 2, true, 2> : (tp == 1 ? nf4_gemv<1, 2, true, 1> : nf4_gemv<1, 2, true, 0>));
      if (n8 == 2)
        return tp == 4 ? nf4_gemv<2, 2, true, 4>
                       : (tp == 2 ? nf4_gemv<2, 2, true, 2> : (tp == 1 ? nf4_gemv<2, 2, true, 1> : nf4_gemv<2, 2, true, 0>));
      return tp == 2 ? nf4_gemv<4, 1, true, 2> : (tp == 1 ? nf4_gemv<4, 1, true, 1> : nf4_gemv<4, 1, true, 0>);
    }
    if (n8 == 1)
      return tp == 4 ? nf4_gemv<1, 2, false, 4>
                     : (tp == 2 ? nf4_gemv<1, 2, false, 2> : (tp == 1 ? nf4_gemv<1, 2, false, 1> : nf4_gemv<1, 2, false, 0>));
    if (n8 == 2)
      return tp == 4 ? nf4_gemv<2, 2, false, 4>
                     : (tp == 2 ? nf4_gemv<2, 2, false, 2> : (tp == 1 ? nf4_gemv<2, 2, false, 1> : nf4_gemv<2, 2, false, 0>));
    return tp == 2 ? nf4_gemv<4, 1, false, 2> : (tp == 1 ? nf4_gemv<4, 1, false, 1> : nf4_gemv<4, 1, false, 0>);
  };
  // one slot per instantiation: (tokens, parts) in {8, 16, 32} x {4, 2, 1, T given}
  // (32 tokens: 4 parts unused), times the dtype
  static PerDeviceOnce attr_done[24];
  const int part_kind = t_parts == 4 ? 0 : (t_parts == 2 ? 1 : (t_parts == 1 ? 2 : 3));
  const int kind = (nt8 == 1 ? 0 : (nt8 == 2 ? 4 : 8)) + part_kind;
  const int slot = kind + (a.f16 ? 12 : 0);
  auto* kernel = kernel_for(nt8, a.f16 != 0, t_parts);
  if (dry_run) return cudaSuccess;
  cudaError_t e = cudaSuccess;
  const int dev = PerDeviceOnce::current();
  if (!attr_done[slot].done(dev)) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kGvMaxDynSmem));
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
