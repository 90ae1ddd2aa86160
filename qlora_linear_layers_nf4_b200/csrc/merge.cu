// Merge of a quantized base with its low-rank adapter, written dense:
//
//   W_merged[n, k] = w'[n, k] + s (B A)[n, k],   s = alpha / r
//
// (qlora-rs src/export.rs, merge_and_export_gguf: W_merged = W_base +
// (B @ A) * scale; "LoRA and QLoRA, mathematically", "The merge math",
// equation 6.3.6.)  w' is the fp32 dequant L[code] * scale; the sum is taken
// in fp32 with one rounding (an FMA of s and the fp32 B A accumulator onto
// w') and then rounded to the output type.
//
// One CTA per 128 x 256 output tile.  B A is a rank-r contraction, so it runs
// on the tensor cores: the tile's B rows (K-major, r contiguous) and A columns
// (MN-major straight from A's [r, K] storage) come by TMA, one tcgen05 MMA
// chain accumulates the 128 x 256 fp32 product in TMEM, and eight epilogue
// warps read it back, dequantize the matching NF4 codes (read once from HBM,
// fetched while the MMAs run), stage each warp's 32 x 32 piece of the merged
// tile in swizzled shared memory and write it with a TMA tensor store, so
// every HBM write is a whole line and no warp waits on another.  The kernel is bound by the output and code bytes;
// the contraction is a small fraction of its time.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kernels.h"
#include "nf4_common.cuh"
#include "tc_common.cuh"

namespace nf4 {
namespace {

using namespace tc;

constexpr int kMgRows = 128;                 // output rows (W rows) per CTA
constexpr int kMgCols = 256;                 // output columns (K) per CTA (TMEM columns)
constexpr int kMgEpiWarps = kMgCols / 32;    // 128 columns per epilogue thread
constexpr int kMgThreads = 64 + 32 * kMgEpiWarps;
constexpr int kMgCtasPerSm = 512 / kMgCols;  // as many as the TMEM columns allow
// Output staging, after the MMAs are done, over the operand buffers: per
// epilogue warp two 32 x 32 buffers (4 KB each, sized for fp32 rows).
constexpr uint32_t kMgStageBytes = 4096;
constexpr uint32_t kMgStagingBytes = kMgEpiWarps * 2 * kMgStageBytes;
constexpr int kMgMaxChunks = 4;              // r <= 256 in 64-wide chunks
constexpr uint32_t kMgBBytes = kMgRows * 128;            // B rows x 64 r (bf16)
constexpr uint32_t kMgABytes = (kMgCols / 64) * 64 * 128; // 64 r x kMgCols k (bf16)
constexpr uint32_t kMgChunkBytes = kMgBBytes + kMgABytes;

struct MergeParams {
  int N, K, r, chunks, bs_shift;
  float s;
  int double_quant;
  int out_kind;        // kMergeBf16, kMergeF32 or kMergeF16
  const uint8_t* codes;
  const uint8_t* absmax_q;
  const float* absmax;
  const float* absmax_scale;
  void* out;
  uint32_t* status;
};

struct MergeShared {
  uint64_t full[kMgMaxChunks];
  uint64_t accum;
  uint32_t tmem_base;
  uint32_t abort_flag;
  float lut[16 * 32];                        // [level][lane] copies: conflict-free lookups
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
// Two merged values as one 32-bit word of the 2-byte output type.
__device__ __forceinline__ uint32_t pack_out2(bool f16, float lo, float hi) {
  return f16 ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi);
}

// Bytes of the operand region: every r chunk, and at least the output staging.
__host__ __device__ constexpr uint32_t merge_region_bytes(int chunks) {
  return uint32_t(chunks) * kMgChunkBytes > kMgStagingBytes ? uint32_t(chunks) * kMgChunkBytes
                                                            : kMgStagingBytes;
}

__global__ void __launch_bounds__(kMgThreads, kMgCtasPerSm)
    nf4_merge_kernel(const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_a,
                     const __grid_constant__ CUtensorMap tm_out, const MergeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  MergeShared* sh = reinterpret_cast<MergeShared*>(smem + merge_region_bytes(p.chunks));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.y * kMgRows;
  const int k0 = blockIdx.x * kMgCols;
  volatile uint32_t* abort_flag = &sh->abort_flag;

  if (threadIdx.x == 0) {
    for (int j = 0; j < kMgMaxChunks; ++j) mbar_init(&sh->full[j], 1);
    mbar_init(&sh->accum, 1);
    sh->abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  for (int i = threadIdx.x; i < 16 * 32; i += blockDim.x) sh->lut[i] = level(i >> 5);
  if (warp == 1) {
    tmem_alloc(&sh->tmem_base, kMgCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;

  if (warp == 0) {
    // ---------------- TMA: every r chunk of the tile's B rows and A columns at once
    if (lane == 0) {
      for (int j = 0; j < p.chunks; ++j) {
        uint8_t* b = smem + j * kMgChunkBytes;
        uint8_t* a = b + kMgBBytes;
        mbar_arrive_expect_tx(&sh->full[j], kMgChunkBytes);
        tma_load_2d(b, &tm_b, &sh->full[j], 64 * j, n0);
#pragma unroll
        for (int g = 0; g < kMgCols / 64; ++g) tma_load_2d(a + g * 8192, &tm_a, &sh->full[j], k0 + 64 * g, 64 * j);
      }
      if (*abort_flag) {
        // unwind (bounded): the copies still in flight land before the CTA exits
        for (int j = 0; j < p.chunks; ++j) {
          uint32_t no_abort = 0;
          mbar_wait(&sh->full[j], 0, &no_abort, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA: D[128 n, 256 k] = sum over r of B[n, r] A[r, k]
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, kMgCols, false, true);
      bool ok = true;
      int issued = 0;
      for (int j = 0; j < p.chunks && ok; ++j) {
        ok = mbar_wait(&sh->full[j], 0, abort_flag, p.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t b_base = smem_u32(smem + j * kMgChunkBytes);
        const uint32_t a_base = b_base + kMgBBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t adesc = smem_desc_sw128(b_base + kk * 32, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(a_base + kk * 2048, 8192, 1024);
          umma_f16(tmem, adesc, bdesc, idesc, (j > 0 || kk > 0) ? 1u : 0u);
        }
        ++issued;
      }
      // one commit, after the last MMA: it covers the whole chain
      if (ok) umma_commit(&sh->accum);
      else if (issued > 0) {
        umma_commit(&sh->accum);
        uint32_t no_abort = 0;
        mbar_wait(&sh->accum, 0, &no_abort, nullptr);
      }
    }
  } else {
    // ---------------- epilogue: one output row, 128 columns per thread
    const int quad = warp & 3;                      // TMEM lanes 32 quad .. + 31
    const int half = (warp - 2) >> 2;               // 128-column part of the tile
    const int row = quad * 32 + lane;
    const int n = n0 + row;
    const int kh = k0 + half * 128;                 // first column of this thread's half
    // The row's codes (64 bytes) and its two block scales are fetched before
    // the accumulator is ready, so their latency hides behind the MMAs.
    uint4 cw[4] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0),
                   make_uint4(0, 0, 0, 0)};
    float scale[2] = {0.0f, 0.0f};
    const bool live = n < p.N && kh < p.K;
    if (live) {
      const uint4* src = reinterpret_cast<const uint4*>(p.codes + (int64_t(n) * p.K + kh) / 2);
#pragma unroll
      for (int c = 0; c < 4; ++c) cw[c] = (kh + 32 * c < p.K) ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
      const float s_g = p.double_quant ? __ldg(p.absmax_scale) : 0.0f;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        if (kh + 64 * j >= p.K) continue;
        const int64_t blk = chunk_block(n, p.K, (kh + 64 * j) / 64, p.bs_shift);
        scale[j] = p.double_quant ? __fmul_rn(float(__ldg(p.absmax_q + blk)), s_g) : __ldg(p.absmax + blk);
      }
    }
    // Each warp stages and stores its own 32 rows, so the warps never wait on
    // one another: two 32 x 32 buffers per warp, one TMA store per piece.
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&sh->accum, 0, abort_flag, p.status));
    tc_fence_after();
    if (ok) {
      const float* lut = sh->lut + lane;
      const bool f16 = p.out_kind == kMergeF16;
      uint8_t* stage = smem + (warp - 2) * 2 * kMgStageBytes;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int k = kh + 32 * c;
        // Stop at the first piece past the last column (warp-uniform), so that
        // every staged piece is stored and the wait below frees the right buffer.
        if (k >= p.K) break;
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + (uint32_t(quad * 32) << 16) + half * 128 + c * 32, v);
        tmem_ld_wait();
        const float sc = scale[c >> 1];
        const uint32_t words[4] = {cw[c].x, cw[c].y, cw[c].z, cw[c].w};
        float m[32];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
#pragma unroll
          for (int bidx = 0; bidx < 4; ++bidx) {
            const uint32_t byte = (words[q] >> (8 * bidx)) & 0xffu;
            const int e = 8 * q + 2 * bidx;          // even element in the high nibble
            const float w0 = __fmul_rn(lut[(byte >> 4) * 32], sc);
            const float w1 = __fmul_rn(lut[(byte & 15u) * 32], sc);
            m[e] = fmaf(p.s, __uint_as_float(v[e]), w0);
            m[e + 1] = fmaf(p.s, __uint_as_float(v[e + 1]), w1);
          }
        }
        // buffer c & 1 is free once the store issued two pieces ago has read it
        uint8_t* buf = stage + (c & 1) * kMgStageBytes;
        if (lane == 0 && c >= 2) bulk_wait_group_read<1>();
        __syncwarp();
        if (p.out_kind == kMergeF32) {   // 128-byte rows, 128-byte swizzle: chunk j at j ^ (lane & 7)
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<float4*>(buf + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                make_float4(m[4 * j], m[4 * j + 1], m[4 * j + 2], m[4 * j + 3]);
        } else {               // 64-byte rows, 64-byte swizzle: chunk j at j ^ ((lane >> 1) & 3)
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(buf + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) =
                make_uint4(pack_out2(f16, m[8 * j], m[8 * j + 1]), pack_out2(f16, m[8 * j + 2], m[8 * j + 3]),
                           pack_out2(f16, m[8 * j + 4], m[8 * j + 5]), pack_out2(f16, m[8 * j + 6], m[8 * j + 7]));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tm_out, buf, k, n0 + quad * 32);   // rows past N are clipped by the map
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
    tmem_dealloc(tmem, kMgCols);
  }
}

}  // namespace

// Dynamic shared memory for `chunks` 64-wide r chunks, padded so that no more
// CTAs share an SM than their TMEM tiles fit (kMgCtasPerSm).
size_t merge_smem_bytes(int chunks) {
  const size_t need = size_t(merge_region_bytes(chunks)) + sizeof(MergeShared) + 1024;
  const size_t floor = (228u * 1024u) / (kMgCtasPerSm + 1) + 1024u;
  return need > floor ? need : floor;
}

cudaError_t launch_merge(const nf4_weight& w, const void* A, const void* B, int r, float alpha,
                         int out_kind, void* out, uint32_t* status, cudaStream_t st, int* launches) {
  static PerDeviceOnce attr_done;
  const int dev = PerDeviceOnce::current();
  if (!attr_done.done(dev)) {
    const cudaError_t e = cudaFuncSetAttribute(nf4_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               int(merge_smem_bytes(kMgMaxChunks)));
    if (e != cudaSuccess) return e;
    attr_done.mark(dev);
  }
  if (r < 1 || r > 64 * kMgMaxChunks) return cudaErrorInvalidValue;
  const size_t smem = merge_smem_bytes((r + 63) / 64);
  const int64_t N = w.rows, K = w.cols;
  CUtensorMap tb, ta, to;
  // B [N, r]: 64-wide r chunks of 128 rows (K-major operand); A [r, K]: 64 r x 64 k boxes
  // (MN-major); out [N, K]: 32 x 128 boxes in the staging layout.
  bool ok = make_map_2d(&tb, B, true, uint64_t(r), uint64_t(N), 64, kMgRows, true);
  ok = ok && make_map_2d(&ta, A, true, uint64_t(K), uint64_t(r), 64, 64, true);
  // (the store copies bytes: a bf16 map serves the f16 output as well)
  ok = ok && (out_kind == kMergeF32
                  ? make_map_2d_f32(&to, out, uint64_t(K), uint64_t(N), 32, 32, CU_TENSOR_MAP_SWIZZLE_128B)
                  : make_map_2d_bf16(&to, out, uint64_t(K), uint64_t(N), 32, 32, CU_TENSOR_MAP_SWIZZLE_64B));
  if (!ok) return cudaErrorInvalidValue;
  MergeParams p;
  p.N = int(N);
  p.K = int(K);
  p.r = r;
  p.chunks = (r + 63) / 64;
  p.bs_shift = log2_block(w.block_size);
  if (p.bs_shift < 0) return cudaErrorInvalidValue;
  p.s = alpha / float(r);
  p.double_quant = w.double_quant;
  p.out_kind = out_kind;
  p.codes = w.codes;
  p.absmax_q = w.absmax_q;
  p.absmax = w.absmax;
  p.absmax_scale = w.absmax_scale;
  p.out = out;
  p.status = status;
  const dim3 grid(unsigned((K + kMgCols - 1) / kMgCols), unsigned((N + kMgRows - 1) / kMgRows));
  NF4_PROF_BEGIN(st, kKMerge);
  nf4_merge_kernel<<<grid, kMgThreads, smem, st>>>(tb, ta, to, p);
  NF4_PROF_END(st, kKMerge);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) ++*launches;
  return e;
}

}  // namespace nf4
