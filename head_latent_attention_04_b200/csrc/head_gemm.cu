// Per-head projections of absorbed MLA on tcgen05 tensor cores.
//
//   mla_absorb_q : q_lat[n,h,:] = W_UK[:,h,:] q_nope[n,h,:]   (M = d_c = 512, K = d = 128)
//   mla_out_uv   : out[n,h,:]   = W_UV[:,h,:]^T o_lat[n,h,:]  (M = d_v = 128, K = d_c = 512)
//
// These are the Step-2 terms of the MLA matrix-absorption notes' order 2
// (2bshkd in section 2.2, 2bhsvk in section 3.2).  With decode batches the token
// count is small, so both are written "swap-AB": a 128-row slice of one head's
// weight is the M operand and the tokens (up to 256 per CTA) the N operand, so
// D[m][n] sits in TMEM with one lane per output feature.  Reading W_UK / W_UV
// (16.8 MB each at 128 heads) dominates, as the izhida.com answer notes for the
// W_V product of a batched GEMV; every CTA therefore puts all (absorb) or most
// (out_uv) of its loads in flight at once.
//
// Epilogue: D is converted to bf16 into shared memory as [token][128 features]
// and written by one TMA store; tokens past n_tokens are clipped by the tensor
// map, so a partial token tile needs no bounds checks.
//
// absorb_q_kernel: one CTA per (128-row tile of W_UK, head, token tile).  K = 128
//   is two 64-wide chunks: one barrier covers the 32 KB weight tile and the
//   tokens' q_nope, then 8 MMAs.  4 x 128 CTAs for a 128-head batch, several
//   per SM.
// out_uv_kernel: one CTA per (head, token tile); K = 512 streams through a ring
//   of up to 8 stages, each 16 KB of W_UV (MN-major: v contiguous) plus the
//   tokens' 64-wide o_lat chunk.  The CTA prefetches its head's W_UV into L2
//   before waiting for the merge kernel, so the weight read overlaps it.
//
// The same two products also run as FP8 (E4M3) block-quantised BMMs
// (mla_absorb_q_fp8, mla_out_uv_fp8, with the weight and row quantisers), in
// the section that follows the bf16 kernels.
#include "mla_internal.h"
#include "ptx.cuh"
#include "tmap.h"

#include <cuda_bf16.h>

#include <algorithm>

namespace mla {
namespace {

using namespace ptx;

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kMaxBN = 256;
constexpr int kATileBytes = kBM * kBK * 2;       // 16 KB: 128 rows x 64 K
constexpr int kMaxRing = 8;
constexpr int kSmemPerSM = 233472;               // 228 KB of shared memory per SM
constexpr int kSmemLimit = 232448;               // per CTA

struct GemmParams {
  int n_tokens, n_heads, bn;
  int stages;   // out_uv ring depth
};

__host__ __device__ constexpr uint32_t tmem_cols_for(int bn) {
  return bn <= 32 ? 32u : bn <= 64 ? 64u : bn <= 128 ? 128u : 256u;
}

// TMEM [128 lanes x bn] fp32 -> bf16 smem tile [bn][128] -> one TMA store at (x, h, n0).
__device__ __forceinline__ void store_tile(uint32_t tmem, uint8_t* s_out, int bn, const CUtensorMap* tm_out,
                                           int x, int h, int n0) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(s_out);
  const int m = warp * 32 + lane;
  for (int c = 0; c < bn; c += 32) {
    uint32_t r[32];
    tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c, r);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (c + j < bn) o[(c + j) * kBM + m] = __float2bfloat16_rn(__uint_as_float(r[j]));
  }
  fence_proxy_async_smem();   // the TMA store reads the tile through the async proxy
  __syncthreads();
  if (threadIdx.x == 0) {
    tma_store_3d(tm_out, s_out, x, h, n0);
    bulk_commit();
    bulk_wait_all<0>();
  }
}

__global__ void __launch_bounds__(128)
absorb_q_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                const __grid_constant__ CUtensorMap tm_out, GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int bn = p.bn;
  uint8_t* sA = smem;                        // 2 chunks x 16 KB (SW128, K-major)
  uint8_t* sB = smem + 2 * kATileBytes;      // 2 chunks x bn rows x 128 B
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + 2 * bn * 128);
  uint64_t* done = full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int mt = blockIdx.x, h = blockIdx.y, n0 = blockIdx.z * bn;
  const uint32_t cols = tmem_cols_for(bn);

  if (threadIdx.x == 0) {
    mbar_init(full, 1);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_out);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();   // set-up above overlaps the previous kernel; global memory only from here
  griddep_launch_dependents();

  if (warp == 0 && lane == 0) {
    mbar_arrive_expect_tx(full, 2 * kATileBytes + 2 * bn * 128);
#pragma unroll
    for (int kc = 0; kc < 2; ++kc) {
      tma_load_3d(sA + kc * kATileBytes, &tm_w, full, kc * kBK, h, mt * kBM);
      tma_load_3d(sB + kc * bn * 128, &tm_x, full, kc * kBK, h, n0);
    }
  } else if (warp == 1 && lane == 0) {
    if (mbar_wait(full, 0, abort_flag)) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16(kBM, bn, 0, 0);
#pragma unroll
      for (int kc = 0; kc < 2; ++kc)
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          mma_ss(tmem, sdesc(smem_u32(sA + kc * kATileBytes) + kk * 32, 16, 1024, kSwizzle128B),
                 sdesc(smem_u32(sB + kc * bn * 128) + kk * 32, 16, 1024, kSwizzle128B), idesc, (kc | kk) != 0);
    } else {
      *abort_flag = 1;
    }
    mma_commit(done);
  }
  __syncwarp();
  // block-uniform: every thread has seen `done` before the tile area is reused for the output
  const bool ok = __syncthreads_and(mbar_wait(done, 0, abort_flag) && !*abort_flag);
  tc_fence_after();
  if (ok) store_tile(tmem, smem, bn, &tm_out, mt * kBM, h, n0);
  tc_fence_before();
  __syncthreads();
  __syncwarp();
  if (warp == 1) tmem_dealloc(tmem, cols);
}

__global__ void __launch_bounds__(128)
out_uv_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
              const __grid_constant__ CUtensorMap tm_out, GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int bn = p.bn, S = p.stages;
  const int stage_bytes = kATileBytes + bn * 128;   // W_UV chunk (two 64-v halves) + o_lat chunk
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * stage_bytes);
  uint64_t* empty = full + kMaxRing;
  uint64_t* done = empty + kMaxRing;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = blockIdx.y, n0 = blockIdx.z * bn;
  const uint32_t cols = tmem_cols_for(bn);
  constexpr int kChunks = 512 / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_out);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, cols);
    tmem_relinquish();
  }
  // This head's W_UV slice (128 KB) into L2 while the previous kernel finishes:
  // a prefetch moves no data into this CTA and reads nothing the previous
  // kernel writes, so it may precede the dependency wait.
  if (warp == 0 && lane < kChunks) {
    tma_prefetch_l2_3d(&tm_w, 0, h, lane * kBK);
    tma_prefetch_l2_3d(&tm_w, 64, h, lane * kBK);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();
  griddep_launch_dependents();

  if (warp == 0 && lane == 0) {
    for (int kc = 0; kc < kChunks; ++kc) {
      const int s = kc % S;
      if (kc >= S && !mbar_wait(&empty[s], ((kc / S) - 1) & 1, abort_flag)) {
        *abort_flag = 1;
        break;
      }
      uint8_t* st = smem + s * stage_bytes;
      mbar_arrive_expect_tx(&full[s], stage_bytes);
      tma_load_3d(st, &tm_w, &full[s], 0, h, kc * kBK);                      // v 0..63
      tma_load_3d(st + kATileBytes / 2, &tm_w, &full[s], 64, h, kc * kBK);   // v 64..127
      tma_load_3d(st + kATileBytes, &tm_x, &full[s], kc * kBK, h, n0);
    }
  } else if (warp == 1 && lane == 0) {
    const uint32_t idesc = idesc_bf16(kBM, bn, 1, 0);
    for (int kc = 0; kc < kChunks; ++kc) {
      const int s = kc % S;
      if (!mbar_wait(&full[s], (kc / S) & 1, abort_flag)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t a0 = smem_u32(smem + s * stage_bytes), b0 = a0 + kATileBytes;
#pragma unroll
      for (int kk = 0; kk < kBK / 16; ++kk)
        mma_ss(tmem, sdesc(a0 + kk * 2048, kATileBytes / 2, 1024, kSwizzle128B),
               sdesc(b0 + kk * 32, 16, 1024, kSwizzle128B), idesc, (kc | kk) != 0);
      mma_commit(&empty[s]);
    }
    mma_commit(done);
  }
  __syncwarp();
  // block-uniform; all loads were consumed by completed MMAs, so the ring is free for the output
  const bool ok = __syncthreads_and(mbar_wait(done, 0, abort_flag) && !*abort_flag);
  tc_fence_after();
  if (ok) store_tile(tmem, smem, bn, &tm_out, 0, h, n0);
  tc_fence_before();
  __syncthreads();
  __syncwarp();
  if (warp == 1) tmem_dealloc(tmem, cols);
}

// Token tile: at most 256, a multiple of 16, tiles of near-equal size.
int token_tile(int n_tokens, int* n_tiles) {
  const int tiles = (n_tokens + kMaxBN - 1) / kMaxBN;
  const int per = (n_tokens + tiles - 1) / tiles;
  *n_tiles = tiles;
  return ((per + 15) / 16) * 16;
}

cudaError_t set_smem_attrs() {
  static cudaError_t e = [] {
    cudaError_t a = cudaFuncSetAttribute(absorb_q_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
    cudaError_t b = cudaFuncSetAttribute(out_uv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
    return a != cudaSuccess ? a : b;
  }();
  return e;
}

// Row-major [N][H][F] bf16 tensor maps: load boxes of 64 features x bn tokens
// (SW128) and store boxes of 128 features x bn tokens (no swizzle).
mla_status_t act_map(CUtensorMap* m, const void* base, int F, int H, int N, int box_f, int bn, bool store) {
  const uint64_t dims[3] = {(uint64_t)F, (uint64_t)H, (uint64_t)N};
  const uint64_t str[2] = {(uint64_t)F * 2, (uint64_t)H * F * 2};
  const uint32_t box[3] = {(uint32_t)box_f, 1, (uint32_t)bn};
  return encode_tmap_bf16(m, base, 3, dims, str, box,
                          store ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B);
}

// Weight [512][H][128] bf16 as (128, H, 512), box {64, 1, box_k}.
mla_status_t weight_map(CUtensorMap* m, const void* base, int H, int box_k) {
  const uint64_t dims[3] = {128, (uint64_t)H, 512};
  const uint64_t str[2] = {128 * 2, (uint64_t)H * 128 * 2};
  const uint32_t box[3] = {64, 1, (uint32_t)box_k};
  return encode_tmap_bf16(m, base, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// ----------------------------------------------------------------- FP8 (E4M3) block-quantised BMMs
// "Lower latency and higher throughput with multi-node DeepSeek deployment",
// sections "Quantization" and "MLA layer": weights carry one scale per
// 128 x 128 block (quantised once, here by quantize_weight_kernel) and
// activations one scale per 128-element vector along K, computed on the fly.
// A block's scale is s = amax / 448 and a value's code is E4M3(x * (448 /
// amax)), rounded to nearest even; an all-zero block takes s = 1.  Products of
// a K-block are summed exactly-rounded in fp32 by the tensor cores and scaled
// by s_act * s_weight afterwards.

constexpr float kE4M3Max = 448.f;

// 128 bf16 (16 x 16 bytes) -> 128 E4M3 codes (32 words, element 4j + i in byte
// i of word j) and the vector's scale.
__device__ __forceinline__ float quant128(const uint4 (&x)[16], uint32_t (&q)[32]) {
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const uint32_t w[4] = {x[k].x, x[k].y, x[k].z, x[k].w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[i] << 16)), fabsf(__uint_as_float(w[i] & 0xFFFF0000u))));
  }
  const float r = amax > 0.f ? __fdiv_rn(kE4M3Max, amax) : 1.f;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const uint32_t w[4] = {x[k].x, x[k].y, x[k].z, x[k].w};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint32_t a = w[2 * i], b = w[2 * i + 1];
      q[2 * k + i] = cvt_e4m3x2(__fmul_rn(__uint_as_float(a << 16), r), __fmul_rn(__uint_as_float(a & 0xFFFF0000u), r)) |
                     (cvt_e4m3x2(__fmul_rn(__uint_as_float(b << 16), r), __fmul_rn(__uint_as_float(b & 0xFFFF0000u), r)) << 16);
    }
  }
  return amax > 0.f ? __fdiv_rn(amax, kE4M3Max) : 1.f;
}

__device__ __forceinline__ void load128(const __nv_bfloat16* src, uint4 (&x)[16]) {
#pragma unroll
  for (int k = 0; k < 16; ++k) x[k] = __ldg(reinterpret_cast<const uint4*>(src) + k);
}

// Codes of one 128-byte row into a K-major SW128 tile (16-byte chunk c of row
// r at chunk c ^ (r & 7)); the tile base is 1024-byte aligned.
__device__ __forceinline__ void put_row_sw128(uint8_t* tile, int r, const uint32_t (&q)[32]) {
  uint8_t* row = tile + r * 128;
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4)) = make_uint4(q[4 * c], q[4 * c + 1], q[4 * c + 2], q[4 * c + 3]);
}

// One 128 x 128 weight block (kb, h) of W [512][H][128] bf16 -> codes and
// scales[h][kb].  kTransposed = false: codes [H][512][128] (W_UK: rows k,
// K = d contiguous); true: codes [H][128][512] (W_UV: rows v, K = k contiguous).
template <bool kTransposed>
__global__ void __launch_bounds__(128) quantize_weight_kernel(const __nv_bfloat16* __restrict__ w, int n_heads,
                                                              uint8_t* __restrict__ codes, float* __restrict__ scales) {
  __shared__ __align__(16) __nv_bfloat16 tile[128][128];
  __shared__ float wmax[4];
  const int kb = blockIdx.x, h = blockIdx.y, t = threadIdx.x;
  uint4 x[16];
  load128(w + ((size_t)(kb * 128 + t) * n_heads + h) * 128, x);
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    *reinterpret_cast<uint4*>(&tile[t][8 * k]) = x[k];
    const uint32_t ws[4] = {x[k].x, x[k].y, x[k].z, x[k].w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(ws[i] << 16)), fabsf(__uint_as_float(ws[i] & 0xFFFF0000u))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((t & 31) == 0) wmax[t >> 5] = amax;
  __syncthreads();
  amax = fmaxf(fmaxf(wmax[0], wmax[1]), fmaxf(wmax[2], wmax[3]));
  const float r = amax > 0.f ? __fdiv_rn(kE4M3Max, amax) : 1.f;
  if (t == 0) scales[h * 4 + kb] = amax > 0.f ? __fdiv_rn(amax, kE4M3Max) : 1.f;
  // thread t writes output row t of the block: W_UK row k = kb*128 + t (over d),
  // or W_UV row v = t (over k in the block, read down the tile's column t)
  uint8_t* dst = kTransposed ? codes + ((size_t)h * 128 + t) * 512 + kb * 128
                             : codes + ((size_t)h * 512 + kb * 128 + t) * 128;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint32_t wds[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float f[4];
      if constexpr (kTransposed) {   // down column t of the tile (consecutive threads, consecutive banks)
#pragma unroll
        for (int i = 0; i < 4; ++i) f[i] = __bfloat162float(tile[16 * c + 4 * j + i][t]);
      } else {                       // this thread's own row, still in registers
        const uint4 v = x[2 * c + j / 2];
        const uint32_t a = (j & 1) ? v.z : v.x, b = (j & 1) ? v.w : v.y;
        f[0] = __uint_as_float(a << 16); f[1] = __uint_as_float(a & 0xFFFF0000u);
        f[2] = __uint_as_float(b << 16); f[3] = __uint_as_float(b & 0xFFFF0000u);
      }
      wds[j] = cvt_e4m3x2(__fmul_rn(f[0], r), __fmul_rn(f[1], r)) | (cvt_e4m3x2(__fmul_rn(f[2], r), __fmul_rn(f[3], r)) << 16);
    }
    reinterpret_cast<uint4*>(dst)[c] = make_uint4(wds[0], wds[1], wds[2], wds[3]);
  }
}

// Rows of 128-element vectors: x [rows][cols] bf16 -> codes [rows][cols] and
// scales [rows][cols / 128], one thread per vector (the on-the-fly activation
// quantisation of the BMM kernels, exposed on its own).
__global__ void quantize_rows_kernel(const __nv_bfloat16* __restrict__ x, long long n_vec,
                                     uint8_t* __restrict__ codes, float* __restrict__ scales) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n_vec; i += (long long)gridDim.x * blockDim.x) {
    uint4 v[16];
    load128(x + i * 128, v);
    uint32_t q[32];
    scales[i] = quant128(v, q);
#pragma unroll
    for (int c = 0; c < 8; ++c)
      reinterpret_cast<uint4*>(codes + i * 128)[c] = make_uint4(q[4 * c], q[4 * c + 1], q[4 * c + 2], q[4 * c + 3]);
  }
}

// New cache rows -> FP8 latent-cache slots (row = 512 E4M3 codes | 4 fp32
// scales | 64 bf16 k_rope, 656 bytes).  Thread = (row, 128-column block): the
// same quantiser as the activations, plus a quarter of the row's k_rope.
constexpr int kKvRow = 576, kF8CacheRow = 656;

__global__ void kv_quantize_fp8_kernel(const __nv_bfloat16* __restrict__ kv, const int32_t* __restrict__ slots,
                                       long long n, uint8_t* __restrict__ pool, long long pool_rows,
                                       int32_t* status) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < 4 * n; i += (long long)gridDim.x * blockDim.x) {
    const long long row = i >> 2;
    const int j = (int)(i & 3);
    const long long slot = slots[row];
    if (slot < 0 || slot >= pool_rows) {
      if (status && j == 0) atomicOr(status, MLA_STATUS_BAD_BLOCK);
      continue;
    }
    const __nv_bfloat16* src = kv + row * kKvRow;
    uint8_t* dst = pool + slot * kF8CacheRow;
    uint4 v[16];
    load128(src + 128 * j, v);
    uint32_t q[32];
    const float s = quant128(v, q);
    if (status && s > 65504.f / kE4M3Max) atomicOr(status, MLA_STATUS_CACHE_RANGE);   // widened in fp16
#pragma unroll
    for (int c = 0; c < 8; ++c)
      reinterpret_cast<uint4*>(dst + 128 * j)[c] = make_uint4(q[4 * c], q[4 * c + 1], q[4 * c + 2], q[4 * c + 3]);
    reinterpret_cast<float*>(dst + 512)[j] = s;
    const uint4* rs = reinterpret_cast<const uint4*>(src + 512) + 2 * j;   // k_rope bytes [32j, 32j + 32)
    uint4* rd = reinterpret_cast<uint4*>(dst + 528) + 2 * j;
    rd[0] = __ldg(rs);
    rd[1] = __ldg(rs + 1);
  }
}

// absorb, FP8: one CTA per (128-row tile of the head's W_UK codes, head, token
// tile).  A = codes [128 k][128 d] (one TMA box, SW128); the tokens' q_nope rows
// arrive by TMA as bf16 (two SW128 chunks of 64 d, as in the bf16 kernel) and
// are quantised from shared memory into a SW128 code tile, four threads per
// row (32 values each, the row maximum combined by shuffles; a token tile is a
// multiple of 16 rows, so every warp is wholly in or out of the loop); K = 128
// in 4 MMAs; epilogue D * s_w[h][tile] * s_q[token], staged over the dead
// operands.  Token tiles of at most 128.
__global__ void __launch_bounds__(128)
absorb_q_fp8_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                    const __grid_constant__ CUtensorMap tm_out, const float* __restrict__ w_scales, GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int bn = p.bn;
  uint8_t* sA = smem;                           // 16 KB of weight codes
  uint8_t* sX = sA + kATileBytes;               // 2 chunks x bn x 128 B of bf16 q_nope
  uint8_t* sB = sX + 2 * bn * 128;              // bn x 128 B of codes
  uint8_t* sOut = smem;                         // bf16 [bn][128], over the operands once the MMAs are done
  const int region = (kATileBytes + 3 * bn * 128) > bn * 256 ? (kATileBytes + 3 * bn * 128) : bn * 256;
  float* s_act = reinterpret_cast<float*>(smem + region);     // [bn]
  uint64_t* full = reinterpret_cast<uint64_t*>(s_act + kMaxBN);
  uint64_t* done = full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int mt = blockIdx.x, h = blockIdx.y, n0 = blockIdx.z * bn;
  const uint32_t cols = tmem_cols_for(bn);
  if (threadIdx.x == 0) {
    mbar_init(full, 1);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_out);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();   // global memory only from here
  griddep_launch_dependents();

  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(full, kATileBytes + 2 * bn * 128);
    tma_load_2d(sA, &tm_w, full, 0, h * 512 + mt * kBM);
    tma_load_3d(sX, &tm_x, full, 0, h, n0);
    tma_load_3d(sX + bn * 128, &tm_x, full, 64, h, n0);
  }
  const bool landed = __all_sync(0xffffffffu, mbar_wait(full, 0, abort_flag));   // warp-uniform: the loop shuffles
  if (landed) {
    // item i: row r = i / 4, values [32 qq, 32 qq + 32) with qq = i % 4 (chunk qq / 2,
    // 16-byte pieces 4 (qq % 2) .. + 3 of that chunk's swizzled row)
    for (int i = threadIdx.x; i < bn * 4; i += 128) {
      const int r = i >> 2, qq = i & 3;
      const uint8_t* row = sX + (qq >> 1) * bn * 128 + r * 128;
      float v[32];
      float amax = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint4 w4 = *reinterpret_cast<const uint4*>(row + ((((qq & 1) * 4 + k) ^ (r & 7)) << 4));
        const uint32_t ws[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          v[8 * k + 2 * j] = __uint_as_float(ws[j] << 16);
          v[8 * k + 2 * j + 1] = __uint_as_float(ws[j] & 0xFFFF0000u);
          amax = fmaxf(amax, fmaxf(fabsf(v[8 * k + 2 * j]), fabsf(v[8 * k + 2 * j + 1])));
        }
      }
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      const float rcp = amax > 0.f ? __fdiv_rn(kE4M3Max, amax) : 1.f;
      uint32_t q[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        q[j] = cvt_e4m3x2(__fmul_rn(v[4 * j], rcp), __fmul_rn(v[4 * j + 1], rcp)) |
               (cvt_e4m3x2(__fmul_rn(v[4 * j + 2], rcp), __fmul_rn(v[4 * j + 3], rcp)) << 16);
      uint8_t* crow = sB + r * 128;   // code pieces 2 qq and 2 qq + 1 of row r
      *reinterpret_cast<uint4*>(crow + (((2 * qq) ^ (r & 7)) << 4)) = make_uint4(q[0], q[1], q[2], q[3]);
      *reinterpret_cast<uint4*>(crow + (((2 * qq + 1) ^ (r & 7)) << 4)) = make_uint4(q[4], q[5], q[6], q[7]);
      if (qq == 0) s_act[r] = amax > 0.f ? __fdiv_rn(amax, kE4M3Max) : 1.f;
    }
  }
  fence_proxy_async_smem();   // the MMAs read the code tile through the async proxy
  const bool all_landed = __syncthreads_and(landed);
  if (warp == 1 && lane == 0) {
    if (all_landed) {
      tc_fence_after();
      const uint32_t idesc = idesc_e4m3(kBM, bn);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)   // K = 128 codes = 128 bytes per row, 32 per MMA
        mma_ss_f8(tmem, sdesc(smem_u32(sA) + kk * 32, 16, 1024, kSwizzle128B),
                  sdesc(smem_u32(sB) + kk * 32, 16, 1024, kSwizzle128B), idesc, kk != 0);
    } else {
      *abort_flag = 1;
    }
    mma_commit(done);
  }
  __syncwarp();
  const bool ok = __syncthreads_and(mbar_wait(done, 0, abort_flag) && !*abort_flag);
  tc_fence_after();
  if (ok) {
    const float s_w = w_scales[h * 4 + mt];
    __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(sOut);
    const int m = warp * 32 + lane;
    for (int c = 0; c < bn; c += 32) {
      uint32_t rr[32];
      tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c, rr);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (c + j < bn) o[(c + j) * kBM + m] = __float2bfloat16_rn(__uint_as_float(rr[j]) * (s_w * s_act[c + j]));
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (threadIdx.x == 0) {
      tma_store_3d(&tm_out, sOut, mt * kBM, h, n0);
      bulk_commit();
      bulk_wait_all<0>();
    }
  }
  tc_fence_before();
  __syncthreads();
  __syncwarp();
  if (warp == 1) tmem_dealloc(tmem, cols);
}

// out_uv, FP8: one CTA per (head, token tile of at most 128).  A = the head's
// W_UV codes [128 v][512 k] as four 16 KB K-blocks, B = the tokens' o_lat rows
// quantised per 128-vector into four SW128 tiles, one TMEM accumulator per
// K-block (4 x bn columns), epilogue sum_kb D_kb * s_w[h][kb] * s_o[token][kb].
__global__ void __launch_bounds__(128)
out_uv_fp8_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_out,
                  const __nv_bfloat16* __restrict__ o_lat, const float* __restrict__ w_scales, GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int bn = p.bn;
  uint8_t* sA = smem;                           // 4 x 16 KB
  uint8_t* sB = sA + 4 * kATileBytes;           // 4 x bn x 128 B
  uint8_t* sOut = smem;                         // bn x 256 B, over the weight tiles once the MMAs are done
  float* s_act = reinterpret_cast<float*>(sB + 4 * bn * 128);   // [4][128]
  uint64_t* full = reinterpret_cast<uint64_t*>(s_act + 4 * 128);
  uint64_t* done = full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = blockIdx.y, n0 = blockIdx.z * bn;
  const uint32_t cols = tmem_cols_for(bn);
  if (threadIdx.x == 0) {
    mbar_init(full, 1);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_out);
  }
  // the head's 64 KB of codes into L2 while the previous kernel finishes (a hint)
  if (warp == 0 && lane < 4) tma_prefetch_l2_2d(&tm_w, lane * 128, h * 128);
  if (warp == 1) {
    tmem_alloc(tmem_slot, 4 * cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();
  griddep_launch_dependents();

  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(full, 4 * kATileBytes);
#pragma unroll
    for (int kb = 0; kb < 4; ++kb) tma_load_2d(sA + kb * kATileBytes, &tm_w, full, kb * 128, h * 128);
  }
  for (int i = threadIdx.x; i < 128 * 4; i += 128) {   // vector (token r, K-block kb)
    const int r = i >> 2, kb = i & 3, n = n0 + r;
    if (r >= bn) {   // past the tile: a zero scale for the epilogue's padding columns
      s_act[kb * 128 + r] = 0.f;
      continue;
    }
    uint32_t q[32];
    float sc = 0.f;
    if (n < p.n_tokens) {
      uint4 x[16];
      load128(o_lat + ((size_t)n * p.n_heads + h) * 512 + kb * 128, x);
      sc = quant128(x, q);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) q[j] = 0;
    }
    put_row_sw128(sB + kb * bn * 128, r, q);
    s_act[kb * 128 + r] = sc;
  }
  fence_proxy_async_smem();
  __syncthreads();
  if (warp == 1 && lane == 0) {
    if (mbar_wait(full, 0, abort_flag)) {
      tc_fence_after();
      const uint32_t idesc = idesc_e4m3(kBM, bn);
#pragma unroll
      for (int kb = 0; kb < 4; ++kb)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss_f8(tmem + kb * cols, sdesc(smem_u32(sA + kb * kATileBytes) + kk * 32, 16, 1024, kSwizzle128B),
                    sdesc(smem_u32(sB + kb * bn * 128) + kk * 32, 16, 1024, kSwizzle128B), idesc, kk != 0);
    } else {
      *abort_flag = 1;
    }
    mma_commit(done);
  }
  __syncwarp();
  const bool ok = __syncthreads_and(mbar_wait(done, 0, abort_flag) && !*abort_flag);
  tc_fence_after();
  if (ok) {
    float s_w[4];
#pragma unroll
    for (int kb = 0; kb < 4; ++kb) s_w[kb] = w_scales[h * 4 + kb];
    __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(sOut);
    const int m = warp * 32 + lane;
    for (int c = 0; c < bn; c += 32) {
      float acc[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) acc[j] = 0.f;
#pragma unroll
      for (int kb = 0; kb < 4; ++kb) {
        uint32_t rr[32];
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + kb * cols + c, rr);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] = fmaf(__uint_as_float(rr[j]), s_w[kb] * s_act[kb * 128 + c + j], acc[j]);
      }
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (c + j < bn) o[(c + j) * kBM + m] = __float2bfloat16_rn(acc[j]);
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (threadIdx.x == 0) {
      tma_store_3d(&tm_out, sOut, 0, h, n0);
      bulk_commit();
      bulk_wait_all<0>();
    }
  }
  tc_fence_before();
  __syncthreads();
  __syncwarp();
  if (warp == 1) tmem_dealloc(tmem, 4 * cols);
}

cudaError_t set_smem_attrs_fp8() {
  static cudaError_t e = [] {
    cudaError_t a = cudaFuncSetAttribute(absorb_q_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
    cudaError_t b = cudaFuncSetAttribute(out_uv_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
    return a != cudaSuccess ? a : b;
  }();
  return e;
}

// Token tile of at most `max_bn`, a multiple of 16, tiles of near-equal size.
int token_tile_max(int n_tokens, int max_bn, int* n_tiles) {
  const int tiles = (n_tokens + max_bn - 1) / max_bn;
  const int per = (n_tokens + tiles - 1) / tiles;
  *n_tiles = tiles;
  return ((per + 15) / 16) * 16;
}

// Shared memory padded so that the CTAs sharing an SM never ask for more than
// its 512 TMEM columns: at most 512 / tmem_cols of them fit by shared memory.
int pad_smem_for_tmem(int smem, int tmem_cols) {
  const int ctas = 512 / tmem_cols;
  const int floor_bytes = kSmemPerSM / (ctas + 1) - 1024 + 1;
  return smem < floor_bytes ? floor_bytes : smem;
}

}  // namespace

mla_status_t launch_absorb_q(const void* q_nope, const void* w_uk, void* q_lat, int n_tokens,
                             int n_heads, void* stream) {
  int tiles = 1;
  const int bn = token_tile(n_tokens, &tiles);
  CUtensorMap tw, tx, to;
  mla_status_t st = weight_map(&tw, w_uk, n_heads, kBM);   // 128 latent rows x 64 d
  if (st == MLA_OK) st = act_map(&tx, q_nope, 128, n_heads, n_tokens, 64, bn, false);
  if (st == MLA_OK) st = act_map(&to, q_lat, 512, n_heads, n_tokens, kBM, bn, true);
  if (st != MLA_OK) return st;
  // shared memory: 1 KB alignment slack + weight tile + token chunks (the output
  // tile reuses them) + barriers, padded so that at most 512 / cols CTAs share an
  // SM and their TMEM allocations always fit together
  const int smem = pad_smem_for_tmem(1024 + 2 * kATileBytes + 2 * bn * 128 + 64, (int)tmem_cols_for(bn));
  GemmParams p{n_tokens, n_heads, bn, 0};
  cudaError_t e = set_smem_attrs();
  if (e == cudaSuccess) {
    e = launch_pdl(absorb_q_kernel, dim3(512 / kBM, n_heads, tiles), dim3(128), smem, stream, tw, tx, to, p);
    if (e == cudaSuccess) e = cudaGetLastError();
  }
  if (e != cudaSuccess) return set_error(MLA_ERR_CUDA, "absorb_q launch: %s", cudaGetErrorString(e));
  return MLA_OK;
}

mla_status_t launch_out_uv(const void* o_lat, const void* w_uv, void* out, int n_tokens,
                           int n_heads, void* stream) {
  int tiles = 1;
  const int bn = token_tile(n_tokens, &tiles);
  CUtensorMap tw, tx, to;
  mla_status_t st = weight_map(&tw, w_uv, n_heads, kBK);   // 64 k rows x 64 v (MN-major)
  if (st == MLA_OK) st = act_map(&tx, o_lat, 512, n_heads, n_tokens, 64, bn, false);
  if (st == MLA_OK) st = act_map(&to, out, 128, n_heads, n_tokens, kBM, bn, true);
  if (st != MLA_OK) return st;
  const int stage_bytes = kATileBytes + bn * 128;
  int stages = (200 * 1024) / stage_bytes;
  if (stages > kMaxRing) stages = kMaxRing;
  const int smem = 1024 + stages * stage_bytes + (2 * kMaxRing + 1) * 8 + 16;
  GemmParams p{n_tokens, n_heads, bn, stages};
  cudaError_t e = set_smem_attrs();
  if (e == cudaSuccess) {
    e = launch_pdl(out_uv_kernel, dim3(1, n_heads, tiles), dim3(128), smem, stream, tw, tx, to, p);
    if (e == cudaSuccess) e = cudaGetLastError();
  }
  if (e != cudaSuccess) return set_error(MLA_ERR_CUDA, "out_uv launch: %s", cudaGetErrorString(e));
  return MLA_OK;
}

mla_status_t launch_quantize_weight_fp8(const void* w, int n_heads, bool transposed, void* codes, float* scales,
                                        void* stream) {
  auto wb = static_cast<const __nv_bfloat16*>(w);
  auto cs = static_cast<uint8_t*>(codes);
  auto st = static_cast<cudaStream_t>(stream);
  if (transposed) quantize_weight_kernel<true><<<dim3(4, n_heads), 128, 0, st>>>(wb, n_heads, cs, scales);
  else quantize_weight_kernel<false><<<dim3(4, n_heads), 128, 0, st>>>(wb, n_heads, cs, scales);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(MLA_ERR_CUDA, "quantize_weight launch: %s", cudaGetErrorString(e));
  return MLA_OK;
}

mla_status_t launch_quantize_rows_fp8(const void* x, long long rows, int cols, void* codes, float* scales,
                                      void* stream) {
  const long long n_vec = rows * (cols / 128);
  if (n_vec == 0) return MLA_OK;
  const long long blocks = (n_vec + 127) / 128;
  quantize_rows_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), 128, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(x), n_vec, static_cast<uint8_t*>(codes), scales);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(MLA_ERR_CUDA, "quantize_rows launch: %s", cudaGetErrorString(e));
  return MLA_OK;
}

mla_status_t launch_kv_quantize_fp8(const void* kv, const int32_t* slots, long long n, void* pool_fp8,
                                   long long pool_rows, int32_t* status, void* stream) {
  if (n == 0) return MLA_OK;
  const long long blocks = (4 * n + 127) / 128;
  kv_quantize_fp8_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), 128, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(kv), slots, n, static_cast<uint8_t*>(pool_fp8), pool_rows, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(MLA_ERR_CUDA, "kv_quantize_fp8 launch: %s", cudaGetErrorString(e));
  return MLA_OK;
}

mla_status_t launch_absorb_q_fp8(const void* q_nope, const void* w_codes, const float* w_scales, void* q_lat,
                                 int n_tokens, int n_heads, void* stream) {
  int tiles = 1;
  const int bn = token_tile_max(n_tokens, 128, &tiles);   // bf16 rows + codes stay within 3 CTAs per SM
  CUtensorMap tw, tx, to;
  const uint64_t wdims[2] = {128, (uint64_t)n_heads * 512};
  const uint64_t wstr[1] = {128};
  const uint32_t wbox[2] = {128, (uint32_t)kBM};
  mla_status_t st = encode_tmap_u8(&tw, w_codes, 2, wdims, wstr, wbox, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st == MLA_OK) st = act_map(&tx, q_nope, 128, n_heads, n_tokens, 64, bn, false);
  if (st == MLA_OK) st = act_map(&to, q_lat, 512, n_heads, n_tokens, kBM, bn, true);
  if (st != MLA_OK) return st;
  const int region = std::max(kATileBytes + 3 * bn * 128, bn * 256);
  const int smem = pad_smem_for_tmem(1024 + region + kMaxBN * 4 + 64, (int)tmem_cols_for(bn));
  GemmParams p{n_tokens, n_heads, bn, 0};
  cudaError_t e = set_smem_attrs_fp8();
  if (e == cudaSuccess) {
    e = launch_pdl(absorb_q_fp8_kernel, dim3(512 / kBM, n_heads, tiles), dim3(128), smem, stream, tw, tx, to,
                   w_scales, p);
    if (e == cudaSuccess) e = cudaGetLastError();
  }
  if (e != cudaSuccess) return set_error(MLA_ERR_CUDA, "absorb_q_fp8 launch: %s", cudaGetErrorString(e));
  return MLA_OK;
}

mla_status_t launch_out_uv_fp8(const void* o_lat, const void* w_codes, const float* w_scales, void* out,
                               int n_tokens, int n_heads, void* stream) {
  int tiles = 1;
  const int bn = token_tile_max(n_tokens, 128, &tiles);   // 4 accumulators of bn columns
  CUtensorMap tw, to;
  const uint64_t wdims[2] = {512, (uint64_t)n_heads * 128};
  const uint64_t wstr[1] = {512};
  const uint32_t wbox[2] = {128, (uint32_t)kBM};
  mla_status_t st = encode_tmap_u8(&tw, w_codes, 2, wdims, wstr, wbox, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st == MLA_OK) st = act_map(&to, out, 128, n_heads, n_tokens, kBM, bn, true);
  if (st != MLA_OK) return st;
  const int smem = pad_smem_for_tmem(1024 + 4 * kATileBytes + 4 * bn * 128 + 4 * 128 * 4 + 64,
                                     4 * (int)tmem_cols_for(bn));
  GemmParams p{n_tokens, n_heads, bn, 0};
  cudaError_t e = set_smem_attrs_fp8();
  if (e == cudaSuccess) {
    e = launch_pdl(out_uv_fp8_kernel, dim3(1, n_heads, tiles), dim3(128), smem, stream, tw, to,
                   static_cast<const __nv_bfloat16*>(o_lat), w_scales, p);
    if (e == cudaSuccess) e = cudaGetLastError();
  }
  if (e != cudaSuccess) return set_error(MLA_ERR_CUDA, "out_uv_fp8 launch: %s", cudaGetErrorString(e));
  return MLA_OK;
}

}  // namespace mla
