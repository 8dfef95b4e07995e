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
#include "mla_internal.h"
#include "ptx.cuh"
#include "tmap.h"

#include <cuda_bf16.h>

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
  int smem = 1024 + 2 * kATileBytes + 2 * bn * 128 + 64;
  const int ctas_per_sm = 512 / (int)tmem_cols_for(bn);
  const int floor_bytes = kSmemPerSM / (ctas_per_sm + 1) - 1024 + 1;
  if (smem < floor_bytes) smem = floor_bytes;
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

}  // namespace mla
