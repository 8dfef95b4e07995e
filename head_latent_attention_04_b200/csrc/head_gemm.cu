// Per-head projections of absorbed MLA on tcgen05 tensor cores.
//
//   mla_absorb_q : q_lat[n,h,:] = W_UK[:,h,:] q_nope[n,h,:]   (M = d_c = 512, K = d = 128)
//   mla_out_uv   : out[n,h,:]   = W_UV[:,h,:]^T o_lat[n,h,:]  (M = d_v = 128, K = d_c = 512)
//
// These are the Step-2 terms of the MLA matrix-absorption notes' order 2
// (2bshkd in section 2.2, 2bhsvk in section 3.2).  With decode batches the token
// count is small, so the GEMM is written "swap-AB": the weight slice of one
// head is the 128-row M operand and the tokens are the N operand (16..128 per
// CTA).  Reading W_UK / W_UV (16.8 MB each at 128 heads) dominates, as the
// izhida.com answer notes for the W_V product of a batched GEMV.
//
// One CTA per (head, token tile), covering all M tiles of that head (4 for
// W_UK, 1 for W_UV), so a 128-head batch runs as a single wave.  Warp 0
// streams (M tile, 64-wide K slice) pairs through a 4-stage TMA ring, warp 1
// issues tcgen05.mma into one TMEM accumulator of 128 lanes x BN columns per
// M tile, and all four warps drain them.
#include "mla_internal.h"
#include "ptx.cuh"
#include "tmap.h"

#include <cuda_bf16.h>

namespace mla {
namespace {

using namespace ptx;

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kStages = 4;
constexpr int kMaxBN = 128;
constexpr int kABytes = kBM * kBK * 2;       // 16 KB
constexpr int kBBytesMax = kMaxBN * kBK * 2; // 16 KB
constexpr int kSmemBytes = kStages * (kABytes + kBBytesMax) + 1024 /*align*/ + 256 /*barriers*/;

struct Params {
  __nv_bfloat16* out;
  int n_tokens;
  int n_heads;
  int m_total;   // 512 (absorb) or 128 (out_uv)
  int k_total;   // 128 (absorb) or 512 (out_uv)
  int bn;        // token tile, multiple of 16, <= 128
};

// kAMn: the weight operand is MN-major in shared memory (W_UV: v contiguous).
template <bool kAMn>
__global__ void __launch_bounds__(128, 1)
head_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kStages * kBBytesMax);
  uint64_t* empty = full + kStages;
  uint64_t* done = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = blockIdx.y, n0 = blockIdx.z * p.bn;
  const int k_chunks = p.k_total / kBK;
  const int m_tiles = p.m_total / kBM;
  const int k_steps = m_tiles * k_chunks;            // (m tile, k chunk) pairs, m-major
  const uint32_t tmem_cols = m_tiles == 1 ? 128u : 512u;
  const uint32_t b_bytes = p.bn * kBK * 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // producer
    for (int ks = 0; ks < k_steps; ++ks) {
      const int s = ks % kStages, mt = ks / k_chunks, kc = ks % k_chunks;
      if (ks >= kStages && !mbar_wait(&empty[s], ((ks / kStages) - 1) & 1, abort_flag)) {
        *abort_flag = 1;
        break;
      }
      mbar_arrive_expect_tx(&full[s], kABytes + b_bytes);
      if (kAMn) {
        // W_UV slice: 64 k-rows of 64 v each, two v halves
        tma_load_3d(sA + s * kABytes, &tmA, &full[s], 0, h, kc * kBK);
        tma_load_3d(sA + s * kABytes + kABytes / 2, &tmA, &full[s], 64, h, kc * kBK);
      } else {
        // W_UK slice: 128 latent rows of 64 d each
        tma_load_3d(sA + s * kABytes, &tmA, &full[s], kc * kBK, h, mt * kBM);
      }
      tma_load_3d(sB + s * kBBytesMax, &tmB, &full[s], kc * kBK, h, n0);
    }
  } else if (warp == 1 && lane == 0) {
    // MMA issuer
    const uint32_t idesc = idesc_bf16(kBM, p.bn, kAMn ? 1 : 0, 0);
    for (int ks = 0; ks < k_steps; ++ks) {
      const int s = ks % kStages, mt = ks / k_chunks, kc = ks % k_chunks;
      if (!mbar_wait(&full[s], (ks / kStages) & 1, abort_flag)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t a0 = smem_u32(sA + s * kABytes), b0 = smem_u32(sB + s * kBBytesMax);
#pragma unroll
      for (int kk = 0; kk < kBK / 16; ++kk) {
        const uint64_t ad = kAMn ? sdesc(a0 + kk * 2048, kABytes / 2, 1024, kSwizzle128B)
                                 : sdesc(a0 + kk * 32, 16, 1024, kSwizzle128B);
        const uint64_t bd = sdesc(b0 + kk * 32, 16, 1024, kSwizzle128B);
        mma_ss(tmem + mt * 128, ad, bd, idesc, (kc | kk) != 0);
      }
      mma_commit(&empty[s]);
    }
    mma_commit(done);
  }
  __syncwarp();

  // epilogue: thread = accumulator lane = output row mt*128 + 32*warp + lane
  const bool ok = __all_sync(0xffffffffu, mbar_wait(done, 0, abort_flag));
  tc_fence_after();
  if (ok) {
    const size_t row_stride = (size_t)p.n_heads * p.m_total;
    for (int mt = 0; mt < m_tiles; ++mt) {
      const int m = mt * kBM + warp * 32 + lane;
      for (int c = 0; c < p.bn; c += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + mt * 128 + c, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int n = n0 + c + j;
          if (c + j < p.bn && n < p.n_tokens)
            p.out[(size_t)n * row_stride + (size_t)h * p.m_total + m] =
                __float2bfloat16_rn(__uint_as_float(r[j]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  __syncwarp();
  if (warp == 1) tmem_dealloc(tmem, tmem_cols);
}

mla_status_t launch_head_gemm(bool a_mn, const void* weight, const void* act, void* out,
                              int n_tokens, int n_heads, int m_total, int k_total, void* stream) {
  const int bn = n_tokens >= kMaxBN ? kMaxBN : ((n_tokens + 15) / 16) * 16;
  CUtensorMap tA, tB;
  // weight [512][H][128] bf16: dims innermost-first (128, H, 512)
  const uint64_t wdims[3] = {128, (uint64_t)n_heads, 512};
  const uint64_t wstr[2] = {128 * 2, (uint64_t)n_heads * 128 * 2};
  const uint32_t wbox_k[3] = {64, 1, 128};   // W_UK: 128 latent rows x 64 d
  const uint32_t wbox_mn[3] = {64, 1, 64};   // W_UV: 64 k rows x 64 v
  mla_status_t st = encode_tmap_bf16(&tA, weight, 3, wdims, wstr, a_mn ? wbox_mn : wbox_k,
                                     CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != MLA_OK) return st;
  // activations [N][H][K] bf16
  const uint64_t adims[3] = {(uint64_t)k_total, (uint64_t)n_heads, (uint64_t)n_tokens};
  const uint64_t astr[2] = {(uint64_t)k_total * 2, (uint64_t)n_heads * k_total * 2};
  const uint32_t abox[3] = {64, 1, (uint32_t)bn};
  st = encode_tmap_bf16(&tB, act, 3, adims, astr, abox, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != MLA_OK) return st;

  Params p{static_cast<__nv_bfloat16*>(out), n_tokens, n_heads, m_total, k_total, bn};
  dim3 grid(1, n_heads, (n_tokens + bn - 1) / bn);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  // Attributes are set once per process (outside any later stream capture).
  static cudaError_t attr_mn = cudaFuncSetAttribute(
      head_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  static cudaError_t attr_k = cudaFuncSetAttribute(
      head_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  e = a_mn ? attr_mn : attr_k;
  if (e == cudaSuccess) {
    if (a_mn)
      head_gemm_kernel<true><<<grid, 128, kSmemBytes, s>>>(tA, tB, p);
    else
      head_gemm_kernel<false><<<grid, 128, kSmemBytes, s>>>(tA, tB, p);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return set_error(MLA_ERR_CUDA, "head_gemm launch: %s", cudaGetErrorString(e));
  return MLA_OK;
}

}  // namespace

mla_status_t launch_absorb_q(const void* q_nope, const void* w_uk, void* q_lat, int n_tokens,
                             int n_heads, void* stream) {
  return launch_head_gemm(false, w_uk, q_nope, q_lat, n_tokens, n_heads, 512, 128, stream);
}

mla_status_t launch_out_uv(const void* o_lat, const void* w_uv, void* out, int n_tokens,
                           int n_heads, void* stream) {
  return launch_head_gemm(true, w_uv, o_lat, out, n_tokens, n_heads, 128, 512, stream);
}

}  // namespace mla
