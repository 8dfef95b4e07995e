// Log-sum-exp merge of split-KV pieces, and a bit-exact page-gather check kernel.
//
// A row cut into pieces i = 1..m by the planner has per-piece normalised
// outputs O_i and natural-log LSEs lse_i.  Softmax over the union of the
// pieces' keys is
//   L = log sum_i exp(lse_i),   o = sum_i exp(lse_i - L) O_i,
// the identity the oracle's split-merge pin checks.
//
// The pieces live in the column-group-major workspace the attention kernel
// writes: element (slot, h, col) of O_i sits at
//   ((slot * 64 + col / 8) * n_heads + h) * 8 + col % 8,
// so that 32 consecutive heads of one 8-column group are 1 KB contiguous.
// HBM-bound.  Thread (h, grp) of a block merges 8-column groups grp,
// grp + 4, ... (G of them) of one row, with consecutive h reading
// consecutive 32-byte groups (coalesced).  The pieces are merged in one pass,
// P at a time with all their loads in flight.  G is picked on the host so that
// the grid is about one wave of the SMs (few rows: small G, many blocks; many
// rows: large G, up to 4), and P = 4 / G, so that every thread keeps 8
// 16-byte words in flight and two blocks fit on an SM.  Blocks of rows that
// were not split exit at once.
#include "mla_internal.h"
#include "plan_format.h"
#include "ptx.cuh"

#include <cuda_bf16.h>
#include <math_constants.h>

namespace mla {
namespace {

constexpr int kCombineThreads = 512;   // 128 heads x 4 column-group lanes

template <int G, int P>
__global__ void __launch_bounds__(kCombineThreads, G == 4 ? 1 : 2)
mla_combine_kernel(const int32_t* __restrict__ plan, const float* __restrict__ o_part,
                   const float* __restrict__ lse_part, __nv_bfloat16* __restrict__ o_lat,
                   float* __restrict__ lse_out, int n_heads) {
  ptx::griddep_wait();   // the attention kernel's partials are complete and visible
  ptx::griddep_launch_dependents();
  const int n = blockIdx.x;
  const int h = threadIdx.x & 127;
  const int grp = threadIdx.x >> 7;
  if (h >= n_heads) return;
  const int32_t* rs = plan + plan[kHdrOffRows];
  const int s0 = rs[n], s1 = rs[n + 1];
  if (s1 <= s0) return;   // row written whole by the attention kernel

  // 8-column group of lane i: g0 + 4 i.  Running maximum of the LSEs, sums
  // rescaled when it grows.
  const int g0 = blockIdx.y * (4 * G) + grp;
  const float4* src = reinterpret_cast<const float4*>(o_part) + ((size_t)g0 * n_heads + h) * 2;
  const size_t slot_stride = (size_t)64 * n_heads * 2;      // float4s per slot
  const size_t lane_stride = (size_t)4 * n_heads * 2;       // float4s between this thread's groups
  float m = -CUDART_INF_F, z = 0.f;
  float4 acc[G][2];
#pragma unroll
  for (int i = 0; i < G; ++i) acc[i][0] = acc[i][1] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = s0; s < s1; s += P) {
    float l[P];
    float4 v[P][G][2];
#pragma unroll
    for (int k = 0; k < P; ++k) {
      const bool in = s + k < s1;
      l[k] = in ? __ldg(lse_part + (size_t)(s + k) * n_heads + h) : -CUDART_INF_F;
#pragma unroll
      for (int i = 0; i < G; ++i)
#pragma unroll
        for (int e = 0; e < 2; ++e)
          v[k][i][e] = in ? __ldg(src + (size_t)(s + k) * slot_stride + i * lane_stride + e)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float lm = l[0];
#pragma unroll
    for (int k = 1; k < P; ++k) lm = fmaxf(lm, l[k]);
    const float m_new = fmaxf(m, lm);
    if (m_new == -CUDART_INF_F) continue;
    const float r = (m == -CUDART_INF_F) ? 0.f : __expf(m - m_new);
    z *= r;
#pragma unroll
    for (int i = 0; i < G; ++i)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        acc[i][e].x *= r; acc[i][e].y *= r; acc[i][e].z *= r; acc[i][e].w *= r;
      }
#pragma unroll
    for (int k = 0; k < P; ++k) {
      const float wgt = (l[k] == -CUDART_INF_F) ? 0.f : __expf(l[k] - m_new);
      z += wgt;
#pragma unroll
      for (int i = 0; i < G; ++i)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          acc[i][e].x += wgt * v[k][i][e].x; acc[i][e].y += wgt * v[k][i][e].y;
          acc[i][e].z += wgt * v[k][i][e].z; acc[i][e].w += wgt * v[k][i][e].w;
        }
    }
    m = m_new;
  }
  const float inv_z = z > 0.f ? 1.f / z : 0.f;
  __nv_bfloat16* dst = o_lat + ((size_t)n * n_heads + h) * 512 + 8 * g0;
#pragma unroll
  for (int i = 0; i < G; ++i)
    *reinterpret_cast<uint4*>(dst + 32 * i) =
        make_uint4(ptx::pack_bf16(acc[i][0].x * inv_z, acc[i][0].y * inv_z),
                   ptx::pack_bf16(acc[i][0].z * inv_z, acc[i][0].w * inv_z),
                   ptx::pack_bf16(acc[i][1].x * inv_z, acc[i][1].y * inv_z),
                   ptx::pack_bf16(acc[i][1].z * inv_z, acc[i][1].w * inv_z));
  if (lse_out && blockIdx.y == 0 && grp == 0)
    lse_out[(size_t)n * n_heads + h] = z > 0.f ? m + __logf(z) : -CUDART_INF_F;
}

__global__ void mla_gather_pages_kernel(const uint4* __restrict__ pool, const int32_t* __restrict__ bt,
                                        int b, int n_pages, int max_blocks, int num_blocks,
                                        uint4* __restrict__ out, int32_t* status) {
  constexpr int kPageVec = 64 * 576 * 2 / 16;   // 16-byte words per page
  const int pg = blockIdx.x;
  if (pg >= n_pages) return;
  const int blk = bt[(size_t)b * max_blocks + pg];
  const bool ok = blk >= 0 && blk < num_blocks;
  if (!ok && threadIdx.x == 0 && status) atomicOr(status, MLA_STATUS_BAD_BLOCK);
  for (int i = threadIdx.x; i < kPageVec; i += blockDim.x)
    out[(size_t)pg * kPageVec + i] = ok ? pool[(size_t)blk * kPageVec + i] : make_uint4(0, 0, 0, 0);
}

}  // namespace

mla_status_t launch_combine(const mla_dims_t& d, const int32_t* plan_dev, int32_t n_rows,
                            const float* o_part, const float* lse_part, void* o_lat,
                            float* lse_out, void* stream) {
  // Column groups per thread: the smallest G with n_rows x 32 / G blocks within
  // about one wave (2 blocks of 512 threads per SM).
  static const int sms = [] {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = 148;
    }
    return n;
  }();
  const long long wave = 2LL * sms;
  int G = 1;
  while (G < 4 && (long long)n_rows * (16 / G) > wave) G *= 2;
  dim3 grid(n_rows, 16 / G);
  auto bf = static_cast<__nv_bfloat16*>(o_lat);
  cudaError_t e;
  switch (G) {
    case 1: e = launch_pdl(mla_combine_kernel<1, 4>, grid, dim3(kCombineThreads), 0, stream, plan_dev, o_part, lse_part, bf, lse_out, d.n_heads); break;
    case 2: e = launch_pdl(mla_combine_kernel<2, 2>, grid, dim3(kCombineThreads), 0, stream, plan_dev, o_part, lse_part, bf, lse_out, d.n_heads); break;
    default: e = launch_pdl(mla_combine_kernel<4, 1>, grid, dim3(kCombineThreads), 0, stream, plan_dev, o_part, lse_part, bf, lse_out, d.n_heads); break;
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(MLA_ERR_CUDA, "combine launch: %s", cudaGetErrorString(e));
  return MLA_OK;
}

mla_status_t launch_gather_pages(const void* kv_pool, const int32_t* block_table, int32_t b,
                                 int32_t n_pages, int32_t max_blocks, int32_t num_blocks, void* out,
                                 int32_t* status, void* stream) {
  if (n_pages <= 0) return MLA_OK;
  mla_gather_pages_kernel<<<n_pages, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(kv_pool), block_table, b, n_pages, max_blocks, num_blocks,
      static_cast<uint4*>(out), status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(MLA_ERR_CUDA, "gather launch: %s", cudaGetErrorString(e));
  return MLA_OK;
}

}  // namespace mla
