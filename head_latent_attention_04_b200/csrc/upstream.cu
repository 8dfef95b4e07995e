// The products upstream of the absorbed decode path, fused on sm_100a.
//
// mla_q_up_absorb: per head h, the query up-projection and the first
//   absorption back to back, q_nope never leaving the SM:
//     q_h     = c^Q W^UQ_h           (notes section 2.1 Step 1, term 2bshdq;
//                                     W^UQ carries the head's RoPE columns too)
//     q_lat_h = q_nope_h W^UK_h^T    (section 2.2 Step 2, term 2bshkd)
//   One CTA per (head, token tile of at most 128).  GEMM 1 (swap-AB: M = 128
//   nope features and, in a second accumulator, the 64 RoPE features;
//   N = tokens; K = 1536) streams W^UQ and c^Q through a three-stage ring.
//   Its nope result is converted to bf16 into shared memory as the B operand
//   of GEMM 2 (M = 512 latent rows in four 128-row tiles, K = 128), whose
//   W^UK tiles load into the drained ring meanwhile; the RoPE part goes out
//   by a TMA store.  W^UQ^T W^UK is never formed (no pre-absorption).
//
// mla_qkv_a_proj: the Perplexity write-up's fused qkv_a_proj (section "MLA
//   layer": q_a_proj and kv_a_proj merged, 30.2 -> 16.7 us on H100): one
//   product of the hidden states x [N][7168] with the concatenated
//   down-projection [W^DQ | W^DKV] (2112 output features) gives c^Q [N][1536]
//   and the cache row [c^KV | k_rope] [N][576].  With decode batches the
//   weight read (30 MB) dominates, so the 112 K-chunks are split over a
//   cluster of CTAs: 8 when the tokens fit one tile of 128 (17 x 8 = 136
//   CTAs), else 4 per tile (17 x 4 x tiles).  Each CTA streams its K-chunks
//   through a ring of at most 104 KB (3 stages at 128 tokens, 5 at 16), so two
//   CTAs share an SM and the whole grid is resident; it accumulates in TMEM,
//   sends row slices of its partial tile to the CTA that owns them through
//   distributed shared memory, and each CTA sums the partials of its 16 or 32
//   rows and writes them.  (One CTA per SM with clusters of 8 left a second
//   wave: a GPC holds only two such clusters.)
#include "mla_internal.h"
#include "ptx.cuh"
#include "tmap.h"

#include <cuda_bf16.h>

namespace mla {
namespace {

using namespace ptx;

constexpr int kT = 128;                // token tile
constexpr int kA = 128 * 64 * 2;       // 16 KB: 128 rows x 64 K (SW128)
constexpr int kQStages = 3;
constexpr int kQLora = 1536, kDimE = 7168, kKvA = 576, kQkvOut = kQLora + kKvA;   // 2112

__host__ __device__ constexpr int ring_stage(int bn) { return 2 * kA + bn * 128; }
// the ring also takes GEMM 2's four W^UK tiles (4 x 32 KB) once GEMM 1 has drained it
__host__ __device__ constexpr int ring_bytes(int bn) {
  return kQStages * ring_stage(bn) > 8 * kA ? kQStages * ring_stage(bn) : 8 * kA;
}

__device__ __forceinline__ void tile_out(uint32_t tmem, uint8_t* s_out, int bn, const CUtensorMap* tm, int x, int h,
                                         int n0) {
  // TMEM [128 lanes][bn] fp32 -> bf16 smem [bn][128] -> one TMA store at (x, h, n0)
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(s_out);
  const int m = warp * 32 + lane;
  for (int c = 0; c < bn; c += 32) {
    uint32_t r[32];
    tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c, r);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (c + j < bn) o[(c + j) * 128 + m] = __float2bfloat16_rn(__uint_as_float(r[j]));
  }
  fence_proxy_async_smem();
  __syncthreads();
  if (threadIdx.x == 0) {
    tma_store_3d(tm, s_out, x, h, n0);
    bulk_commit();
    bulk_wait_all<0>();
  }
  __syncthreads();
}

struct QUpParams {
  int n_tokens, bn;
};

__global__ void __launch_bounds__(128, 1)
q_up_absorb_kernel(const __grid_constant__ CUtensorMap tm_uq, const __grid_constant__ CUtensorMap tm_cq,
                   const __grid_constant__ CUtensorMap tm_uk, const __grid_constant__ CUtensorMap tm_qlat,
                   const __grid_constant__ CUtensorMap tm_qrope, const QUpParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int bn = p.bn;
  const int stage = ring_stage(bn);
  uint8_t* ring = smem;                                   // kQStages x stage; later W^UK (4 x 32 KB)
  uint8_t* sB2 = smem + ring_bytes(bn);                   // q_nope bf16: 2 chunks x bn x 128 B (SW128)
  uint8_t* sR = sB2 + 2 * bn * 128;                       // q_rope bf16 [bn][64]
  uint64_t* full = reinterpret_cast<uint64_t*>(sR + bn * 128);
  uint64_t* empty = full + kQStages;
  uint64_t* done1 = empty + kQStages;
  uint64_t* wfull = done1 + 1;
  uint64_t* done2 = wfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done2 + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = blockIdx.y, n0 = blockIdx.z * bn;
  const uint32_t cols = bn <= 32 ? 128u : bn <= 64 ? 256u : 512u;   // four bn-wide accumulators
  constexpr int kChunks = kQLora / 64;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done1, 1);
    mbar_init(wfull, 1);
    mbar_init(done2, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_uq);
    prefetch_tmap(&tm_cq);
    prefetch_tmap(&tm_uk);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();
  griddep_launch_dependents();

  // ---------------- GEMM 1: D_nope [128 x bn] at column 0, D_rope [128 x bn] at column bn
  if (warp == 0 && lane == 0) {
    for (int kc = 0; kc < kChunks; ++kc) {
      const int s = kc % kQStages;
      if (kc >= kQStages && !mbar_wait(&empty[s], ((kc / kQStages) - 1) & 1, abort_flag)) {
        *abort_flag = 1;
        break;
      }
      uint8_t* st = ring + s * stage;
      mbar_arrive_expect_tx(&full[s], kA + kA / 2 + bn * 128);
      tma_load_3d(st, &tm_uq, &full[s], 0, h, kc * 64);             // nope features 0..63 (MN-major)
      tma_load_3d(st + kA / 2, &tm_uq, &full[s], 64, h, kc * 64);   // nope features 64..127
      tma_load_3d(st + kA, &tm_uq, &full[s], 128, h, kc * 64);      // RoPE features 0..63
      tma_load_2d(st + 2 * kA, &tm_cq, &full[s], kc * 64, n0);      // c^Q: bn tokens x 64
    }
    // GEMM 2's W^UK tiles go into the ring once GEMM 1 has drained it
    if (!*abort_flag && mbar_wait(done1, 0, abort_flag)) {
      mbar_arrive_expect_tx(wfull, 4 * 2 * kA);
      for (int m = 0; m < 4; ++m)
        for (int c = 0; c < 2; ++c)
          tma_load_3d(ring + m * 2 * kA + c * kA, &tm_uk, wfull, 64 * c, h, 128 * m);
    } else {
      *abort_flag = 1;
    }
  } else if (warp == 1 && lane == 0) {
    const uint32_t idesc = idesc_bf16(128, bn, 1, 0);
    for (int kc = 0; kc < kChunks; ++kc) {
      const int s = kc % kQStages;
      if (!mbar_wait(&full[s], (kc / kQStages) & 1, abort_flag)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t a0 = smem_u32(ring + s * stage), b0 = a0 + 2 * kA;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t bd = sdesc(b0 + kk * 32, 16, 1024, kSwizzle128B);
        mma_ss(tmem, sdesc(a0 + kk * 2048, kA / 2, 1024, kSwizzle128B), bd, idesc, (kc | kk) != 0);
        // the RoPE tile's rows 64..127 read stale shared memory; those rows are not used
        mma_ss(tmem + bn, sdesc(a0 + kA + kk * 2048, kA / 2, 1024, kSwizzle128B), bd, idesc, (kc | kk) != 0);
      }
      mma_commit(&empty[s]);
    }
    mma_commit(done1);
  }
  __syncwarp();
  bool ok = __syncthreads_and(mbar_wait(done1, 0, abort_flag) && !*abort_flag);
  tc_fence_after();

  // ---------------- q_nope -> bf16 B operand of GEMM 2; q_rope -> its output
  if (ok) {
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const int d = warp * 32 + lane;                       // feature row = TMEM lane
    for (int c = 0; c < bn; c += 32) {
      uint32_t r[32];
      tmem_ld32(tmem + lane_base + c, r);
      tmem_ld_wait();
      uint8_t* base = sB2 + (d >> 6) * (bn * 128) + 2 * (d & 7);
      const int u = (d & 63) >> 3;                         // 16-byte unit of the 128-byte row
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int t = c + j;
        if (t < bn)
          *reinterpret_cast<__nv_bfloat16*>(base + t * 128 + ((u ^ (t & 7)) << 4)) = __float2bfloat16_rn(__uint_as_float(r[j]));
      }
    }
    if (warp < 2) {                                        // RoPE features 0..63 live in lanes 0..63
      for (int c = 0; c < bn; c += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + bn + c, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c + j < bn)
            reinterpret_cast<__nv_bfloat16*>(sR)[(c + j) * 64 + d] = __float2bfloat16_rn(__uint_as_float(r[j]));
      }
    } else {
      uint32_t r[32];   // the other quarters take part in the aligned loads of their lanes
      for (int c = 0; c < bn; c += 32) {
        tmem_ld32(tmem + lane_base + bn + c, r);
        tmem_ld_wait();
      }
    }
    fence_proxy_async_smem();   // sB2 is read by the tensor cores, sR by the TMA store
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  if (ok && threadIdx.x == 0) {
    tma_store_3d(&tm_qrope, sR, 0, h, n0);
    bulk_commit();
  }

  // ---------------- GEMM 2: q_lat^T tile m [128 latent rows x bn] at column m * bn
  if (ok && warp == 1 && lane == 0) {
    if (mbar_wait(wfull, 0, abort_flag)) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16(128, bn, 0, 0);
      for (int m = 0; m < 4; ++m)
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tmem + m * bn, sdesc(smem_u32(ring + m * 2 * kA + c * kA) + kk * 32, 16, 1024, kSwizzle128B),
                   sdesc(smem_u32(sB2 + c * bn * 128) + kk * 32, 16, 1024, kSwizzle128B), idesc, (c | kk) != 0);
    } else {
      *abort_flag = 1;
    }
    mma_commit(done2);
  }
  __syncwarp();
  ok = __syncthreads_and(ok && mbar_wait(done2, 0, abort_flag) && !*abort_flag);
  tc_fence_after();
  if (ok)
    for (int m = 0; m < 4; ++m) tile_out(tmem + m * bn, ring, bn, &tm_qlat, 128 * m, h, n0);
  if (threadIdx.x == 0) bulk_wait_all<0>();   // the q_rope store has read sR
  tc_fence_before();
  __syncthreads();
  __syncwarp();
  if (warp == 1) tmem_dealloc(tmem, cols);
}

// ----------------------------------------------------------------- fused qkv_a_proj
// KS CTAs of a cluster, one K range each: 8 for token tiles of up to 128
// tokens when the batch has one tile (136 CTAs), 4 when it has more (17 x 4 x
// tiles CTAs).  Either way the ring stays under half of an SM's shared memory,
// so two CTAs share an SM and every cluster of the grid is resident at once.
constexpr int kQkvChunks = kDimE / 64;       // 112
constexpr int kQkvMaxStages = 8;
constexpr int kQkvRingBudget = 104 * 1024;   // the ring takes as many stages as fit
constexpr int kQkvT = 128;                   // token tile

struct QkvParams {
  __nv_bfloat16* c_q;    // [N][1536]
  __nv_bfloat16* kv_a;   // [N][576]
  int n_tokens, bn, stages, region;   // region: bytes of the ring / receive area before the barriers
};

template <int KS>
__global__ void __cluster_dims__(1, 1, KS) __launch_bounds__(128, 1)
qkv_a_proj_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                  const QkvParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int bn = p.bn, S = p.stages;
  const int stage = kA + bn * 128;
  uint8_t* ring = smem;                    // later: the partial slices received from the cluster
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.region);
  uint64_t* empty = full + kQkvMaxStages;
  uint64_t* done = empty + kQkvMaxStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const int mt = blockIdx.x, n0 = blockIdx.y * bn;
  const uint32_t cols = bn <= 32 ? 32u : bn <= 64 ? 64u : 128u;
  constexpr int kPer = kQkvChunks / KS;       // K chunks per CTA (14 or 28)
  constexpr int kRowsPer = 128 / KS;          // output rows reduced and written by each CTA
  const int kc0 = (int)rank * kPer;

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
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();
  griddep_launch_dependents();

  if (warp == 0 && lane == 0) {
    for (int i = 0; i < kPer; ++i) {
      const int s = i % S;
      if (i >= S && !mbar_wait(&empty[s], ((i / S) - 1) & 1, abort_flag)) {
        *abort_flag = 1;
        break;
      }
      uint8_t* st = ring + s * stage;
      mbar_arrive_expect_tx(&full[s], stage);
      tma_load_2d(st, &tm_w, &full[s], (kc0 + i) * 64, mt * 128);    // 128 output rows x 64 K
      tma_load_2d(st + kA, &tm_x, &full[s], (kc0 + i) * 64, n0);     // bn tokens x 64 K
    }
  } else if (warp == 1 && lane == 0) {
    const uint32_t idesc = idesc_bf16(128, bn, 0, 0);
    for (int i = 0; i < kPer; ++i) {
      const int s = i % S;
      if (!mbar_wait(&full[s], (i / S) & 1, abort_flag)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t a0 = smem_u32(ring + s * stage), b0 = a0 + kA;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(tmem, sdesc(a0 + kk * 32, 16, 1024, kSwizzle128B), sdesc(b0 + kk * 32, 16, 1024, kSwizzle128B), idesc,
               (i | kk) != 0);
      mma_commit(&empty[s]);
    }
    mma_commit(done);
  }
  __syncwarp();
  const bool ok = __syncthreads_and(mbar_wait(done, 0, abort_flag) && !*abort_flag);
  tc_fence_after();
  cluster_sync();   // every CTA of the cluster is done with its ring before slices land in it

  // ---------------- exchange: row m of the partial tile goes to CTA m / kRowsPer, slot `rank`
  // receive area: [KS slots][kRowsPer rows][bn] fp32 in the (drained) ring
  float* recv = reinterpret_cast<float*>(ring);
  if (ok) {
    const int m = warp * 32 + lane;
    const uint32_t dst = mapa(smem_u32(recv + ((size_t)rank * kRowsPer + m % kRowsPer) * bn), (uint32_t)(m / kRowsPer));
    for (int c = 0; c < bn; c += 32) {
      uint32_t r[32];
      tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c, r);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; j += 4)
        if (c + j < bn)
          asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst + 4u * (c + j)), "r"(r[j]),
                       "r"(r[j + 1]), "r"(r[j + 2]), "r"(r[j + 3])
                       : "memory");
    }
  }
  tc_fence_before();
  cluster_sync();   // every slice has landed (release / acquire at cluster scope)
  if (ok) {
    // thread t: token n0 + t, rows kRowsPer rank .. kRowsPer (rank + 1) - 1 of the tile, 16 at a time
    const int f_base = mt * 128 + kRowsPer * (int)rank;   // first output feature of this slice
    for (int t = threadIdx.x; t < bn && f_base < kQkvOut; t += 128) {
      const int n = n0 + t;
      if (n >= p.n_tokens) continue;
#pragma unroll 1
      for (int hf = 0; hf < kRowsPer / 16; ++hf) {
        float acc[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] = 0.f;
#pragma unroll 1
        for (int sl = 0; sl < KS; ++sl)
#pragma unroll
          for (int i = 0; i < 16; ++i) acc[i] += recv[((size_t)sl * kRowsPer + 16 * hf + i) * bn + t];
        const int f0 = f_base + 16 * hf;
        uint32_t pk[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) pk[i] = pack_bf16(acc[2 * i], acc[2 * i + 1]);
        __nv_bfloat16* dst = f0 < kQLora ? p.c_q + (size_t)n * kQLora + f0 : p.kv_a + (size_t)n * kKvA + (f0 - kQLora);
        reinterpret_cast<uint4*>(dst)[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        reinterpret_cast<uint4*>(dst)[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  __syncwarp();
  if (warp == 1) tmem_dealloc(tmem, cols);
  cluster_sync();
}

cudaError_t upstream_attrs(int smem_q, int smem_qkv) {
  static cudaError_t e = [=] {
    cudaError_t a = cudaFuncSetAttribute(q_up_absorb_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
    cudaError_t b = cudaFuncSetAttribute(qkv_a_proj_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
    cudaError_t c = cudaFuncSetAttribute(qkv_a_proj_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
    return a != cudaSuccess ? a : b != cudaSuccess ? b : c;
  }();
  (void)smem_q;
  (void)smem_qkv;
  return e;
}

int tile_tokens(int n, int* tiles) {
  *tiles = (n + kT - 1) / kT;
  const int per = (n + *tiles - 1) / *tiles;
  return ((per + 15) / 16) * 16;
}

}  // namespace

mla_status_t launch_q_up_absorb(const void* c_q, const void* w_uq, const void* w_uk, void* q_lat, void* q_rope,
                                int n_tokens, int n_heads, void* stream) {
  int tiles = 1;
  const int bn = tile_tokens(n_tokens, &tiles);
  CUtensorMap tuq, tcq, tuk, tql, tqr;
  {
    const uint64_t dims[3] = {192, (uint64_t)n_heads, kQLora};
    const uint64_t str[2] = {192 * 2, (uint64_t)n_heads * 192 * 2};
    const uint32_t box[3] = {64, 1, 64};
    mla_status_t st = encode_tmap_bf16(&tuq, w_uq, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != MLA_OK) return st;
  }
  {
    const uint64_t dims[2] = {kQLora, (uint64_t)n_tokens};
    const uint64_t str[1] = {kQLora * 2};
    const uint32_t box[2] = {64, (uint32_t)bn};
    mla_status_t st = encode_tmap_bf16(&tcq, c_q, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != MLA_OK) return st;
  }
  {
    const uint64_t dims[3] = {128, (uint64_t)n_heads, 512};
    const uint64_t str[2] = {128 * 2, (uint64_t)n_heads * 128 * 2};
    const uint32_t box[3] = {64, 1, 128};
    mla_status_t st = encode_tmap_bf16(&tuk, w_uk, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != MLA_OK) return st;
  }
  {
    const uint64_t dims[3] = {512, (uint64_t)n_heads, (uint64_t)n_tokens};
    const uint64_t str[2] = {512 * 2, (uint64_t)n_heads * 512 * 2};
    const uint32_t box[3] = {128, 1, (uint32_t)bn};
    mla_status_t st = encode_tmap_bf16(&tql, q_lat, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != MLA_OK) return st;
  }
  {
    const uint64_t dims[3] = {64, (uint64_t)n_heads, (uint64_t)n_tokens};
    const uint64_t str[2] = {64 * 2, (uint64_t)n_heads * 64 * 2};
    const uint32_t box[3] = {64, 1, (uint32_t)bn};
    mla_status_t st = encode_tmap_bf16(&tqr, q_rope, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != MLA_OK) return st;
  }
  const int smem = 1024 + ring_bytes(bn) + 3 * bn * 128 + 256;
  QUpParams p{n_tokens, bn};
  cudaError_t e = upstream_attrs(0, 0);
  if (e == cudaSuccess) {
    e = launch_pdl(q_up_absorb_kernel, dim3(1, n_heads, tiles), dim3(128), smem, stream, tuq, tcq, tuk, tql, tqr, p);
    if (e == cudaSuccess) e = cudaGetLastError();
  }
  if (e != cudaSuccess) return set_error(MLA_ERR_CUDA, "q_up_absorb launch: %s", cudaGetErrorString(e));
  return MLA_OK;
}

mla_status_t launch_qkv_a_proj(const void* x, const void* w, void* c_q, void* kv_a, int n_tokens, void* stream) {
  const int tiles = (n_tokens + kQkvT - 1) / kQkvT;
  const int per = (n_tokens + tiles - 1) / tiles;
  const int bn = ((per + 15) / 16) * 16;    // near-equal token tiles of at most 128, multiples of 16
  const int ks = tiles == 1 ? 8 : 4;
  CUtensorMap tw, tx;
  {
    const uint64_t dims[2] = {kDimE, kQkvOut};
    const uint64_t str[1] = {kDimE * 2};
    const uint32_t box[2] = {64, 128};
    mla_status_t st = encode_tmap_bf16(&tw, w, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != MLA_OK) return st;
  }
  {
    const uint64_t dims[2] = {kDimE, (uint64_t)n_tokens};
    const uint64_t str[1] = {kDimE * 2};
    const uint32_t box[2] = {64, (uint32_t)bn};
    mla_status_t st = encode_tmap_bf16(&tx, x, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != MLA_OK) return st;
  }
  const int stage = kA + bn * 128;
  int stages = kQkvRingBudget / stage;
  if (stages > kQkvMaxStages) stages = kQkvMaxStages;
  const int ring = stages * stage;
  const int recv = 128 * bn * 4;            // KS slots x (128 / KS) rows x bn fp32
  const int region = ring > recv ? ring : recv;
  const int smem = 1024 + region + 256;
  QkvParams p{static_cast<__nv_bfloat16*>(c_q), static_cast<__nv_bfloat16*>(kv_a), n_tokens, bn, stages, region};
  cudaError_t e = upstream_attrs(0, 0);
  if (e == cudaSuccess) {
    const dim3 grid((kQkvOut + 127) / 128, tiles, ks);
    e = ks == 8 ? launch_pdl(qkv_a_proj_kernel<8>, grid, dim3(128), smem, stream, tw, tx, p)
                : launch_pdl(qkv_a_proj_kernel<4>, grid, dim3(128), smem, stream, tw, tx, p);
    if (e == cudaSuccess) e = cudaGetLastError();
  }
  if (e != cudaSuccess) return set_error(MLA_ERR_CUDA, "qkv_a_proj launch: %s", cudaGetErrorString(e));
  return MLA_OK;
}

}  // namespace mla
