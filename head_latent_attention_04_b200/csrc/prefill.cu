// Prefill / chunked prefill of MLA in order 1 ("MHA form") on sm_100a.
//
// "MLA Matrix Absorption Analysis" section 2.4.1 compares the evaluation
// orders of the first absorption: when the query length equals the key
// length (t = s, prefill) order 1 needs fewer FLOPs than the absorbed order
// (by 98304 s^2 at DeepSeek-V3 widths); the Perplexity write-up's future-work
// section names prefill in the up-projected form and chunked prefill.  So
// prefill up-projects the latent cache once per sequence,
//   K[t,h,:] = W_UK[:,h,:]^T c_KV[t]     (notes section 2.1 Step 2)
//   V[t,h,:] = W_UV[:,h,:]^T c_KV[t]     (notes section 3.1 Step 1)
// and runs causal multi-head attention with the RoPE key shared by all heads:
//   logit[i,h,t] = scale (q_nope[i,h] . K[t,h] + q_rope[i,h] . k_rope[t])
//   out[i,h,:]   = sum_t softmax_t(logit) V[t,h,:]     over t <= T - s + i
// (the s new tokens of a chunk are already in the cache and sit at positions
// T - s .. T - 1, so a chunk of s < T tokens is chunked prefill).
//
// up_proj_kernel: one CTA per (128-token tile, head) makes both K and V from one
//   staged c_KV tile: a tcgen05 GEMM with M = 128 tokens (two cache pages, read
//   through the block table by TMA from the (column, row, block) view of the
//   pool), N = 256 (the head's 128 W_UK and 128 W_UV features), K = 512 latent
//   columns streamed through a two-stage ring (two CTAs per SM); tokens on
//   TMEM lanes, so each thread packs its token's rows in the SW128 layout of
//   the output boxes and four TMA stores write K and V [T][h][128] bf16.
// prefill_attn_kernel: one CTA per (128-query tile, head).  Warp 0 stages
//   K + k_rope and V tiles of 128 keys through a three-stage and a two-stage
//   ring (a K stage is released by its QK product, a V stage by its PV
//   product); the softmax warps put the Q tile into TMEM once; warp 1 issues
//   S = Q K^T (M = 128 queries, N = 128 keys, K = 192: 8 MMAs on K, 4 on
//   k_rope, A = Q from TMEM) into a single S buffer; warp 2 issues
//   O += P V (M = 128, N = 128, K = 128 keys: 8 MMAs) from two P buffers;
//   warps 3-10 run the online softmax, two threads per query row (TMEM lane
//   quarter = warp % 4, one 64-key half each, their maxima and sums combined
//   through shared memory), with the causal mask on the diagonal tiles and a
//   lazy reference maximum, and write the normalised rows.
// TMEM (512 columns): S [0,128) fp32, P [128,192) and [192,256) bf16 pairs,
// O [256,384) fp32, Q [384,480) bf16 pairs.
#include "mla_internal.h"
#include "ptx.cuh"
#include "tmap.h"

#include <cuda_bf16.h>
#include <math_constants.h>

namespace mla {
namespace {

using namespace ptx;

constexpr int kTile = 128;                 // tokens per tile (queries, keys, up-projection)
constexpr int kChunk = kTile * 128;        // 16 KB: 128 rows x 64 bf16 (SW128)
constexpr int kUpStages = 2;            // 97 KB: two CTAs per SM, so one's epilogue overlaps the other's loads
constexpr int kUpABytes = kChunk;          // c_KV chunk: 128 tokens x 64 latent columns (two pages, SW128)
constexpr int kUpBBytes = 4 * kChunk / 2;  // W_UK | W_UV chunk: 64 latent rows x 256 features (four SW128 blocks)
constexpr int kUpStageBytes = kUpABytes + kUpBBytes;
constexpr int kUpSmem = 1024 + kUpStages * kUpStageBytes + 256;

struct UpParams {
  const int32_t* block_row;   // the sequence's block-table row
  int T, n_pages, num_blocks;
};

__global__ void __launch_bounds__(128)
up_proj_kernel(const __grid_constant__ CUtensorMap tm_wk, const __grid_constant__ CUtensorMap tm_wv,
               const __grid_constant__ CUtensorMap tm_pool, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const UpParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kUpStages * kUpStageBytes);
  uint64_t* empty = full + kUpStages;
  uint64_t* done = empty + kUpStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int t0 = blockIdx.x * kTile, h = blockIdx.y;
  constexpr int kChunks = 512 / 64;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kUpStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_wk);
    prefetch_tmap(&tm_wv);
    prefetch_tmap(&tm_pool);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * kTile);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();
  griddep_launch_dependents();

  if (warp == 0 && lane == 0) {
    // block ids of the tile's two pages (pages past the sequence: block 0, clipped at the store)
    int blk[2];
    for (int q = 0; q < 2; ++q) {
      const int pg = t0 / 64 + q;
      int b = pg < p.n_pages ? p.block_row[pg] : 0;
      blk[q] = (b < 0 || b >= p.num_blocks) ? 0 : b;
    }
    for (int kc = 0; kc < kChunks; ++kc) {
      const int s = kc % kUpStages;
      if (kc >= kUpStages && !mbar_wait(&empty[s], ((kc / kUpStages) - 1) & 1, abort_flag)) {
        *abort_flag = 1;
        break;
      }
      uint8_t* st = smem + s * kUpStageBytes;
      uint8_t* sb = st + kUpABytes;
      mbar_arrive_expect_tx(&full[s], kUpStageBytes);
      tma_load_3d(st, &tm_pool, &full[s], kc * 64, 0, blk[0]);                   // tokens 0..63
      tma_load_3d(st + kChunk / 2, &tm_pool, &full[s], kc * 64, 0, blk[1]);      // tokens 64..127
      tma_load_3d(sb, &tm_wk, &full[s], 0, h, kc * 64);                          // K features 0..63
      tma_load_3d(sb + kChunk / 2, &tm_wk, &full[s], 64, h, kc * 64);            // K features 64..127
      tma_load_3d(sb + kChunk, &tm_wv, &full[s], 0, h, kc * 64);                 // V features 0..63
      tma_load_3d(sb + 3 * kChunk / 2, &tm_wv, &full[s], 64, h, kc * 64);        // V features 64..127
    }
  } else if (warp == 1 && lane == 0) {
    // D[token][K features | V features] += c_KV[token][k] W[k][feature]: M = 128 tokens
    // (A K-major), N = 256 (B MN-major, four 64-feature blocks 8 KB apart)
    const uint32_t idesc = idesc_bf16(128, 2 * kTile, 0, 1);
    for (int kc = 0; kc < kChunks; ++kc) {
      const int s = kc % kUpStages;
      if (!mbar_wait(&full[s], (kc / kUpStages) & 1, abort_flag)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t a0 = smem_u32(smem + s * kUpStageBytes), b0 = a0 + kUpABytes;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(tmem, sdesc(a0 + kk * 32, 16, 1024, kSwizzle128B),
               sdesc(b0 + kk * 2048, kChunk / 2, 1024, kSwizzle128B), idesc, (kc | kk) != 0);
      mma_commit(&empty[s]);
    }
    mma_commit(done);
  }
  __syncwarp();
  const bool ok = __syncthreads_and(mbar_wait(done, 0, abort_flag) && !*abort_flag);
  tc_fence_after();
  if (ok) {
    // TMEM lane = token, column = feature: each thread packs its token's 64-feature
    // blocks to bf16 in the SW128 layout of the output boxes (the stage memory is
    // free: every load landed and every product that read it completed)
    const int r = warp * 32 + lane;
#pragma unroll 1
    for (int blkf = 0; blkf < 4; ++blkf) {
      uint8_t* dst = smem + blkf * kChunk + r * 128;
#pragma unroll 1
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + blkf * 64 + hh * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int chunk = hh * 4 + c;   // 16-byte chunk of the 128-byte row
          st_shared_v4(smem_u32(dst + ((chunk ^ (r & 7)) << 4)),
                       make_uint4(pack_bf16(__uint_as_float(v[8 * c]), __uint_as_float(v[8 * c + 1])),
                                  pack_bf16(__uint_as_float(v[8 * c + 2]), __uint_as_float(v[8 * c + 3])),
                                  pack_bf16(__uint_as_float(v[8 * c + 4]), __uint_as_float(v[8 * c + 5])),
                                  pack_bf16(__uint_as_float(v[8 * c + 6]), __uint_as_float(v[8 * c + 7]))));
        }
      }
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  if (ok && threadIdx.x == 0) {
    // rows past T are clipped by the stores
    tma_store_3d(&tm_k, smem, 0, h, t0);
    tma_store_3d(&tm_k, smem + kChunk, 64, h, t0);
    tma_store_3d(&tm_v, smem + 2 * kChunk, 0, h, t0);
    tma_store_3d(&tm_v, smem + 3 * kChunk, 64, h, t0);
    bulk_commit();
    bulk_wait_all<0>();
  }
  __syncwarp();
  if (warp == 1) tmem_dealloc(tmem, 2 * kTile);
}

// ----------------------------------------------------------------- causal attention
constexpr int kAttThreads = 352;            // 11 warps
constexpr int kSoftWarp0 = 3;               // softmax: warps 3 .. 10, two per TMEM lane quarter
constexpr int kSoftWarps = 8;
constexpr int kKStageBytes = 3 * kChunk;    // K (two 64-d chunks) + k_rope (one 64-col chunk), 48 KB
constexpr int kVStageBytes = 2 * kChunk;    // V as two 64-v chunks (MN-major B), 32 KB
constexpr int kKStages = 3, kVStages = 2;
constexpr int kOffK = 0;
constexpr int kOffV = kOffK + kKStages * kKStageBytes;
constexpr int kOffPMax = kOffV + kVStages * kVStageBytes;          // fp32 [2 tiles][2 halves][128] half-row maxima
constexpr int kOffLSum = kOffPMax + 4 * kTile * 4;                  // fp32 [2 halves][128] half-row sums
constexpr int kOffBar = kOffLSum + 2 * kTile * 4;
constexpr uint32_t kTS = 0, kTP = 128, kTO = 256, kTQ = 384, kTCols = 512;   // Q: 96 columns of bf16 pairs
constexpr float kRescale = 8.0f;            // log2 units

struct AttBars {
  uint64_t q_full, k_full[kKStages], k_empty[kKStages], v_full[kVStages], v_empty[kVStages];
  uint64_t s_full, s_read, p_full[2], o_full[2], o_done;
  uint64_t qk_done, pv_done;
  uint64_t pmax[2][4];   // the two softmax warps of lane quarter q posted their tile-b half-row maxima
  uint64_t lsum[4];      // ... and, at the end, their half-row sums
  uint32_t tmem_base;
  int abort;
};
constexpr int kAttSmem = kOffBar + (int)sizeof(AttBars) + 1024;

struct AttParams {
  const __nv_bfloat16* q_nope;   // [s][H][128]
  const __nv_bfloat16* q_rope;   // [s][H][64]
  const int32_t* block_row;
  __nv_bfloat16* out;      // [s][H][128]
  float* lse;              // [s][H] or null
  int T, s, n_heads, n_pages, num_blocks;
  float scale_log2;
};

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float y;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(a), "f"(b), "f"(c));
  return y;
}

__global__ void __launch_bounds__(kAttThreads, 1)
prefill_attn_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_pool, const AttParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem + kOffK;
  uint8_t* sV = smem + kOffV;
  AttBars* bars = reinterpret_cast<AttBars*>(smem + kOffBar);
  int* abort_flag = &bars->abort;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int qt = blockIdx.x, h = blockIdx.y;
  const int q0 = qt * kTile;                              // first query of the tile (chunk index)
  const int pos0 = p.T - p.s;                             // position of chunk query 0
  const int last_q = min(q0 + kTile, p.s) - 1;
  const int n_tiles = (pos0 + last_q) / kTile + 1;        // key tiles up to the causal limit

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, kSoftWarps);   // Q rows stored into TMEM by the softmax warps
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_read, kSoftWarps);
    mbar_init(&bars->p_full[0], kSoftWarps);
    mbar_init(&bars->p_full[1], kSoftWarps);
    for (int q = 0; q < 4; ++q) {
      mbar_init(&bars->pmax[0][q], 2);
      mbar_init(&bars->pmax[1][q], 2);
      mbar_init(&bars->lsum[q], 2);
    }
    mbar_init(&bars->o_full[0], 1);
    mbar_init(&bars->o_full[1], 1);
    mbar_init(&bars->o_done, 1);
    mbar_init(&bars->qk_done, 1);
    mbar_init(&bars->pv_done, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, kTCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  griddep_wait();
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // K (with k_rope) and V of a tile are separate rings: a K stage is free
      // once its QK product completed, a V stage once its PV product did, so
      // the next K tile loads a whole softmax earlier than a joint stage would.
      int jk = 0, jv = 0;   // tiles whose K / V loads were issued
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j % kKStages, sv = j % kVStages;
        if (j >= kKStages && !mbar_wait(&bars->k_empty[s], ((j / kKStages) - 1) & 1, abort_flag)) {
          *abort_flag = 1;
          break;
        }
        int blk[2];
        for (int q = 0; q < 2; ++q) {
          const int pg = 2 * j + q;
          const int b = pg < p.n_pages ? p.block_row[pg] : 0;
          blk[q] = (b < 0 || b >= p.num_blocks) ? 0 : b;
        }
        uint8_t* st = sK + s * kKStageBytes;
        mbar_arrive_expect_tx(&bars->k_full[s], kKStageBytes);
        tma_load_3d(st, &tm_k, &bars->k_full[s], 0, h, j * kTile);          // keys past T: zero fill
        tma_load_3d(st + kChunk, &tm_k, &bars->k_full[s], 64, h, j * kTile);
        tma_load_3d(st + 2 * kChunk, &tm_pool, &bars->k_full[s], 512, 0, blk[0]);   // k_rope, keys 0..63
        tma_load_3d(st + 2 * kChunk + kChunk / 2, &tm_pool, &bars->k_full[s], 512, 0, blk[1]);
        jk = j + 1;
        if (j >= kVStages && !mbar_wait(&bars->v_empty[sv], ((j / kVStages) - 1) & 1, abort_flag)) {
          *abort_flag = 1;
          break;
        }
        uint8_t* sv_st = sV + sv * kVStageBytes;
        mbar_arrive_expect_tx(&bars->v_full[sv], kVStageBytes);
        tma_load_3d(sv_st, &tm_v, &bars->v_full[sv], 0, h, j * kTile);
        tma_load_3d(sv_st + kChunk, &tm_v, &bars->v_full[sv], 64, h, j * kTile);
        jv = j + 1;
      }
      // every issued load must land before the CTA exits
      for (int k = jk - 1; k >= 0 && k >= jk - kKStages; --k)
        mbar_drain(&bars->k_full[k % kKStages], (k / kKStages) & 1);
      for (int k = jv - 1; k >= 0 && k >= jv - kVStages; --k)
        mbar_drain(&bars->v_full[k % kVStages], (k / kVStages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ QK issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, kTile, 0, 0);
      bool ok = mbar_wait(&bars->q_full, 0, abort_flag);
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int s = j % kKStages;
        if (!mbar_wait(&bars->k_full[s], (j / kKStages) & 1, abort_flag) ||
            (j > 0 && !mbar_wait(&bars->s_read, (j - 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sK + s * kKStageBytes);
#pragma unroll
        for (int t = 0; t < 12; ++t) {   // K = 192 in steps of 16: chunk t / 4 (nope, nope, rope); A = Q from TMEM
          const uint32_t off = (t >> 2) * kChunk + (t & 3) * 32;
          mma_ts(tmem + kTS, tmem + kTQ + 8 * t, sdesc(k_addr + off, 16, 1024, kSwizzle128B), idesc, t != 0);
        }
        mma_commit(&bars->k_empty[s]);
        mma_commit(&bars->s_full);
      }
      if (!ok) *abort_flag = 1;
      mma_commit(&bars->qk_done);
      mbar_drain(&bars->qk_done, 0);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ PV issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, 128, 0, 1);
      bool ok = true;
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j % kVStages;
        if (!mbar_wait(&bars->v_full[s], (j / kVStages) & 1, abort_flag) ||
            !mbar_wait(&bars->p_full[j & 1], (j >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sV + s * kVStageBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)   // 128 keys in steps of 16
          mma_ts(tmem + kTO, tmem + kTP + 64 * (j & 1) + 8 * kk,
                 sdesc(v_addr + kk * 2048, kChunk, 1024, kSwizzle128B), idesc, (j | kk) != 0);
        mma_commit(&bars->v_empty[s]);
        mma_commit(&bars->o_full[j & 1]);
      }
      if (ok) mma_commit(&bars->o_done);
      else *abort_flag = 1;
      mma_commit(&bars->pv_done);
      mbar_drain(&bars->pv_done, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax (8 warps)
    // Thread = (query row r, key half c): keys [64c, 64c + 64) of each tile and
    // output columns [64c, 64c + 64).  The two halves of a row combine their
    // maxima per tile and their sums at the end through shared memory, in the
    // same order, so both take the same rescaling decisions.
    const int quarter = warp & 3;
    const int c = (warp - kSoftWarp0) >> 2;
    const int r = quarter * 32 + lane;                 // query row of the tile = TMEM lane
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    float* s_pmax = reinterpret_cast<float*>(smem + kOffPMax);
    float* s_lsum = reinterpret_cast<float*>(smem + kOffLSum);
    const int qpos = pos0 + q0 + r;                    // position of this query (keys <= qpos visible)
    const float sl2 = p.scale_log2;
    {
      // the tile's query rows into TMEM (A operand of QK): half 0 the q_nope row
      // (64 columns of bf16 pairs), half 1 the q_rope row (32 columns)
      const int q = q0 + r;
      const uint4 zero = make_uint4(0, 0, 0, 0);
      if (c == 0) {
        const uint4* src = reinterpret_cast<const uint4*>(p.q_nope + ((size_t)q * p.n_heads + h) * 128);
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t v[32];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint4 x = q < p.s ? __ldg(src + 8 * hh + k) : zero;
            v[4 * k] = x.x; v[4 * k + 1] = x.y; v[4 * k + 2] = x.z; v[4 * k + 3] = x.w;
          }
          tmem_st32(tmem + lane_addr + kTQ + 32 * hh, v);
        }
      } else {
        const uint4* src = reinterpret_cast<const uint4*>(p.q_rope + ((size_t)q * p.n_heads + h) * 64);
        uint32_t v[32];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint4 x = q < p.s ? __ldg(src + k) : zero;
          v[4 * k] = x.x; v[4 * k + 1] = x.y; v[4 * k + 2] = x.z; v[4 * k + 3] = x.w;
        }
        tmem_st32(tmem + lane_addr + kTQ + 64, v);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->q_full);
    }
    float m_ref = -CUDART_INF_F, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int b = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full, j & 1, abort_flag))) { ok = false; break; }
      tc_fence_after();
      uint32_t v[64];
      tmem_ld32(tmem + lane_addr + kTS + 64 * c, *reinterpret_cast<uint32_t(*)[32]>(v));
      tmem_ld32(tmem + lane_addr + kTS + 64 * c + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->s_read);
      // causal mask: key j * 128 + 64c + k is visible iff <= qpos (which also
      // excludes keys >= T); only the tiles that reach past some row's last
      // visible key take it.  Maxima are taken on the raw scores (the scale is
      // positive, so the scaled maximum is the same rounded value).
      const int vis = qpos - j * kTile - 64 * c;       // columns [0, vis] of this half visible
      const bool full = __all_sync(0xffffffffu, vis >= 63);
      if (!full) {
#pragma unroll
        for (int k = 0; k < 64; ++k)
          if (k > vis) v[k] = __float_as_uint(-CUDART_INF_F);
      }
      float mq[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
      for (int k = 0; k < 64; k += 8)
#pragma unroll
        for (int a = 0; a < 4; ++a)
          mq[a] = max3f(mq[a], __uint_as_float(v[k + 2 * a]), __uint_as_float(v[k + 2 * a + 1]));
      const float mloc = max3f(mq[0], mq[1], fmaxf(mq[2], mq[3]));
      s_pmax[(b * 2 + c) * kTile + r] = mloc;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->pmax[b][quarter]);
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->pmax[b][quarter], (j >> 1) & 1, abort_flag))) { ok = false; break; }
      const float mx = fmaxf(mloc, s_pmax[(b * 2 + (c ^ 1)) * kTile + r]) * sl2;
      const float m_new = fmaxf(m_ref, mx);
      const bool move = (m_ref == -CUDART_INF_F) ? (m_new != -CUDART_INF_F) : (m_new > m_ref + kRescale);
      float alpha = 1.f;
      if (move) {
        alpha = (m_ref == -CUDART_INF_F) ? 0.f : ex2f(m_ref - m_new);
        m_ref = m_new;
      }
      const float nb = (m_ref == -CUDART_INF_F) ? 0.f : -m_ref;
      const float2 sl2x2 = make_float2(sl2, sl2), nbx2 = make_float2(nb, nb);
      uint32_t pk[32];
      float2 ps[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float2 x = __ffma2_rn(make_float2(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1])), sl2x2, nbx2);
        const float e0 = ex2f(x.x), e1 = ex2f(x.y);
        pk[k] = pack_bf16(e0, e1);
        ps[k & 1] = __fadd2_rn(ps[k & 1], make_float2(e0, e1));
      }
      l_run = l_run * alpha + ((ps[0].x + ps[1].x) + (ps[0].y + ps[1].y));
      // P buffer j & 1 is free once the PV product of tile j - 2 completed
      if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait(&bars->o_full[j & 1], ((j >> 1) - 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      if (__any_sync(0xffffffffu, move && j > 0)) {
        // rescale this half's O columns: the PV product of tile j - 1 must have landed
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_full[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float a = (move && j > 0) ? alpha : 1.f;
#pragma unroll 1
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_addr + kTO + 64 * c + 32 * cc, o);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * a);
          tmem_st32(tmem + lane_addr + kTO + 64 * c + 32 * cc, o);
        }
        tmem_st_wait();
      }
      tmem_st32(tmem + lane_addr + kTP + 64 * (j & 1) + 32 * c, pk);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[j & 1]);
    }
    if (ok && !__all_sync(0xffffffffu, mbar_wait(&bars->o_done, 0, abort_flag))) ok = false;
    if (ok) {
      s_lsum[c * kTile + r] = l_run;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->lsum[quarter]);
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->lsum[quarter], 0, abort_flag))) ok = false;
    }
    if (ok) {
      tc_fence_after();
      l_run = s_lsum[r] + s_lsum[kTile + r];           // same order in both halves
      const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
      const int q = q0 + r;
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_addr + kTO + 64 * c + 32 * cc, o);
        tmem_ld_wait();
        if (q < p.s) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + ((size_t)q * p.n_heads + h) * 128 + 64 * c + 32 * cc);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            dst[k] = make_uint4(pack_bf16(__uint_as_float(o[8 * k]) * inv_l, __uint_as_float(o[8 * k + 1]) * inv_l),
                                pack_bf16(__uint_as_float(o[8 * k + 2]) * inv_l, __uint_as_float(o[8 * k + 3]) * inv_l),
                                pack_bf16(__uint_as_float(o[8 * k + 4]) * inv_l, __uint_as_float(o[8 * k + 5]) * inv_l),
                                pack_bf16(__uint_as_float(o[8 * k + 6]) * inv_l, __uint_as_float(o[8 * k + 7]) * inv_l));
        }
      }
      if (c == 0 && q < p.s && p.lse)
        p.lse[(size_t)q * p.n_heads + h] = l_run > 0.f ? (m_ref + __log2f(l_run)) * 0.6931471805599453f : -CUDART_INF_F;
    } else {
      *abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  __syncwarp();
  if (warp == 1) tmem_dealloc(tmem, kTCols);
}

cudaError_t prefill_attrs() {
  static cudaError_t e = [] {
    cudaError_t a = cudaFuncSetAttribute(up_proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kUpSmem);
    cudaError_t b = cudaFuncSetAttribute(prefill_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttSmem);
    return a != cudaSuccess ? a : b;
  }();
  return e;
}

// [N][H][F] bf16 viewed as (F, H, N): boxes of 64 features x 128 rows (SW128), or a
// store box of 128 features x 128 rows (no swizzle).
mla_status_t rows_map(CUtensorMap* m, const void* base, int F, int H, int N) {
  const uint64_t dims[3] = {(uint64_t)F, (uint64_t)H, (uint64_t)N};
  const uint64_t str[2] = {(uint64_t)F * 2, (uint64_t)H * F * 2};
  const uint32_t box[3] = {64, 1, (uint32_t)kTile};
  return encode_tmap_bf16(m, base, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// The cache pool as (column, row within the block, block), boxes of 64 columns x 64 rows.
mla_status_t pool_map(CUtensorMap* m, const void* pool, int num_blocks) {
  const uint64_t dims[3] = {576, 64, (uint64_t)num_blocks};
  const uint64_t str[2] = {576 * 2, 64 * 576 * 2};
  const uint32_t box[3] = {64, 64, 1};
  return encode_tmap_bf16(m, pool, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

mla_status_t launch_prefill_up_proj(const void* kv_pool, const int32_t* block_row, int T, int num_blocks,
                                    const void* w_uk, const void* w_uv, int n_heads, void* k_out, void* v_out,
                                    void* stream) {
  CUtensorMap twk, twv, tpool, tk, tv;
  const uint64_t wdims[3] = {128, (uint64_t)n_heads, 512};
  const uint64_t wstr[2] = {128 * 2, (uint64_t)n_heads * 128 * 2};
  const uint32_t wbox[3] = {64, 1, 64};
  mla_status_t st = encode_tmap_bf16(&twk, w_uk, 3, wdims, wstr, wbox, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st == MLA_OK) st = encode_tmap_bf16(&twv, w_uv, 3, wdims, wstr, wbox, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st == MLA_OK) st = pool_map(&tpool, kv_pool, num_blocks);
  if (st == MLA_OK) st = rows_map(&tk, k_out, 128, n_heads, T);
  if (st == MLA_OK) st = rows_map(&tv, v_out, 128, n_heads, T);
  if (st != MLA_OK) return st;
  UpParams p{block_row, T, (T + 63) / 64, num_blocks};
  cudaError_t e = prefill_attrs();
  if (e == cudaSuccess) {
    e = launch_pdl(up_proj_kernel, dim3((T + kTile - 1) / kTile, n_heads), dim3(128), kUpSmem, stream, twk, twv,
                   tpool, tk, tv, p);
    if (e == cudaSuccess) e = cudaGetLastError();
  }
  if (e != cudaSuccess) return set_error(MLA_ERR_CUDA, "prefill up-projection launch: %s", cudaGetErrorString(e));
  return MLA_OK;
}

mla_status_t launch_prefill_attn(const void* q_nope, const void* q_rope, const void* k, const void* v,
                                 const void* kv_pool, const int32_t* block_row, int T, int s, int n_heads,
                                 int num_blocks, float scale, void* out, float* lse, void* stream) {
  CUtensorMap tk, tv, tpool;
  mla_status_t st = rows_map(&tk, k, 128, n_heads, T);
  if (st == MLA_OK) st = rows_map(&tv, v, 128, n_heads, T);
  if (st == MLA_OK) st = pool_map(&tpool, kv_pool, num_blocks);
  if (st != MLA_OK) return st;
  AttParams p{static_cast<const __nv_bfloat16*>(q_nope), static_cast<const __nv_bfloat16*>(q_rope), block_row,
              static_cast<__nv_bfloat16*>(out), lse, T, s, n_heads, (T + 63) / 64, num_blocks,
              scale * 1.4426950408889634f};
  cudaError_t e = prefill_attrs();
  if (e == cudaSuccess) {
    e = launch_pdl(prefill_attn_kernel, dim3((s + kTile - 1) / kTile, n_heads), dim3(kAttThreads), kAttSmem, stream,
                   tk, tv, tpool, p);
    if (e == cudaSuccess) e = cudaGetLastError();
  }
  if (e != cudaSuccess) return set_error(MLA_ERR_CUDA, "prefill attention launch: %s", cudaGetErrorString(e));
  return MLA_OK;
}

}  // namespace mla
