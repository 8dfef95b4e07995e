// Absorbed MLA decode attention on sm_100a (tcgen05 + TMEM + TMA + 2-CTA clusters).
//
// What it computes, per query row (token n, head h), over keys t < kv_len:
//   logit_t = scale * (q_lat[n,h,:] . c_KV[t,:] + q_rope[n,h,:] . k_rope[t,:])
//   o_lat[n,h,:] = sum_t softmax(logit)_t c_KV[t,:]
// i.e. Step 3 of order 2 of the first absorption (term 2bhstk) plus the
// RoPE-MQA score, then Step 1 of order 2 of the second absorption (2bhskt),
// in the notation of "MLA Matrix Absorption Analysis" (sections 2.2, 3.2).  The
// RoPE term of the izhida.com answer is the extra 64-wide shared key.
//
// Why this shape on B200.  The 128 heads of a query share one cache stream,
// so S = [q_lat | q_rope] [c_KV | k_rope]^T (M = 128 heads, N = 64 keys,
// K = 576) and O += P c_KV (M = 128, N = 512, K = 64) are dense contractions
// for the tensor cores.  O for 128 heads x 512 latent columns in fp32 is
// exactly one SM's 512 TMEM columns, leaving no room for S.  So a cluster of
// two CTAs splits the latent dimension: CTA r owns latent columns
// [256r, 256r + 256) and RoPE columns [32r, 32r + 32).  Each CTA stages only
// its half of every cache row (each byte is read from HBM once) and computes
// a partial score over its 288 columns.  The partial scores, scaled to log2
// units (scale * log2(e)), are rounded to fp16 and exchanged through
// distributed shared memory (one bulk copy per page, counted on the
// receiver's mbarrier); both CTAs then add fp16(S0) + fp16(S1) as fp16 pairs,
// which is bit-identical in the pair, so both take the same softmax
// decisions.  Each CTA accumulates its 256 output columns.
//
// TMEM (512 columns): O [0,256) fp32, S [256,320) fp32 (released as soon as
// the sender has read it), two P buffers [320,352) and [352,384) bf16 (A
// operand of the PV product; page g uses buffer g & 1, so the softmax of a
// page never waits for the previous page's PV product), q_lat half [384,512)
// as bf16 pairs (A operand of QK).  Shared memory holds five 36 KB stages of
// cache rows, one fp16 score tile each way (own, peer), both read right after
// they land, and the q_rope half (A operand of the two RoPE MMAs).
//
// Warp roles (512 threads): warp 0 TMA producer; warp 1 QK issuer and TMEM
// owner; warp 2 PV issuer (two issuing threads, so a page waiting for its
// softmax never holds back the next QK, and the tensor pipe takes work from
// both); warps 3-6 score sender and q_lat loader (one thread per row);
// warps 7-14 softmax / correction / epilogue (two warps per TMEM lane
// quarter, one per 32-key half); warp 15 copies each page's score tile to
// the peer (one thread), so no sender waits on a copy.  The grid
// is persistent: one cluster per SM pair, each walking the (row, page range)
// items the host plan gives it.  Every wait is bounded (200 ms by default,
// mla_set_wait_limit_ns); on expiry the CTA sets MLA_STATUS_TIMEOUT, stops its
// peer, drains the copies and products it issued and returns without trapping.
//
// FP8 latent cache (mla_decode_attn_fp8cache).  A token row is then 656
// bytes: c_KV as 512 E4M3 codes, one fp32 scale per 128-column block, and
// k_rope in bf16 (the block scheme of "Lower latency and higher throughput
// with multi-node DeepSeek deployment", section "Quantization", applied to
// the cached activation).  The producer loads a CTA's two code blocks, their
// scales and its RoPE columns raw (21 KB of HBM per half page instead of
// 36 KB), and the four sender warps widen the stage in place to the layout
// above in fp16 (code x scale, one fp16 multiply per pair of codes: two
// instructions per pair, where a bf16 result would take six), two pages ahead
// of the QK product.  The latent products then run as kind::f16 with fp16
// operands: q_lat is rounded to fp16 when it is loaded, P is written as fp16
// pairs; the RoPE products stay bf16.  Everything else is the bf16 kernel.
#include "mla_internal.h"
#include "plan_format.h"
#include "ptx.cuh"
#include "tmap.h"

#include <cuda_bf16.h>
#include <math_constants.h>

#include <atomic>

namespace mla {
namespace {

using namespace ptx;

constexpr int kPage = 64;
constexpr int kRows = 128;
constexpr int kStages = 5;
constexpr int kChunkBytes = kPage * 128;                     // 64 keys x 64 latent cols (SW128)
constexpr int kRopeBytes = kPage * 64;                       // 64 keys x 32 rope cols (SW64)
constexpr int kStageBytes = 4 * kChunkBytes + kRopeBytes;    // 36 KB: half a page
// FP8 cache row: [512 E4M3 codes | 4 fp32 scales | 64 bf16 k_rope].  Raw stage
// layout: code block h of this CTA (128 bytes per key, SW128) in chunk 2h + 1;
// the scales of keys [16w, 16w + 16) (16 bytes each) at 2048 w, inside the rows
// of chunk 0 that sender warp w alone rewrites; RoPE where the bf16 stage has it.
constexpr int kF8Row = 656, kF8ScaleOff = 512, kF8RopeOff = 528;
constexpr int kF8ScaleKeys = 16;
constexpr int kF8StageTx = 2 * kChunkBytes + (kPage / kF8ScaleKeys) * kF8ScaleKeys * 16 + kRopeBytes;
constexpr int kXRow = 64 * 2;                                // fp16 score row, 16B chunks XOR (row & 7)
constexpr int kXBytes = kRows * kXRow;                       // one score tile (16 KB)

constexpr int kOffKV = 0;
constexpr int kOffXPeer = kOffKV + kStages * kStageBytes;   // peer's partial scores (one tile)
constexpr int kOffXOwn = kOffXPeer + kXBytes;                // own partial scores (fp16, one tile)
constexpr int kOffPMax = kOffXOwn + kXBytes;                 // fp32 [2 pages][2 halves][128] half-row maxima
constexpr int kOffLSum = kOffPMax + 4 * kRows * 4;     // fp32 [2 items][2 halves][128] half-row sums
constexpr int kOffQRope = kOffLSum + 4 * kRows * 4;    // bf16 q_rope half, 128 rows x 64 B (SW64, A of QK)
constexpr int kOffBar = kOffQRope + kRows * 64;

constexpr int kThreads = 512;            // 16 warps
constexpr int kSoftWarp0 = 7, kCopyWarp = 15;   // senders are warps 3 .. 6
constexpr int kSoftWarps = 8;

constexpr uint32_t kTmemO = 0, kTmemS = 256, kTmemP = 320, kTmemQ = 384, kTmemCols = 512;   // P: two 32-column buffers
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;   // log2 units: rescale O only when the max grows by > 2^8

struct DecodeParams {
  const __nv_bfloat16* q_lat;   // [N][H][512]
  const __nv_bfloat16* q_rope;  // [N][H][64]
  const int32_t* block_table;   // [B][max_blocks]
  const int32_t* seq_lens;      // [B]
  const int32_t* plan;
  const int32_t* draft_masks;   // [B][s_q] visibility of the drafts (bit j: draft j), or null
  float* o_part;                // [slots][H][512]
  float* lse_part;              // [slots][H]
  __nv_bfloat16* o_lat;         // [N][H][512]
  float* lse_out;               // [N][H] or null
  int32_t* status;
  int n_heads, max_blocks, num_blocks, s_q, causal, B, n_rows, num_clusters;
  float scale_log2;             // scale * log2(e)
  uint64_t wait_ns;             // limit of every protocol wait (drains of issued work use the default)
};

struct Bars {
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t kv_conv[kStages];   // FP8 cache: the stage has been widened to bf16 (4 sender warps)
  uint64_t q_full, q_empty;
  uint64_t s_full;       // QK product of the current page is in S
  uint64_t s_read;       // the sender has read S (the next QK may overwrite it)
  uint64_t own_full;     // own fp16 partial-score tile written (4 sender warps)
  uint64_t own_free;     // own tile read by the softmax (8 warps) and by its bulk copy (1)
  uint64_t x_recv;       // peer's fp16 partial scores landed in the peer tile (1 arrival + 16 KB tx)
  uint64_t x_sendok;     // peer has read its peer tile, which this CTA may refill (8 remote arrivals)
  uint64_t p_full;       // P written (O rescaled if needed), 8 softmax warps
  uint64_t o_full[2];     // PV product of a page complete, per P buffer (page g uses buffer g & 1)
  uint64_t o_done;        // every PV product of the current item complete (epilogue)
  uint64_t o_free, qk_done, pv_done;
  uint64_t pmax[2][4];   // the two softmax warps of row quarter q posted their page-b half-row maxima
  uint64_t lsum[4];      // the two softmax warps of row quarter q posted their half-row sums (per item)
  uint32_t tmem_base;    // TMEM allocation
  uint32_t sent_count;   // score tiles this CTA has copied to its peer
  WaitCtl wc;            // abort flag and wait limit of every role
};
constexpr int kSmemBytes = kOffBar + (int)sizeof(Bars) + 1024;

__device__ __forceinline__ void report(int32_t* status, int bits) {
  if (status) atomicOr(status, bits);
}

// Suspend-time hint of the pipeline waits (0: no hint, spin).
constexpr uint32_t kWaitHintNs = 0;

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile WaitCtl* wc) {
  return __all_sync(0xffffffffu, mbar_wait<false, kWaitHintNs>(bar, parity, wc));
}
// For data the peer CTA's bulk copy wrote: its complete_tx releases at cluster
// scope, so the waiter must acquire at cluster scope to see the bytes.
__device__ __forceinline__ bool warp_wait_cluster(uint64_t* bar, uint32_t parity, volatile WaitCtl* wc) {
  return __all_sync(0xffffffffu, mbar_wait<true, kWaitHintNs>(bar, parity, wc));
}

// The plan fixes each row's key count (kv_len) from the host seq_lens it was
// made with.  True if the device seq_lens (T of the item's sequence) now give
// another count: the softmax then masks every key of the item, so the row is
// written as zeros with LSE -inf, and MLA_STATUS_BAD_SEQLEN is reported.
__device__ __forceinline__ bool item_stale(const int32_t* w, int T, const DecodeParams& p) {
  const int want = p.causal ? T - p.s_q + 1 + w[kItQi] : T;
  return want != w[kItKvLen];
}

// Keys of the item's last page that are attended (1 .. 64).  When fewer than
// 64, that page is loaded shifted: its first `attended` keys land in stage
// rows [64 - attended, 64) and the rows above them are the TMA's zero fill
// (a negative row coordinate), so no stale or non-finite cache row past the
// key count ever reaches the P.c_KV product (where 0 * Inf would be NaN).
__device__ __forceinline__ int last_page_keys(const int32_t* w) {
  return w[kItKvLen] - (w[kItPageEnd] - 1) * kPage;
}

// fp16 pair sum and maximum (round to nearest even; the maximum of -inf and x is x).
__device__ __forceinline__ uint32_t hadd2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t hmax2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// (a.lo + c, a.hi + c) in fp32 for an fp16 pair a: the mixed-precision add
// takes the fp16 operand exactly and rounds the sum once.
__device__ __forceinline__ void add_f16x2_to_f32(uint32_t a, float c, float& lo, float& hi) {
  asm("{\n\t.reg .f16 a0, a1;\n\t"
      "mov.b32 {a0, a1}, %2;\n\t"
      "add.rn.f32.f16 %0, a0, %3;\n\tadd.rn.f32.f16 %1, a1, %3;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(a), "f"(c));
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// kFp8: the cache pool holds FP8 rows (tm_kv = the codes as bytes, tm_scale =
// the scales as bytes, tm_rope = the bf16 RoPE columns); otherwise bf16 rows
// (tm_kv = the latent columns, tm_rope = the RoPE columns, tm_scale unused).
// kTree: p.draft_masks gives each query's view of the drafted tokens (an
// instance of its own, so the other instances' softmax loop carries no mask
// code: its instruction footprint was measured to cost 1-2 %).
template <bool kFp8, bool kTree>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
mla_decode_kernel(const __grid_constant__ CUtensorMap tm_kv, const __grid_constant__ CUtensorMap tm_rope,
                  const __grid_constant__ CUtensorMap tm_scale, const DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_kv = smem + kOffKV;
  uint8_t* s_xpeer = smem + kOffXPeer;
  uint8_t* s_xown = smem + kOffXOwn;
  float* s_pmax = reinterpret_cast<float*>(smem + kOffPMax);
  float* s_lsum = reinterpret_cast<float*>(smem + kOffLSum);
  uint8_t* s_qrope = smem + kOffQRope;
  Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
  uint32_t* tmem_slot = &bars->tmem_base;
  volatile WaitCtl* wc = &bars->wc;
  volatile uint32_t* sent_count = &bars->sent_count;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank(), peer = rank ^ 1u;
  const int cid = (int)cluster_id_x();
  // A role that gives up stops both CTAs of the pair (the peer would otherwise
  // wait for score tiles that never come): it raises its own flag and the
  // peer's, so after the final cluster barrier both flags tell the same story.
  auto give_up = [&]() {
    wc->abort = 1;
    st_cluster_u32(mapa(smem_u32((const void*)&wc->abort), peer), 1u);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
      if (kFp8) mbar_init(&bars->kv_conv[s], 4);
    }
    mbar_init(&bars->q_full, 4);       // the 4 q_lat / q_rope loader warps
    mbar_init(&bars->q_empty, 1);
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_read, 4);
    mbar_init(&bars->own_full, 4);
    mbar_init(&bars->own_free, kSoftWarps + 1);
    mbar_init(&bars->x_recv, 1);
    mbar_init(&bars->x_sendok, kSoftWarps);
    mbar_init(&bars->p_full, kSoftWarps);
    mbar_arrive_expect_tx(&bars->x_recv, kXBytes);   // armed for page 0
    mbar_init(&bars->o_full[0], 1);
    mbar_init(&bars->o_full[1], 1);
    mbar_init(&bars->o_done, 1);
    mbar_init(&bars->o_free, kSoftWarps);
    mbar_init(&bars->qk_done, 1);
    mbar_init(&bars->pv_done, 1);
    for (int q = 0; q < 4; ++q) {
      mbar_init(&bars->pmax[0][q], 2);
      mbar_init(&bars->pmax[1][q], 2);
      mbar_init(&bars->lsum[q], 2);
    }
    wc->abort = 0;
    wc->limit_ns = p.wait_ns;
    *sent_count = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_kv);
    prefetch_tmap(&tm_rope);
    if (kFp8) prefetch_tmap(&tm_scale);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // peer barriers and flags initialised before any remote access
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();   // set-up above overlaps the previous kernel; global memory only from here
  griddep_launch_dependents();

  // The section offsets follow from the cluster count, so the cluster's item
  // range is read without first waiting for the header (checked alongside).
  // The plan must match the launch (uniform over the grid).
  const int32_t* plan = p.plan;
  const int off_cluster = kPlanHeaderWords, off_items = kPlanHeaderWords + p.num_clusters + 1;
  const int32_t* items = plan + off_items;
  const int it_begin_raw = plan[off_cluster + cid], it_end_raw = plan[off_cluster + cid + 1];
  const bool plan_ok = plan[kHdrMagic] == kPlanMagic && plan[kHdrNumClusters] == p.num_clusters &&
                       plan[kHdrNumRows] == p.n_rows && plan[kHdrHeads] == p.n_heads &&
                       plan[kHdrB] == p.B && plan[kHdrSq] == p.s_q &&
                       plan[kHdrMaxBlocks] == p.max_blocks && plan[kHdrCausal] == (p.causal ? 1 : 0) &&
                       plan[kHdrOffCluster] == off_cluster && plan[kHdrOffItems] == off_items;
  const int it_begin = plan_ok ? it_begin_raw : 0;
  const int it_end = plan_ok ? it_end_raw : 0;
  if (!plan_ok && threadIdx.x == 0 && rank == 0 && cid == 0) report(p.status, MLA_STATUS_BAD_PLAN);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // Lane 0 waits and issues; the whole warp fetches block ids 32 pages at a
    // time with one coalesced load, so a page's TMA never waits on its own
    // block-table read.  (An L2 prefetch of the blocks a few pages ahead was
    // measured slower at distances 2 to 12.)
    int g = 0;
    bool fail = false;
    for (int it = it_begin; it < it_end && !fail; ++it) {
      if (__any_sync(0xffffffffu, wc->abort != 0)) break;   // warp-uniform
      const int32_t* w = items + (size_t)it * kItemWords;
      const int b = w[kItB], pb = w[kItPageBegin], pe = w[kItPageEnd];
      const int shift = kPage - min(last_page_keys(w), kPage);   // zero-filled rows of the last page
      int my_blk = pb + lane < pe ? p.block_table[(size_t)b * p.max_blocks + pb + lane] : 0;
      if (lane == 0 && it + 1 < it_end) {   // the next item's query rows, so that its loaders read them from L2
        const size_t nrow = (size_t)items[(size_t)(it + 1) * kItemWords + kItRow];
        bulk_prefetch_l2(p.q_lat + nrow * p.n_heads * 512, (uint32_t)p.n_heads * 1024u);
        bulk_prefetch_l2(p.q_rope + nrow * p.n_heads * 64, (uint32_t)p.n_heads * 128u);
      }
      for (int pg = pb; pg < pe && !fail; ++pg, ++g) {
        const int rel = pg - pb;
        if ((rel & 31) == 0 && rel > 0) {
          const int q = pg + lane;
          my_blk = q < pe ? p.block_table[(size_t)b * p.max_blocks + q] : 0;
        }
        int blk = __shfl_sync(0xffffffffu, my_blk, rel & 31);
        if (lane == 0) {
          const int s = g % kStages;
          if (g >= kStages && !mbar_wait<false, kWaitHintNs>(&bars->kv_empty[s], ((g / kStages) - 1) & 1, wc)) {
            fail = true;
          } else {
            if (blk < 0 || blk >= p.num_blocks) {
              report(p.status, MLA_STATUS_BAD_BLOCK);
              blk = 0;
            }
            uint8_t* st = s_kv + s * kStageBytes;
            const int y = pg + 1 == pe ? -shift : 0;   // first row of the block to load
            if constexpr (kFp8) {
              mbar_arrive_expect_tx(&bars->kv_full[s], kF8StageTx);
#pragma unroll
              for (int h = 0; h < 2; ++h)
                tma_load_3d(st + (2 * h + 1) * kChunkBytes, &tm_kv, &bars->kv_full[s], 256 * rank + 128 * h, y, blk);
#pragma unroll
              for (int w4 = 0; w4 < kPage / kF8ScaleKeys; ++w4)
                tma_load_3d(st + 2048 * w4, &tm_scale, &bars->kv_full[s], 0, y + kF8ScaleKeys * w4, blk);
              tma_load_3d(st + 4 * kChunkBytes, &tm_rope, &bars->kv_full[s], 32 * rank, y, blk);
            } else {
              mbar_arrive_expect_tx(&bars->kv_full[s], kStageBytes);   // zero-filled bytes count too
#pragma unroll
              for (int c = 0; c < 4; ++c)
                tma_load_3d(st + c * kChunkBytes, &tm_kv, &bars->kv_full[s], 256 * rank + 64 * c, y, blk);
              tma_load_3d(st + 4 * kChunkBytes, &tm_rope, &bars->kv_full[s], 512 + 32 * rank, y, blk);
            }
          }
        }
        fail = __shfl_sync(0xffffffffu, fail, 0);
        if (fail) break;   // this page was not issued
      }
    }
    if (lane == 0) {
      if (fail) {
        give_up();
        report(p.status, MLA_STATUS_TIMEOUT);
      }
      // every issued load must land before the CTA may exit
      for (int k = g - 1; k >= 0 && k >= g - kStages; --k)
        mbar_drain(&bars->kv_full[k % kStages], (k / kStages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ QK issuer
    // S = [q_lat | q_rope] . [c_KV | k_rope]^T over this CTA's 288 columns:
    // M = 128 rows, N = 64 keys, 16 MMAs with A = q_lat and 2 with A = q_rope,
    // both from TMEM.  S is single-buffered; the sender frees it (s_read) as
    // soon as it has copied the product out.  The whole warp runs the loop
    // (descriptors stay warp-uniform) and one elected lane issues.
    const uint32_t idesc_qk = idesc_bf16(128, 64, 0, 0);                                // RoPE half
    const uint32_t idesc_lat = kFp8 ? idesc_f16(128, 64, 0, 0) : idesc_qk;              // latent half
    const uint64_t kv_desc0 = sdesc(smem_u32(s_kv), 16, 1024, kSwizzle128B);
    const uint64_t kr_desc0 = sdesc(smem_u32(s_kv) + 4 * kChunkBytes, 16, 512, kSwizzle64B);
    const uint64_t qr_desc = sdesc(smem_u32(s_qrope), 16, 512, kSwizzle64B);
    bool ok = true;
    int g = 0;
    for (int it = it_begin; ok && it < it_end; ++it) {
      const int32_t* w = items + (size_t)it * kItemWords;
      const int n = w[kItPageEnd] - w[kItPageBegin];
      if (!warp_wait(&bars->q_full, (it - it_begin) & 1, wc)) { ok = false; break; }
      for (int j = 0; j < n; ++j, ++g) {
        const int s = g % kStages;
        if (!warp_wait(&bars->kv_full[s], (g / kStages) & 1, wc) ||
            (kFp8 && !warp_wait(&bars->kv_conv[s], (g / kStages) & 1, wc)) ||
            (g > 0 && !warp_wait(&bars->s_read, (g - 1) & 1, wc))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t kvd = kv_desc0 + (uint64_t)((s * kStageBytes) >> 4);
        const uint64_t krd = kr_desc0 + (uint64_t)((s * kStageBytes) >> 4);
#pragma unroll
        for (int t = 0; t < 16; ++t)   // latent half: K = 256 in steps of 16, A = q_lat from TMEM
          mma_ts_elect(tmem + kTmemS, tmem + kTmemQ + 8 * t,
                       kvd + (uint64_t)(((t >> 2) * kChunkBytes + (t & 3) * 32) >> 4), idesc_lat, t != 0);
#pragma unroll
        for (int t = 0; t < 2; ++t)    // RoPE half: K = 32, A = q_rope from shared memory
          mma_ss_elect(tmem + kTmemS, qr_desc + (uint64_t)(t * 2), krd + (uint64_t)(t * 2), idesc_qk, 1);
        mma_commit_elect(&bars->s_full);
      }
      if (ok) mma_commit_elect(&bars->q_empty);   // q_lat and q_rope (TMEM) may be replaced
    }
    if (!ok && lane == 0) {
      give_up();
      report(p.status, MLA_STATUS_TIMEOUT);
    }
    __syncwarp();
    mma_commit_elect(&bars->qk_done);
    mbar_drain(&bars->qk_done, 0);   // no MMA may still write TMEM at dealloc
  } else if (warp == 2) {
    // ------------------------------------------------------------ PV issuer
    // O += P . c_KV: M = 128 rows, N = 256 latent columns, K = 64 keys in 4
    // MMAs, A = P (bf16 pairs) from TMEM buffer g & 1, B = the stage's c_KV
    // half (MN-major).  Warp-wide loop, one elected lane issues.
    const uint32_t idesc_pv = kFp8 ? idesc_f16(128, 256, 0, 1) : idesc_bf16(128, 256, 0, 1);
    const uint64_t v_desc0 = sdesc(smem_u32(s_kv), kChunkBytes, 1024, kSwizzle128B);
    bool ok = true;
    int g = 0;
    for (int it = it_begin; ok && it < it_end; ++it) {
      const int32_t* w = items + (size_t)it * kItemWords;
      const int n = w[kItPageEnd] - w[kItPageBegin];
      const int ii = it - it_begin;
      for (int j = 0; j < n; ++j, ++g) {
        const int s = g % kStages;
        if (!warp_wait(&bars->p_full, g & 1, wc) ||
            (j == 0 && ii > 0 && !warp_wait(&bars->o_free, (ii - 1) & 1, wc))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t vd = v_desc0 + (uint64_t)((s * kStageBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)   // 64 keys in steps of 16; P (bf16 pairs) from TMEM
          mma_ts_elect(tmem + kTmemO, tmem + kTmemP + 32 * (g & 1) + 8 * kk, vd + (uint64_t)(kk * (2048 >> 4)),
                       idesc_pv, (j | kk) != 0);
        mma_commit_elect(&bars->kv_empty[s]);
        mma_commit_elect(&bars->o_full[g & 1]);
      }
      // o_full alone cannot tell the last page's completion from the one before
      // (a parity wait sees one phase at a time), so the epilogue waits on this
      if (ok) mma_commit_elect(&bars->o_done);
    }
    if (!ok && lane == 0) {
      give_up();
      report(p.status, MLA_STATUS_TIMEOUT);
    }
    __syncwarp();
    mma_commit_elect(&bars->pv_done);
    mbar_drain(&bars->pv_done, 0);
  } else if (warp < kSoftWarp0) {
    // ------------------------------------------------------------ query loader and score sender (4 warps)
    // At each item start the thread of row r copies its 256 q_lat columns and
    // its 32 q_rope columns into TMEM (A operands of the QK product) once the
    // previous item's last QK has completed; the producer has prefetched those
    // rows into L2.  Per page it reads this CTA's partial scores (its 288
    // columns) as soon as the QK product lands, frees S, rounds to fp16 into
    // the own tile, and the copy warp pushes that tile to the peer's tile with a
    // bulk copy that completes on the peer's x_recv.  Thread = one row, 64
    // keys; 16-byte chunks XOR-swizzled by (row & 7).
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const float sl2 = p.scale_log2;
    // FP8 cache: widen stage gg to fp16 in place.  Thread = (key cr, code
    // block ch).  Its 128 codes sit in chunk 2ch + 1, row cr; it writes the
    // block's 128 fp16 columns to chunks 2ch (codes 0-63) and 2ch + 1 (codes
    // 64-127, over its own codes, all read by then), so no thread overwrites
    // bytes another thread still reads, except the scales in chunk 0: read
    // first, then the warp syncs.  Page g + 1 is widened before page g's
    // scores are awaited (pages 0 and 1 before page 0's), that is, right after
    // page g - 1's scores have gone out: neither the score exchange nor the
    // next QK product waits for it.
    auto widen = [&](int gg) -> bool {
      const int s = gg % kStages;
      if (!warp_wait(&bars->kv_full[s], (gg / kStages) & 1, wc)) return false;
      const int w4 = warp - 3, ch = lane >> 4;
      // (recomputed per call: kept live across the sender loop they cost registers)
      int cr;
      asm volatile("mov.b32 %0, %1;" : "=r"(cr) : "r"(kF8ScaleKeys * w4 + (lane & 15)));
      const uint32_t st = smem_u32(s_kv + s * kStageBytes);
      const uint32_t s2 = pack_f16(ld_shared_f32(st + 2048 * w4 + (lane & 15) * 16 + (2 * rank + ch) * 4), 0.f);
      __syncwarp();   // lanes 0 and 1 overwrite the warp's scales below
      const uint32_t sc2 = __byte_perm(s2, 0, 0x1010);   // (s, s) in fp16
      const uint32_t row = st + 2 * ch * kChunkBytes + cr * 128;
#pragma unroll 1
      for (int hb = 0; hb < 2; ++hb) {   // codes [64 hb, 64 hb + 64) -> fp16 chunk 2ch + hb
        uint4 raw[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) raw[k] = ld_shared_v4(row + kChunkBytes + (((4 * hb + k) ^ (cr & 7)) << 4));
#pragma unroll
        for (int k = 0; k < 4; ++k) {   // 16 codes -> fp16 16-byte chunks 2k, 2k + 1
          const uint32_t wd[4] = {raw[k].x, raw[k].y, raw[k].z, raw[k].w};
          uint32_t o[8];
#pragma unroll
          for (int i = 0; i < 4; ++i) dequant_e4m3x4_f16(wd[i], sc2, o[2 * i], o[2 * i + 1]);
          const uint32_t a = row + hb * kChunkBytes;
          st_shared_v4(a + (((2 * k) ^ (cr & 7)) << 4), make_uint4(o[0], o[1], o[2], o[3]));
          st_shared_v4(a + (((2 * k + 1) ^ (cr & 7)) << 4), make_uint4(o[4], o[5], o[6], o[7]));
        }
      }
      fence_proxy_async_smem();   // read by the tensor cores
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->kv_conv[s]);
      return true;
    };
    int g = 0;
    int pages_total = 0, widened = 0;   // FP8 cache: this cluster's pages, and those widened so far
    if constexpr (kFp8) {
      for (int it = it_begin; it < it_end; ++it)
        pages_total += items[(size_t)it * kItemWords + kItPageEnd] - items[(size_t)it * kItemWords + kItPageBegin];
    }
    for (int it = it_begin; it < it_end; ++it) {
      const int32_t* w = items + (size_t)it * kItemWords;
      const int ii = it - it_begin;
      if (ii > 0 && !warp_wait(&bars->q_empty, (ii - 1) & 1, wc)) goto sender_fail;
      {
        {
          const uint4* rsrc = reinterpret_cast<const uint4*>(p.q_rope + ((size_t)w[kItRow] * p.n_heads + r) * 64 +
                                                             32 * rank);
          // row r of the K-major A tile, 64 bytes: 16-byte chunk k at (k ^ ((r >> 1) & 3))
          // (the 64-byte swizzle the MMA descriptor names)
          uint4 q[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) q[k] = r < p.n_heads ? __ldg(rsrc + k) : make_uint4(0, 0, 0, 0);
          const uint32_t dst = smem_u32(s_qrope) + r * 64;
#pragma unroll
          for (int k = 0; k < 4; ++k) st_shared_v4(dst + ((k ^ ((r >> 1) & 3)) << 4), q[k]);
          fence_proxy_async_smem();   // read by the tensor cores
        }
        const uint4* src = reinterpret_cast<const uint4*>(p.q_lat + ((size_t)w[kItRow] * p.n_heads + r) * 512 +
                                                          256 * rank);
        if constexpr (kFp8) {   // the latent products take fp16 operands: 32 columns at a time
#pragma unroll 1
          for (int hq = 0; hq < 4; ++hq) {
            uint32_t v[32];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint4 q = r < p.n_heads ? __ldg(src + 8 * hq + k) : make_uint4(0, 0, 0, 0);
              v[4 * k] = bf16x2_to_f16x2(q.x); v[4 * k + 1] = bf16x2_to_f16x2(q.y);
              v[4 * k + 2] = bf16x2_to_f16x2(q.z); v[4 * k + 3] = bf16x2_to_f16x2(q.w);
            }
            tmem_st32(tmem + lane_addr + kTmemQ + 32 * hq, v);
          }
        } else {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t v[64];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const uint4 q = r < p.n_heads ? __ldg(src + 16 * hh + k) : make_uint4(0, 0, 0, 0);
              v[4 * k] = q.x; v[4 * k + 1] = q.y; v[4 * k + 2] = q.z; v[4 * k + 3] = q.w;
            }
            tmem_st32(tmem + lane_addr + kTmemQ + 64 * hh, *reinterpret_cast<uint32_t(*)[32]>(v));
            tmem_st32(tmem + lane_addr + kTmemQ + 64 * hh + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->q_full);
      }
      const int n = w[kItPageEnd] - w[kItPageBegin];
      for (int j = 0; j < n; ++j, ++g) {
        if constexpr (kFp8) {   // pages up to g + 1: at g = 0 pages 0 and 1, then one per page
          for (; widened < min(g + 2, pages_total); ++widened)
            if (!widen(widened)) goto sender_fail;
        }
        uint32_t v[64];
        if (!warp_wait(&bars->s_full, g & 1, wc)) goto sender_fail;
        tc_fence_after();
        tmem_ld32(tmem + lane_addr + kTmemS, *reinterpret_cast<uint32_t(*)[32]>(v));
        tmem_ld32(tmem + lane_addr + kTmemS + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_read);
        uint32_t hv[32];
#pragma unroll
        for (int k = 0; k < 32; ++k)   // scaled to log2 units, then rounded to fp16
          hv[k] = pack_f16(__uint_as_float(v[2 * k]) * sl2, __uint_as_float(v[2 * k + 1]) * sl2);
        // single tile: page g - 1's own tile must have been read by the softmax and the copy
        if (g >= 1 && !warp_wait(&bars->own_free, (g - 1) & 1, wc)) goto sender_fail;
        {
          uint8_t* own = s_xown + r * kXRow;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            *reinterpret_cast<uint4*>(own + ((k ^ (r & 7)) << 4)) =
                make_uint4(hv[4 * k], hv[4 * k + 1], hv[4 * k + 2], hv[4 * k + 3]);
        }
        fence_proxy_async_smem();   // the copy warp's bulk copy reads the tile through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->own_full);
      }
    }
    goto sender_done;
  sender_fail:
    give_up();
    if (lane == 0) report(p.status, MLA_STATUS_TIMEOUT);
  sender_done:;
  } else if (warp == kCopyWarp) {
    // ------------------------------------------------------------ score copy (one thread)
    // Per page: one bulk copy of the own fp16 tile to the peer's tile,
    // completing on the peer's x_recv, once the 4 sender warps have written
    // it and the peer has read page g - 1 out of its tile.  The own tile may
    // be rewritten once the copy has read it (own_free).  A warp of its own,
    // so that waiting for the copy never holds back the next page's score read.
    if (lane == 0) {
      const uint32_t x_peer = mapa(smem_u32(s_xpeer), peer);
      const uint32_t x_recv_peer = mapa(smem_u32(&bars->x_recv), peer);
      uint32_t sent = 0;
      bool ok = true;
      int g = 0;
      for (int it = it_begin; ok && it < it_end; ++it) {
        const int32_t* w = items + (size_t)it * kItemWords;
        const int n = w[kItPageEnd] - w[kItPageBegin];
        for (int j = 0; j < n; ++j, ++g) {
          if (!mbar_wait<false, kWaitHintNs>(&bars->own_full, g & 1, wc) ||
              (g >= 1 && !mbar_wait<false, kWaitHintNs>(&bars->x_sendok, (g - 1) & 1, wc))) {
            ok = false;
            break;
          }
          bulk_copy_to_peer(x_peer, smem_u32(s_xown), kXBytes, x_recv_peer);
          bulk_commit();
          *sent_count = ++sent;
          bulk_wait_read<0>();
          mbar_arrive(&bars->own_free);
        }
      }
      if (!ok) {
        give_up();
        report(p.status, MLA_STATUS_TIMEOUT);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue (8 warps)
    // Thread = (row r, key half c): keys [32c, 32c+32) of each page, output
    // columns [128c, 128c+128) of this CTA's 256.
    const int quarter = warp & 3;
    const int c = (warp - kSoftWarp0) >> 2;
    const int r = quarter * 32 + lane;
    const int tid = threadIdx.x - kSoftWarp0 * 32;    // 0 .. 255
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const uint32_t x_sendok_peer = mapa(smem_u32(&bars->x_sendok), peer);
    bool out_of_range = false;   // a fp16 partial overflowed: a reference max of +Inf, or a NaN sum
    // The sequence length of the next item is loaded one item ahead, so that
    // the stale-plan check never waits for memory at an item boundary.
    // So is the next item's draft mask, when drafts form a tree.
    constexpr bool tree = kTree;
    int T_next = 0, m_next = 0;
    if (it_begin < it_end) {
      const int32_t* w0 = items + (size_t)it_begin * kItemWords;
      T_next = p.seq_lens[w0[kItB]];
      if (tree) m_next = p.draft_masks[w0[kItRow]];
    }
    int g = 0;
    for (int it = it_begin; it < it_end; ++it) {
      const int32_t* w = items + (size_t)it * kItemWords;
      const int row = w[kItRow], slot = w[kItSlot], pb = w[kItPageBegin];
      const int n = w[kItPageEnd] - pb;
      const int ii = it - it_begin;
      const bool stale = item_stale(w, T_next, p);
      const uint32_t drafts_seen = (uint32_t)m_next;
      if (it + 1 < it_end) {
        const int32_t* w1 = items + (size_t)(it + 1) * kItemWords;
        T_next = p.seq_lens[w1[kItB]];
        if (tree) m_next = p.draft_masks[w1[kItRow]];
      }
      // key index of the first draft (the plan of a tree batch is not causal: kv_len = T)
      const int first_draft = w[kItKvLen] - p.s_q;
      if (stale && tid == 0 && rank == 0) report(p.status, MLA_STATUS_BAD_SEQLEN);
      // keys masked in the item's last page: the zero-filled rows of its shifted load
      const int shift_last = kPage - min(last_page_keys(w), kPage);

      float m_ref = -CUDART_INF_F, l_run = 0.f;
      for (int j = 0; j < n; ++j) {
        const int gj = g + j, b = gj & 1;
        // full score = fp16(own partial) + fp16(peer partial), identical in both CTAs.
        // The own tile is read (and released) first: it lands before the peer's.
        uint4 po[4], pr[4];
        const uint32_t off_base = (uint32_t)(4 * c);
        if (!warp_wait(&bars->own_full, gj & 1, wc)) goto softmax_fail;
        {
          const uint8_t* orow = s_xown + r * kXRow;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            po[k] = *reinterpret_cast<const uint4*>(orow + (((off_base + k) ^ (r & 7)) << 4));
          uint32_t bar_addr = smem_u32(&bars->own_free);
          // arrive only after the own tile was read (one word of each 16-byte load)
          asm volatile("" : "+r"(bar_addr) : "r"(po[0].x ^ po[1].x ^ po[2].x ^ po[3].x));
          __syncwarp();
          if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar_addr) : "memory");
        }
        if (!warp_wait_cluster(&bars->x_recv, gj & 1, wc)) goto softmax_fail;
        {
          const uint8_t* xrow = s_xpeer + r * kXRow;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            pr[k] = *reinterpret_cast<const uint4*>(xrow + (((off_base + k) ^ (r & 7)) << 4));
          // the peer tile is consumed: re-arm x_recv for page gj + 1, then let the peer refill it
          uint32_t ok_addr = x_sendok_peer;
          asm volatile("" : "+r"(ok_addr) : "r"(pr[0].x ^ pr[1].x ^ pr[2].x ^ pr[3].x));
          __syncwarp();
          if (lane == 0) {
            if (warp == kSoftWarp0) mbar_arrive_expect_tx(&bars->x_recv, kXBytes);
            mbar_arrive_relaxed_cluster(ok_addr);
          }
        }
        // scores in log2 units: fp16(own) + fp16(peer), summed as fp16 pairs
        uint32_t s2[16];
        {
          const uint32_t* ow = reinterpret_cast<const uint32_t*>(po);
          const uint32_t* pw = reinterpret_cast<const uint32_t*>(pr);
#pragma unroll
          for (int k = 0; k < 16; ++k) s2[k] = hadd2(ow[k], pw[k]);
        }
        // masked keys [0, lo) of this page (-inf): the last page's zero fill, or
        // all of them when the device seq_lens disagree with the plan
        const int lo = stale ? kPage : (j == n - 1 ? shift_last : 0);
        if (lo > 32 * c) {
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            if (32 * c + 2 * k < lo) s2[k] = (s2[k] & 0xffff0000u) | 0xfc00u;
            if (32 * c + 2 * k + 1 < lo) s2[k] = (s2[k] & 0x0000ffffu) | 0xfc000000u;
          }
        }
        if constexpr (tree) {
          // draft keys: column col holds key (page start + col - shift); draft
          // d = key - first_draft is visible iff bit d of this row's mask is set
          const int col0 = first_draft - ((pb + j) * kPage - (j == n - 1 ? shift_last : 0));
          if (col0 < 32 * c + 32) {
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const int d0 = 32 * c + 2 * k - col0, d1 = d0 + 1;
              if (d0 >= 0 && !((drafts_seen >> d0) & 1u)) s2[k] = (s2[k] & 0xffff0000u) | 0xfc00u;
              if (d1 >= 0 && !((drafts_seen >> d1) & 1u)) s2[k] = (s2[k] & 0x0000ffffu) | 0xfc000000u;
            }
          }
        }
        float mloc;
        {
          uint32_t t[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) t[k] = hmax2(s2[k], s2[k + 8]);
#pragma unroll
          for (int k = 0; k < 4; ++k) t[k] = hmax2(t[k], t[k + 4]);
          t[0] = hmax2(hmax2(t[0], t[2]), hmax2(t[1], t[3]));
          const float2 m2 = unpack_f16x2(t[0]);
          mloc = fmaxf(m2.x, m2.y);
        }
        s_pmax[(b * 2 + c) * kRows + r] = mloc;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->pmax[b][quarter]);
        if (!warp_wait(&bars->pmax[b][quarter], (gj >> 1) & 1, wc)) goto softmax_fail;
        const float mx = fmaxf(mloc, s_pmax[(b * 2 + (c ^ 1)) * kRows + r]);

        // lazy reference max (log2 domain): move it only when the row max grows by > 2^8
        const float m_new = fmaxf(m_ref, mx);
        const bool move = (m_ref == -CUDART_INF_F) ? (m_new != -CUDART_INF_F)
                                                   : (m_new > m_ref + kRescaleThreshold);
        float alpha = 1.f;
        if (move) {
          alpha = (m_ref == -CUDART_INF_F) ? 0.f : ex2(m_ref - m_new);
          m_ref = m_new;
        }
        const float nb = (m_ref == -CUDART_INF_F) ? 0.f : -m_ref;
        uint32_t pk[16];
        float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          float x0, x1;
          add_f16x2_to_f32(s2[k], nb, x0, x1);   // exact score + nb, rounded once
          const float e0 = ex2(x0), e1 = ex2(x1);
          pk[k] = kFp8 ? pack_f16(e0, e1) : pack_bf16(e0, e1);
          ps[k & 3] += e0 + e1;
        }
        l_run = l_run * alpha + ((ps[0] + ps[1]) + (ps[2] + ps[3]));

        // P buffer gj & 1 is free once the PV product of page gj - 2 has completed
        if (gj >= 2 && !warp_wait(&bars->o_full[gj & 1], ((gj >> 1) - 1) & 1, wc)) goto softmax_fail;
        if (__any_sync(0xffffffffu, move && j > 0)) {
          // rescaling O: the PV product of page gj - 1 (same item) must have landed
          if (!warp_wait(&bars->o_full[(gj - 1) & 1], ((gj - 1) >> 1) & 1, wc)) goto softmax_fail;
          tc_fence_after();
          const float a = (move && j > 0) ? alpha : 1.f;
#pragma unroll 1
          for (int q = 0; q < 4; ++q) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_addr + kTmemO + 128 * c + 32 * q, o);
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * a);
            tmem_st32(tmem + lane_addr + kTmemO + 128 * c + 32 * q, o);
          }
          tmem_st_wait();
        }
        tmem_st16(tmem + lane_addr + kTmemP + 32 * (gj & 1) + 16 * c, pk);   // keys [32c, 32c+32), bf16 pairs
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full);
      }

      // epilogue: O / l  ->  o_lat (whole row) or the row's partial slot.  A
      // stale item has P = 0 throughout: its row is written as zeros.
      {
        if (!warp_wait(&bars->o_done, ii & 1, wc)) goto softmax_fail;
        tc_fence_after();
        float* ls = s_lsum + (ii & 1) * 2 * kRows;    // [item parity][half][row]
        ls[c * kRows + r] = l_run;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->lsum[quarter]);
        if (!warp_wait(&bars->lsum[quarter], ii & 1, wc)) goto softmax_fail;
        l_run = ls[r] + ls[kRows + r];             // same order in both halves
        out_of_range |= (m_ref == CUDART_INF_F) | (l_run != l_run);
        const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
        const bool valid = r < p.n_heads;
        const bool o_lat_32b = (reinterpret_cast<uintptr_t>(p.o_lat) & 31) == 0;
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_addr + kTmemO + 128 * c + 32 * q, o);
          tmem_ld_wait();
          if (!valid) continue;
          const int col = 256 * rank + 128 * c + 32 * q;
          if (slot < 0) {
            uint32_t pk[16];
#pragma unroll
            for (int k = 0; k < 16; ++k)
              pk[k] = pack_bf16(__uint_as_float(o[2 * k]) * inv_l, __uint_as_float(o[2 * k + 1]) * inv_l);
            __nv_bfloat16* dst = p.o_lat + ((size_t)row * p.n_heads + r) * 512 + col;
            if (o_lat_32b) {   // one full 32-byte sector per store
              st_global_v8(dst, pk[0], pk[1], pk[2], pk[3], pk[4], pk[5], pk[6], pk[7]);
              st_global_v8(dst + 16, pk[8], pk[9], pk[10], pk[11], pk[12], pk[13], pk[14], pk[15]);
            } else {
#pragma unroll
              for (int k = 0; k < 4; ++k)
                reinterpret_cast<uint4*>(dst)[k] = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
            }
          } else {
            // column-group-major partials, 8 columns (32 bytes) per group: a warp's
            // 32 rows of one group are 1 KB contiguous, and a reader of one row
            // gets whole 32-byte sectors
            float* dst = p.o_part + (((size_t)slot * 64 + col / 8) * p.n_heads + r) * 8;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              uint32_t v[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) v[e] = __float_as_uint(__uint_as_float(o[8 * k + e]) * inv_l);
              st_global_v8(dst + (size_t)k * p.n_heads * 8, v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]);
            }
          }
        }
        if (valid && rank == 0 && c == 0) {
          const float lse = (l_run > 0.f) ? (m_ref + __log2f(l_run)) * kLn2 : -CUDART_INF_F;
          if (slot >= 0) p.lse_part[(size_t)slot * p.n_heads + r] = lse;
          else if (p.lse_out) p.lse_out[(size_t)row * p.n_heads + r] = lse;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->o_free);
      }
      g += n;
    }
    goto softmax_done;
  softmax_fail:
    give_up();
    if (lane == 0) report(p.status, MLA_STATUS_TIMEOUT);
  softmax_done:
    if (__any_sync(0xffffffffu, out_of_range) && lane == 0 && rank == 0) report(p.status, MLA_STATUS_SCORE_RANGE);
  }

  tc_fence_before();
  __syncthreads();
  __syncwarp();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
  __syncwarp();
  cluster_sync();   // no CTA leaves while its peer may still write into its shared memory
  // After a give-up, roles may have left their loops with the peer's last
  // score tile still on its way here.  A give-up raises both CTAs' flags
  // before its CTA reaches the barrier above, so after it both flags agree
  // and both CTAs take the same branch.  A copy is only sent after the
  // receiver consumed the previous one, so at most the peer's last copy is
  // outstanding: wait (default limit) for its phase, which lands because it
  // was issued, then meet the peer once more.
  {
    // (addresses recomputed here rather than kept live through the roles)
    Bars* b = reinterpret_cast<Bars*>(((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023)) + kOffBar);
    if (*reinterpret_cast<volatile int*>(&b->wc.abort) != 0) {
      if (threadIdx.x == 0) {
        const uint32_t sent_by_peer = ld_cluster_u32(mapa(smem_u32(&b->sent_count), cluster_ctarank() ^ 1u));
        if (sent_by_peer > 0) mbar_drain<true>(&b->x_recv, (sent_by_peer - 1) & 1);
      }
      __syncwarp();
      cluster_sync();
    }
  }
}

std::atomic<uint64_t> g_wait_limit_ns{kWaitLimitNs};

// Set once per process, so that later launches can be captured in a CUDA graph.
template <bool kFp8, bool kTree>
cudaError_t decode_smem_attr() {
  static cudaError_t e =
      cudaFuncSetAttribute(mla_decode_kernel<kFp8, kTree>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  return e;
}

template <bool kFp8, bool kTree>
mla_status_t launch_decode_impl(const mla_dims_t& d, const void* q_lat, const void* q_rope,
                                const void* kv_pool, const int32_t* block_table,
                                const int32_t* seq_lens, const int32_t* draft_masks, const int32_t* plan_dev,
                                int32_t num_clusters, float* o_part, float* lse_part,
                                void* o_lat, float* lse_out, int32_t* status, void* stream) {
  // The pool as (column, row within the block, block): a box may start at a
  // negative row, which the TMA fills with zeros (the shifted last page).
  CUtensorMap tm_kv, tm_rope, tm_scale;
  mla_status_t st;
  if constexpr (kFp8) {
    const uint64_t rstr[2] = {kF8Row, (uint64_t)kPage * kF8Row};
    const uint64_t cdims[3] = {512, (uint64_t)kPage, (uint64_t)d.num_blocks};
    const uint32_t box_c[3] = {128, kPage, 1};
    st = encode_tmap_u8(&tm_kv, kv_pool, 3, cdims, rstr, box_c, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != MLA_OK) return st;
    const uint64_t sdims[3] = {16, (uint64_t)kPage, (uint64_t)d.num_blocks};
    const uint32_t box_s[3] = {16, kF8ScaleKeys, 1};
    st = encode_tmap_u8(&tm_scale, static_cast<const uint8_t*>(kv_pool) + kF8ScaleOff, 3, sdims, rstr, box_s,
                        CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != MLA_OK) return st;
    const uint64_t rdims[3] = {64, (uint64_t)kPage, (uint64_t)d.num_blocks};
    const uint32_t box_r[3] = {32, kPage, 1};
    st = encode_tmap_bf16(&tm_rope, static_cast<const uint8_t*>(kv_pool) + kF8RopeOff, 3, rdims, rstr, box_r,
                          CU_TENSOR_MAP_SWIZZLE_64B);
    if (st != MLA_OK) return st;
  } else {
    const uint64_t pdims[3] = {576, (uint64_t)kPage, (uint64_t)d.num_blocks};
    const uint64_t pstr[2] = {576 * 2, (uint64_t)kPage * 576 * 2};
    const uint32_t box_kv[3] = {64, kPage, 1};
    const uint32_t box_rope[3] = {32, kPage, 1};
    st = encode_tmap_bf16(&tm_kv, kv_pool, 3, pdims, pstr, box_kv, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != MLA_OK) return st;
    st = encode_tmap_bf16(&tm_rope, kv_pool, 3, pdims, pstr, box_rope, CU_TENSOR_MAP_SWIZZLE_64B);
    if (st != MLA_OK) return st;
    tm_scale = tm_rope;   // unused
  }
  const int N = d.B * d.s_q;

  DecodeParams p;
  p.q_lat = static_cast<const __nv_bfloat16*>(q_lat);
  p.q_rope = static_cast<const __nv_bfloat16*>(q_rope);
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.plan = plan_dev;
  p.draft_masks = draft_masks;
  p.o_part = o_part;
  p.lse_part = lse_part;
  p.o_lat = static_cast<__nv_bfloat16*>(o_lat);
  p.lse_out = lse_out;
  p.status = status;
  p.n_heads = d.n_heads;
  p.max_blocks = d.max_blocks_per_seq;
  p.num_blocks = d.num_blocks;
  p.s_q = d.s_q;
  p.causal = d.causal;
  p.B = d.B;
  p.n_rows = N;
  p.num_clusters = num_clusters;
  p.scale_log2 = d.scale * 1.4426950408889634f;
  p.wait_ns = g_wait_limit_ns.load(std::memory_order_relaxed);

  cudaError_t e = decode_smem_attr<kFp8, kTree>();
  if (e == cudaSuccess) {
    e = launch_pdl(mla_decode_kernel<kFp8, kTree>, dim3(2 * num_clusters), dim3(kThreads), kSmemBytes, stream, tm_kv,
                   tm_rope, tm_scale, p);
    if (e == cudaSuccess) e = cudaGetLastError();
  }
  if (e != cudaSuccess) return set_error(MLA_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
  return MLA_OK;
}

}  // namespace

mla_status_t launch_decode_attn(const mla_dims_t& d, const void* q_lat, const void* q_rope,
                                const void* kv_pool, const int32_t* block_table,
                                const int32_t* seq_lens, const int32_t* draft_masks, const int32_t* plan_dev,
                                int32_t num_clusters, float* o_part, float* lse_part,
                                void* o_lat, float* lse_out, int32_t* status, void* stream) {
  if (draft_masks)
    return launch_decode_impl<false, true>(d, q_lat, q_rope, kv_pool, block_table, seq_lens, draft_masks, plan_dev,
                                           num_clusters, o_part, lse_part, o_lat, lse_out, status, stream);
  return launch_decode_impl<false, false>(d, q_lat, q_rope, kv_pool, block_table, seq_lens, nullptr, plan_dev,
                                          num_clusters, o_part, lse_part, o_lat, lse_out, status, stream);
}

mla_status_t launch_decode_attn_fp8cache(const mla_dims_t& d, const void* q_lat, const void* q_rope,
                                         const void* kv_pool_fp8, const int32_t* block_table,
                                         const int32_t* seq_lens, const int32_t* plan_dev, int32_t num_clusters,
                                         float* o_part, float* lse_part, void* o_lat, float* lse_out,
                                         int32_t* status, void* stream) {
  return launch_decode_impl<true, false>(d, q_lat, q_rope, kv_pool_fp8, block_table, seq_lens, nullptr, plan_dev,
                                         num_clusters, o_part, lse_part, o_lat, lse_out, status, stream);
}

void set_decode_wait_limit_ns(int64_t ns) {
  g_wait_limit_ns.store(ns > 0 ? (uint64_t)ns : kWaitLimitNs, std::memory_order_relaxed);
}

mla_status_t decode_max_clusters(int32_t* n) {
  cudaError_t e = decode_smem_attr<false, false>();
  if (e != cudaSuccess) return set_error(MLA_ERR_CUDA, "max clusters: %s", cudaGetErrorString(e));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int count = 0;
  e = cudaOccupancyMaxActiveClusters(&count, mla_decode_kernel<false, false>, &cfg);
  if (e != cudaSuccess || count <= 0) {
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    count = sms / 2;
    cudaGetLastError();
  }
  *n = count;
  return MLA_OK;
}

}  // namespace mla
