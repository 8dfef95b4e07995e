/*
 * mla.h -- C ABI of the B200 (sm_100a) absorbed MLA decode library (libmla).
 *
 * The library computes one decode step of DeepSeek-V2/V3 Multi-head Latent
 * Attention (MLA) in the absorbed evaluation order ("order 2") of the MLA
 * matrix-absorption notes (wkq9411.github.io, "MLA Matrix Absorption
 * Analysis", section 2.2 for the logits and section 3.2 for the output):
 *
 *   q_lat[n,h,:] = sum_d q_nope[n,h,d] * W_UK[:,h,d]                mla_absorb_q
 *   logit[n,h,t] = scale * (q_lat[n,h].c_KV[t] + q_rope[n,h].k_rope[t])
 *   p = softmax_t(logit), o_lat[n,h,:] = sum_t p[t] c_KV[t]          mla_decode_attn
 *                                                                   (+ mla_combine)
 *   out[n,h,:]   = sum_k o_lat[n,h,k] * W_UV[k,h,:]                  mla_out_uv
 *
 * K = W_UK c_KV and V = W_UV c_KV are never formed, nor are W_UQ^T W_UK or
 * W_O W_UV.  The RoPE key is the extra multi-query term of the izhida.com
 * answer "How is DeepSeek-V2's inference cost computed?": one 64-wide
 * post-rotation key per token, shared by all heads, whose score is added.
 *
 * Conventions (every entry point):
 *   - bf16 is IEEE bfloat16 stored as uint16; fp32 is IEEE float.
 *   - All tensor arguments are CALLER-OWNED DEVICE pointers (plan_host and
 *     seq_lens_host excepted), contiguous row-major, 16-byte aligned.  The
 *     library never allocates, frees or retains device memory.
 *   - `stream` is a cudaStream_t (passed as void*); every device call is
 *     asynchronous on it.  Host-side validation happens before any launch.
 *   - Return value: MLA_OK or an error code; mla_last_error_string() gives a
 *     thread-local message for the last failing call.  Nothing aborts,
 *     throws or traps across this boundary.
 *   - Device-detected faults (a block id outside [0, num_blocks), a wait
 *     that ran past its time limit) set bits of the optional int32 *status
 *     word (atomic OR) and skip or substitute the affected work; they never
 *     trap.  Pass NULL to skip status reporting.
 *
 * Shapes: n_tokens N = B * s_q query rows; row n = b * s_q + i.
 * Supported: d_nope = 128, d_rope = 64, d_c = 512, d_v = 128, page_size = 64,
 * 1 <= s_q <= 8, 1 <= n_heads <= 128.  Other shapes return MLA_ERR_UNSUPPORTED.
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,        /* null/misaligned pointer, bad size, inconsistent plan */
  MLA_ERR_UNSUPPORTED = 2,        /* shape outside the supported set */
  MLA_ERR_WORKSPACE_TOO_SMALL = 3,
  MLA_ERR_CUDA = 4,               /* a CUDA runtime call failed (message has the CUDA error) */
  MLA_ERR_TIMEOUT = 5
} mla_status_t;

/* Bits set in the device status word. */
#define MLA_STATUS_BAD_BLOCK   0x1   /* block_table entry outside [0, num_blocks): block 0 used */
#define MLA_STATUS_TIMEOUT     0x2   /* a bounded device wait expired; outputs are invalid */
#define MLA_STATUS_BAD_SEQLEN  0x4   /* a row's device seq_lens disagrees with the plan: row skipped */
#define MLA_STATUS_BAD_PLAN    0x8   /* the plan was made for other dims or another cluster count:
                                        nothing computed */
#define MLA_STATUS_SCORE_RANGE 0x10  /* a partial score of an attended key left the fp16 range
                                        (|x| > 65504) or was not a number: outputs are invalid */
#define MLA_STATUS_CACHE_RANGE 0x20  /* mla_kv_quantize_fp8: a 128-column block of c_KV has
                                        amax > 65504, beyond what mla_decode_attn_fp8cache widens
                                        (fp16); the row is written but must not be attended */

/* Problem dimensions of one decode batch. */
typedef struct {
  int32_t B;                  /* sequences */
  int32_t s_q;                /* new query tokens per sequence: 1, or up to 8 speculative (MTP) */
  int32_t n_heads;            /* h */
  int32_t d_nope;             /* 128 */
  int32_t d_rope;             /* 64 */
  int32_t d_c;                /* 512 (latent width of c_KV) */
  int32_t d_v;                /* 128 */
  int32_t page_size;          /* 64 tokens per cache block */
  int32_t max_blocks_per_seq; /* columns of block_table */
  int32_t num_blocks;         /* blocks in the cache pool */
  float scale;                /* softmax scale, e.g. 1/sqrt(d_nope + d_rope) */
  int32_t causal;             /* s_q > 1: 1 = query i attends t <= T - s_q + i; 0 = all T */
} mla_dims_t;

/* Library version (major * 10000 + minor * 100 + patch). */
int32_t mla_version(void);

/* Thread-local message of the last failing call on this thread ("" if none). */
const char* mla_last_error_string(void);

/*
 * mla_absorb_q -- first absorption, order 2, Step 2 of the notes' section 2.2:
 * the per-head contraction q_lat = q_nope^T W_UK (term 2bshkd of FLOPs_order2).
 *   q_nope  bf16 [n_tokens][n_heads][128]   (device, read)
 *   w_uk    bf16 [512][n_heads][128]        (device, read; (k, h, d) as in section 2.1)
 *   q_lat   bf16 [n_tokens][n_heads][512]   (device, written; fp32 accumulation, RNE to bf16)
 * 1 <= n_tokens <= 65536.
 */
mla_status_t mla_absorb_q(const void* q_nope, const void* w_uk, void* q_lat,
                          int32_t n_tokens, int32_t n_heads, void* stream);

/*
 * mla_out_uv -- second absorption, order 2, Step 2 of the notes' section 3.2:
 * out = W_UV applied per head to the latent output (term 2bhsvk of FLOPs_order2).
 *   o_lat   bf16 [n_tokens][n_heads][512]   (device, read)
 *   w_uv    bf16 [512][n_heads][128]        (device, read; (k, h, v) as in section 3.1)
 *   out     bf16 [n_tokens][n_heads][128]   (device, written; fp32 accumulation)
 */
mla_status_t mla_out_uv(const void* o_lat, const void* w_uv, void* out,
                        int32_t n_tokens, int32_t n_heads, void* stream);

/*
 * FP8 block-quantised projections ("Lower latency and higher throughput with
 * multi-node DeepSeek deployment", sections "Quantization" and "MLA layer":
 * k_b_proj and v_b_proj as FP8 block-quantised BMMs).  Weights are quantised
 * once, with one fp32 scale per 128 x 128 block of each head's matrix;
 * activations are quantised on the fly inside the BMMs, with one scale per
 * 128-element vector along K.  The format is E4M3 (largest finite 448).  A
 * block's scale is s = amax / 448 (s = 1 for an all-zero block) and a value's
 * code is E4M3(x * (448 / amax)), rounded to nearest even and saturated.  Each
 * K-block's code products are summed in fp32 by the tensor cores, then
 * scaled by s_act * s_weight; the outputs are bf16 (RNE).
 *
 * mla_quantize_w_uk_fp8: w_uk bf16 [512][n_heads][128] (read) ->
 *   w_codes E4M3 [n_heads][512][128] (written; per head, rows k, K = d
 *   contiguous) and w_scales fp32 [n_heads][4] (written; block k / 128).
 * mla_quantize_w_uv_fp8: w_uv bf16 [512][n_heads][128] (read) ->
 *   w_codes E4M3 [n_heads][128][512] (written; per head, rows v, K = k
 *   contiguous) and w_scales fp32 [n_heads][4] (written; block k / 128).
 * mla_quantize_rows_fp8: x bf16 [rows][cols] (cols a multiple of 128) ->
 *   codes E4M3 [rows][cols] and scales fp32 [rows][cols / 128]: the same
 *   per-vector quantisation the BMMs apply to their activations.
 * mla_absorb_q_fp8: as mla_absorb_q, with the weight given as codes and
 *   scales from mla_quantize_w_uk_fp8; q_nope is quantised per (token, head).
 * mla_out_uv_fp8: as mla_out_uv, with codes and scales from
 *   mla_quantize_w_uv_fp8; o_lat is quantised per (token, head, 128 columns).
 * Codes are bytes; every pointer is a device pointer (16-byte aligned except
 * the scale arrays, which need 4).  1 <= n_heads <= 128, 1 <= n_tokens <= 65536.
 */
mla_status_t mla_quantize_w_uk_fp8(const void* w_uk, int32_t n_heads, void* w_codes, float* w_scales,
                                   void* stream);
mla_status_t mla_quantize_w_uv_fp8(const void* w_uv, int32_t n_heads, void* w_codes, float* w_scales,
                                   void* stream);
mla_status_t mla_quantize_rows_fp8(const void* x, int64_t rows, int32_t cols, void* codes, float* scales,
                                   void* stream);
mla_status_t mla_absorb_q_fp8(const void* q_nope, const void* w_uk_codes, const float* w_uk_scales, void* q_lat,
                              int32_t n_tokens, int32_t n_heads, void* stream);
mla_status_t mla_out_uv_fp8(const void* o_lat, const void* w_uv_codes, const float* w_uv_scales, void* out,
                            int32_t n_tokens, int32_t n_heads, void* stream);

/*
 * Split-KV planning (host only, deterministic).  The decode kernel is a
 * persistent grid of 2-CTA clusters; each cluster walks a contiguous range of
 * the flattened (sequence, page) work list of one query position, so a long
 * sequence is split across clusters and a cluster can cover several short
 * ones.  Ranges are equal in pages plus a fixed cost of five pages for every
 * row a range starts.  Pieces of a split row are merged by mla_combine.
 *
 * mla_plan_size: upper bounds for the plan (int32 words, in bytes) and for
 *   the two workspace arrays, o_part (slots x n_heads x 512 fp32) and
 *   lse_part fp32 [slots][n_heads], for `num_clusters` clusters.
 * mla_plan: writes the plan into caller memory `plan_host` (plan_bytes from
 *   mla_plan_size); the caller copies it to the device unchanged.  Fails with
 *   MLA_ERR_INVALID_ARG if some seq_lens_host[b] < s_q or > max_blocks*64.
 *   *num_slots receives the number of partial-output slots used.
 * mla_max_clusters: how many decode clusters the current device runs at once
 *   (the natural `num_clusters`).
 */
mla_status_t mla_max_clusters(int32_t* num_clusters);
mla_status_t mla_plan_size(const mla_dims_t* dims, int32_t num_clusters, size_t* plan_bytes,
                           size_t* o_part_bytes, size_t* lse_part_bytes);
mla_status_t mla_plan(const mla_dims_t* dims, const int32_t* seq_lens_host, int32_t num_clusters,
                      void* plan_host, size_t plan_bytes, int32_t* num_slots);

/*
 * mla_decode_attn -- the attention core: scores of the absorbed query
 * [q_lat | q_rope] against the paged [c_KV | k_rope] cache (notes section 2.2
 * Step 3, term 2bhstk, plus the RoPE term), softmax over t, and the weighted
 * sum of c_KV (notes section 3.2 Step 1, term 2bhskt).
 *   q_lat        bf16 [N][n_heads][512]     (from mla_absorb_q)
 *   q_rope       bf16 [N][n_heads][64]      (post-rotation)
 *   kv_pool      bf16 [num_blocks][64][576] (token row = c_KV (512) | k_rope (64))
 *   block_table  int32 [B][max_blocks_per_seq]
 *   seq_lens     int32 [B]  T_b, counting the s_q new tokens.  A plan is valid for the
 *                lengths it was made from: the kernel compares each row's key count
 *                with these device values, and a row that disagrees is skipped
 *                (written as zeros with LSE -inf) and MLA_STATUS_BAD_SEQLEN is
 *                set.  A decode loop whose lengths grow every step makes a new
 *                plan (mla_plan, host only, microseconds) and copies it each step.
 *   plan_dev     the plan from mla_plan, copied to the device
 *   num_clusters the num_clusters the plan was built for (grid = 2 * num_clusters CTAs)
 *   o_part       fp32, slots x n_heads x 512  workspace (split rows), 32-byte
 *                aligned; element (slot, h, col) at
 *                ((slot*64 + col/8)*n_heads + h)*8 + col%8, so that the stores
 *                of 32 rows are contiguous and a reader of one row gets whole
 *                32-byte sectors
 *   lse_part     fp32 [slots][n_heads]        workspace
 *   o_lat        bf16 [N][n_heads][512]       rows not split are written here
 *   lse_out      fp32 [N][n_heads] or NULL    natural-log LSE of the scaled logits
 *   status       int32 [1] or NULL
 * Rows that the plan splits are completed by mla_combine.
 *
 * Numerics: the two CTAs of a cluster each score half of the 576 columns and
 * exchange their partial scores rounded to fp16; a partial of an attended key
 * beyond the fp16 range sets MLA_STATUS_SCORE_RANGE.  Cache rows past a row's
 * key count (page tails, other queries' keys) may hold anything, NaN and Inf
 * included: the kernel zeroes them in shared memory before the P.c_KV product.
 */
mla_status_t mla_decode_attn(const mla_dims_t* dims, const void* q_lat, const void* q_rope,
                             const void* kv_pool, const int32_t* block_table,
                             const int32_t* seq_lens, const void* plan_dev, int32_t num_clusters,
                             float* o_part, float* lse_part, void* o_lat, float* lse_out,
                             int32_t* status, void* stream);

/*
 * mla_decode_attn_tree -- mla_decode_attn for drafted tokens that form a tree
 * (EAGLE-style speculative decoding, named as future work in "Lower latency
 * and higher throughput with multi-node DeepSeek deployment", section
 * "Будущая работа": several tokens drafted as a tree instead of a chain).
 * Query i of sequence b attends every committed key t < T_b - s_q and the
 * drafts its mask allows:
 *   draft_masks  int32 [B][s_q] (device): bit j of draft_masks[b * s_q + i]
 *                set = key T_b - s_q + j (draft j) is visible to query i.
 *                For a tree, row i holds i's ancestors and i itself; the
 *                causal rule is the chain's masks (bits 0 .. i).
 * The plan must be made with dims->causal = 0 (every row covers all T_b
 * keys; MLA_ERR_INVALID_ARG otherwise).  A row whose mask and prefix leave
 * no key visible is written as zeros with LSE -inf.  1 <= s_q <= 8.  All
 * other arguments and outputs are those of mla_decode_attn; mla_combine
 * completes split rows as usual.
 */
mla_status_t mla_decode_attn_tree(const mla_dims_t* dims, const void* q_lat, const void* q_rope,
                                  const void* kv_pool, const int32_t* block_table, const int32_t* seq_lens,
                                  const int32_t* draft_masks, const void* plan_dev, int32_t num_clusters,
                                  float* o_part, float* lse_part, void* o_lat, float* lse_out,
                                  int32_t* status, void* stream);

/*
 * mla_decode_attn_fp8cache -- mla_decode_attn on an FP8 latent cache.  The
 * pages quantise activations in 128-element blocks with one scale each ("Lower
 * latency and higher throughput with multi-node DeepSeek deployment", section
 * "Quantization"); applied to the cached c_KV row that halves the bytes the
 * decode streams per token (656 instead of 1152), the cache-size argument of
 * the izhida.com answer.  Token row layout (656 bytes, 16-byte multiple):
 *   bytes [0, 512)    E4M3 codes of c_KV[t, 0..511]
 *   bytes [512, 528)  fp32 scales s_0..s_3, c_KV[t, c] = code[c] * s_{c / 128}
 *   bytes [528, 656)  k_rope[t, 0..63] in bf16 (not quantised)
 *   kv_pool_fp8  uint8 [num_blocks][64][656], 16-byte aligned (mla_kv_quantize_fp8 writes it)
 * Numerics: the kernel widens every staged row to fp16 (code * fp16(scale),
 * rounded once), rounds q_lat to fp16 and writes P as fp16, and runs the
 * latent products on those fp16 operands (fp32 accumulation); the RoPE
 * products are bf16 as in mla_decode_attn.  Blocks need amax <= 65504 (see
 * MLA_STATUS_CACHE_RANGE) and q_lat |x| <= 65504 (beyond, the scores become
 * infinite and MLA_STATUS_SCORE_RANGE is set).  All other arguments, outputs,
 * status bits and the plan are those of mla_decode_attn; mla_combine
 * completes split rows.  No draft-tree masks.
 */
mla_status_t mla_decode_attn_fp8cache(const mla_dims_t* dims, const void* q_lat, const void* q_rope,
                                      const void* kv_pool_fp8, const int32_t* block_table,
                                      const int32_t* seq_lens, const void* plan_dev, int32_t num_clusters,
                                      float* o_part, float* lse_part, void* o_lat, float* lse_out,
                                      int32_t* status, void* stream);

/*
 * mla_kv_quantize_fp8 -- write cache rows into FP8 pool slots (the layout of
 * mla_decode_attn_fp8cache).  Per 128-column block of c_KV: amax = max |x|,
 * s = amax / 448, code = E4M3(x * (448 / amax)) rounded to nearest even and
 * saturated (an all-zero block takes s = 1); k_rope is copied.
 *   kv        bf16 [n][576]  rows c_KV (512) | k_rope (64), 16-byte aligned
 *   slots     int32 [n]      destination of row i: block * 64 + row in the block (4-byte aligned)
 *   pool_fp8  uint8 [num_blocks][64][656]
 *   status    int32 [1] or NULL: MLA_STATUS_BAD_BLOCK when a slot lies outside
 *             the pool (that row is not written); MLA_STATUS_CACHE_RANGE when a
 *             block's amax exceeds 65504 (written, but not attendable)
 * Rows with equal slots race (one of them wins).
 */
mla_status_t mla_kv_quantize_fp8(const void* kv, const int32_t* slots, int64_t n, void* pool_fp8,
                                 int32_t num_blocks, int32_t* status, void* stream);

/*
 * mla_combine -- log-sum-exp merge of the split pieces of each split row:
 *   L = log sum_i exp(lse_i),  o_lat = sum_i exp(lse_i - L) * O_i.
 * Reads o_part/lse_part written by mla_decode_attn with the same plan, writes
 * o_lat bf16 [N][n_heads][512] and (if non-NULL) lse_out for split rows only.
 */
mla_status_t mla_combine(const mla_dims_t* dims, const void* plan_dev, const float* o_part, const float* lse_part, void* o_lat,
                         float* lse_out, void* stream);

/*
 * mla_decode_attn_combine_noalloc -- mla_decode_attn followed by mla_combine,
 * for callers that cannot allocate device memory.  There is no counterpart in
 * the paper; it exists for deployment.
 *
 * Some callers may not call cudaMalloc while they run: a serving runtime that
 * reserves nearly all HBM for its paged KV-cache pool at start-up and only
 * hands kernels buffers it planned for, or a plugin invoked where allocation
 * is forbidden.  Such a caller cannot supply the o_part / lse_part workspace
 * or a device copy of the plan that the two calls above take.  This entry
 * point takes the HOST plan (from mla_plan) and keeps the plan copy and the
 * split-KV partial outputs in a fixed device array owned by the library:
 *   - its size is mla_noalloc_scratch_bytes() (32 MiB); a batch whose plan
 *     needs more returns MLA_ERR_WORKSPACE_TOO_SMALL and launches nothing;
 *   - every GPU that loads the library holds that array until the process
 *     exits;
 *   - the first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture;
 *   - it allocates nothing and frees nothing;
 *   - all calls share the array, and it keeps the last call's contents
 *     (nothing in it needs to start at zero); calls that overlap on the GPU
 *     race on it, so serialise them;
 *   - the plan is copied to the array with cudaMemcpyAsync on `stream`: from
 *     pageable memory the call returns once the bytes are staged, but from
 *     pinned memory the copy may still be reading plan_host after the call
 *     returns, so do not overwrite it until the stream has passed this call;
 *   - `stream` must belong to the current device (MLA_ERR_INVALID_ARG
 *     otherwise): the array used is the current device's.
 * The plan is checked against dims and num_clusters on the host before any
 * copy (magic word, cluster count, B, s_q, n_heads, max_blocks_per_seq,
 * causal, and that plan_bytes covers it); a mismatch is MLA_ERR_INVALID_ARG.
 * The other arguments mean what they mean for mla_decode_attn / mla_combine;
 * o_lat (and lse_out if non-NULL) receive the finished rows.
 */
mla_status_t mla_decode_attn_combine_noalloc(const mla_dims_t* dims, const void* q_lat,
                                             const void* q_rope, const void* kv_pool,
                                             const int32_t* block_table, const int32_t* seq_lens,
                                             const void* plan_host, size_t plan_bytes,
                                             int32_t num_clusters, void* o_lat, float* lse_out,
                                             int32_t* status, void* stream);

/*
 * Upstream of the absorbed path, fused.
 *
 * mla_qkv_a_proj -- the Perplexity write-up's qkv_a_proj ("MLA layer": q_a_proj
 * and kv_a_proj merged into one product): for the hidden states of N tokens,
 *   c_q  = x W^DQ   and   kv_a = x W^DKV = [c_KV | k_rope (before rotation)]
 *   x        bf16 [N][7168]           (DeepSeek-V3 model width)
 *   w_qkv_a  bf16 [2112][7168]        rows 0..1535 = W^DQ^T, rows 1536..2111 = W^DKV^T
 *   c_q      bf16 [N][1536] (written), kv_a bf16 [N][576] (written; the cache row)
 * fp32 accumulation; one launch (the K range is split over a cluster of 8
 * CTAs and reduced through distributed shared memory).  1 <= N <= 65536.
 *
 * mla_q_up_absorb -- the query up-projection feeding the first absorption
 * without q_nope leaving the SM ("MLA Matrix Absorption Analysis" section 2.2
 * Steps 1-2, terms 2bshdq and 2bshkd):
 *   q[n,h,:]     = sum_j c_q[n,j] W_UQ[j,h,:]           (128 nope + 64 RoPE columns)
 *   q_lat[n,h,:] = sum_d q[n,h,d] W_UK[:,h,d]            (d < 128)
 *   c_q    bf16 [N][1536], w_uq bf16 [1536][n_heads][192] (q, h, d + R), w_uk bf16 [512][n_heads][128]
 *   q_lat  bf16 [N][n_heads][512] (written), q_rope bf16 [N][n_heads][64] (written, before rotation)
 * W_UQ^T W_UK is never formed.  1 <= N <= 65536, 1 <= n_heads <= 128.
 */
mla_status_t mla_qkv_a_proj(const void* x, const void* w_qkv_a, void* c_q, void* kv_a, int32_t n_tokens,
                            void* stream);
mla_status_t mla_q_up_absorb(const void* c_q, const void* w_uq, const void* w_uk, void* q_lat, void* q_rope,
                             int32_t n_tokens, int32_t n_heads, void* stream);

/*
 * Prefill and chunked prefill in order 1 ("MHA form").  "MLA Matrix
 * Absorption Analysis" section 2.4.1: when the query length equals the key
 * length (t = s) the un-absorbed order 1 needs fewer FLOPs than the absorbed
 * order 2 (by 98304 s^2 at DeepSeek-V3 widths), and the Perplexity write-up's
 * future-work section names prefill in the up-projected form and chunked
 * prefill.  One sequence per call; its cache rows are read through its
 * block-table row (int32 [ceil(T / 64)], device), as in decode.
 *
 * mla_prefill_up_proj -- K and V of the sequence's first T tokens:
 *   K[t,h,:] = W_UK[:,h,:]^T c_KV[t]   (notes section 2.1 Step 2)
 *   V[t,h,:] = W_UV[:,h,:]^T c_KV[t]   (notes section 3.1 Step 1)
 *   k_out, v_out   bf16 [T][n_heads][128] (device, written; fp32 accumulation)
 *   w_uk, w_uv     bf16 [512][n_heads][128]
 *
 * mla_prefill_attn -- causal attention of the chunk's s query tokens (the last
 * s of the T cached tokens, positions T - s .. T - 1; s = T is a full
 * prefill, s < T a chunk after a prefix) over K, V and the cached RoPE keys:
 *   logit[i,h,t] = scale (q_nope[i,h] . K[t,h] + q_rope[i,h] . k_rope[t])
 *   out[i,h,:]   = sum_{t <= T - s + i} softmax_t(logit) V[t,h,:]
 *   q_nope bf16 [s][n_heads][128], q_rope bf16 [s][n_heads][64] (post-rotation)
 *   k, v   bf16 [T][n_heads][128] from mla_prefill_up_proj
 *   out    bf16 [s][n_heads][128] (written), lse fp32 [s][n_heads] or NULL
 * 1 <= s <= T <= 2^22, 1 <= n_heads <= 128.
 */
mla_status_t mla_prefill_up_proj(const void* kv_pool, const int32_t* block_table_row, int32_t T, int32_t num_blocks,
                                 const void* w_uk, const void* w_uv, int32_t n_heads, void* k_out, void* v_out,
                                 void* stream);
mla_status_t mla_prefill_attn(const void* q_nope, const void* q_rope, const void* k, const void* v,
                              const void* kv_pool, const int32_t* block_table_row, int32_t T, int32_t s,
                              int32_t n_heads, int32_t num_blocks, float scale, void* out, float* lse, void* stream);

/* Size in bytes of the device array mla_decode_attn_combine_noalloc works in. */
size_t mla_noalloc_scratch_bytes(void);

/*
 * mla_set_wait_limit_ns -- upper bound, in nanoseconds of GPU global time, on
 * each wait of the decode kernel's pipeline roles for every decode launch
 * made after the call (process-wide).  Default 200 ms; ns <= 0 restores it.
 * When a wait runs past the bound the kernel sets MLA_STATUS_TIMEOUT, stops
 * both CTAs of the cluster, waits (with the default bound) for the copies and
 * tensor-core products it has already issued, frees its tensor memory and
 * returns; the context stays usable.  A tiny bound makes the time-out path run
 * on purpose, which is what the failure-detection test does.
 */
void mla_set_wait_limit_ns(int64_t ns);

/*
 * mla_debug_gather_pages -- copies the cache rows of sequence b, in token
 * order, through block_table into out bf16 [n_pages*64][576] (bit-exact page
 * indexing check; not on the decode path).  Out-of-range block ids set
 * MLA_STATUS_BAD_BLOCK and write zeros.
 */
mla_status_t mla_debug_gather_pages(const void* kv_pool, const int32_t* block_table, int32_t b,
                                    int32_t n_pages, int32_t max_blocks_per_seq, int32_t num_blocks,
                                    void* out, int32_t* status, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MLA_H_ */
