// Exported C ABI of libmla: argument validation, error reporting, planning and launches.
#include "mla_internal.h"
#include "plan_format.h"
#include "tmap.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>

namespace mla {

static thread_local char g_err[512] = "";

mla_status_t set_error(mla_status_t code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

void clear_error() { g_err[0] = '\0'; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

static mla_status_t encode_tmap(CUtensorMap* map, CUtensorMapDataType type, const void* base, int rank,
                                const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                                CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return set_error(MLA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t d[5], s[4];
  cuuint32_t b[5], e[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    e[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) s[i] = strides_bytes[i];
  CUresult r = fn(map, type, (cuuint32_t)rank, const_cast<void*>(base), d, s,
                  b, e, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(MLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MLA_OK;
}

mla_status_t encode_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                              const uint64_t* strides_bytes, const uint32_t* box,
                              CUtensorMapSwizzle swizzle) {
  return encode_tmap(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, rank, dims, strides_bytes, box, swizzle);
}

mla_status_t encode_tmap_u8(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                            const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swizzle) {
  return encode_tmap(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, rank, dims, strides_bytes, box, swizzle);
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static mla_status_t check_ptr(const void* p, const char* name) {
  if (!p) return set_error(MLA_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned16(p)) return set_error(MLA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return MLA_OK;
}

static mla_status_t check_dims(const mla_dims_t* d) {
  if (!d) return set_error(MLA_ERR_INVALID_ARG, "dims is NULL");
  if (d->B < 1 || d->num_blocks < 1 || d->max_blocks_per_seq < 1)
    return set_error(MLA_ERR_INVALID_ARG, "B, num_blocks and max_blocks_per_seq must be >= 1");
  if (d->d_nope != 128 || d->d_rope != 64 || d->d_c != 512 || d->d_v != 128 || d->page_size != 64)
    return set_error(MLA_ERR_UNSUPPORTED,
                     "only d_nope=128, d_rope=64, d_c=512, d_v=128, page_size=64 are supported");
  if (d->s_q < 1 || d->s_q > 8) return set_error(MLA_ERR_UNSUPPORTED, "s_q must be in [1, 8]");
  if (d->n_heads < 1 || d->n_heads > 128) return set_error(MLA_ERR_UNSUPPORTED, "n_heads must be in [1, 128]");
  if (!(d->scale > 0.f) || d->scale != d->scale) return set_error(MLA_ERR_INVALID_ARG, "scale must be > 0");
  if ((int64_t)d->num_blocks * 64 > INT32_MAX) return set_error(MLA_ERR_UNSUPPORTED, "pool too large");
  if ((int64_t)d->B * d->s_q > 65536) return set_error(MLA_ERR_UNSUPPORTED, "more than 65536 query rows");
  return MLA_OK;
}

static mla_status_t check_tokens(int n_tokens, int n_heads) {
  if (n_tokens < 1 || n_tokens > 65536) return set_error(MLA_ERR_UNSUPPORTED, "n_tokens must be in [1, 65536]");
  if (n_heads < 1 || n_heads > 128) return set_error(MLA_ERR_UNSUPPORTED, "n_heads must be in [1, 128]");
  return MLA_OK;
}

}  // namespace mla

using namespace mla;

#define MLA_TRY(x)                     \
  do {                                 \
    mla_status_t _s = (x);             \
    if (_s != MLA_OK) return _s;       \
  } while (0)

extern "C" {

int32_t mla_version(void) { return 100; }

const char* mla_last_error_string(void) { return g_err; }

mla_status_t mla_absorb_q(const void* q_nope, const void* w_uk, void* q_lat, int32_t n_tokens,
                          int32_t n_heads, void* stream) {
  clear_error();
  MLA_TRY(check_tokens(n_tokens, n_heads));
  MLA_TRY(check_ptr(q_nope, "q_nope"));
  MLA_TRY(check_ptr(w_uk, "w_uk"));
  MLA_TRY(check_ptr(q_lat, "q_lat"));
  return launch_absorb_q(q_nope, w_uk, q_lat, n_tokens, n_heads, stream);
}

mla_status_t mla_out_uv(const void* o_lat, const void* w_uv, void* out, int32_t n_tokens,
                        int32_t n_heads, void* stream) {
  clear_error();
  MLA_TRY(check_tokens(n_tokens, n_heads));
  MLA_TRY(check_ptr(o_lat, "o_lat"));
  MLA_TRY(check_ptr(w_uv, "w_uv"));
  MLA_TRY(check_ptr(out, "out"));
  return launch_out_uv(o_lat, w_uv, out, n_tokens, n_heads, stream);
}

mla_status_t mla_quantize_w_uk_fp8(const void* w_uk, int32_t n_heads, void* w_codes, float* w_scales,
                                   void* stream) {
  clear_error();
  if (n_heads < 1 || n_heads > 128) return set_error(MLA_ERR_UNSUPPORTED, "n_heads must be in [1, 128]");
  MLA_TRY(check_ptr(w_uk, "w_uk"));
  MLA_TRY(check_ptr(w_codes, "w_codes"));
  if (!w_scales) return set_error(MLA_ERR_INVALID_ARG, "w_scales is NULL");
  return launch_quantize_weight_fp8(w_uk, n_heads, false, w_codes, w_scales, stream);
}

mla_status_t mla_quantize_w_uv_fp8(const void* w_uv, int32_t n_heads, void* w_codes, float* w_scales,
                                   void* stream) {
  clear_error();
  if (n_heads < 1 || n_heads > 128) return set_error(MLA_ERR_UNSUPPORTED, "n_heads must be in [1, 128]");
  MLA_TRY(check_ptr(w_uv, "w_uv"));
  MLA_TRY(check_ptr(w_codes, "w_codes"));
  if (!w_scales) return set_error(MLA_ERR_INVALID_ARG, "w_scales is NULL");
  return launch_quantize_weight_fp8(w_uv, n_heads, true, w_codes, w_scales, stream);
}

mla_status_t mla_quantize_rows_fp8(const void* x, int64_t rows, int32_t cols, void* codes, float* scales,
                                   void* stream) {
  clear_error();
  if (rows < 0) return set_error(MLA_ERR_INVALID_ARG, "rows must be >= 0");
  if (cols < 128 || cols % 128 != 0) return set_error(MLA_ERR_UNSUPPORTED, "cols must be a positive multiple of 128");
  if (rows == 0) return MLA_OK;
  MLA_TRY(check_ptr(x, "x"));
  MLA_TRY(check_ptr(codes, "codes"));
  if (!scales) return set_error(MLA_ERR_INVALID_ARG, "scales is NULL");
  return launch_quantize_rows_fp8(x, rows, cols, codes, scales, stream);
}

mla_status_t mla_absorb_q_fp8(const void* q_nope, const void* w_uk_codes, const float* w_uk_scales, void* q_lat,
                              int32_t n_tokens, int32_t n_heads, void* stream) {
  clear_error();
  MLA_TRY(check_tokens(n_tokens, n_heads));
  MLA_TRY(check_ptr(q_nope, "q_nope"));
  MLA_TRY(check_ptr(w_uk_codes, "w_uk_codes"));
  MLA_TRY(check_ptr(q_lat, "q_lat"));
  if (!w_uk_scales) return set_error(MLA_ERR_INVALID_ARG, "w_uk_scales is NULL");
  return launch_absorb_q_fp8(q_nope, w_uk_codes, w_uk_scales, q_lat, n_tokens, n_heads, stream);
}

mla_status_t mla_out_uv_fp8(const void* o_lat, const void* w_uv_codes, const float* w_uv_scales, void* out,
                            int32_t n_tokens, int32_t n_heads, void* stream) {
  clear_error();
  MLA_TRY(check_tokens(n_tokens, n_heads));
  MLA_TRY(check_ptr(o_lat, "o_lat"));
  MLA_TRY(check_ptr(w_uv_codes, "w_uv_codes"));
  MLA_TRY(check_ptr(out, "out"));
  if (!w_uv_scales) return set_error(MLA_ERR_INVALID_ARG, "w_uv_scales is NULL");
  return launch_out_uv_fp8(o_lat, w_uv_codes, w_uv_scales, out, n_tokens, n_heads, stream);
}

mla_status_t mla_max_clusters(int32_t* num_clusters) {
  clear_error();
  if (!num_clusters) return set_error(MLA_ERR_INVALID_ARG, "num_clusters is NULL");
  return decode_max_clusters(num_clusters);
}

mla_status_t mla_plan_size(const mla_dims_t* dims, int32_t num_clusters, size_t* plan_bytes,
                           size_t* o_part_bytes, size_t* lse_part_bytes) {
  clear_error();
  MLA_TRY(check_dims(dims));
  if (num_clusters < 1 || num_clusters > 4096)
    return set_error(MLA_ERR_INVALID_ARG, "num_clusters must be in [1, 4096]");
  const int32_t N = dims->B * dims->s_q;
  const int64_t slots = plan_slots_upper_bound(num_clusters, N);
  if (plan_bytes) *plan_bytes = (size_t)plan_words_upper_bound(num_clusters, N) * 4;
  if (o_part_bytes) *o_part_bytes = (size_t)slots * dims->n_heads * 512 * 4;
  if (lse_part_bytes) *lse_part_bytes = (size_t)slots * dims->n_heads * 4;
  return MLA_OK;
}

mla_status_t mla_plan(const mla_dims_t* dims, const int32_t* seq_lens_host, int32_t num_clusters,
                      void* plan_host, size_t plan_bytes, int32_t* num_slots) {
  clear_error();
  MLA_TRY(check_dims(dims));
  if (!seq_lens_host || !plan_host) return set_error(MLA_ERR_INVALID_ARG, "NULL host buffer");
  if (num_clusters < 1 || num_clusters > 4096)
    return set_error(MLA_ERR_INVALID_ARG, "num_clusters must be in [1, 4096]");
  if ((reinterpret_cast<uintptr_t>(plan_host) & 3u) != 0)
    return set_error(MLA_ERR_INVALID_ARG, "plan_host must be 4-byte aligned");
  return build_plan(*dims, seq_lens_host, num_clusters, static_cast<int32_t*>(plan_host),
                    (int64_t)(plan_bytes / 4), num_slots);
}

mla_status_t mla_decode_attn(const mla_dims_t* dims, const void* q_lat, const void* q_rope,
                             const void* kv_pool, const int32_t* block_table,
                             const int32_t* seq_lens, const void* plan_dev, int32_t num_clusters,
                             float* o_part, float* lse_part, void* o_lat, float* lse_out,
                             int32_t* status, void* stream) {
  clear_error();
  MLA_TRY(check_dims(dims));
  MLA_TRY(check_ptr(q_lat, "q_lat"));
  MLA_TRY(check_ptr(q_rope, "q_rope"));
  MLA_TRY(check_ptr(kv_pool, "kv_pool"));
  MLA_TRY(check_ptr(block_table, "block_table"));
  MLA_TRY(check_ptr(seq_lens, "seq_lens"));
  MLA_TRY(check_ptr(plan_dev, "plan_dev"));
  MLA_TRY(check_ptr(o_lat, "o_lat"));
  if (num_clusters < 1 || num_clusters > 4096)
    return set_error(MLA_ERR_INVALID_ARG, "num_clusters must be in [1, 4096]");
  // o_part / lse_part may be NULL only when the plan splits no row; the kernel
  // checks slots against the plan, the host cannot see the device plan here.
  if ((o_part && (reinterpret_cast<uintptr_t>(o_part) & 31u)) || (lse_part && (reinterpret_cast<uintptr_t>(lse_part) & 3u)))
    return set_error(MLA_ERR_INVALID_ARG, "o_part must be 32-byte aligned, lse_part 4-byte aligned");
  return launch_decode_attn(*dims, q_lat, q_rope, kv_pool, block_table, seq_lens, nullptr,
                            static_cast<const int32_t*>(plan_dev), num_clusters, o_part, lse_part,
                            o_lat, lse_out, status, stream);
}

mla_status_t mla_decode_attn_tree(const mla_dims_t* dims, const void* q_lat, const void* q_rope,
                                  const void* kv_pool, const int32_t* block_table, const int32_t* seq_lens,
                                  const int32_t* draft_masks, const void* plan_dev, int32_t num_clusters,
                                  float* o_part, float* lse_part, void* o_lat, float* lse_out,
                                  int32_t* status, void* stream) {
  clear_error();
  MLA_TRY(check_dims(dims));
  if (dims->causal != 0)
    return set_error(MLA_ERR_INVALID_ARG, "draft-tree attention needs dims->causal = 0 (plan with kv_len = T)");
  MLA_TRY(check_ptr(q_lat, "q_lat"));
  MLA_TRY(check_ptr(q_rope, "q_rope"));
  MLA_TRY(check_ptr(kv_pool, "kv_pool"));
  MLA_TRY(check_ptr(block_table, "block_table"));
  MLA_TRY(check_ptr(seq_lens, "seq_lens"));
  MLA_TRY(check_ptr(draft_masks, "draft_masks"));
  MLA_TRY(check_ptr(plan_dev, "plan_dev"));
  MLA_TRY(check_ptr(o_lat, "o_lat"));
  if (num_clusters < 1 || num_clusters > 4096)
    return set_error(MLA_ERR_INVALID_ARG, "num_clusters must be in [1, 4096]");
  if ((o_part && (reinterpret_cast<uintptr_t>(o_part) & 31u)) || (lse_part && (reinterpret_cast<uintptr_t>(lse_part) & 3u)))
    return set_error(MLA_ERR_INVALID_ARG, "o_part must be 32-byte aligned, lse_part 4-byte aligned");
  return launch_decode_attn(*dims, q_lat, q_rope, kv_pool, block_table, seq_lens, draft_masks,
                            static_cast<const int32_t*>(plan_dev), num_clusters, o_part, lse_part,
                            o_lat, lse_out, status, stream);
}

mla_status_t mla_decode_attn_fp8cache(const mla_dims_t* dims, const void* q_lat, const void* q_rope,
                                      const void* kv_pool_fp8, const int32_t* block_table,
                                      const int32_t* seq_lens, const void* plan_dev, int32_t num_clusters,
                                      float* o_part, float* lse_part, void* o_lat, float* lse_out,
                                      int32_t* status, void* stream) {
  clear_error();
  MLA_TRY(check_dims(dims));
  MLA_TRY(check_ptr(q_lat, "q_lat"));
  MLA_TRY(check_ptr(q_rope, "q_rope"));
  MLA_TRY(check_ptr(kv_pool_fp8, "kv_pool_fp8"));
  MLA_TRY(check_ptr(block_table, "block_table"));
  MLA_TRY(check_ptr(seq_lens, "seq_lens"));
  MLA_TRY(check_ptr(plan_dev, "plan_dev"));
  MLA_TRY(check_ptr(o_lat, "o_lat"));
  if (num_clusters < 1 || num_clusters > 4096)
    return set_error(MLA_ERR_INVALID_ARG, "num_clusters must be in [1, 4096]");
  if ((o_part && (reinterpret_cast<uintptr_t>(o_part) & 31u)) || (lse_part && (reinterpret_cast<uintptr_t>(lse_part) & 3u)))
    return set_error(MLA_ERR_INVALID_ARG, "o_part must be 32-byte aligned, lse_part 4-byte aligned");
  return launch_decode_attn_fp8cache(*dims, q_lat, q_rope, kv_pool_fp8, block_table, seq_lens,
                                     static_cast<const int32_t*>(plan_dev), num_clusters, o_part, lse_part,
                                     o_lat, lse_out, status, stream);
}

mla_status_t mla_kv_quantize_fp8(const void* kv, const int32_t* slots, int64_t n, void* pool_fp8,
                                 int32_t num_blocks, int32_t* status, void* stream) {
  clear_error();
  if (n < 0 || num_blocks < 1) return set_error(MLA_ERR_INVALID_ARG, "n must be >= 0 and num_blocks >= 1");
  if (n == 0) return MLA_OK;
  MLA_TRY(check_ptr(kv, "kv"));
  if (!slots || (reinterpret_cast<uintptr_t>(slots) & 3u))
    return set_error(MLA_ERR_INVALID_ARG, "slots is NULL or not 4-byte aligned");
  MLA_TRY(check_ptr(pool_fp8, "pool_fp8"));
  return launch_kv_quantize_fp8(kv, slots, n, pool_fp8, (long long)num_blocks * 64, status, stream);
}

mla_status_t mla_combine(const mla_dims_t* dims, const void* plan_dev, const float* o_part,
                         const float* lse_part, void* o_lat, float* lse_out, void* stream) {
  clear_error();
  MLA_TRY(check_dims(dims));
  MLA_TRY(check_ptr(plan_dev, "plan_dev"));
  MLA_TRY(check_ptr(o_lat, "o_lat"));
  if (!o_part || !lse_part) return set_error(MLA_ERR_INVALID_ARG, "o_part / lse_part is NULL");
  return launch_combine(*dims, static_cast<const int32_t*>(plan_dev), dims->B * dims->s_q, o_part,
                        lse_part, o_lat, lse_out, stream);
}

mla_status_t mla_decode_attn_combine_noalloc(const mla_dims_t* dims, const void* q_lat, const void* q_rope,
                                              const void* kv_pool, const int32_t* block_table,
                                              const int32_t* seq_lens, const void* plan_host,
                                              size_t plan_bytes, int32_t num_clusters, void* o_lat,
                                              float* lse_out, int32_t* status, void* stream) {
  clear_error();
  MLA_TRY(check_dims(dims));
  MLA_TRY(check_ptr(q_lat, "q_lat"));
  MLA_TRY(check_ptr(q_rope, "q_rope"));
  MLA_TRY(check_ptr(kv_pool, "kv_pool"));
  MLA_TRY(check_ptr(block_table, "block_table"));
  MLA_TRY(check_ptr(seq_lens, "seq_lens"));
  MLA_TRY(check_ptr(o_lat, "o_lat"));
  if (!plan_host || (reinterpret_cast<uintptr_t>(plan_host) & 3u))
    return set_error(MLA_ERR_INVALID_ARG, "plan_host is NULL or not 4-byte aligned");
  if (num_clusters < 1 || num_clusters > 4096)
    return set_error(MLA_ERR_INVALID_ARG, "num_clusters must be in [1, 4096]");
  return decode_attn_combine_noalloc(*dims, q_lat, q_rope, kv_pool, block_table, seq_lens, plan_host,
                                     plan_bytes, num_clusters, o_lat, lse_out, status, stream);
}

size_t mla_noalloc_scratch_bytes(void) { return noalloc_scratch_bytes(); }

mla_status_t mla_q_up_absorb(const void* c_q, const void* w_uq, const void* w_uk, void* q_lat, void* q_rope,
                             int32_t n_tokens, int32_t n_heads, void* stream) {
  clear_error();
  MLA_TRY(check_tokens(n_tokens, n_heads));
  MLA_TRY(check_ptr(c_q, "c_q"));
  MLA_TRY(check_ptr(w_uq, "w_uq"));
  MLA_TRY(check_ptr(w_uk, "w_uk"));
  MLA_TRY(check_ptr(q_lat, "q_lat"));
  MLA_TRY(check_ptr(q_rope, "q_rope"));
  return launch_q_up_absorb(c_q, w_uq, w_uk, q_lat, q_rope, n_tokens, n_heads, stream);
}

mla_status_t mla_qkv_a_proj(const void* x, const void* w_qkv_a, void* c_q, void* kv_a, int32_t n_tokens,
                            void* stream) {
  clear_error();
  if (n_tokens < 1 || n_tokens > 65536) return set_error(MLA_ERR_UNSUPPORTED, "n_tokens must be in [1, 65536]");
  MLA_TRY(check_ptr(x, "x"));
  MLA_TRY(check_ptr(w_qkv_a, "w_qkv_a"));
  MLA_TRY(check_ptr(c_q, "c_q"));
  MLA_TRY(check_ptr(kv_a, "kv_a"));
  return launch_qkv_a_proj(x, w_qkv_a, c_q, kv_a, n_tokens, stream);
}

static mla_status_t check_prefill(int T, int s, int n_heads, int num_blocks) {
  if (n_heads < 1 || n_heads > 128) return set_error(MLA_ERR_UNSUPPORTED, "n_heads must be in [1, 128]");
  if (T < 1 || T > (1 << 22)) return set_error(MLA_ERR_UNSUPPORTED, "T must be in [1, 2^22]");
  if (s < 1 || s > T) return set_error(MLA_ERR_INVALID_ARG, "s must be in [1, T]");
  if (num_blocks < 1 || (int64_t)num_blocks * 64 > INT32_MAX)
    return set_error(MLA_ERR_INVALID_ARG, "num_blocks out of range");
  return MLA_OK;
}

mla_status_t mla_prefill_up_proj(const void* kv_pool, const int32_t* block_table_row, int32_t T, int32_t num_blocks,
                                 const void* w_uk, const void* w_uv, int32_t n_heads, void* k_out, void* v_out,
                                 void* stream) {
  clear_error();
  MLA_TRY(check_prefill(T, 1, n_heads, num_blocks));
  MLA_TRY(check_ptr(kv_pool, "kv_pool"));
  MLA_TRY(check_ptr(block_table_row, "block_table_row"));
  MLA_TRY(check_ptr(w_uk, "w_uk"));
  MLA_TRY(check_ptr(w_uv, "w_uv"));
  MLA_TRY(check_ptr(k_out, "k_out"));
  MLA_TRY(check_ptr(v_out, "v_out"));
  return launch_prefill_up_proj(kv_pool, block_table_row, T, num_blocks, w_uk, w_uv, n_heads, k_out, v_out, stream);
}

mla_status_t mla_prefill_attn(const void* q_nope, const void* q_rope, const void* k, const void* v,
                              const void* kv_pool, const int32_t* block_table_row, int32_t T, int32_t s,
                              int32_t n_heads, int32_t num_blocks, float scale, void* out, float* lse, void* stream) {
  clear_error();
  MLA_TRY(check_prefill(T, s, n_heads, num_blocks));
  if (!(scale > 0.f) || scale != scale) return set_error(MLA_ERR_INVALID_ARG, "scale must be > 0");
  MLA_TRY(check_ptr(q_nope, "q_nope"));
  MLA_TRY(check_ptr(q_rope, "q_rope"));
  MLA_TRY(check_ptr(k, "k"));
  MLA_TRY(check_ptr(v, "v"));
  MLA_TRY(check_ptr(kv_pool, "kv_pool"));
  MLA_TRY(check_ptr(block_table_row, "block_table_row"));
  MLA_TRY(check_ptr(out, "out"));
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return set_error(MLA_ERR_INVALID_ARG, "lse must be 4-byte aligned");
  return launch_prefill_attn(q_nope, q_rope, k, v, kv_pool, block_table_row, T, s, n_heads, num_blocks, scale, out,
                             lse, stream);
}

void mla_set_wait_limit_ns(int64_t ns) { set_decode_wait_limit_ns(ns); }

mla_status_t mla_debug_gather_pages(const void* kv_pool, const int32_t* block_table, int32_t b,
                                    int32_t n_pages, int32_t max_blocks_per_seq, int32_t num_blocks,
                                    void* out, int32_t* status, void* stream) {
  clear_error();
  MLA_TRY(check_ptr(kv_pool, "kv_pool"));
  MLA_TRY(check_ptr(block_table, "block_table"));
  MLA_TRY(check_ptr(out, "out"));
  if (b < 0 || n_pages < 0 || n_pages > max_blocks_per_seq || num_blocks < 1)
    return set_error(MLA_ERR_INVALID_ARG, "bad gather arguments");
  return launch_gather_pages(kv_pool, block_table, b, n_pages, max_blocks_per_seq, num_blocks, out,
                             status, stream);
}

}  // extern "C"
