// Internal declarations shared by the library's translation units.
#pragma once
#include "../../include/mla.h"

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

namespace mla {

// Launches `kernel` with programmatic stream serialization: it may begin its
// set-up while the previous kernel in the stream is still running (every
// kernel of the library calls ptx::griddep_wait() before touching global memory).
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, void* stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Records a printf-style message in the thread-local error slot; returns `code`.
mla_status_t set_error(mla_status_t code, const char* fmt, ...);
void clear_error();

mla_status_t build_plan(const mla_dims_t& d, const int32_t* seq_lens, int32_t num_clusters,
                        int32_t* plan, int64_t plan_words, int32_t* num_slots_out);

// Kernel launchers (defined in the .cu files); each returns MLA_OK or MLA_ERR_CUDA.
mla_status_t launch_absorb_q(const void* q_nope, const void* w_uk, void* q_lat, int n_tokens,
                             int n_heads, void* stream);
mla_status_t launch_out_uv(const void* o_lat, const void* w_uv, void* out, int n_tokens,
                           int n_heads, void* stream);
mla_status_t launch_quantize_weight_fp8(const void* w, int n_heads, bool transposed, void* codes, float* scales,
                                        void* stream);
mla_status_t launch_quantize_rows_fp8(const void* x, long long rows, int cols, void* codes, float* scales,
                                      void* stream);
mla_status_t launch_absorb_q_fp8(const void* q_nope, const void* w_codes, const float* w_scales, void* q_lat,
                                 int n_tokens, int n_heads, void* stream);
mla_status_t launch_out_uv_fp8(const void* o_lat, const void* w_codes, const float* w_scales, void* out,
                               int n_tokens, int n_heads, void* stream);
mla_status_t launch_decode_attn(const mla_dims_t& d, const void* q_lat, const void* q_rope,
                                const void* kv_pool, const int32_t* block_table,
                                const int32_t* seq_lens, const int32_t* draft_masks, const int32_t* plan_dev,
                                int32_t num_clusters, float* o_part, float* lse_part,
                                void* o_lat, float* lse_out, int32_t* status, void* stream);
// The same kernel on an FP8 latent cache (rows of 656 bytes: 512 E4M3 codes,
// 4 fp32 block scales, 64 bf16 k_rope).  No draft-tree masks.
mla_status_t launch_decode_attn_fp8cache(const mla_dims_t& d, const void* q_lat, const void* q_rope,
                                         const void* kv_pool_fp8, const int32_t* block_table,
                                         const int32_t* seq_lens, const int32_t* plan_dev, int32_t num_clusters,
                                         float* o_part, float* lse_part, void* o_lat, float* lse_out,
                                         int32_t* status, void* stream);
// bf16 cache rows [n][576] -> FP8 pool slots (flat token index block * 64 + row).
mla_status_t launch_kv_quantize_fp8(const void* kv, const int32_t* slots, long long n, void* pool_fp8,
                                   long long pool_rows, int32_t* status, void* stream);
mla_status_t launch_combine(const mla_dims_t& d, const int32_t* plan_dev, int32_t n_rows,
                            const float* o_part, const float* lse_part, void* o_lat,
                            float* lse_out, void* stream);
mla_status_t launch_prefill_up_proj(const void* kv_pool, const int32_t* block_row, int T, int num_blocks,
                                    const void* w_uk, const void* w_uv, int n_heads, void* k_out, void* v_out,
                                    void* stream);
mla_status_t launch_prefill_attn(const void* q_nope, const void* q_rope, const void* k, const void* v,
                                 const void* kv_pool, const int32_t* block_row, int T, int s, int n_heads,
                                 int num_blocks, float scale, void* out, float* lse, void* stream);
mla_status_t launch_q_up_absorb(const void* c_q, const void* w_uq, const void* w_uk, void* q_lat, void* q_rope,
                                int n_tokens, int n_heads, void* stream);
mla_status_t launch_qkv_a_proj(const void* x, const void* w, void* c_q, void* kv_a, int n_tokens, void* stream);
mla_status_t launch_gather_pages(const void* kv_pool, const int32_t* block_table, int32_t b,
                                 int32_t n_pages, int32_t max_blocks, int32_t num_blocks, void* out,
                                 int32_t* status, void* stream);
mla_status_t decode_max_clusters(int32_t* n);
void set_decode_wait_limit_ns(int64_t ns);
mla_status_t decode_attn_combine_noalloc(const mla_dims_t& d, const void* q_lat, const void* q_rope,
                                         const void* kv_pool, const int32_t* block_table,
                                         const int32_t* seq_lens, const void* plan_host,
                                         size_t plan_bytes, int32_t num_clusters, void* o_lat,
                                         float* lse_out, int32_t* status, void* stream);
size_t noalloc_scratch_bytes();

}  // namespace mla
