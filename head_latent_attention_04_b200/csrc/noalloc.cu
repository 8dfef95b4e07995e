// Allocation-free decode entry point: attention + log-sum-exp merge with the
// split-KV workspace in a fixed, library-owned device array.
//
// Who needs this: callers that must not allocate device memory while they
// run -- for example a serving runtime that reserves nearly all HBM for its
// paged KV-cache pool at start-up and hands kernels only what it planned
// for, or a plugin that is invoked from a context where cudaMalloc is not
// allowed.  Those callers cannot provide the o_part / lse_part workspace
// that mla_decode_attn and mla_combine expect, nor a device copy of the plan.
//
// This file holds that workspace as a file-scope __device__ array of
// kScratchBytes.  Every GPU that loads the library reserves it until the
// process exits.  Host code cannot use the array's name as a device address
// (it is a host-side stand-in), so the first call on each device looks the
// real address up with cudaGetSymbolAddress, with that device current, and
// caches it.  Make that first call before any stream capture.
//
// The plan is copied into the array with cudaMemcpyAsync on the caller's
// stream; from pinned host memory that copy may still be reading plan_host
// after the call returns.
//
// All calls share the one array, which keeps whatever the last call left in
// it.  Nothing in it needs to start at zero: the attention kernel writes every
// partial slot the plan uses before the merge reads it.  Calls whose work can
// overlap on the GPU (two streams, or two threads launching at once) race on
// the array and give wrong results; serialise them.
#include "mla_internal.h"
#include "plan_format.h"

#include <cuda_runtime.h>

#include <mutex>

namespace mla {
namespace {

// 32 MiB: the plan and the partial outputs of e.g. a 32-sequence, 128-head,
// 4096-token batch split over 74 clusters (104 slots, about 27 MB) fit.
constexpr size_t kScratchBytes = 32u << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// The array of the current device, which must also be the device of `stream`
// (the plan copy and both kernels run there).
mla_status_t scratch_for_current_device(cudaStream_t stream, void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_error(MLA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  int stream_dev = dev;
  e = cudaStreamGetDevice(stream, &stream_dev);
  if (e != cudaSuccess) return set_error(MLA_ERR_CUDA, "cudaStreamGetDevice: %s", cudaGetErrorString(e));
  if (stream_dev != dev)
    return set_error(MLA_ERR_INVALID_ARG, "stream belongs to device %d but device %d is current", stream_dev, dev);
  if (dev < 0 || dev >= kMaxDevices) return set_error(MLA_ERR_UNSUPPORTED, "device index %d too large", dev);
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return set_error(MLA_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MLA_OK;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace

size_t noalloc_scratch_bytes() { return kScratchBytes; }

mla_status_t decode_attn_combine_noalloc(const mla_dims_t& d, const void* q_lat, const void* q_rope,
                                         const void* kv_pool, const int32_t* block_table,
                                         const int32_t* seq_lens, const void* plan_host,
                                         size_t plan_bytes, int32_t num_clusters, void* o_lat,
                                         float* lse_out, int32_t* status, void* stream) {
  const int32_t* plan = static_cast<const int32_t*>(plan_host);
  if (plan_bytes < kPlanHeaderWords * 4 || plan[kHdrMagic] != kPlanMagic)
    return set_error(MLA_ERR_INVALID_ARG, "plan_host is not a plan made by mla_plan");
  if (plan[kHdrNumClusters] != num_clusters || plan[kHdrB] != d.B || plan[kHdrSq] != d.s_q ||
      plan[kHdrNumRows] != d.B * d.s_q || plan[kHdrHeads] != d.n_heads ||
      plan[kHdrMaxBlocks] != d.max_blocks_per_seq || plan[kHdrCausal] != (d.causal ? 1 : 0))
    return set_error(MLA_ERR_INVALID_ARG, "plan was made for other dims or another cluster count");
  const int64_t words_signed = plan[kHdrTotalWords];
  if (words_signed < kPlanHeaderWords || plan[kHdrNumSlots] < 0)
    return set_error(MLA_ERR_INVALID_ARG, "plan_host is not a plan made by mla_plan");
  const size_t words = (size_t)words_signed;
  if (words * 4 > plan_bytes) return set_error(MLA_ERR_INVALID_ARG, "plan_bytes smaller than the plan");
  const size_t slots = (size_t)plan[kHdrNumSlots];
  const size_t plan_region = round_up(words * 4, 256);
  const size_t lse_region = round_up(slots * d.n_heads * sizeof(float), 256);
  const size_t opart_region = slots * d.n_heads * 512 * sizeof(float);
  const size_t need = plan_region + lse_region + opart_region;
  if (need > kScratchBytes)
    return set_error(MLA_ERR_WORKSPACE_TOO_SMALL,
                     "this batch needs %zu bytes of scratch; the allocation-free entry point has %zu "
                     "(use mla_decode_attn + mla_combine with caller workspace, or fewer clusters)",
                     need, kScratchBytes);

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* base = nullptr;
  mla_status_t st = scratch_for_current_device(s, &base);
  if (st != MLA_OK) return st;
  unsigned char* b = static_cast<unsigned char*>(base);
  int32_t* plan_dev = reinterpret_cast<int32_t*>(b);
  float* lse_part = reinterpret_cast<float*>(b + plan_region);
  float* o_part = reinterpret_cast<float*>(b + plan_region + lse_region);

  cudaError_t e = cudaMemcpyAsync(plan_dev, plan_host, words * 4, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return set_error(MLA_ERR_CUDA, "plan copy: %s", cudaGetErrorString(e));
  st = launch_decode_attn(d, q_lat, q_rope, kv_pool, block_table, seq_lens, nullptr, plan_dev, num_clusters, o_part,
                          lse_part, o_lat, lse_out, status, stream);
  if (st != MLA_OK) return st;
  if (slots > 0)
    st = launch_combine(d, plan_dev, d.B * d.s_q, o_part, lse_part, o_lat, lse_out, stream);
  return st;
}

}  // namespace mla
