// kvq_decode_attn_noalloc: decode attention + merge with a fixed, library-owned scratch.
//
// Some callers cannot allocate device memory at decode time: an inference runtime that
// pre-plans every buffer before serving, a process running under a memory pool that
// forbids new allocations, or a host that calls in from a context where cudaMalloc is
// not permitted.  This entry point runs the same split-KV kernel, with its in-kernel
// merge, as kvq_decode_attn given an output pointer, but keeps the partials and merge
// words in a static device array owned by the library, so the caller passes only
// inputs and outputs.
#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

// Every GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[KVQ_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array on the current device.  In host code the symbol
// name is only a host-side stand-in, never a device address, so it is looked up with
// cudaGetSymbolAddress, with the device current, on every call: nothing is cached that a
// reset or a recreated context could leave stale.  The first lookup on a device is its
// set-up (it may load the library's device code there).
int scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return KVQ_ERR_CUDA;
  *out = p;
  return KVQ_OK;
}

}  // namespace
}  // namespace kvq

using namespace kvq;

extern "C" int kvq_decode_attn_noalloc(const kvq_cache_desc* desc, const void* q, int32_t batch,
                                       int32_t num_q_heads, const void* k_codes,
                                       const void* k_scales, const void* v_codes,
                                       const void* v_scales, const int32_t* page_table,
                                       int32_t max_pages, const int32_t* seq_lens,
                                       int32_t max_seq_len, float sm_scale, float tau,
                                       int32_t split_tokens, uint32_t options,
                                       unsigned long long* stats, float* out, void* stream) {
  if (!desc || !out) return KVQ_ERR_INVALID_ARG;
  const int32_t L = kvq_resolve_split(desc, batch, num_q_heads, max_seq_len, split_tokens, options);
  if (L < 0) return L;
  const size_t need = kvq_workspace_size(batch, num_q_heads, desc->head_dim, max_seq_len, L);
  if (need == 0 || need > (size_t)KVQ_NOALLOC_SCRATCH_BYTES) return KVQ_ERR_WORKSPACE;
  void* ws = nullptr;
  int st = scratch_address(&ws);
  if (st != KVQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the flag word and the merge words start at zero for every call; the launch
  // counter in the header (bytes 8..15) keeps counting, so that no exchange entry left
  // by an earlier call carries the tag of this one
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), s) != cudaSuccess ||
      cudaMemsetAsync(static_cast<uint8_t*>(ws) + kWorkspaceHeader, 0, counters_bytes(batch, num_q_heads),
                      s) != cudaSuccess)
    return KVQ_ERR_CUDA;
  // the merge runs inside the decode kernel (output pointer given)
  return kvq_decode_attn(desc, q, batch, num_q_heads, k_codes, k_scales, v_codes, v_scales,
                         page_table, max_pages, seq_lens, max_seq_len, sm_scale, tau, L, options,
                         ws, need, stats, out, stream);
}

extern "C" int kvq_noalloc_read_flags(uint32_t* flags, void* stream) {
  if (!flags) return KVQ_ERR_INVALID_ARG;
  void* ws = nullptr;
  const int st = scratch_address(&ws);
  if (st != KVQ_OK) return st;
  // the flag word is word 0 of the scratch, as of a workspace
  return kvq_read_device_flags(ws, flags, stream);
}
