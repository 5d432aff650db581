// Internal interfaces between the C-ABI layer (kvq_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

constexpr int kTile = 64;  // positions per K tile / per TMA box

struct DecodeArgs {
  kvq_cache_desc desc;
  const void* q;
  int batch, num_q_heads, group;
  const void* k_codes;
  const void* k_scales;
  const void* v_codes;
  const void* v_scales;
  const int32_t* page_table;
  int max_pages;
  const int32_t* seq_lens;
  int max_seq_len;
  float sm_scale, tau;
  int split_tokens;   // resolved, multiple of kTile
  int max_splits;     // ceil(max_seq_len / split_tokens)
  void* workspace;
  unsigned long long* arrive;  // [batch][num_kv_heads] exchange arrival words (kArriveStep per launch)
  unsigned long long* zflag;  // [batch][num_kv_heads] output rows cleared (launch tag)
  unsigned long long* epoch;  // launch counter in the workspace header (exchange tags)
  float* part_o;      // partials, see below
  float* part_m;
  float* part_l;
  ulonglong2* xch;    // tagged (m, l) each split publishes for the others
                      // [batch][num_q_heads][max_splits]
  unsigned long long* stats;
  float* out;         // non-null: merge in the same kernel and write the output
  int cluster;        // consecutive splits per thread-block cluster (1, 2, 4 or 8)
  int shared_max;     // the splits of a cluster share one running maximum
  int global_max;     // every split of a (sequence, KV head) uses the maximum over all of them
  int grid;           // CTAs launched (a multiple of cluster)
  int units_per_seq;  // cluster groups of one (sequence, KV head) at max_seq_len
  int group_merge;    // every unit has its own CTA: the splits of a (sequence, KV head)
                      // exchange (m, l) and each adds its share into the output
  int v_early;        // tau > 0: copy each V tile together with its K tile (every row,
                      // kept or not) instead of only the kept rows after the skip test
};

// Workspace: a 256-byte header (word 0: KVQ_FLAG_* bits; bytes 8..15: the launch
// counter that tags the exchange entries); the merge words (u64 "output rows cleared"
// flags, then u64 exchange arrival counts, each
// [batch][num_q_heads] of which [batch][num_kv_heads] are used, together rounded up to 256
// bytes); then, one slot per split:
//   (m, l) exchange [batch][num_q_heads][max_splits] 2 x u64, each word a fp32 value
//   under a 32-bit launch tag (what the splits of a (sequence, KV head) publish to one
//   another)
//   o [batch][num_q_heads][max_splits][head_dim] fp32 (unnormalized)
//   m [batch][num_q_heads][max_splits] fp32 (running maximum, log2 units)
//   l [batch][num_q_heads][max_splits] fp32
size_t partials_bytes(int batch, int num_q_heads, int head_dim, int max_splits);
__host__ __device__ inline size_t counters_bytes(int batch, int num_q_heads) {
  return ((size_t)batch * num_q_heads * (2 * sizeof(uint64_t)) + 255) / 256 * 256;
}

// x2 == nullptr: one plane pair; otherwise the second pair (x2, codes2, scales2) in the
// same launch.
int launch_quantize(const kvq_cache_desc& desc, const void* x, const void* x2, int n_tok,
                    const int32_t* slots, void* codes, void* scales, void* codes2, void* scales2,
                    cudaStream_t stream);
int launch_selftest_wait(void* workspace, long long max_cycles, cudaStream_t stream);
int launch_combine(const kvq_cache_desc& desc, const void* workspace, int batch, int num_q_heads,
                   int max_seq_len, int split_tokens, int max_splits, const int32_t* seq_lens,
                   float* out, cudaStream_t stream);

int device_sm_count();

}  // namespace kvq
