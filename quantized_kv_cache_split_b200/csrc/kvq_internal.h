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
  unsigned long long* stats;
  int num_sms;
};

// Partials inside the workspace (after the 256-byte header):
//   o [batch][num_q_heads][max_splits][head_dim] fp32 (unnormalized)
//   m [batch][num_q_heads][max_splits] fp32 (running maximum, log2 units)
//   l [batch][num_q_heads][max_splits] fp32
size_t partials_bytes(int batch, int num_q_heads, int head_dim, int max_splits);

int launch_quantize(const kvq_cache_desc& desc, const void* x, int n_tok, const int32_t* slots,
                    void* codes, void* scales, cudaStream_t stream);
int launch_decode(const DecodeArgs& a, cudaStream_t stream);
int launch_combine(const kvq_cache_desc& desc, const void* workspace, int batch, int num_q_heads,
                   int max_seq_len, int split_tokens, int max_splits, const int32_t* seq_lens,
                   float* out, cudaStream_t stream);

int device_sm_count();

}  // namespace kvq
