// C-ABI entry points of libkvq: argument validation, then one launch each.
// Nothing here allocates device memory or keeps per-call state.
#include <math.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "kvq_decode2.h"
#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {

size_t partials_bytes(int batch, int num_q_heads, int head_dim, int max_splits) {
  const size_t units = (size_t)batch * num_q_heads * max_splits;
  return units * (16 + ((size_t)head_dim + 2) * sizeof(float));  // (m, l) exchange, o, m, l
}

int device_sm_count() {
  static std::mutex mu;
  static std::vector<int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  std::lock_guard<std::mutex> lock(mu);
  if ((int)cache.size() <= dev) cache.resize(dev + 1, 0);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    cache[dev] = n;
  }
  return cache[dev];
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_desc(const kvq_cache_desc* d) {
  if (!d) return KVQ_ERR_INVALID_ARG;
  if (d->fmt != KVQ_FMT_Q8_0 && d->fmt != KVQ_FMT_Q4_0 && d->fmt != KVQ_FMT_LUT4 &&
      d->fmt != KVQ_FMT_NVFP4)
    return KVQ_ERR_UNSUPPORTED;
  if (d->head_dim != 64 && d->head_dim != 128) return KVQ_ERR_UNSUPPORTED;
  if (d->num_kv_heads < 1 || d->num_pages < 1) return KVQ_ERR_INVALID_ARG;
  if (d->page_size < 64 || d->page_size % 64 != 0) return KVQ_ERR_UNSUPPORTED;
  if ((int64_t)d->num_pages * d->num_kv_heads * d->page_size > 0x7fffffffLL)
    return KVQ_ERR_UNSUPPORTED;  // rows are addressed with 32-bit indices
  if (d->fmt == KVQ_FMT_LUT4 && (!d->codebook || !d->signs)) return KVQ_ERR_INVALID_ARG;
  if (d->fmt == KVQ_FMT_LUT4 && (reinterpret_cast<uintptr_t>(d->signs) & 7u)) return KVQ_ERR_INVALID_ARG;
  return KVQ_OK;
}

int max_splits_for(int max_seq_len, int split_tokens) {
  return (max_seq_len + split_tokens - 1) / split_tokens;
}

constexpr int kMinSplits = 32;         // splits per (sequence, KV head) at the least
constexpr int kMinSplitTokens = 128;   // positions per split at the least (automatic choice)

int cluster_for(int max_splits) { return max_splits >= 4 ? 4 : max_splits >= 2 ? 2 : 1; }

// Split length L of a request (the device is queried only when split_tokens == 0).
int resolve_split_len(const kvq_cache_desc* desc, int batch, int num_q_heads, int max_seq_len,
                      int split_tokens, uint32_t options, int* L_out) {
  int st = check_desc(desc);
  if (st != KVQ_OK) return st;
  if (batch < 0 || num_q_heads < 1 || max_seq_len < 0 || split_tokens < 0)
    return KVQ_ERR_INVALID_ARG;
  if (options & ~(KVQ_OPT_SHARED_MAX | KVQ_OPT_GLOBAL_MAX | KVQ_OPT_V_KEPT_ONLY | KVQ_OPT_V_WITH_K))
    return KVQ_ERR_INVALID_ARG;
  if ((options & KVQ_OPT_SHARED_MAX) && (options & KVQ_OPT_GLOBAL_MAX)) return KVQ_ERR_INVALID_ARG;
  if ((options & KVQ_OPT_V_KEPT_ONLY) && (options & KVQ_OPT_V_WITH_K)) return KVQ_ERR_INVALID_ARG;
  int L;
  if (split_tokens > 0) {
    L = std::min(split_tokens, KVQ_MAX_SPLIT_TOKENS);
  } else if (options & KVQ_OPT_SHARED_MAX) {
    // clusters of 4 splits sharing their running maximum: about one split per CTA slot of
    // the device if every sequence were max_seq_len long
    const int64_t pairs = (int64_t)std::max(batch, 1) * desc->num_kv_heads;
    const int cap4 = decode2_capacity(desc->fmt, desc->head_dim, 4, KVQ_MAX_SPLIT_TOKENS);
    const int cap1 = decode2_capacity(desc->fmt, desc->head_dim, 1, KVQ_MAX_SPLIT_TOKENS);
    if (cap1 <= 0) return KVQ_ERR_CUDA;
    const int64_t ctas_per_pair = cap4 > 0 ? 4 * std::max<int64_t>(1, cap4 / pairs)
                                           : std::max<int64_t>(1, cap1 / pairs);
    L = (int)std::min<int64_t>((std::max(max_seq_len, 1) + ctas_per_pair - 1) / ctas_per_pair,
                               KVQ_MAX_SPLIT_TOKENS);
  } else {
    // Splits per (sequence, KV head): enough to give every SM a CTA of 16 warps, and at
    // least kMinSplits (short contexts: more and smaller CTAs, each a shorter chain; the
    // kernel's CTA follows the split, one warp per tile).  Then the shortest length from
    // there whose units all fit on the device at once, so that the splits merge inside
    // the kernel.
    const int64_t pairs = (int64_t)std::max(batch, 1) * desc->num_kv_heads;
    const int64_t n = std::max(max_seq_len, 1);
    const int cap16 = decode2_capacity(desc->fmt, desc->head_dim, 1, KVQ_MAX_SPLIT_TOKENS);
    if (cap16 <= 0) return KVQ_ERR_CUDA;
    const int64_t S = std::max<int64_t>(cap16 / pairs, kMinSplits);
    int64_t l = (n + S - 1) / S;
    l = std::min<int64_t>(std::max<int64_t>((l + kTile - 1) / kTile * kTile, kMinSplitTokens),
                          KVQ_MAX_SPLIT_TOKENS);
    bool fits = false;
    for (;; l += kTile) {
      const int cap = decode2_capacity(desc->fmt, desc->head_dim, 1, (int)l);
      if (cap <= 0) return KVQ_ERR_CUDA;
      fits = pairs * ((n + l - 1) / l) <= cap;
      if (fits || l >= KVQ_MAX_SPLIT_TOKENS) break;
    }
    // More splits than CTAs even at the longest split: the CTAs loop over the units, and
    // two CTAs of half the size per SM (splits of 8 tiles) overlap one's copies with the
    // other's arithmetic (measured faster than one CTA of 16 warps looping)
    L = fits ? (int)l : KVQ_MAX_SPLIT_TOKENS / 2;
  }
  L = (L + kTile - 1) / kTile * kTile;
  *L_out = std::max(kTile, std::min(L, KVQ_MAX_SPLIT_TOKENS));
  return KVQ_OK;
}

// Splits per thread-block cluster: 1 unless the splits share their running maximum;
// then 4 when a sequence can have 4 or more splits, else 2 (smaller when the device
// cannot hold such clusters).  Also the clusters that fit on the device at once.
int resolve_cluster(const kvq_cache_desc* desc, int max_seq_len, int L, uint32_t options,
                    int* cs_out, int* cap_out) {
  int CS = (options & KVQ_OPT_SHARED_MAX) ? cluster_for(max_splits_for(std::max(max_seq_len, 1), L)) : 1;
  for (; CS >= 1; CS >>= 1) {
    const int cap = decode2_capacity(desc->fmt, desc->head_dim, CS, L);
    if (cap > 0) {
      *cs_out = CS;
      *cap_out = cap;
      return KVQ_OK;
    }
  }
  return KVQ_ERR_CUDA;
}

}  // namespace
}  // namespace kvq

using namespace kvq;

extern "C" {

size_t kvq_code_row_bytes(int32_t fmt, int32_t head_dim) {
  if (head_dim != 64 && head_dim != 128) return 0;
  if (fmt == KVQ_FMT_Q8_0) return (size_t)head_dim;
  if (fmt == KVQ_FMT_Q4_0 || fmt == KVQ_FMT_LUT4 || fmt == KVQ_FMT_NVFP4) return (size_t)head_dim / 2;
  return 0;
}

size_t kvq_scale_row_count(int32_t fmt, int32_t head_dim) {
  if (head_dim != 64 && head_dim != 128) return 0;
  if (fmt == KVQ_FMT_Q8_0 || fmt == KVQ_FMT_Q4_0) return (size_t)head_dim / 32;
  if (fmt == KVQ_FMT_LUT4) return 1;
  if (fmt == KVQ_FMT_NVFP4) return ((size_t)head_dim / 16 + 4 + 7) / 8 * 4;  // bytes / 2
  return 0;
}

int kvq_quantize(const kvq_cache_desc* desc, const void* x, int32_t n_tokens,
                 const int32_t* slots, void* codes, void* scales, void* stream) {
  int st = check_desc(desc);
  if (st != KVQ_OK) return st;
  if (n_tokens < 0) return KVQ_ERR_INVALID_ARG;
  if (n_tokens == 0) return KVQ_OK;
  if (!x || !codes || !scales) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(scales) || (reinterpret_cast<uintptr_t>(x) & 1u))
    return KVQ_ERR_INVALID_ARG;
  if (!slots && (int64_t)n_tokens > (int64_t)desc->num_pages * desc->page_size)
    return KVQ_ERR_INVALID_ARG;
  return launch_quantize(*desc, x, nullptr, n_tokens, slots, codes, scales, nullptr, nullptr,
                         static_cast<cudaStream_t>(stream));
}

int kvq_quantize_kv(const kvq_cache_desc* desc, const void* k, const void* v, int32_t n_tokens,
                    const int32_t* slots, void* k_codes, void* k_scales, void* v_codes,
                    void* v_scales, void* stream) {
  int st = check_desc(desc);
  if (st != KVQ_OK) return st;
  if (n_tokens < 0) return KVQ_ERR_INVALID_ARG;
  if (n_tokens == 0) return KVQ_OK;
  if (!k || !v || !k_codes || !k_scales || !v_codes || !v_scales) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(k_codes) || !aligned16(k_scales) || !aligned16(v_codes) || !aligned16(v_scales) ||
      (reinterpret_cast<uintptr_t>(k) & 1u) || (reinterpret_cast<uintptr_t>(v) & 1u))
    return KVQ_ERR_INVALID_ARG;
  if (!slots && (int64_t)n_tokens > (int64_t)desc->num_pages * desc->page_size)
    return KVQ_ERR_INVALID_ARG;
  return launch_quantize(*desc, k, v, n_tokens, slots, k_codes, k_scales, v_codes, v_scales,
                         static_cast<cudaStream_t>(stream));
}

int32_t kvq_resolve_split(const kvq_cache_desc* desc, int32_t batch, int32_t num_q_heads,
                          int32_t max_seq_len, int32_t split_tokens, uint32_t options) {
  int L = 0;
  const int st = resolve_split_len(desc, batch, num_q_heads, max_seq_len, split_tokens, options, &L);
  return st != KVQ_OK ? st : L;
}

int32_t kvq_resolve_cluster(const kvq_cache_desc* desc, int32_t batch, int32_t num_q_heads,
                            int32_t max_seq_len, int32_t split_tokens, uint32_t options) {
  int L = 0, CS = 0, cap = 0;
  int st = resolve_split_len(desc, batch, num_q_heads, max_seq_len, split_tokens, options, &L);
  if (st != KVQ_OK) return st;
  st = resolve_cluster(desc, max_seq_len, L, options, &CS, &cap);
  return st != KVQ_OK ? st : CS;
}

size_t kvq_workspace_size(int32_t batch, int32_t num_q_heads, int32_t head_dim,
                          int32_t max_seq_len, int32_t split_tokens) {
  if (batch < 0 || num_q_heads < 0 || head_dim <= 0 || max_seq_len < 0 || split_tokens <= 0)
    return 0;
  return kWorkspaceHeader + counters_bytes(batch, num_q_heads) +
         partials_bytes(batch, num_q_heads, head_dim, max_splits_for(max_seq_len, split_tokens));
}

int kvq_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
  if (!workspace || workspace_bytes < kWorkspaceHeader) return KVQ_ERR_WORKSPACE;
  return cudaMemsetAsync(workspace, 0, workspace_bytes, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? KVQ_OK
             : KVQ_ERR_CUDA;
}

int kvq_selftest_wait(void* workspace, size_t workspace_bytes, long long max_cycles, void* stream) {
  if (!workspace || max_cycles <= 0 || !aligned16(workspace)) return KVQ_ERR_INVALID_ARG;
  if (workspace_bytes < kWorkspaceHeader) return KVQ_ERR_WORKSPACE;
  return launch_selftest_wait(workspace, max_cycles, static_cast<cudaStream_t>(stream));
}

int kvq_read_device_flags(const void* workspace, uint32_t* flags, void* stream) {
  if (!workspace || !flags) return KVQ_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return KVQ_ERR_CUDA;
  if (cudaMemcpy(flags, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost) != cudaSuccess)
    return KVQ_ERR_CUDA;
  return KVQ_OK;
}

int kvq_decode_attn(const kvq_cache_desc* desc, const void* q, int32_t batch,
                    int32_t num_q_heads, const void* k_codes, const void* k_scales,
                    const void* v_codes, const void* v_scales, const int32_t* page_table,
                    int32_t max_pages, const int32_t* seq_lens, int32_t max_seq_len,
                    float sm_scale, float tau, int32_t split_tokens, uint32_t options,
                    void* workspace, size_t workspace_bytes, unsigned long long* stats,
                    float* out, void* stream) {
  int st = check_desc(desc);
  if (st != KVQ_OK) return st;
  if (batch < 0 || num_q_heads < 1 || max_pages < 1 || max_seq_len < 0) return KVQ_ERR_INVALID_ARG;
  if (batch > KVQ_MAX_BATCH) return KVQ_ERR_UNSUPPORTED;
  if (num_q_heads % desc->num_kv_heads != 0) return KVQ_ERR_INVALID_ARG;
  const int group = num_q_heads / desc->num_kv_heads;
  if (group > KVQ_MAX_GROUP) return KVQ_ERR_UNSUPPORTED;
  if (!(tau >= 0.0f) || !isfinite(sm_scale)) return KVQ_ERR_INVALID_ARG;
  if (!q || !k_codes || !k_scales || !v_codes || !v_scales || !seq_lens || !workspace)
    return KVQ_ERR_INVALID_ARG;
  if (!aligned16(k_codes) || !aligned16(k_scales) || !aligned16(v_codes) || !aligned16(v_scales) ||
      !aligned16(workspace) || !aligned16(q) || !aligned16(out))
    return KVQ_ERR_INVALID_ARG;
  if (!page_table && (int64_t)batch * max_pages > desc->num_pages) return KVQ_ERR_INVALID_ARG;
  int L = 0;
  st = resolve_split_len(desc, batch, num_q_heads, max_seq_len, split_tokens, options, &L);
  if (st != KVQ_OK) return st;
  if (max_splits_for(max_seq_len, L) > KVQ_MAX_SPLITS) return KVQ_ERR_UNSUPPORTED;
  const size_t need = kvq_workspace_size(batch, num_q_heads, desc->head_dim, max_seq_len, L);
  if (workspace_bytes < need) return KVQ_ERR_WORKSPACE;
  if (batch == 0) return KVQ_OK;
  if (max_seq_len == 0) {  // no positions anywhere: the output is zero
    if (out && cudaMemsetAsync(out, 0, (size_t)batch * num_q_heads * desc->head_dim * sizeof(float),
                               static_cast<cudaStream_t>(stream)) != cudaSuccess)
      return KVQ_ERR_CUDA;
    return KVQ_OK;
  }
  int CS = 1, capacity = 0;
  st = resolve_cluster(desc, max_seq_len, L, options, &CS, &capacity);
  if (st != KVQ_OK) return st;
  DecodeArgs a;
  a.desc = *desc;
  a.q = q;
  a.batch = batch;
  a.num_q_heads = num_q_heads;
  a.group = group;
  a.k_codes = k_codes;
  a.k_scales = k_scales;
  a.v_codes = v_codes;
  a.v_scales = v_scales;
  a.page_table = page_table;
  a.max_pages = max_pages;
  a.seq_lens = seq_lens;
  a.max_seq_len = max_seq_len;
  a.sm_scale = sm_scale;
  a.tau = tau;
  a.split_tokens = L;
  a.max_splits = max_splits_for(max_seq_len, L);
  a.workspace = workspace;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.zflag = reinterpret_cast<unsigned long long*>(ws + kWorkspaceHeader);
  a.arrive = a.zflag + (size_t)batch * num_q_heads;
  a.epoch = reinterpret_cast<unsigned long long*>(ws + kEpochOffset);
  a.group_merge = 0;  // decided at launch
  const size_t n_part = (size_t)batch * num_q_heads * a.max_splits;
  a.xch = reinterpret_cast<ulonglong2*>(ws + kWorkspaceHeader + counters_bytes(batch, num_q_heads));
  a.part_o = reinterpret_cast<float*>(a.xch + n_part);
  a.part_m = a.part_o + n_part * desc->head_dim;
  a.part_l = a.part_m + n_part;
  a.stats = stats;
  a.out = out;
  a.cluster = CS;
  a.shared_max = (options & KVQ_OPT_SHARED_MAX) ? 1 : 0;
  a.global_max = (options & KVQ_OPT_GLOBAL_MAX) ? 1 : 0;
  // clusters: at most one per (sequence, KV head, group of CS splits), at most what fits
  a.units_per_seq = (a.max_splits + CS - 1) / CS;
  const int64_t groups = (int64_t)batch * desc->num_kv_heads * a.units_per_seq;
  // the maximum over all splits needs every split on its own CTA at once
  if (a.global_max && groups > capacity) return KVQ_ERR_UNSUPPORTED;
  a.grid = (int)std::min<int64_t>(groups, capacity) * CS;
  // At these sizes the step is bound by latency and instruction issue, not by bytes, so
  // by default V comes with K (no second DRAM round trip)
  a.v_early = (options & KVQ_OPT_V_KEPT_ONLY) ? 0 : 1;
  // The merge: inside the decode kernel when every group of splits has its own CTAs at
  // once (the splits exchange (m, l) and add their shares into the output); otherwise every
  // split writes its partial to the workspace and the combine kernel merges them, one CTA
  // per (sequence, query head), which measured faster than the last finisher of each
  // (sequence, KV head) merging alone.
  const bool combine_after = out && groups > capacity;
  st = launch_decode2(a, static_cast<cudaStream_t>(stream));
  if (st != KVQ_OK || !combine_after) return st;
  return launch_combine(*desc, workspace, batch, num_q_heads, max_seq_len, L, a.max_splits, seq_lens, out,
                        static_cast<cudaStream_t>(stream));
}

int kvq_combine(const kvq_cache_desc* desc, const void* workspace, int32_t batch,
                int32_t num_q_heads, int32_t max_seq_len, int32_t split_tokens, uint32_t options,
                const int32_t* seq_lens, float* out, void* stream) {
  int st = check_desc(desc);
  if (st != KVQ_OK) return st;
  if (batch < 0 || num_q_heads < 1 || max_seq_len < 0) return KVQ_ERR_INVALID_ARG;
  if (!workspace || !seq_lens || !out) return KVQ_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) & 15u) return KVQ_ERR_INVALID_ARG;
  int L = 0;
  st = resolve_split_len(desc, batch, num_q_heads, max_seq_len, split_tokens, options, &L);
  if (st != KVQ_OK) return st;
  if (max_splits_for(max_seq_len, L) > KVQ_MAX_SPLITS) return KVQ_ERR_UNSUPPORTED;
  if (batch == 0) return KVQ_OK;
  return launch_combine(*desc, workspace, batch, num_q_heads, std::max(max_seq_len, 0), L,
                        max_splits_for(max_seq_len, L), seq_lens, out,
                        static_cast<cudaStream_t>(stream));
}

// Lloyd's iteration for N(0, sigma^2): thresholds at midpoints, centroids at the
// conditional means sigma * (phi(a) - phi(b)) / (Phi(b) - Phi(a)).
int kvq_lloyd_max_codebook(int32_t levels, double sigma, uint16_t* out_fp16) {
  if (levels < 2 || levels > 256 || !(sigma > 0.0) || !out_fp16) return KVQ_ERR_INVALID_ARG;
  const double inv_sqrt2pi = 0.3989422804014327;
  auto pdf = [&](double z) { return isinf(z) ? 0.0 : inv_sqrt2pi * exp(-0.5 * z * z); };
  auto cdf = [&](double z) {
    if (isinf(z)) return z > 0 ? 1.0 : 0.0;
    return 0.5 * erfc(-z * 0.7071067811865476);
  };
  std::vector<double> cen(levels), nxt(levels), edge(levels + 1);
  for (int i = 0; i < levels; ++i) cen[i] = -2.0 + 4.0 * i / (levels - 1);  // unit-variance start
  for (int iter = 0; iter < 200000; ++iter) {
    edge[0] = -INFINITY;
    edge[levels] = INFINITY;
    for (int i = 1; i < levels; ++i) edge[i] = 0.5 * (cen[i - 1] + cen[i]);
    for (int i = 0; i < levels; ++i) {
      const double mass = cdf(edge[i + 1]) - cdf(edge[i]);
      nxt[i] = (pdf(edge[i]) - pdf(edge[i + 1])) / mass;
    }
    double move = 0.0;
    for (int i = 0; i < levels; ++i) {
      const double v = 0.5 * (nxt[i] - nxt[levels - 1 - i]);  // keep it exactly symmetric
      move = std::max(move, fabs(v - cen[i]));
      cen[i] = v;
    }
    if (move < 1e-13) break;
  }
  for (int i = 0; i < levels; ++i) {
    const __half h = __double2half(cen[i] * sigma);
    out_fp16[i] = __half_as_ushort(h);
  }
  return KVQ_OK;
}

const char* kvq_status_string(int status) {
  switch (status) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID_ARG: return "invalid argument";
    case KVQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case KVQ_ERR_CUDA: return "CUDA error";
    case KVQ_ERR_WORKSPACE: return "workspace too small";
    case KVQ_ERR_DEVICE: return "device-side fault reported";
    default: return "unknown status";
  }
}

}  // extern "C"
