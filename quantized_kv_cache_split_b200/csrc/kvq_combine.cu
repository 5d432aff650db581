// Log-sum-exp merge of split-KV partials (flash-decoding combine).
//   M = max_s m_s,  out = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s
// (m is kept in log2 units by the decode kernel).  For the rotated lut4 format
// the merged vector is rotated back: out = s .* (c * H * out').
// The decode kernel leaves one partial per split, so sequence b has ceil(n_b / L) of them.
// One CTA of 512 threads per (sequence, query head): the partial maxima and weights
// are computed one partial per thread, then 512/head_dim thread groups each sum a
// share of the partials with several loads in flight, and the groups are added.
#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kCombineThreads = 512;
constexpr int kMaxCombineSplits = KVQ_MAX_SPLITS;  // splits per sequence merged by one CTA


template <int D, bool ROT>
__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(const uint8_t* __restrict__ ws, int batch, int hq, int max_seq_len,
               int split_tokens, int max_splits, const int32_t* __restrict__ seq_lens,
               const int8_t* __restrict__ signs, float* __restrict__ out) {
  constexpr int kGroups = kCombineThreads / D;  // thread groups splitting the split range
  __shared__ float wsh[kMaxCombineSplits];
  __shared__ float part[kGroups][D];
  __shared__ float red[32];
  const int bh = blockIdx.x;
  const int b = bh / hq;
  const int tid = threadIdx.x;
  const size_t n_part = (size_t)batch * hq * max_splits;
  // the partials follow the header, the merge words and the (m, l) exchange entries
  const float* o = reinterpret_cast<const float*>(ws + kWorkspaceHeader + counters_bytes(batch, hq) +
                                                  16 * n_part);
  const float* m = o + n_part * D;
  const float* l = m + n_part;
  const int n = max(0, min(seq_lens[b], max_seq_len));
  const int ns = (n + split_tokens - 1) / split_tokens;
  const size_t u0 = (size_t)bh * max_splits;
  // 1. maxima and weights: one split per thread (strided), loads all in flight
  float M = -INFINITY;
  for (int s = tid; s < ns; s += kCombineThreads) M = fmaxf(M, m[u0 + s]);
#pragma unroll
  for (int off = 16; off; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  if ((tid & 31) == 0) red[tid >> 5] = M;
  __syncthreads();
  M = red[0];
  for (int w = 1; w < kCombineThreads / 32; ++w) M = fmaxf(M, red[w]);
  float dl = 0.f;
  for (int s = tid; s < ns; s += kCombineThreads) {
    const float wgt = ex2(m[u0 + s] - M);
    wsh[s] = wgt;
    dl = fmaf(wgt, l[u0 + s], dl);
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) dl += __shfl_xor_sync(0xffffffffu, dl, off);
  __syncthreads();
  if ((tid & 31) == 0) red[tid >> 5] = dl;
  __syncthreads();
  float den = 0.f;
  for (int w = 0; w < kCombineThreads / 32; ++w) den += red[w];
  // 2. weighted sum of the partial outputs: group gi takes splits gi, gi + kGroups, ...
  const int gi = tid / D, d = tid - gi * D;
  float acc = 0.f;
  int s = gi;
  for (; s + 3 * kGroups < ns; s += 4 * kGroups) {
    const float v0 = o[(u0 + s) * D + d], v1 = o[(u0 + s + kGroups) * D + d];
    const float v2 = o[(u0 + s + 2 * kGroups) * D + d], v3 = o[(u0 + s + 3 * kGroups) * D + d];
    acc = fmaf(wsh[s], v0, acc);
    acc = fmaf(wsh[s + kGroups], v1, acc);
    acc = fmaf(wsh[s + 2 * kGroups], v2, acc);
    acc = fmaf(wsh[s + 3 * kGroups], v3, acc);
  }
  for (; s < ns; s += kGroups) acc = fmaf(wsh[s], o[(u0 + s) * D + d], acc);
  part[gi][d] = acc;
  __syncthreads();
  if (tid < D) {
    float num = 0.f;
#pragma unroll
    for (int g2 = 0; g2 < kGroups; ++g2) num += part[g2][tid];
    part[0][tid] = ns > 0 ? num / den : 0.f;
  }
  __syncthreads();
  if constexpr (ROT) {
    if (tid < 32) {
      constexpr int K = D / 32;
      float y[K];
#pragma unroll
      for (int k = 0; k < K; ++k) y[k] = part[0][32 * k + tid];
#pragma unroll
      for (int hb = 1; hb < 32; hb <<= 1) {
        const bool upper = (tid & hb) != 0;
#pragma unroll
        for (int k = 0; k < K; ++k) {
          const float t = __shfl_xor_sync(0xffffffffu, y[k], hb);
          y[k] = upper ? (t - y[k]) : (y[k] + t);
        }
      }
#pragma unroll
      for (int k = 0; k + 1 < K; k += 2) {
        const float u = y[k], v = y[k + 1];
        y[k] = u + v; y[k + 1] = u - v;
      }
      if (K == 4) {
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const float u = y[k], v = y[k + 2];
          y[k] = u + v; y[k + 2] = u - v;
        }
      }
      const float cs = D == 64 ? 0.125f : 0.08838834764831845f;  // 1/sqrt(D)
#pragma unroll
      for (int k = 0; k < K; ++k) part[1 % kGroups][32 * k + tid] = y[k] * cs * (float)signs[32 * k + tid];
    }
    __syncthreads();
    if (tid < D) out[(size_t)bh * D + tid] = part[1 % kGroups][tid];
  } else {
    if (tid < D) out[(size_t)bh * D + tid] = part[0][tid];
  }
}

}  // namespace

int launch_combine(const kvq_cache_desc& desc, const void* workspace, int batch, int num_q_heads,
                   int max_seq_len, int split_tokens, int max_splits, const int32_t* seq_lens, float* out, cudaStream_t stream) {
  const int64_t blocks = (int64_t)batch * num_q_heads;
  if (blocks <= 0) return KVQ_OK;
  if (blocks > 0x7fffffffLL) return KVQ_ERR_UNSUPPORTED;
  const uint8_t* ws = static_cast<const uint8_t*>(workspace);
  if (max_splits > kMaxCombineSplits) return KVQ_ERR_UNSUPPORTED;
  const bool rot = desc.fmt == KVQ_FMT_LUT4;
#define KVQ_COMBINE(DIM, ROT)                                                            \
  combine_kernel<DIM, ROT><<<(unsigned)blocks, kCombineThreads, 0, stream>>>(            \
      ws, batch, num_q_heads, max_seq_len, split_tokens, max_splits, seq_lens,           \
      desc.signs, out)
  if (desc.head_dim == 128) {
    if (rot) KVQ_COMBINE(128, true); else KVQ_COMBINE(128, false);
  } else if (desc.head_dim == 64) {
    if (rot) KVQ_COMBINE(64, true); else KVQ_COMBINE(64, false);
  } else {
    return KVQ_ERR_UNSUPPORTED;
  }
#undef KVQ_COMBINE
  return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

}  // namespace kvq
