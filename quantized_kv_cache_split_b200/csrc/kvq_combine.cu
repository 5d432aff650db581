// Log-sum-exp merge of split-KV partials (flash-decoding combine).
//   M = max_s m_s,  out = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s
// (m is kept in log2 units by the decode kernel).  For the rotated lut4 format
// the merged vector is rotated back: out = s .* (c * H * out').
// One CTA of head_dim threads per (sequence, query head); thread d owns dim d.
#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

template <int D, bool ROT>
__global__ void __launch_bounds__(128)
combine_kernel(const uint8_t* __restrict__ ws, int batch, int hq, int max_seq_len, int page_cap,
               int split_tokens, int max_splits, const int32_t* __restrict__ seq_lens,
               const int8_t* __restrict__ signs, float* __restrict__ out) {
  __shared__ float vec[D];
  const int bh = blockIdx.x;
  const int b = bh / hq;
  const int d = threadIdx.x;
  const float* o = reinterpret_cast<const float*>(ws + kWorkspaceHeader);
  const size_t n_part = (size_t)batch * hq * max_splits;
  const float* m = o + n_part * D;
  const float* l = m + n_part;
  const int n = max(0, min(seq_lens[b], min(max_seq_len, page_cap)));
  const int ns = (n + split_tokens - 1) / split_tokens;
  const size_t u0 = (size_t)bh * max_splits;
  float M = -INFINITY;
  for (int s = 0; s < ns; ++s) M = fmaxf(M, m[u0 + s]);
  float num = 0.f, den = 0.f;
  for (int s = 0; s < ns; ++s) {
    const float w = ex2(m[u0 + s] - M);
    den = fmaf(w, l[u0 + s], den);
    num = fmaf(w, o[(u0 + s) * D + d], num);
  }
  float res = ns > 0 ? num / den : 0.f;
  if constexpr (ROT) {
    vec[d] = res;
    __syncthreads();
    if (d < 32) {
      constexpr int K = D / 32;
      float y[K];
#pragma unroll
      for (int k = 0; k < K; ++k) y[k] = vec[32 * k + d];
#pragma unroll
      for (int hb = 1; hb < 32; hb <<= 1) {
        const bool upper = (d & hb) != 0;
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
      const float cs = rsqrtf((float)D);
#pragma unroll
      for (int k = 0; k < K; ++k) vec[32 * k + d] = y[k] * cs * (float)signs[32 * k + d];
    }
    __syncthreads();
    res = vec[d];
  }
  out[(size_t)bh * D + d] = res;
}

}  // namespace

int launch_combine(const kvq_cache_desc& desc, const void* workspace, int batch, int num_q_heads,
                   int max_seq_len, int split_tokens, int max_splits, const int32_t* seq_lens,
                   float* out, cudaStream_t stream) {
  const int64_t blocks = (int64_t)batch * num_q_heads;
  if (blocks <= 0) return KVQ_OK;
  if (blocks > 0x7fffffffLL) return KVQ_ERR_UNSUPPORTED;
  const uint8_t* ws = static_cast<const uint8_t*>(workspace);
  const int cap = (int)std::min<int64_t>((int64_t)max_seq_len, 0x7fffffff);
  const bool rot = desc.fmt == KVQ_FMT_LUT4;
#define KVQ_COMBINE(DIM, ROT)                                                            \
  combine_kernel<DIM, ROT><<<(unsigned)blocks, DIM, 0, stream>>>(                        \
      ws, batch, num_q_heads, max_seq_len, cap, split_tokens, max_splits, seq_lens,      \
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
