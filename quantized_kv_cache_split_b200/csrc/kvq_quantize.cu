// Cache writers: fp16 K/V vectors -> q8_0 / q4_0 / rotated lut4 blocks.
//
// One warp per (token, KV head) vector.  Lane l holds elements l, l+32, l+64,
// l+96 (head_dim 128) or l, l+32 (head_dim 64), so a 32-element block is one
// warp-wide reduction and every store is coalesced.  All arithmetic uses the
// IEEE round-to-nearest-even intrinsics (__fdiv_rn, __fadd_rn, __fmul_rn,
// __fsqrt_rn), which the compiler never contracts into FMAs: the codes are the
// bit-exact result of the fp32 formulas stated in kvq.h.
#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kWarpsPerBlock = 8;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ int64_t slot_row(int64_t slot, int page_size, int hkv, int h) {
  const int64_t page = slot / page_size;
  const int64_t off = slot - page * page_size;
  return (page * hkv + h) * page_size + off;
}

// q8_0: d = amax/127, q = round-half-away(x/d) clamped to [-127, 127].
template <int D>
__global__ void __launch_bounds__(32 * kWarpsPerBlock)
quant_q8_0_kernel(const __half* __restrict__ x, int n_tok, int hkv, const int32_t* __restrict__ slots,
                  int page_size, int8_t* __restrict__ codes, __half* __restrict__ scales) {
  constexpr int NB = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t vec = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  if (vec >= (int64_t)n_tok * hkv) return;
  const int64_t tok = vec / hkv;
  const int h = (int)(vec - tok * hkv);
  const int64_t slot = slots ? (int64_t)slots[tok] : tok;
  const int64_t row = slot_row(slot, page_size, hkv, h);
  const __half* xv = x + vec * D;
  float d_mine = 0.f;
#pragma unroll
  for (int m = 0; m < NB; ++m) {
    const float v = __half2float(xv[32 * m + lane]);
    const float amax = warp_max(fabsf(v));
    const float d = __fdiv_rn(amax, 127.0f);
    int q = 0;
    if (d != 0.0f) {
      q = (int)roundf(__fdiv_rn(v, d));
      q = max(-127, min(127, q));
    }
    codes[row * D + 32 * m + lane] = (int8_t)q;
    if (lane == m) d_mine = d;
  }
  if (lane < NB) scales[row * NB + lane] = __float2half_rn(d_mine);
}

// q4_0: m = signed element of largest |x| (lowest index on ties), d = m/-8,
// q = min(15, floor(x/d + 8.5)); q = 8 when d == 0.
template <int D>
__global__ void __launch_bounds__(32 * kWarpsPerBlock)
quant_q4_0_kernel(const __half* __restrict__ x, int n_tok, int hkv, const int32_t* __restrict__ slots,
                  int page_size, uint8_t* __restrict__ codes, __half* __restrict__ scales) {
  constexpr int NB = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t vec = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  if (vec >= (int64_t)n_tok * hkv) return;
  const int64_t tok = vec / hkv;
  const int h = (int)(vec - tok * hkv);
  const int64_t slot = slots ? (int64_t)slots[tok] : tok;
  const int64_t row = slot_row(slot, page_size, hkv, h);
  const __half* xv = x + vec * D;
  float d_mine = 0.f;
#pragma unroll
  for (int m = 0; m < NB; ++m) {
    const float v = __half2float(xv[32 * m + lane]);
    // argmax of |v| with the lowest lane winning ties; carry the signed value.
    float best = fabsf(v), val = v;
    int idx = lane;
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const float ov = __shfl_xor_sync(0xffffffffu, val, o);
      const int oi = __shfl_xor_sync(0xffffffffu, idx, o);
      if (ob > best || (ob == best && oi < idx)) { best = ob; val = ov; idx = oi; }
    }
    const float d = __fdiv_rn(val, -8.0f);
    int q = 8;
    if (d != 0.0f) {
      const float t = __fadd_rn(__fdiv_rn(v, d), 8.5f);
      q = min(15, (int)floorf(t));
    }
    const int hi = __shfl_down_sync(0xffffffffu, q, 1);
    if ((lane & 1) == 0) codes[row * (D / 2) + 16 * m + (lane >> 1)] = (uint8_t)(q | (hi << 4));
    if (lane == m) d_mine = d;
  }
  if (lane < NB) scales[row * NB + lane] = __float2half_rn(d_mine);
}

// lut4: y = c * H (s .* x) (butterflies h = 1, 2, ..., D/2 in fp32), n = |y| by a
// pairwise tree (strides D/2 ... 1), u = y / n, idx = #{k : u > t_k},
// t_k = (c_k + c_{k+1}) * 0.5 from the fp16 codebook.
template <int D>
__global__ void __launch_bounds__(32 * kWarpsPerBlock)
quant_lut4_kernel(const __half* __restrict__ x, int n_tok, int hkv, const int32_t* __restrict__ slots,
                  int page_size, const uint16_t* __restrict__ codebook,
                  const int8_t* __restrict__ signs, uint8_t* __restrict__ codes,
                  __half* __restrict__ norms) {
  constexpr int K = D / 32;  // elements per lane
  __shared__ float thr[15];
  if (threadIdx.x < 15) {
    const float c0 = __half2float(__ushort_as_half(codebook[threadIdx.x]));
    const float c1 = __half2float(__ushort_as_half(codebook[threadIdx.x + 1]));
    thr[threadIdx.x] = __fmul_rn(__fadd_rn(c0, c1), 0.5f);
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t vec = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  if (vec >= (int64_t)n_tok * hkv) return;
  const int64_t tok = vec / hkv;
  const int h = (int)(vec - tok * hkv);
  const int64_t slot = slots ? (int64_t)slots[tok] : tok;
  const int64_t row = slot_row(slot, page_size, hkv, h);
  const __half* xv = x + vec * D;

  float y[K];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int i = 32 * k + lane;
    y[k] = __fmul_rn(__half2float(xv[i]), (float)signs[i]);
  }
  // cross-lane stages h = 1..16: the lower index keeps a+b, the upper a-b.
#pragma unroll
  for (int hb = 1; hb < 32; hb <<= 1) {
    const bool upper = (lane & hb) != 0;
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const float o = __shfl_xor_sync(0xffffffffu, y[k], hb);
      y[k] = upper ? __fsub_rn(o, y[k]) : __fadd_rn(y[k], o);
    }
  }
  // in-lane stages h = 32 (k pairs 0-1, 2-3) and h = 64 (k pairs 0-2, 1-3)
  if (K >= 2) {
#pragma unroll
    for (int k = 0; k < K; k += 2) {
      const float a = y[k], b = y[k + 1];
      y[k] = __fadd_rn(a, b);
      y[k + 1] = __fsub_rn(a, b);
    }
  }
  if (K == 4) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float a = y[k], b = y[k + 2];
      y[k] = __fadd_rn(a, b);
      y[k + 2] = __fsub_rn(a, b);
    }
  }
  const float c = (float)(1.0 / sqrt((double)D));
#pragma unroll
  for (int k = 0; k < K; ++k) y[k] = __fmul_rn(y[k], c);

  // sum of squares: strides 64, 32 in-lane, then 16..1 across lanes
  float sq;
  if (K == 4) {
    const float t0 = __fadd_rn(__fmul_rn(y[0], y[0]), __fmul_rn(y[2], y[2]));
    const float t1 = __fadd_rn(__fmul_rn(y[1], y[1]), __fmul_rn(y[3], y[3]));
    sq = __fadd_rn(t0, t1);
  } else {
    sq = __fadd_rn(__fmul_rn(y[0], y[0]), __fmul_rn(y[1], y[1]));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) sq = __fadd_rn(sq, __shfl_xor_sync(0xffffffffu, sq, o));
  const float n = __fsqrt_rn(sq);

#pragma unroll
  for (int k = 0; k < K; ++k) {
    const float u = (n == 0.0f) ? 0.0f : __fdiv_rn(y[k], n);
    int idx = 0;
#pragma unroll
    for (int t = 0; t < 15; ++t) idx += (u > thr[t]) ? 1 : 0;
    const int hi = __shfl_down_sync(0xffffffffu, idx, 1);
    if ((lane & 1) == 0) codes[row * (D / 2) + 16 * k + (lane >> 1)] = (uint8_t)(idx | (hi << 4));
  }
  if (lane == 0) norms[row] = __float2half_rn(n);
}

}  // namespace

int launch_quantize(const kvq_cache_desc& desc, const void* x, int n_tok, const int32_t* slots,
                    void* codes, void* scales, cudaStream_t stream) {
  const int64_t vecs = (int64_t)n_tok * desc.num_kv_heads;
  const int64_t blocks = (vecs + kWarpsPerBlock - 1) / kWarpsPerBlock;
  if (blocks > 0x7fffffffLL) return KVQ_ERR_UNSUPPORTED;
  const dim3 grid((unsigned)blocks), block(32 * kWarpsPerBlock);
  const __half* xh = static_cast<const __half*>(x);
  const int hkv = desc.num_kv_heads, ps = desc.page_size;
#define KVQ_QUANT_CASE(FMT, DIM, KERNEL, ...)                                     \
  if (desc.fmt == FMT && desc.head_dim == DIM) {                                  \
    KERNEL<DIM><<<grid, block, 0, stream>>>(xh, n_tok, hkv, slots, ps, __VA_ARGS__); \
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;             \
  }
  KVQ_QUANT_CASE(KVQ_FMT_Q8_0, 64, quant_q8_0_kernel, (int8_t*)codes, (__half*)scales)
  KVQ_QUANT_CASE(KVQ_FMT_Q8_0, 128, quant_q8_0_kernel, (int8_t*)codes, (__half*)scales)
  KVQ_QUANT_CASE(KVQ_FMT_Q4_0, 64, quant_q4_0_kernel, (uint8_t*)codes, (__half*)scales)
  KVQ_QUANT_CASE(KVQ_FMT_Q4_0, 128, quant_q4_0_kernel, (uint8_t*)codes, (__half*)scales)
  KVQ_QUANT_CASE(KVQ_FMT_LUT4, 64, quant_lut4_kernel, desc.codebook, desc.signs, (uint8_t*)codes,
                 (__half*)scales)
  KVQ_QUANT_CASE(KVQ_FMT_LUT4, 128, quant_lut4_kernel, desc.codebook, desc.signs,
                 (uint8_t*)codes, (__half*)scales)
#undef KVQ_QUANT_CASE
  return KVQ_ERR_UNSUPPORTED;
}

}  // namespace kvq
