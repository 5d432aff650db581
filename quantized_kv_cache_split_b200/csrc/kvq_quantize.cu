// Cache writers: fp16 K/V vectors -> q8_0 / q4_0 / rotated lut4 / nvfp4 blocks.
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
quant_q8_0_kernel(const __half* __restrict__ x, const __half* __restrict__ x2, int n_tok, int hkv,
                  const int32_t* __restrict__ slots, int page_size, int8_t* __restrict__ codes,
                  __half* __restrict__ scales, int8_t* __restrict__ codes2, __half* __restrict__ scales2) {
  if (blockIdx.y) {  // the second plane pair (V of a K + V write)
    x = x2;
    codes = codes2;
    scales = scales2;
  }
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
quant_q4_0_kernel(const __half* __restrict__ x, const __half* __restrict__ x2, int n_tok, int hkv,
                  const int32_t* __restrict__ slots, int page_size, uint8_t* __restrict__ codes,
                  __half* __restrict__ scales, uint8_t* __restrict__ codes2, __half* __restrict__ scales2) {
  if (blockIdx.y) {  // the second plane pair (V of a K + V write)
    x = x2;
    codes = codes2;
    scales = scales2;
  }
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
quant_lut4_kernel(const __half* __restrict__ x, const __half* __restrict__ x2, int n_tok, int hkv,
                  const int32_t* __restrict__ slots, int page_size, const uint16_t* __restrict__ codebook,
                  const int8_t* __restrict__ signs, uint8_t* __restrict__ codes,
                  __half* __restrict__ norms, uint8_t* __restrict__ codes2, __half* __restrict__ norms2) {
  if (blockIdx.y) {  // the second plane pair (V of a K + V write)
    x = x2;
    codes = codes2;
    norms = norms2;
  }
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

// ------------------------------------------------------------------ nvfp4
// E2M1 magnitude code of |v|: the number of decision points passed, where the points
// are the midpoints 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5 between the values 0, 0.5, 1,
// 1.5, 2, 3, 4, 6, and a value on a midpoint goes to the even code (round to nearest
// even); above 6 it stays at 6 (saturation).  The sign bit follows the sign of v.
__device__ __forceinline__ uint32_t e2m1_code(float v) {
  const float a = fabsf(v);
  const float mid[7] = {0.25f, 0.75f, 1.25f, 1.75f, 2.5f, 3.5f, 5.0f};
  uint32_t c = 0;
#pragma unroll
  for (int k = 0; k < 7; ++k) c += (a > mid[k] || (a == mid[k] && (k & 1))) ? 1u : 0u;
  return c | (signbit(v) ? 8u : 0u);
}

// E4M3 code of t >= 0: round to nearest even on the 3-bit mantissa, saturating at 448.
__device__ __forceinline__ uint32_t e4m3_code(float t) {
  if (!(t < 448.0f)) return 126u;                    // 448 and beyond (also NaN): 448
  if (t < 0.015625f) {                               // below 2^-6: subnormal steps of 2^-9
    const int m = __float2int_rn(__fmul_rn(t, 512.0f));  // exact scaling, ties to even
    return (uint32_t)m;                              // m == 8 is the smallest normal, code 8
  }
  const uint32_t bits = __float_as_uint(t);
  int e = (int)((bits >> 23) & 0xffu) - 127 + 7;     // biased E4M3 exponent, 1 .. 15
  uint32_t q = (bits >> 20) & 7u;
  const uint32_t rem = bits & 0xfffffu, half = 0x80000u;
  if (rem > half || (rem == half && (q & 1u))) ++q;
  if (q == 8u) { q = 0; ++e; }
  if (e > 15 || (e == 15 && q == 7u)) return 126u;
  return ((uint32_t)e << 3) | q;
}

__device__ __forceinline__ float e4m3_value(uint32_t code) {
  const int e = (int)(code >> 3) & 15, m = (int)(code & 7u);
  return e ? ldexpf((float)(8 + m), e - 10) : ldexpf((float)m, -9);
}

__device__ __forceinline__ float half_warp_max(float v) {
#pragma unroll
  for (int o = 8; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// nvfp4: g = amax/2688 over the vector; per 16-element block s = e4m3(amax_b / (6 g));
// code = e2m1(x / (g s)).  Lane l holds elements l + 32 m, so block 2m + (l >> 4) is a
// half-warp.  Scale row: the E4M3 bytes, then g (fp32), then zero padding.
template <int D>
__global__ void __launch_bounds__(32 * kWarpsPerBlock)
quant_nvfp4_kernel(const __half* __restrict__ x, const __half* __restrict__ x2, int n_tok, int hkv,
                   const int32_t* __restrict__ slots, int page_size, uint8_t* __restrict__ codes,
                   uint8_t* __restrict__ scales, uint8_t* __restrict__ codes2, uint8_t* __restrict__ scales2) {
  if (blockIdx.y) {  // the second plane pair (V of a K + V write)
    x = x2;
    codes = codes2;
    scales = scales2;
  }
  constexpr int NM = D / 32;
  constexpr int SROWB = (D / 16 + 4 + 7) / 8 * 8;  // scale row bytes
  const int lane = threadIdx.x & 31;
  const int64_t vec = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  if (vec >= (int64_t)n_tok * hkv) return;
  const int64_t tok = vec / hkv;
  const int h = (int)(vec - tok * hkv);
  const int64_t slot = slots ? (int64_t)slots[tok] : tok;
  const int64_t row = slot_row(slot, page_size, hkv, h);
  const __half* xv = x + vec * D;
  float v[NM];
  float amax = 0.f;
#pragma unroll
  for (int m = 0; m < NM; ++m) {
    v[m] = __half2float(xv[32 * m + lane]);
    amax = fmaxf(amax, fabsf(v[m]));
  }
  amax = warp_max(amax);
  const float g = __fdiv_rn(amax, 2688.0f);
  const float six_g = __fmul_rn(6.0f, g);
  uint8_t* srow = scales + row * SROWB;
#pragma unroll
  for (int m = 0; m < NM; ++m) {
    const float amax_b = half_warp_max(fabsf(v[m]));
    const float t = six_g > 0.f ? __fdiv_rn(amax_b, six_g) : 0.f;
    const uint32_t sc = e4m3_code(t);
    const float den = __fmul_rn(g, e4m3_value(sc));
    const uint32_t q = den > 0.f ? e2m1_code(__fdiv_rn(v[m], den)) : 0u;
    const uint32_t hi = __shfl_down_sync(0xffffffffu, q, 1);
    if ((lane & 1) == 0) codes[row * (D / 2) + 16 * m + (lane >> 1)] = (uint8_t)(q | (hi << 4));
    if ((lane & 15) == 0) srow[2 * m + (lane >> 4)] = (uint8_t)sc;
  }
  if (lane == 0) *reinterpret_cast<float*>(srow + D / 16) = g;
  if (lane == 1 && SROWB > D / 16 + 4) *reinterpret_cast<uint32_t*>(srow + D / 16 + 4) = 0u;
}

}  // namespace

int launch_quantize(const kvq_cache_desc& desc, const void* x, const void* x2, int n_tok,
                    const int32_t* slots, void* codes, void* scales, void* codes2, void* scales2,
                    cudaStream_t stream) {
  const int64_t vecs = (int64_t)n_tok * desc.num_kv_heads;
  const int64_t blocks = (vecs + kWarpsPerBlock - 1) / kWarpsPerBlock;
  if (blocks > 0x7fffffffLL) return KVQ_ERR_UNSUPPORTED;
  // y = 0: the first plane pair; y = 1: the second (K and V in one launch)
  const dim3 grid((unsigned)blocks, x2 ? 2u : 1u), block(32 * kWarpsPerBlock);
  const __half* xh = static_cast<const __half*>(x);
  const __half* xh2 = static_cast<const __half*>(x2);
  const int hkv = desc.num_kv_heads, ps = desc.page_size;
#define KVQ_QUANT_CASE(FMT, DIM, KERNEL, ...)                                            \
  if (desc.fmt == FMT && desc.head_dim == DIM) {                                         \
    KERNEL<DIM><<<grid, block, 0, stream>>>(xh, xh2, n_tok, hkv, slots, ps, __VA_ARGS__); \
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;                    \
  }
  KVQ_QUANT_CASE(KVQ_FMT_Q8_0, 64, quant_q8_0_kernel, (int8_t*)codes, (__half*)scales, (int8_t*)codes2,
                 (__half*)scales2)
  KVQ_QUANT_CASE(KVQ_FMT_Q8_0, 128, quant_q8_0_kernel, (int8_t*)codes, (__half*)scales, (int8_t*)codes2,
                 (__half*)scales2)
  KVQ_QUANT_CASE(KVQ_FMT_Q4_0, 64, quant_q4_0_kernel, (uint8_t*)codes, (__half*)scales, (uint8_t*)codes2,
                 (__half*)scales2)
  KVQ_QUANT_CASE(KVQ_FMT_Q4_0, 128, quant_q4_0_kernel, (uint8_t*)codes, (__half*)scales, (uint8_t*)codes2,
                 (__half*)scales2)
  KVQ_QUANT_CASE(KVQ_FMT_LUT4, 64, quant_lut4_kernel, desc.codebook, desc.signs, (uint8_t*)codes,
                 (__half*)scales, (uint8_t*)codes2, (__half*)scales2)
  KVQ_QUANT_CASE(KVQ_FMT_LUT4, 128, quant_lut4_kernel, desc.codebook, desc.signs, (uint8_t*)codes,
                 (__half*)scales, (uint8_t*)codes2, (__half*)scales2)
  KVQ_QUANT_CASE(KVQ_FMT_NVFP4, 64, quant_nvfp4_kernel, (uint8_t*)codes, (uint8_t*)scales, (uint8_t*)codes2,
                 (uint8_t*)scales2)
  KVQ_QUANT_CASE(KVQ_FMT_NVFP4, 128, quant_nvfp4_kernel, (uint8_t*)codes, (uint8_t*)scales, (uint8_t*)codes2,
                 (uint8_t*)scales2)
#undef KVQ_QUANT_CASE
  return KVQ_ERR_UNSUPPORTED;
}

}  // namespace kvq
