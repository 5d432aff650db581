// Device code shared by the decode kernels (sm_100a): the per-format layout constants,
// the centroid / E2M1 lookups, the K-tile scoring job on the tensor cores (mma.sync
// m16n8k16: positions x heads x head_dim), the V dequantization of raw code words, the
// query fragments (lut4: the query rotated by the same random-sign Walsh-Hadamard
// transform as the cache) and the tagged (m, l) exchange reductions.
//
// Method: tproger.ru, "Пропуск 90% работы по деквантизации ускорил декодирование LLM",
// section "Решение — не ускорять, а пропускать" (weights from K first, V work skipped
// below the threshold) and "FAQ" (K is always dequantized).
#pragma once

#include <cuda_fp8.h>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {
constexpr float kPScale = 16384.0f;      // p is stored in fp16 as p * 2^14
constexpr float kPUnscale = 1.0f / 16384.0f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kMagic = 0x64006400u;    // fp16 1024 in both halves (unit mantissa step 1)
constexpr uint32_t kMagic64 = 0x54005400u;  // fp16 64: mantissa bits 4..7 then count in units of 1


template <int FMT, int D>
struct Cfg {
  static constexpr bool kQ8 = FMT == KVQ_FMT_Q8_0;
  static constexpr bool kQ4 = FMT == KVQ_FMT_Q4_0;
  static constexpr bool kLut = FMT == KVQ_FMT_LUT4;
  static constexpr bool kNv = FMT == KVQ_FMT_NVFP4;      // E2M1 codes, E4M3 scales per 16
  static constexpr int CROW = kQ8 ? D : D / 2;          // code bytes per row
  // fp16 slots per scale row (nvfp4: E4M3 bytes, fp32 vector scale, padding)
  static constexpr int NSC = kLut ? 1 : kNv ? (D / 16 + 4 + 7) / 8 * 4 : D / 32;
  static constexpr int SROW = 2 * NSC;                   // scale bytes per row
  static constexpr int NBLK = D / 32;
  static constexpr int KSTEPS = D / 16;
  // XOR swizzle of 16-byte chunks within a K code row: chunk ^= (row >> SWZ_SHIFT) & SWZ_MASK
  static constexpr int SWZ_SHIFT = CROW == 128 ? 0 : CROW == 64 ? 1 : 2;
  static constexpr int SWZ_MASK = CROW / 16 - 1;
  // V pass: thread (r, c) owns dims E*r .. E*r + E - 1
  static constexpr int E = D / 8;
  static constexpr int MT = D / 16;                      // m-tiles (16 dims each)
  static constexpr int NE = MT * 4;                      // accumulator registers per thread
  static constexpr int RAWB = kQ8 ? E : E / 2;           // code bytes per position per thread
  static constexpr int NWORD = RAWB / 4;
  // q8_0 / q4_0 V pass: codes enter the MMA as magic-number fp16 (code + offset) read
  // with transposing matrix loads, the scale rides on the weights (see vg_mag)
  static constexpr bool kMag = kQ8 || kQ4;
  static_assert(CROW % 16 == 0 && (CROW == 128 || CROW == 64 || CROW == 32), "row size");
};

// ------------------------------------------------------------------ LUT lookups
// 16 fp16 centroids held as 4 registers of low bytes and 4 of high bytes; a
// lookup of four 4-bit indices is two byte-permutes per byte plane and a select.
struct Lut {
  uint32_t lo[4], hi[4];
};

// sel: four indices in the low 16 bits (nibble k -> output byte k);
// mask: 0xff in output byte k when index k >= 8.
__device__ __forceinline__ void lut_lookup4(const Lut& t, uint32_t sel, uint32_t mask, uint32_t& L,
                                            uint32_t& H) {
  const uint32_t s = sel & 0x7777u;
  const uint32_t la = prmt(t.lo[0], t.lo[1], s), lb = prmt(t.lo[2], t.lo[3], s);
  const uint32_t ha = prmt(t.hi[0], t.hi[1], s), hb = prmt(t.hi[2], t.hi[3], s);
  L = (la & ~mask) | (lb & mask);
  H = (ha & ~mask) | (hb & mask);
}
// byte masks for nibbles 0-3 / 4-7 of x: replicate bit 3 of each nibble
__device__ __forceinline__ uint32_t nib_mask_lo(uint32_t x) { return prmt(x << 4, x, 0xD9C8u); }
__device__ __forceinline__ uint32_t nib_mask_hi(uint32_t x) { return prmt(x << 4, x, 0xFBEAu); }

// An E4M3 byte as an fp16 pair (s, s) (exact).
__device__ __forceinline__ __half2 e4m3_pair(uint32_t b) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(b | (b << 8)), __NV_E4M3);
  return *reinterpret_cast<const __half2*>(&h);
}
__device__ __forceinline__ float e4m3_float(uint32_t b) { return __low2float(e4m3_pair(b)); }
__device__ __forceinline__ uint32_t hmul2u(uint32_t a, __half2 b) {
  return h2_as_u32(__hmul2(u32_as_h2(a), b));
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  return h2_as_u32(__floats2half2_rn(lo, hi));
}

// ------------------------------------------------------------------ K job
// Raw scores (before sm_scale) of 16 positions (rows row0, row0 + 8 of this lane)
// x 8 heads.  q8_0 / q4_0: codes enter the MMA as fp16 (code + offset); the
// accumulator starts at -corr (the offset's contribution for this lane's heads) so
// each block's sum is exactly sum_d q_d * code_d, then the block scale multiplies it.
template <int FMT, int D>
__device__ __forceinline__ void k_job_scores(const uint8_t* __restrict__ codes,
                                             const uint8_t* __restrict__ sc, int row0,
                                             const uint32_t (&qf)[D / 16][2],
                                             const uint32_t (&ql)[D / 16][2],
                                             const float (&corr)[D / 32][2], const Lut& lut,
                                             int c, float (&s)[4]) {
  using C = Cfg<FMT, D>;
  const int row1 = row0 + 8;
  const uint8_t* p0 = codes + row0 * C::CROW + (c << 2);
  const uint8_t* p1 = codes + row1 * C::CROW + (c << 2);
  const int sw0 = (row0 >> C::SWZ_SHIFT) & C::SWZ_MASK;
  const int sw1 = (row1 >> C::SWZ_SHIFT) & C::SWZ_MASK;
  s[0] = s[1] = s[2] = s[3] = 0.f;
  if constexpr (C::kQ8 || C::kQ4) {
    float2 d0f[C::NBLK / 2 > 0 ? C::NBLK / 2 : 1], d1f[C::NBLK / 2 > 0 ? C::NBLK / 2 : 1];
    if constexpr (C::NBLK == 4) {
      const uint2 u0 = *reinterpret_cast<const uint2*>(sc + row0 * C::SROW);
      const uint2 u1 = *reinterpret_cast<const uint2*>(sc + row1 * C::SROW);
      d0f[0] = __half22float2(u32_as_h2(u0.x)); d0f[1] = __half22float2(u32_as_h2(u0.y));
      d1f[0] = __half22float2(u32_as_h2(u1.x)); d1f[1] = __half22float2(u32_as_h2(u1.y));
    } else {
      d0f[0] = __half22float2(u32_as_h2(lds32(sc + row0 * C::SROW)));
      d1f[0] = __half22float2(u32_as_h2(lds32(sc + row1 * C::SROW)));
    }
#pragma unroll
    for (int m = 0; m < C::NBLK; ++m) {
      float t[4] = {-corr[m][0], -corr[m][1], -corr[m][0], -corr[m][1]};
      if constexpr (C::kQ8) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int ks = 2 * m + j;  // chunk ks of the row holds dims 16 ks .. 16 ks + 15
          const uint32_t x0 = lds32(p0 + ((ks ^ sw0) << 4)) ^ 0x80808080u;
          const uint32_t x1 = lds32(p1 + ((ks ^ sw1) << 4)) ^ 0x80808080u;
          // (byte + 128) | fp16(1024): code + 1152, exact
          mma16816(t, prmt(x0, 0x64646464u, 0x4240u), prmt(x1, 0x64646464u, 0x4240u),
                   prmt(x0, 0x64646464u, 0x4341u), prmt(x1, 0x64646464u, 0x4341u), qf[ks][0],
                   qf[ks][1]);
        }
      } else {
        const uint32_t x0 = lds32(p0 + ((m ^ sw0) << 4));
        const uint32_t x1 = lds32(p1 + ((m ^ sw1) << 4));
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const uint32_t y0 = x0 >> (8 * j), y1 = x1 >> (8 * j);
          // even nibbles: 1024 + n; odd nibbles (bits 4..7): 64 + n
          mma16816(t, (y0 & 0x000F000Fu) | kMagic, (y1 & 0x000F000Fu) | kMagic,
                   (y0 & 0x00F000F0u) | kMagic64, (y1 & 0x00F000F0u) | kMagic64,
                   qf[2 * m + j][0], qf[2 * m + j][1]);
        }
      }
      const float d0 = (m & 1) ? d0f[m >> 1].y : d0f[m >> 1].x;
      const float d1 = (m & 1) ? d1f[m >> 1].y : d1f[m >> 1].x;
      s[0] = fmaf(d0, t[0], s[0]); s[1] = fmaf(d0, t[1], s[1]);
      s[2] = fmaf(d1, t[2], s[2]); s[3] = fmaf(d1, t[3], s[3]);
    }
  } else if constexpr (C::kLut) {
    // lut4: centroid lookups; the query carries hi + lo fp16 parts.
#pragma unroll
    for (int m = 0; m < C::NBLK; ++m) {
      const uint32_t x0 = lds32(p0 + ((m ^ sw0) << 4));
      const uint32_t x1 = lds32(p1 + ((m ^ sw1) << 4));
      uint32_t L0, H0, L1, H1, L2, H2, L3, H3;
      lut_lookup4(lut, x0, nib_mask_lo(x0), L0, H0);          // row0 dims +0..3
      lut_lookup4(lut, x0 >> 16, nib_mask_hi(x0), L1, H1);    // row0 dims +4..7
      lut_lookup4(lut, x1, nib_mask_lo(x1), L2, H2);          // row1 dims +0..3
      lut_lookup4(lut, x1 >> 16, nib_mask_hi(x1), L3, H3);    // row1 dims +4..7
      const uint32_t a0 = prmt(L0, H0, 0x5140u), a2 = prmt(L0, H0, 0x7362u);
      const uint32_t a1 = prmt(L2, H2, 0x5140u), a3 = prmt(L2, H2, 0x7362u);
      mma16816(s, a0, a1, a2, a3, qf[2 * m][0], qf[2 * m][1]);
      mma16816(s, a0, a1, a2, a3, ql[2 * m][0], ql[2 * m][1]);
      const uint32_t b0 = prmt(L1, H1, 0x5140u), b2 = prmt(L1, H1, 0x7362u);
      const uint32_t b1 = prmt(L3, H3, 0x5140u), b3 = prmt(L3, H3, 0x7362u);
      mma16816(s, b0, b1, b2, b3, qf[2 * m + 1][0], qf[2 * m + 1][1]);
      mma16816(s, b0, b1, b2, b3, ql[2 * m + 1][0], ql[2 * m + 1][1]);
    }
    const float n0 = __half2float(*reinterpret_cast<const __half*>(sc + row0 * 2));
    const float n1 = __half2float(*reinterpret_cast<const __half*>(sc + row1 * 2));
    s[0] *= n0; s[1] *= n0; s[2] *= n1; s[3] *= n1;
  } else {
    // nvfp4: E2M1 values from the table; the lane's 8 dims of chunk m lie in 16-block
    // 2m + c/2, whose E4M3 scale multiplies them in fp16 (exact: an E2M1 value times an
    // E4M3 value is representable); the fp32 vector scale multiplies the score.
    const uint8_t* s0p = sc + row0 * C::SROW;
    const uint8_t* s1p = sc + row1 * C::SROW;
#pragma unroll
    for (int m = 0; m < C::NBLK; ++m) {
      const uint32_t x0 = lds32(p0 + ((m ^ sw0) << 4));
      const uint32_t x1 = lds32(p1 + ((m ^ sw1) << 4));
      const int blk = 2 * m + (c >> 1);
      const __half2 sc0 = e4m3_pair(s0p[blk]), sc1 = e4m3_pair(s1p[blk]);
      uint32_t L0, H0, L1, H1, L2, H2, L3, H3;
      lut_lookup4(lut, x0, nib_mask_lo(x0), L0, H0);          // row0 dims +0..3
      lut_lookup4(lut, x0 >> 16, nib_mask_hi(x0), L1, H1);    // row0 dims +4..7
      lut_lookup4(lut, x1, nib_mask_lo(x1), L2, H2);          // row1 dims +0..3
      lut_lookup4(lut, x1 >> 16, nib_mask_hi(x1), L3, H3);    // row1 dims +4..7
      const uint32_t a0 = hmul2u(prmt(L0, H0, 0x5140u), sc0), a2 = hmul2u(prmt(L0, H0, 0x7362u), sc0);
      const uint32_t a1 = hmul2u(prmt(L2, H2, 0x5140u), sc1), a3 = hmul2u(prmt(L2, H2, 0x7362u), sc1);
      mma16816(s, a0, a1, a2, a3, qf[2 * m][0], qf[2 * m][1]);
      const uint32_t b0 = hmul2u(prmt(L1, H1, 0x5140u), sc0), b2 = hmul2u(prmt(L1, H1, 0x7362u), sc0);
      const uint32_t b1 = hmul2u(prmt(L3, H3, 0x5140u), sc1), b3 = hmul2u(prmt(L3, H3, 0x7362u), sc1);
      mma16816(s, b0, b1, b2, b3, qf[2 * m + 1][0], qf[2 * m + 1][1]);
    }
    const float g0 = *reinterpret_cast<const float*>(s0p + D / 16);
    const float g1 = *reinterpret_cast<const float*>(s1p + D / 16);
    s[0] *= g0; s[1] *= g0; s[2] *= g1; s[3] *= g1;
  }
}

// ------------------------------------------------------------------ V pass
// Dequantize the raw bits of two positions (a, b) into half2 (a, b) pairs, one per
// dim owned by this thread (E of them), in dim order.
template <int FMT, int D>
__device__ __forceinline__ void v_dequant_pair(const uint32_t (&ra)[Cfg<FMT, D>::NWORD],
                                               const uint32_t (&rb)[Cfg<FMT, D>::NWORD],
                                               const Lut& lut, uint32_t (&e)[Cfg<FMT, D>::E]) {
  using C = Cfg<FMT, D>;
#pragma unroll
  for (int k = 0; k < C::NWORD; ++k) {
    const uint32_t wa = ra[k], wb = rb[k];
    if constexpr (C::kQ8) {
      // 4 int8 codes per word -> 4 dims
      const __half2 bias = __half2half2(__ushort_as_half(0x6480));  // 1152
      const uint32_t xa = wa ^ 0x80808080u, xb = wb ^ 0x80808080u;
      const uint32_t t01 = prmt(xa, xb, 0x5140u), t23 = prmt(xa, xb, 0x7362u);
      e[4 * k + 0] = h2_as_u32(__hsub2(u32_as_h2(prmt(t01, 0x64646464u, 0x4140u)), bias));
      e[4 * k + 1] = h2_as_u32(__hsub2(u32_as_h2(prmt(t01, 0x64646464u, 0x4342u)), bias));
      e[4 * k + 2] = h2_as_u32(__hsub2(u32_as_h2(prmt(t23, 0x64646464u, 0x4140u)), bias));
      e[4 * k + 3] = h2_as_u32(__hsub2(u32_as_h2(prmt(t23, 0x64646464u, 0x4342u)), bias));
    } else if constexpr (C::kQ4) {
      // 8 nibbles per word -> 8 dims; x_lo holds dims 0-3 of both positions, x_hi dims 4-7
      const __half2 b1032 = __half2half2(__ushort_as_half(0x6408));  // 1032
      const __half2 b72 = __half2half2(__ushort_as_half(0x5480));    // 72
#pragma unroll
      for (int hlf = 0; hlf < 2; ++hlf) {
        const uint32_t x = hlf ? prmt(wa, wb, 0x7632u) : prmt(wa, wb, 0x5410u);
        const uint32_t y = x >> 8;
        e[8 * k + 4 * hlf + 0] = h2_as_u32(__hsub2(u32_as_h2((x & 0x000F000Fu) | kMagic), b1032));
        e[8 * k + 4 * hlf + 1] = h2_as_u32(__hsub2(u32_as_h2((x & 0x00F000F0u) | kMagic64), b72));
        e[8 * k + 4 * hlf + 2] = h2_as_u32(__hsub2(u32_as_h2((y & 0x000F000Fu) | kMagic), b1032));
        e[8 * k + 4 * hlf + 3] = h2_as_u32(__hsub2(u32_as_h2((y & 0x00F000F0u) | kMagic64), b72));
      }
    } else {
#pragma unroll
      for (int hlf = 0; hlf < 2; ++hlf) {
        const uint32_t x = hlf ? prmt(wa, wb, 0x7632u) : prmt(wa, wb, 0x5410u);
        uint32_t La, Ha, Lb, Hb;
        lut_lookup4(lut, x, nib_mask_lo(x), La, Ha);
        lut_lookup4(lut, x >> 16, nib_mask_hi(x), Lb, Hb);
        const uint32_t ta01 = prmt(La, Ha, 0x5140u), tb01 = prmt(Lb, Hb, 0x5140u);
        const uint32_t ta23 = prmt(La, Ha, 0x7362u), tb23 = prmt(Lb, Hb, 0x7362u);
        e[8 * k + 4 * hlf + 0] = prmt(ta01, tb01, 0x5410u);
        e[8 * k + 4 * hlf + 1] = prmt(ta01, tb01, 0x7632u);
        e[8 * k + 4 * hlf + 2] = prmt(ta23, tb23, 0x5410u);
        e[8 * k + 4 * hlf + 3] = prmt(ta23, tb23, 0x7632u);
      }
    }
  }
}

template <int FMT, int D>
__device__ __forceinline__ void v_raw(const uint8_t* p, uint32_t (&w)[Cfg<FMT, D>::NWORD]) {
  using C = Cfg<FMT, D>;
  if constexpr (C::NWORD == 4) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    w[0] = u.x; w[1] = u.y; w[2] = u.z; w[3] = u.w;
  } else if constexpr (C::NWORD == 2) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    w[0] = u.x; w[1] = u.y;
  } else {
    w[0] = lds32(p);
  }
}

// (M, L) of the exchange entries e[u] this lane takes: u = first + step * t (t < T) in
// every pass of T * step entries, u < n, none when !active; M is their maximum and L
// their denominators rescaled to it.  Each pass waits until all its entries carry this
// launch's tag (its loads all in flight together); false if that took longer than
// `limit` SM cycles.  Warp-uniform: every lane of the warp calls it with the same n.
template <int T>
__device__ __forceinline__ bool xch_reduce(const ulonglong2* e, int first, int step, int n,
                                           bool active, uint32_t tag, float& M, float& L,
                                           long long limit = kWaitCycles, int sleep_ns = 32) {
  M = -INFINITY;
  L = 0.f;
  for (int ub = 0; ub < n; ub += T * step) {
    float mv[T], lv[T];
    const long long t0 = clock64();
    for (;;) {
      bool all = true;
#pragma unroll
      for (int t = 0; t < T; ++t) {
        const int u = ub + first + step * t;
        mv[t] = -INFINITY;
        lv[t] = 0.f;
        if (active && u < n)
          all &= xch_load(e + u, tag, mv[t], lv[t]);
      }
      if (__all_sync(0xffffffffu, all)) break;
      if (__any_sync(0xffffffffu, clock64() - t0 > limit)) return false;
      __nanosleep(sleep_ns);
    }
    float bm = M;
#pragma unroll
    for (int t = 0; t < T; ++t) bm = fmaxf(bm, mv[t]);
    float ds = (M == -INFINITY) ? 0.f : L * ex2(M - bm);
#pragma unroll
    for (int t = 0; t < T; ++t)
      if (mv[t] != -INFINITY) ds = fmaf(ex2(mv[t] - bm), lv[t], ds);
    M = bm;
    L = ds;
  }
  return true;
}

// Combine (M, L) across the lanes that differ in bits 1 .. max_off of the lane index.
__device__ __forceinline__ void xch_combine(float& M, float& L, int max_off) {
  for (int o = 1; o <= max_off; o <<= 1) {
    const float Mo = __shfl_xor_sync(0xffffffffu, M, o);
    const float Lo = __shfl_xor_sync(0xffffffffu, L, o);
    const float nm = fmaxf(M, Mo);
    L = (M == -INFINITY ? 0.f : L * ex2(M - nm)) + (Mo == -INFINITY ? 0.f : Lo * ex2(Mo - nm));
    M = nm;
  }
}

// bit 4r set iff any of bits 4r .. 4r+3 of a ballot is set (one row per 4-lane group)
__device__ __forceinline__ uint32_t rows_of(uint32_t bal) {
  uint32_t x = bal | (bal >> 1);
  x |= x >> 2;
  return x & 0x11111111u;
}

// ------------------------------------------------------------------ query fragments
// Lane (r, c) of every warp builds, from the fp16 query words it loaded (zeros for a
// head the group does not have), the B fragments of the K pass for query head r, plus the offset correction of its accumulator heads 2c, 2c + 1
// (q8_0 / q4_0) or the fp16 low parts of the rotated query (lut4).  The dims a lane
// needs mirror how each format's A fragment is unpacked from one 32-bit word of codes:
//   q8_0  k-step ks: dims 16 ks + 4c + {0, 2 | 1, 3}
//   q4_0  k-step 2m + j: dims 32m + 8c + 2j + {0, 4 | 1, 5}
//   lut4  k-step 2m + j: dims 32m + 8c + 4j + {0, 1 | 2, 3}
// The raw query words a lane needs (loaded early, so that they lead the copy queue),
// and for lut4 the rotation signs of its dims.
template <int D>
struct QRaw {
  uint32_t w[D / 8];
  uint32_t sg[D / 16];
};

template <int FMT, int D>
__device__ __forceinline__ void load_query(const __half* __restrict__ qh,
                                           const int8_t* __restrict__ signs, int c, QRaw<D>& q) {
  using C = Cfg<FMT, D>;
#pragma unroll
  for (int i = 0; i < D / 8; ++i) q.w[i] = 0u;
#pragma unroll
  for (int i = 0; i < D / 16; ++i) q.sg[i] = 0u;
  if (qh) {
    if constexpr (C::kQ8) {
#pragma unroll
      for (int ks = 0; ks < C::KSTEPS; ++ks) {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(qh + 16 * ks + 4 * c));
        q.w[2 * ks] = u.x;
        q.w[2 * ks + 1] = u.y;
      }
    } else {
#pragma unroll
      for (int m = 0; m < C::NBLK; ++m) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(qh + 32 * m + 8 * c));
        q.w[4 * m] = u.x; q.w[4 * m + 1] = u.y; q.w[4 * m + 2] = u.z; q.w[4 * m + 3] = u.w;
      }
    }
  }
  if constexpr (C::kLut) {
#pragma unroll
    for (int m = 0; m < C::NBLK; ++m) {
      const uint2 u = __ldg(reinterpret_cast<const uint2*>(signs + 32 * m + 8 * c));
      q.sg[2 * m] = u.x;
      q.sg[2 * m + 1] = u.y;
    }
  }
}

template <int FMT, int D>
__device__ __forceinline__ void build_query(const QRaw<D>& q, int c,
                                            uint32_t (&qf)[D / 16][2], uint32_t (&ql)[D / 16][2],
                                            float (&corr)[D / 32][2]) {
  using C = Cfg<FMT, D>;
  if constexpr (C::kNv) {
    // the query as it is (no rotation, no offset): k-step 2m + j takes halves 4j .. 4j + 3
    // of the lane's 8 dims 32m + 8c .. 32m + 8c + 7
#pragma unroll
    for (int m = 0; m < C::NBLK; ++m) {
      qf[2 * m][0] = q.w[4 * m];
      qf[2 * m][1] = q.w[4 * m + 1];
      qf[2 * m + 1][0] = q.w[4 * m + 2];
      qf[2 * m + 1][1] = q.w[4 * m + 3];
      ql[2 * m][0] = ql[2 * m][1] = ql[2 * m + 1][0] = ql[2 * m + 1][1] = 0u;
      corr[m][0] = corr[m][1] = 0.f;
    }
  } else if constexpr (!C::kLut) {
    float part[C::NBLK];
#pragma unroll
    for (int m = 0; m < C::NBLK; ++m) {
      if constexpr (C::kQ4) {
        const uint4 u = make_uint4(q.w[4 * m], q.w[4 * m + 1], q.w[4 * m + 2], q.w[4 * m + 3]);
        qf[2 * m][0] = prmt(u.x, u.z, 0x5410u);
        qf[2 * m][1] = prmt(u.x, u.z, 0x7632u);
        qf[2 * m + 1][0] = prmt(u.y, u.w, 0x5410u);
        qf[2 * m + 1][1] = prmt(u.y, u.w, 0x7632u);
        // dims 32m + 8c + i: even i enter the MMA as 1024 + n, odd i as 64 + n; both
        // decode as n - 8, so the offsets are 1032 and 72
        const float2 f0 = __half22float2(u32_as_h2(u.x)), f1 = __half22float2(u32_as_h2(u.y));
        const float2 f2 = __half22float2(u32_as_h2(u.z)), f3 = __half22float2(u32_as_h2(u.w));
        part[m] = 1032.f * ((f0.x + f1.x) + (f2.x + f3.x)) + 72.f * ((f0.y + f1.y) + (f2.y + f3.y));
      } else {
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int ks = 2 * m + j;
          const uint2 u = make_uint2(q.w[2 * ks], q.w[2 * ks + 1]);
          qf[ks][0] = prmt(u.x, u.y, 0x5410u);
          qf[ks][1] = prmt(u.x, u.y, 0x7632u);
          const float2 f0 = __half22float2(u32_as_h2(u.x)), f1 = __half22float2(u32_as_h2(u.y));
          s += (f0.x + f0.y) + (f1.x + f1.y);
        }
        part[m] = 1152.f * s;  // codes enter as 1152 + q
      }
      ql[2 * m][0] = ql[2 * m][1] = ql[2 * m + 1][0] = ql[2 * m + 1][1] = 0;
    }
    // sum over the four lanes of head r, then fetch heads 2c, 2c + 1
#pragma unroll
    for (int m = 0; m < C::NBLK; ++m) {
      float v = part[m];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      corr[m][0] = __shfl_sync(0xffffffffu, v, 8 * c);
      corr[m][1] = __shfl_sync(0xffffffffu, v, 8 * c + 4);
    }
  } else {
    // q' = (1/sqrt(D)) H (s .* q), Sylvester H.  Lane c of head r holds dims
    // 32m + 8c + i: index bits 0-2 are i (in the lane), bits 3-4 are c (lanes c ^ 1,
    // c ^ 2), bits 5-6 are m (in the lane).
    float y[C::NBLK][8];
#pragma unroll
    for (int m = 0; m < C::NBLK; ++m) {
      const uint2 sg = make_uint2(q.sg[2 * m], q.sg[2 * m + 1]);
      const uint32_t w[4] = {q.w[4 * m], q.w[4 * m + 1], q.w[4 * m + 2], q.w[4 * m + 3]};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float2 f = __half22float2(u32_as_h2(w[i >> 1]));
        const int8_t sgn = static_cast<int8_t>(((i < 4 ? sg.x : sg.y) >> (8 * (i & 3))) & 0xffu);
        y[m][i] = ((i & 1) ? f.y : f.x) * (float)sgn;
      }
    }
#pragma unroll
    for (int h = 1; h < 8; h <<= 1)
#pragma unroll
      for (int m = 0; m < C::NBLK; ++m)
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (!(i & h)) {
            const float p = y[m][i], q = y[m][i + h];
            y[m][i] = p + q;
            y[m][i + h] = p - q;
          }
#pragma unroll
    for (int bit = 1; bit < 4; bit <<= 1) {
      const bool upper = (c & bit) != 0;
#pragma unroll
      for (int m = 0; m < C::NBLK; ++m)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float o = __shfl_xor_sync(0xffffffffu, y[m][i], bit);
          y[m][i] = upper ? (o - y[m][i]) : (y[m][i] + o);
        }
    }
#pragma unroll
    for (int h = 1; h < C::NBLK; h <<= 1)
#pragma unroll
      for (int m = 0; m < C::NBLK; ++m)
        if (!(m & h)) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float p = y[m][i], q = y[m + h][i];
            y[m][i] = p + q;
            y[m + h][i] = p - q;
          }
        }
    const float cs = D == 64 ? 0.125f : 0.08838834764831845f;  // 1/sqrt(D)
#pragma unroll
    for (int m = 0; m < C::NBLK; ++m) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float v0 = y[m][4 * j] * cs, v1 = y[m][4 * j + 1] * cs;
        const float v2 = y[m][4 * j + 2] * cs, v3 = y[m][4 * j + 3] * cs;
        const __half2 h01 = __floats2half2_rn(v0, v1), h23 = __floats2half2_rn(v2, v3);
        qf[2 * m + j][0] = h2_as_u32(h01);
        qf[2 * m + j][1] = h2_as_u32(h23);
        ql[2 * m + j][0] = pack_h2(v0 - __low2float(h01), v1 - __high2float(h01));
        ql[2 * m + j][1] = pack_h2(v2 - __low2float(h23), v3 - __high2float(h23));
      }
      corr[m][0] = corr[m][1] = 0.f;
    }
  }
}


// Chunk swizzle of a staged row (K tiles and V rows alike): 16-byte chunk cc of row `row`
// sits at chunk position cc ^ swz(row).
template <int FMT, int D>
__device__ __forceinline__ int swz(int row) {
  using C = Cfg<FMT, D>;
  return (row >> C::SWZ_SHIFT) & C::SWZ_MASK;
}

// Stage the V rows row0 .. row0 + rows - 1 of a tile (rows = 64, or 32 for a half tile):
}  // namespace
}  // namespace kvq
