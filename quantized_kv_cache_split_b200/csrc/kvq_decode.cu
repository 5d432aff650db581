// Split-KV decode attention with sparse V dequantization (sm_100a).
//
// Method (tproger.ru, "Пропуск 90% работы по деквантизации ускорил
// декодирование LLM", section "Решение — не ускорять, а пропускать"): the
// softmax weights come from K before any V work, so V dequantization and
// accumulation are skipped for every position whose weight exp(s - m_running)
// is below tau.  Section "FAQ": K itself is always dequantized.
//
// One CTA (4 warps) per SM runs a persistent loop over work units
// (sequence b, KV head, split of <= 1024 positions).  Per unit:
//   K pass  64-position K tiles (codes + block scales) stream into a ring of
//           shared-memory stages through TMA (2-D tensor copy with hardware
//           swizzle for the codes, 1-D bulk copy for the scales), issued up to
//           STAGES tiles ahead by one thread and running on into the next unit.
//           Each warp dequantizes 16 positions in registers and multiplies them
//           with the query group on the tensor cores (mma m16n8k16: positions x
//           heads x head_dim); block scales / vector norms are applied to the
//           fp32 score, so integer codes enter the MMA exactly.  Scores (log2
//           units) go to shared memory; the running maximum is kept per head.
//   weights Once every K tile of the unit is folded in, m_running is the unit's
//           maximum.  p = 2^(s - m); l sums every p; (position, head) pairs with
//           p < tau are dropped; positions kept by any head of the group are
//           compacted (warp ballot + prefix) into a list, with their p values
//           (fp16, pre-scaled by 2^14) transposed per head.
//   V pass  Only listed positions are fetched (cp.async 16-byte gathers of their
//           V rows and scales, four 64-row batches in flight), dequantized in
//           registers and accumulated on the tensor cores (dims x heads x
//           positions).  Skipped positions cost no HBM read, no dequant, no MMA.
//   output  Unnormalized o, m (log2 units) and l of the unit go to the
//           workspace; kvq_combine merges the units of a sequence.
#include <cudaTypedefs.h>

#include <mutex>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kLmax = KVQ_MAX_SPLIT_TOKENS;
constexpr int kMaxTiles = kLmax / kTile;
constexpr int kPktStride = kLmax + 8;   // halves per head row of the compacted weights
constexpr float kPScale = 16384.0f;     // p is stored in fp16 as p * 2^14
constexpr float kPUnscale = 1.0f / 16384.0f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kMagic = 0x64006400u;  // fp16 1024.0 in both halves

template <int FMT, int D>
struct Cfg {
  static constexpr bool kQ8 = FMT == KVQ_FMT_Q8_0;
  static constexpr bool kQ4 = FMT == KVQ_FMT_Q4_0;
  static constexpr bool kLut = FMT == KVQ_FMT_LUT4;
  static constexpr int CROW = kQ8 ? D : D / 2;          // code bytes per row
  static constexpr int NSC = kLut ? 1 : D / 32;          // fp16 per scale row
  static constexpr int SROW = 2 * NSC;                   // scale bytes per row
  static constexpr int NBLK = D / 32;
  static constexpr int KSTEPS = D / 16;
  static constexpr int STAGE_CODE = kTile * CROW;
  static constexpr int STAGE_SC = kTile * SROW;
  static constexpr int STAGE_BYTES = (STAGE_CODE + STAGE_SC + 1023) / 1024 * 1024;
  static constexpr int STAGES = STAGE_BYTES <= 5120 ? 16 : 12;
  // TMA swizzle of the codes: 16-byte chunk index ^= (row >> SWZ_SHIFT) & SWZ_MASK
  static constexpr int SWZ_SHIFT = CROW == 128 ? 0 : CROW == 64 ? 1 : 2;
  static constexpr int SWZ_MASK = CROW / 16 - 1;
  // V pass
  static constexpr int VB = 64;               // positions per gather batch
  static constexpr int NVB = 4;               // batches in flight
  static constexpr int VSTRIDE = CROW + 16;   // padded row stride of the V staging buffer
  static constexpr int VDW = D / kWarps;      // dims per warp
  static constexpr int E = VDW / 8;           // dims per thread
  static constexpr int MT = VDW / 16;         // m-tiles per warp
  static_assert(CROW % 16 == 0 && (CROW == 128 || CROW == 64 || CROW == 32), "row size");
};

template <int FMT, int D>
struct Layout {
  using C = Cfg<FMT, D>;
  static constexpr size_t stage = 0;
  static constexpr size_t S = stage + (size_t)C::STAGES * C::STAGE_BYTES;  // float [kLmax][8]
  static constexpr size_t pkt = S + (size_t)kLmax * 8 * 4;                  // half [8][kPktStride]
  static constexpr size_t list = pkt + (size_t)8 * kPktStride * 2;          // u16 [kLmax]
  static constexpr size_t vbuf = list + (size_t)kLmax * 2;                  // [NVB][VB][VSTRIDE]
  static constexpr size_t vsc = vbuf + (size_t)C::NVB * C::VB * C::VSTRIDE;  // [NVB][VB][8]
  static constexpr size_t q = vsc + (size_t)C::NVB * C::VB * 8;             // float [8][D]
  static constexpr size_t rows = q + (size_t)8 * D * 4;                     // int [kMaxTiles]
  static constexpr size_t stage_row = rows + kMaxTiles * 4;                 // int [STAGES]
  static constexpr size_t red = stage_row + C::STAGES * 4;                  // float [3][kWarps][8]
  static constexpr size_t cnt = red + 3 * kWarps * 8 * 4;                   // int [8]
  static constexpr size_t bars = (cnt + 8 * 4 + 7) / 8 * 8;                 // u64 [STAGES]
  static constexpr size_t prefix = bars + C::STAGES * 8;                    // int [MAX_BATCH + 1]
  static constexpr size_t total = prefix + (KVQ_MAX_BATCH + 1) * 4;
  static constexpr size_t alloc = total + 1024;  // slack for aligning the base to 1024
};

struct Item {
  int b, kvh, split, t0, n_tok;
};

__device__ __forceinline__ int clamp_len(const DecodeArgs& a, int b) {
  const int cap = min(a.max_seq_len, a.max_pages * a.desc.page_size);
  const int n = a.seq_lens[b];
  return max(0, min(n, cap));
}

__device__ __forceinline__ Item decode_item(const DecodeArgs& a, const int* prefix, int it) {
  const int hkv = a.desc.num_kv_heads;
  Item I;
  const int sg = it / hkv;
  I.kvh = it - sg * hkv;
  int lo = 0, hi = a.batch;  // largest b with prefix[b] <= sg
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= sg) lo = mid; else hi = mid;
  }
  I.b = lo;
  I.split = sg - prefix[lo];
  I.t0 = I.split * a.split_tokens;
  I.n_tok = min(a.split_tokens, clamp_len(a, lo) - I.t0);
  return I;
}

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

// ------------------------------------------------------------------ query fragments
// Physical dims feeding the B fragment of k-step ks for tid-in-group c, in the
// order (reg0.lo, reg0.hi, reg1.lo, reg1.hi).  They mirror how each format's
// A fragment is unpacked from one 32-bit word of codes.
template <int FMT>
__device__ __forceinline__ void k_dims(int ks, int c, int (&d)[4]) {
  if (FMT == KVQ_FMT_Q8_0) {
    const int base = 16 * ks + 4 * c;  // bytes b0..b3 -> (b0, b2) and (b1, b3)
    d[0] = base; d[1] = base + 2; d[2] = base + 1; d[3] = base + 3;
  } else if (FMT == KVQ_FMT_Q4_0) {
    const int base = 32 * (ks >> 1) + 8 * c + 2 * (ks & 1);  // nibble pairs (n, n+4)
    d[0] = base; d[1] = base + 4; d[2] = base + 1; d[3] = base + 5;
  } else {
    const int base = 32 * (ks >> 1) + 8 * c + 4 * (ks & 1);  // consecutive nibbles
    d[0] = base; d[1] = base + 1; d[2] = base + 2; d[3] = base + 3;
  }
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  return h2_as_u32(__floats2half2_rn(lo, hi));
}

// ------------------------------------------------------------------ K tile
// Scores of 16 positions (rows row0, row0 + 8 of this lane) x 8 heads.
template <int FMT, int D>
__device__ __forceinline__ void k_tile_scores(const uint8_t* __restrict__ codes,
                                              const uint8_t* __restrict__ sc, int row0,
                                              const uint32_t (&qf)[D / 16][2],
                                              const uint32_t (&ql)[D / 16][2], const Lut& lut,
                                              int c, float (&s)[4]) {
  using C = Cfg<FMT, D>;
  const int row1 = row0 + 8;
  const uint8_t* p0 = codes + row0 * C::CROW + (c << 2);
  const uint8_t* p1 = codes + row1 * C::CROW + (c << 2);
  const int sw0 = (row0 >> C::SWZ_SHIFT) & C::SWZ_MASK;
  const int sw1 = (row1 >> C::SWZ_SHIFT) & C::SWZ_MASK;
  s[0] = s[1] = s[2] = s[3] = 0.f;
  if constexpr (C::kQ8) {
    // scales of the two rows: NBLK fp16 each
    uint32_t d0w[2], d1w[2];
    if constexpr (C::NBLK == 4) {
      const uint2 u0 = *reinterpret_cast<const uint2*>(sc + row0 * C::SROW);
      const uint2 u1 = *reinterpret_cast<const uint2*>(sc + row1 * C::SROW);
      d0w[0] = u0.x; d0w[1] = u0.y; d1w[0] = u1.x; d1w[1] = u1.y;
    } else {
      d0w[0] = lds32(sc + row0 * C::SROW); d1w[0] = lds32(sc + row1 * C::SROW);
      d0w[1] = d1w[1] = 0;
    }
    const __half2 bias = __half2half2(__ushort_as_half(0x6480));  // 1152
#pragma unroll
    for (int m = 0; m < C::NBLK; ++m) {
      float t[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int ks = 2 * m + j;  // chunk ks of the row holds dims 16 ks .. 16 ks + 15
        const uint32_t x0 = lds32(p0 + ((ks ^ sw0) << 4)) ^ 0x80808080u;
        const uint32_t x1 = lds32(p1 + ((ks ^ sw1) << 4)) ^ 0x80808080u;
        const uint32_t a0 = h2_as_u32(__hsub2(u32_as_h2(prmt(x0, 0x64646464u, 0x4240u)), bias));
        const uint32_t a1 = h2_as_u32(__hsub2(u32_as_h2(prmt(x1, 0x64646464u, 0x4240u)), bias));
        const uint32_t a2 = h2_as_u32(__hsub2(u32_as_h2(prmt(x0, 0x64646464u, 0x4341u)), bias));
        const uint32_t a3 = h2_as_u32(__hsub2(u32_as_h2(prmt(x1, 0x64646464u, 0x4341u)), bias));
        mma16816(t, a0, a1, a2, a3, qf[ks][0], qf[ks][1]);
      }
      const uint32_t w0 = d0w[m >> 1], w1 = d1w[m >> 1];
      const float d0 = __half2float(__ushort_as_half((uint16_t)((m & 1) ? (w0 >> 16) : w0)));
      const float d1 = __half2float(__ushort_as_half((uint16_t)((m & 1) ? (w1 >> 16) : w1)));
      s[0] = fmaf(d0, t[0], s[0]); s[1] = fmaf(d0, t[1], s[1]);
      s[2] = fmaf(d1, t[2], s[2]); s[3] = fmaf(d1, t[3], s[3]);
    }
  } else if constexpr (C::kQ4) {
    uint32_t d0w[2], d1w[2];
    if constexpr (C::NBLK == 4) {
      const uint2 u0 = *reinterpret_cast<const uint2*>(sc + row0 * C::SROW);
      const uint2 u1 = *reinterpret_cast<const uint2*>(sc + row1 * C::SROW);
      d0w[0] = u0.x; d0w[1] = u0.y; d1w[0] = u1.x; d1w[1] = u1.y;
    } else {
      d0w[0] = lds32(sc + row0 * C::SROW); d1w[0] = lds32(sc + row1 * C::SROW);
      d0w[1] = d1w[1] = 0;
    }
    const __half2 b1032 = __half2half2(__ushort_as_half(0x6408));       // 1032
    const __half2 inv16 = __half2half2(__ushort_as_half(0x2C00));       // 1/16
    const __half2 m72 = __half2half2(__ushort_as_half(0xD480));         // -72
#pragma unroll
    for (int m = 0; m < C::NBLK; ++m) {
      const uint32_t x0 = lds32(p0 + ((m ^ sw0) << 4));
      const uint32_t x1 = lds32(p1 + ((m ^ sw1) << 4));
      float t[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const uint32_t y0 = x0 >> (8 * j), y1 = x1 >> (8 * j);
        // (n_{2j}, n_{2j+4}) and 16 * (n_{2j+1}, n_{2j+5}) as fp16, then minus 8
        const uint32_t a0 = h2_as_u32(__hsub2(u32_as_h2((y0 & 0x000F000Fu) | kMagic), b1032));
        const uint32_t a1 = h2_as_u32(__hsub2(u32_as_h2((y1 & 0x000F000Fu) | kMagic), b1032));
        const uint32_t a2 =
            h2_as_u32(__hfma2(u32_as_h2((y0 & 0x00F000F0u) | kMagic), inv16, m72));
        const uint32_t a3 =
            h2_as_u32(__hfma2(u32_as_h2((y1 & 0x00F000F0u) | kMagic), inv16, m72));
        mma16816(t, a0, a1, a2, a3, qf[2 * m + j][0], qf[2 * m + j][1]);
      }
      const uint32_t w0 = d0w[m >> 1], w1 = d1w[m >> 1];
      const float d0 = __half2float(__ushort_as_half((uint16_t)((m & 1) ? (w0 >> 16) : w0)));
      const float d1 = __half2float(__ushort_as_half((uint16_t)((m & 1) ? (w1 >> 16) : w1)));
      s[0] = fmaf(d0, t[0], s[0]); s[1] = fmaf(d0, t[1], s[1]);
      s[2] = fmaf(d1, t[2], s[2]); s[3] = fmaf(d1, t[3], s[3]);
    }
  } else {
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
      // k-step 2m: dims +0..3, k-step 2m+1: dims +4..7
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
  }
}

// ------------------------------------------------------------------ V batch
// Accumulate o[dims of this warp][8 heads] += v_hat^T p over one staged batch.
template <int FMT, int D>
__device__ __forceinline__ void v_dequant_pair(uint32_t ra, uint32_t rb, const Lut& lut,
                                               uint32_t (&e)[Cfg<FMT, D>::E]) {
  using C = Cfg<FMT, D>;
  if constexpr (C::kQ8) {
    const __half2 bias = __half2half2(__ushort_as_half(0x6480));  // 1152
    if constexpr (C::E == 4) {
      const uint32_t wa = ra ^ 0x80808080u, wb = rb ^ 0x80808080u;
      const uint32_t t01 = prmt(wa, wb, 0x5140u), t23 = prmt(wa, wb, 0x7362u);
      e[0] = h2_as_u32(__hsub2(u32_as_h2(prmt(t01, 0x64646464u, 0x4140u)), bias));
      e[1] = h2_as_u32(__hsub2(u32_as_h2(prmt(t01, 0x64646464u, 0x4342u)), bias));
      e[2] = h2_as_u32(__hsub2(u32_as_h2(prmt(t23, 0x64646464u, 0x4140u)), bias));
      e[3] = h2_as_u32(__hsub2(u32_as_h2(prmt(t23, 0x64646464u, 0x4342u)), bias));
    } else {
      const uint32_t t = prmt(ra ^ 0x8080u, rb ^ 0x8080u, 0x5140u);
      e[0] = h2_as_u32(__hsub2(u32_as_h2(prmt(t, 0x64646464u, 0x4140u)), bias));
      e[1] = h2_as_u32(__hsub2(u32_as_h2(prmt(t, 0x64646464u, 0x4342u)), bias));
    }
  } else if constexpr (C::kQ4) {
    const __half2 b1032 = __half2half2(__ushort_as_half(0x6408));
    const __half2 inv16 = __half2half2(__ushort_as_half(0x2C00));
    const __half2 m72 = __half2half2(__ushort_as_half(0xD480));
    const uint32_t x = (C::E == 4) ? prmt(ra, rb, 0x5410u) : prmt(ra, rb, 0x0400u);
    e[0] = h2_as_u32(__hsub2(u32_as_h2((x & 0x000F000Fu) | kMagic), b1032));
    e[1] = h2_as_u32(__hfma2(u32_as_h2((x & 0x00F000F0u) | kMagic), inv16, m72));
    if constexpr (C::E == 4) {
      const uint32_t y = x >> 8;
      e[2] = h2_as_u32(__hsub2(u32_as_h2((y & 0x000F000Fu) | kMagic), b1032));
      e[3] = h2_as_u32(__hfma2(u32_as_h2((y & 0x00F000F0u) | kMagic), inv16, m72));
    }
  } else {
    if constexpr (C::E == 4) {
      const uint32_t x = prmt(ra, rb, 0x5410u);  // low half: a's 4 nibbles, high: b's
      uint32_t La, Ha, Lb, Hb;
      lut_lookup4(lut, x, nib_mask_lo(x), La, Ha);
      lut_lookup4(lut, x >> 16, nib_mask_hi(x), Lb, Hb);
      const uint32_t ta01 = prmt(La, Ha, 0x5140u), tb01 = prmt(Lb, Hb, 0x5140u);
      const uint32_t ta23 = prmt(La, Ha, 0x7362u), tb23 = prmt(Lb, Hb, 0x7362u);
      e[0] = prmt(ta01, tb01, 0x5410u);
      e[1] = prmt(ta01, tb01, 0x7632u);
      e[2] = prmt(ta23, tb23, 0x5410u);
      e[3] = prmt(ta23, tb23, 0x7632u);
    } else {
      const uint32_t x = prmt(ra, rb, 0x0040u);  // nibbles: a0 a1 b0 b1
      uint32_t L, H;
      lut_lookup4(lut, x, nib_mask_lo(x), L, H);
      e[0] = prmt(L, H, 0x6240u);
      e[1] = prmt(L, H, 0x7351u);
    }
  }
}

template <int FMT, int D>
__device__ __forceinline__ uint32_t v_raw(const uint8_t* row, int boff) {
  using C = Cfg<FMT, D>;
  if constexpr (C::kQ8) {
    if constexpr (C::E == 4) return lds32(row + boff);
    else return lds16(row + boff);
  } else {
    if constexpr (C::E == 4) return lds16(row + boff);
    else return lds8(row + boff);
  }
}

template <int FMT, int D>
__device__ __forceinline__ __half v_scale(const uint8_t* vs, const uint16_t* list, int s_begin,
                                          int slot, int n_in, int blk) {
  using C = Cfg<FMT, D>;
  if (slot >= n_in) return __ushort_as_half(0);
  if constexpr (C::kLut) {
    const int tok = list[s_begin + slot];
    return *reinterpret_cast<const __half*>(vs + slot * 8 + 2 * (tok & 1));
  } else {
    return *reinterpret_cast<const __half*>(vs + slot * 8 + 2 * blk);
  }
}

template <int FMT, int D>
__device__ __forceinline__ void v_batch(const uint8_t* __restrict__ vb, const uint8_t* __restrict__ vs,
                                        const __half* __restrict__ pkt,
                                        const uint16_t* __restrict__ list, int s_begin, int n_in,
                                        int warp, int lane, const Lut& lut,
                                        float (&acc)[Cfg<FMT, D>::MT][4]) {
  using C = Cfg<FMT, D>;
  const int r = lane >> 2, c = lane & 3;
  const int dim0 = warp * C::VDW + C::E * r;
  const int boff = C::kQ8 ? dim0 : dim0 / 2;
  const int blk = (warp * C::VDW) / 32;
  const __half* prow = pkt + r * kPktStride + s_begin;
#pragma unroll
  for (int ks = 0; ks < C::VB / 16; ++ks) {
    if (ks * 16 >= n_in) break;
    const int sa = ks * 16 + 2 * c, sc = sa + 8;
    const uint32_t b0 = lds32(prow + sa);
    const uint32_t b1 = lds32(prow + sc);
    const __half2 dab = __halves2half2(v_scale<FMT, D>(vs, list, s_begin, sa, n_in, blk),
                                       v_scale<FMT, D>(vs, list, s_begin, sa + 1, n_in, blk));
    const __half2 dcd = __halves2half2(v_scale<FMT, D>(vs, list, s_begin, sc, n_in, blk),
                                       v_scale<FMT, D>(vs, list, s_begin, sc + 1, n_in, blk));
    uint32_t eab[C::E], ecd[C::E];
    v_dequant_pair<FMT, D>(v_raw<FMT, D>(vb + sa * C::VSTRIDE, boff),
                           v_raw<FMT, D>(vb + (sa + 1) * C::VSTRIDE, boff), lut, eab);
    v_dequant_pair<FMT, D>(v_raw<FMT, D>(vb + sc * C::VSTRIDE, boff),
                           v_raw<FMT, D>(vb + (sc + 1) * C::VSTRIDE, boff), lut, ecd);
#pragma unroll
    for (int e = 0; e < C::E; ++e) {
      eab[e] = h2_as_u32(__hmul2(u32_as_h2(eab[e]), dab));
      ecd[e] = h2_as_u32(__hmul2(u32_as_h2(ecd[e]), dcd));
    }
#pragma unroll
    for (int mt = 0; mt < C::MT; ++mt)
      mma16816(acc[mt], eab[2 * mt], eab[2 * mt + 1], ecd[2 * mt], ecd[2 * mt + 1], b0, b1);
  }
}

// ------------------------------------------------------------------ the kernel
template <int FMT, int D>
__global__ void __launch_bounds__(kThreads, 1)
decode_kernel(const __grid_constant__ CUtensorMap tmap_k, const DecodeArgs a) {
  using C = Cfg<FMT, D>;
  using LY = Layout<FMT, D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* stages = smem + LY::stage;
  float* S = reinterpret_cast<float*>(smem + LY::S);
  __half* pkt = reinterpret_cast<__half*>(smem + LY::pkt);
  uint16_t* list = reinterpret_cast<uint16_t*>(smem + LY::list);
  uint8_t* vbuf = smem + LY::vbuf;
  uint8_t* vsc = smem + LY::vsc;
  float* qs = reinterpret_cast<float*>(smem + LY::q);
  int* item_rows = reinterpret_cast<int*>(smem + LY::rows);
  int* stage_row = reinterpret_cast<int*>(smem + LY::stage_row);
  float* red = reinterpret_cast<float*>(smem + LY::red);
  int* cnt = reinterpret_cast<int*>(smem + LY::cnt);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + LY::bars);
  int* prefix = reinterpret_cast<int*>(smem + LY::prefix);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = lane >> 2, c = lane & 3;
  uint32_t* flags = reinterpret_cast<uint32_t*>(a.workspace);
  const int hkv = a.desc.num_kv_heads, G = a.group, P = a.desc.page_size, Ls = a.split_tokens;
  const int B = a.batch, Hq = a.num_q_heads;

  // ---- work list: splits per sequence, exclusive prefix
  for (int b = tid; b < B; b += kThreads) {
    const int n = a.seq_lens[b];
    const int cap = min(a.max_seq_len, a.max_pages * P);
    if (n < 0 || n > cap) set_flag(flags, KVQ_FLAG_BAD_SEQLEN);
    const int nc = max(0, min(n, cap));
    prefix[b + 1] = (nc + Ls - 1) / Ls;
  }
  if (tid == 0) {
    prefix[0] = 0;
    for (int i = 0; i < C::STAGES; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
    prefetch_tensormap(&tmap_k);
  }
  __syncthreads();
  if (warp == 0) {
    int run = 0;
    for (int base = 1; base <= B; base += 32) {
      const int i = base + lane;
      int v = (i <= B) ? prefix[i] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
      }
      if (i <= B) prefix[i] = v + run;
      run += __shfl_sync(0xffffffffu, v, 31);
    }
  }
  __syncthreads();
  const int total_items = prefix[B] * hkv;
  if ((int)blockIdx.x >= total_items) return;

  // ---- lut4 tables (registers)
  Lut lut;
  if constexpr (C::kLut) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t e = a.desc.codebook[4 * i + j];
        lo |= (e & 0xffu) << (8 * j);
        hi |= (e >> 8) << (8 * j);
      }
      lut.lo[i] = lo; lut.hi[i] = hi;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) lut.lo[i] = lut.hi[i] = 0;
  }

  // ---- producer state (thread 0): next tile to issue
  int p_k = 0, p_t = 0, p_g = 0;
  Item p_item;
  p_item.n_tok = 0;
  const uint8_t* ksc = static_cast<const uint8_t*>(a.k_scales);
  auto producer_fill = [&](int limit) {
    while (p_g < limit) {
      if (p_t * kTile >= p_item.n_tok) {  // advance to the next work unit
        const int it = blockIdx.x + p_k * gridDim.x;
        if (it >= total_items) return;
        p_item = decode_item(a, prefix, it);
        ++p_k;
        p_t = 0;
      }
      const int stage = p_g % C::STAGES;
      uint8_t* dst = stages + (size_t)stage * C::STAGE_BYTES;
      const int tok0 = p_item.t0 + p_t * kTile;
      const int lp = tok0 / P, off = tok0 - lp * P;
      const int page = a.page_table ? a.page_table[(size_t)p_item.b * a.max_pages + lp]
                                    : p_item.b * a.max_pages + lp;
      if (page >= 0 && page < a.desc.num_pages) {
        const int row0 = (page * hkv + p_item.kvh) * P + off;
        mbar_arrive_expect_tx(&bars[stage], C::STAGE_CODE + C::STAGE_SC);
        tma_load_2d(dst, &tmap_k, 0, row0, &bars[stage]);
        bulk_load(dst + C::STAGE_CODE, ksc + (size_t)row0 * C::SROW, C::STAGE_SC, &bars[stage]);
        stage_row[stage] = row0;
      } else {
        set_flag(flags, KVQ_FLAG_BAD_PAGE);
        stage_row[stage] = -1;
        mbar_arrive(&bars[stage]);  // completes the phase with no bytes
      }
      ++p_t;
      ++p_g;
    }
  };
  if (tid == 0) producer_fill(C::STAGES);

  const float qk_scale = a.sm_scale * kLog2e;
  const __half* qg = static_cast<const __half*>(a.q);
  const uint8_t* vcodes = static_cast<const uint8_t*>(a.v_codes);
  const uint8_t* vscales = static_cast<const uint8_t*>(a.v_scales);
  float* ws_o = reinterpret_cast<float*>(static_cast<uint8_t*>(a.workspace) + kWorkspaceHeader);
  const size_t n_part = (size_t)B * Hq * a.max_splits;
  float* ws_m = ws_o + n_part * D;
  float* ws_l = ws_m + n_part;

  int g = 0;  // K tiles consumed by this CTA
  for (int k = 0;; ++k) {
    const int it = blockIdx.x + k * gridDim.x;
    if (it >= total_items) break;
    const Item I = decode_item(a, prefix, it);
    const int ntiles = (I.n_tok + kTile - 1) / kTile;

    // ---- query group -> shared (fp32), rotated for lut4
    for (int i = tid; i < 8 * D; i += kThreads) {
      const int h = i / D, d = i - h * D;
      qs[i] = (h < G) ? __half2float(qg[((size_t)I.b * Hq + I.kvh * G + h) * D + d]) : 0.f;
    }
    __syncthreads();
    if constexpr (C::kLut) {
      // q' = c * H * (s .* q), butterflies in fp32; warp w rotates heads w and w + 4
      constexpr int K = D / 32;
      for (int h = warp; h < 8; h += kWarps) {
        float y[K];
#pragma unroll
        for (int kk = 0; kk < K; ++kk) {
          const int i = 32 * kk + lane;
          y[kk] = qs[h * D + i] * (float)a.desc.signs[i];
        }
#pragma unroll
        for (int hb = 1; hb < 32; hb <<= 1) {
          const bool upper = (lane & hb) != 0;
#pragma unroll
          for (int kk = 0; kk < K; ++kk) {
            const float o = __shfl_xor_sync(0xffffffffu, y[kk], hb);
            y[kk] = upper ? (o - y[kk]) : (y[kk] + o);
          }
        }
#pragma unroll
        for (int kk = 0; kk + 1 < K; kk += 2) {
          const float u = y[kk], v = y[kk + 1];
          y[kk] = u + v; y[kk + 1] = u - v;
        }
        if (K == 4) {
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            const float u = y[kk], v = y[kk + 2];
            y[kk] = u + v; y[kk + 2] = u - v;
          }
        }
        const float cs = rsqrtf((float)D);
#pragma unroll
        for (int kk = 0; kk < K; ++kk) qs[h * D + 32 * kk + lane] = y[kk] * cs;
      }
      __syncthreads();
    }
    uint32_t qf[C::KSTEPS][2], ql[C::KSTEPS][2];
#pragma unroll
    for (int ks = 0; ks < C::KSTEPS; ++ks) {
      int d[4];
      k_dims<FMT>(ks, c, d);
      const float v0 = qs[r * D + d[0]], v1 = qs[r * D + d[1]];
      const float v2 = qs[r * D + d[2]], v3 = qs[r * D + d[3]];
      const __half2 h01 = __floats2half2_rn(v0, v1), h23 = __floats2half2_rn(v2, v3);
      qf[ks][0] = h2_as_u32(h01);
      qf[ks][1] = h2_as_u32(h23);
      if constexpr (C::kLut) {
        ql[ks][0] = pack_h2(v0 - __low2float(h01), v1 - __high2float(h01));
        ql[ks][1] = pack_h2(v2 - __low2float(h23), v3 - __high2float(h23));
      } else {
        ql[ks][0] = ql[ks][1] = 0;
      }
    }

    // ---- K pass
    float mx0 = -INFINITY, mx1 = -INFINITY;
    for (int t = 0; t < ntiles; ++t) {
      const int stage = g % C::STAGES;
      const bool ok = mbar_wait_bounded(&bars[stage], (uint32_t)(g / C::STAGES) & 1u);
      if (ok) {
        const uint8_t* base = stages + (size_t)stage * C::STAGE_BYTES;
        const int row0 = 16 * warp + r;
        float s[4];
        k_tile_scores<FMT, D>(base, base + C::STAGE_CODE, row0, qf, ql, lut, c, s);
        const int p0 = t * kTile + row0, p1 = p0 + 8;
        const bool v0 = p0 < I.n_tok, v1 = p1 < I.n_tok;
        const float s0 = v0 ? s[0] * qk_scale : -INFINITY, s1 = v0 ? s[1] * qk_scale : -INFINITY;
        const float s2 = v1 ? s[2] * qk_scale : -INFINITY, s3 = v1 ? s[3] * qk_scale : -INFINITY;
        *reinterpret_cast<float2*>(S + p0 * 8 + 2 * c) = make_float2(s0, s1);
        *reinterpret_cast<float2*>(S + p1 * 8 + 2 * c) = make_float2(s2, s3);
        mx0 = fmaxf(mx0, fmaxf(s0, s2));
        mx1 = fmaxf(mx1, fmaxf(s1, s3));
      }
      if (tid == 0) item_rows[t] = stage_row[stage];
      if (__syncthreads_or(!ok)) {
        if (tid == 0) set_flag(flags, KVQ_FLAG_TIMEOUT);
        return;
      }
      if (tid == 0) producer_fill(g + 1 + C::STAGES);
      ++g;
    }

    // ---- running maximum of the unit, per head
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    if (r == 0) {
      red[warp * 8 + 2 * c] = mx0;
      red[warp * 8 + 2 * c + 1] = mx1;
    }
    __syncthreads();
    float mh[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      float v = red[h];
#pragma unroll
      for (int w = 1; w < kWarps; ++w) v = fmaxf(v, red[w * 8 + h]);
      mh[h] = v;
    }

    // ---- weights, skip decision, compaction of kept positions
    float lsum[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) lsum[h] = 0.f;
    int nskip = 0, kept_base = 0;
    for (int base = 0; base < I.n_tok; base += kThreads) {
      const int tok = base + tid;
      bool any = false;
      float pk[8];
      if (tok < I.n_tok) {
        const float4 sa = *reinterpret_cast<const float4*>(S + tok * 8);
        const float4 sb = *reinterpret_cast<const float4*>(S + tok * 8 + 4);
        const float sv[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          pk[h] = 0.f;
          if (h < G) {
            const float p = ex2(sv[h] - mh[h]);
            lsum[h] += p;
            const bool keep = p >= a.tau;
            any |= keep;
            nskip += keep ? 0 : 1;
            pk[h] = keep ? p : 0.f;
          }
        }
      }
      const unsigned bal = __ballot_sync(0xffffffffu, any);
      if (lane == 0) cnt[warp] = __popc(bal);
      __syncthreads();
      int wbase = kept_base;
      for (int w = 0; w < warp; ++w) wbase += cnt[w];
      int total = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) total += cnt[w];
      if (any) {
        const int slot = wbase + __popc(bal & ((1u << lane) - 1u));
        list[slot] = (uint16_t)tok;
#pragma unroll
        for (int h = 0; h < 8; ++h) pkt[h * kPktStride + slot] = __float2half_rn(pk[h] * kPScale);
      }
      kept_base += total;
      __syncthreads();
    }
    const int n_kept = kept_base;
    // zero the compacted weights up to the next multiple of 16 (partial MMA k-steps)
    {
      const int pad_end = (n_kept + 15) & ~15;
      for (int i = tid; i < 8 * 16; i += kThreads) {
        const int h = i >> 4, sl = n_kept + (i & 15);
        if (sl < pad_end) pkt[h * kPktStride + sl] = __ushort_as_half(0);
      }
    }
    // denominators
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      float v = lsum[h];
#pragma unroll
      for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      lsum[h] = v;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) nskip += __shfl_xor_sync(0xffffffffu, nskip, o);
    if (lane == 0) {
#pragma unroll
      for (int h = 0; h < 8; ++h) red[64 + warp * 8 + h] = lsum[h];
      cnt[4 + warp] = nskip;
    }
    __syncthreads();

    // ---- V pass over the kept positions only
    float acc[C::MT][4];
#pragma unroll
    for (int mt = 0; mt < C::MT; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
    const int nb = (n_kept + C::VB - 1) / C::VB;
    auto issue_v = [&](int bi) {
      const int buf = bi % C::NVB;
      const int s_begin = bi * C::VB;
      uint8_t* vb = vbuf + (size_t)buf * C::VB * C::VSTRIDE;
      uint8_t* vs = vsc + (size_t)buf * C::VB * 8;
      constexpr int CPR = C::CROW / 16;
      for (int ch = tid; ch < C::VB * CPR; ch += kThreads) {
        const int sl = ch / CPR, cc = ch - sl * CPR;
        const int slot = s_begin + sl;
        if (slot < n_kept) {
          const int tok = list[slot];
          const int rb = item_rows[tok >> 6];
          if (rb >= 0) {
            const size_t row = (size_t)rb + (tok & 63);
            cp_async16(vb + sl * C::VSTRIDE + cc * 16, vcodes + row * C::CROW + cc * 16);
          }
        }
      }
      if (tid < C::VB) {
        const int slot = s_begin + tid;
        if (slot < n_kept) {
          const int tok = list[slot];
          const int rb = item_rows[tok >> 6];
          if (rb >= 0) {
            const size_t row = (size_t)rb + (tok & 63);
            if constexpr (C::kLut) cp_async4(vs + tid * 8, vscales + (row & ~(size_t)1) * 2);
            else if constexpr (C::SROW == 8) cp_async8(vs + tid * 8, vscales + row * 8);
            else cp_async4(vs + tid * 8, vscales + row * 4);
          }
        }
      }
    };
#pragma unroll
    for (int i = 0; i < C::NVB; ++i) {
      if (i < nb) issue_v(i);
      cp_async_commit();
    }
    for (int bi = 0; bi < nb; ++bi) {
      cp_async_wait<C::NVB - 1>();
      __syncthreads();
      const int buf = bi % C::NVB;
      const int s_begin = bi * C::VB;
      v_batch<FMT, D>(vbuf + (size_t)buf * C::VB * C::VSTRIDE, vsc + (size_t)buf * C::VB * 8, pkt,
                      list, s_begin, min(C::VB, n_kept - s_begin), warp, lane, lut, acc);
      __syncthreads();
      if (bi + C::NVB < nb) issue_v(bi + C::NVB);
      cp_async_commit();
    }
    cp_async_wait<0>();

    // ---- unit epilogue: o (unnormalized), m (log2 units), l
    {
      const size_t unit0 = ((size_t)I.b * Hq + (size_t)I.kvh * G) * a.max_splits + I.split;
      const int dim0 = warp * C::VDW + C::E * r;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int h = 2 * c + hh;
        if (h < G) {
          float* dst = ws_o + (unit0 + (size_t)h * a.max_splits) * D + dim0;
          if constexpr (C::E == 4) {
            *reinterpret_cast<float4*>(dst) =
                make_float4(acc[0][hh] * kPUnscale, acc[0][2 + hh] * kPUnscale,
                            acc[1][hh] * kPUnscale, acc[1][2 + hh] * kPUnscale);
          } else {
            *reinterpret_cast<float2*>(dst) =
                make_float2(acc[0][hh] * kPUnscale, acc[0][2 + hh] * kPUnscale);
          }
        }
      }
      if (tid < G) {
        float l = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) l += red[64 + w * 8 + tid];
        float mt = red[tid];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) mt = fmaxf(mt, red[w * 8 + tid]);
        const size_t u = unit0 + (size_t)tid * a.max_splits;
        ws_m[u] = mt;
        ws_l[u] = l;
      }
      if (tid == 0 && a.stats) {
        int ns = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) ns += cnt[4 + w];
        atomicAdd(&a.stats[0], (unsigned long long)I.n_tok * G);
        atomicAdd(&a.stats[1], (unsigned long long)ns);
        atomicAdd(&a.stats[2], (unsigned long long)n_kept);
        atomicAdd(&a.stats[3], (unsigned long long)(I.n_tok - n_kept));
      }
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

template <int FMT, int D>
int launch_decode_t(const DecodeArgs& a, cudaStream_t stream) {
  using C = Cfg<FMT, D>;
  using LY = Layout<FMT, D>;
  auto encode = tensor_map_encoder();
  if (!encode) return KVQ_ERR_CUDA;
  CUtensorMap tmap;
  const uint64_t rows = (uint64_t)a.desc.num_pages * a.desc.num_kv_heads * a.desc.page_size;
  cuuint64_t dims[2] = {(cuuint64_t)C::CROW, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)C::CROW};
  cuuint32_t box[2] = {(cuuint32_t)C::CROW, (cuuint32_t)kTile};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle swz = C::CROW == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                 : C::CROW == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                 : CU_TENSOR_MAP_SWIZZLE_32B;
  if (encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(a.k_codes), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return KVQ_ERR_CUDA;
  auto kern = decode_kernel<FMT, D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)LY::alloc) !=
      cudaSuccess)
    return KVQ_ERR_CUDA;
  // upper bound on work units: every sequence as long as max_seq_len
  const int64_t units = (int64_t)a.batch * a.desc.num_kv_heads * a.max_splits;
  const int grid = (int)std::min<int64_t>(units, a.num_sms);
  if (grid <= 0) return KVQ_OK;
  kern<<<grid, kThreads, LY::alloc, stream>>>(tmap, a);
  return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

}  // namespace

int launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  const int f = a.desc.fmt, d = a.desc.head_dim;
  if (f == KVQ_FMT_Q8_0 && d == 128) return launch_decode_t<KVQ_FMT_Q8_0, 128>(a, stream);
  if (f == KVQ_FMT_Q8_0 && d == 64) return launch_decode_t<KVQ_FMT_Q8_0, 64>(a, stream);
  if (f == KVQ_FMT_Q4_0 && d == 128) return launch_decode_t<KVQ_FMT_Q4_0, 128>(a, stream);
  if (f == KVQ_FMT_Q4_0 && d == 64) return launch_decode_t<KVQ_FMT_Q4_0, 64>(a, stream);
  if (f == KVQ_FMT_LUT4 && d == 128) return launch_decode_t<KVQ_FMT_LUT4, 128>(a, stream);
  if (f == KVQ_FMT_LUT4 && d == 64) return launch_decode_t<KVQ_FMT_LUT4, 64>(a, stream);
  return KVQ_ERR_UNSUPPORTED;
}

}  // namespace kvq
