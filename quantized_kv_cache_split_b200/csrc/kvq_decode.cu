// Split-KV decode attention with sparse V dequantization (sm_100a).
//
// Method (tproger.ru, "Пропуск 90% работы по деквантизации ускорил
// декодирование LLM", section "Решение — не ускорять, а пропускать"): the
// softmax weights come from K before any V work, so V dequantization and
// accumulation are skipped for every position whose weight exp(s - m_running)
// is below tau.  Section "FAQ": K itself is always dequantized.
//
// Persistent CTAs (one per SM, 16 warps) loop over work units (sequence b, KV
// head, split of <= 1024 positions = at most 16 tiles of 64 positions).
//   K fetch   Warp w owns tile w of the unit.  At the start of the unit it streams
//             the tile's codes and block scales into its private shared buffer with
//             16-byte cp.async copies (an XOR swizzle on the codes keeps the MMA
//             fragment reads free of bank conflicts); nothing waits on another warp.
//             (Measured on B200: per-operation costs make 4 KB bulk/TMA copies run at
//             a fraction of what many 16-byte async copies reach.)
//   K pass    Once its copies land, the warp scores its 64 positions x 8 query heads
//             on the tensor cores (mma m16n8k16: positions x heads x head_dim).  Codes
//             enter the MMA as magic-number fp16 values (code + a fixed offset); the
//             offset's contribution, a per-(head, block) constant of the query, is
//             preloaded into the accumulator, and the block scale / vector norm is
//             applied to the fp32 score.
//   weights   After one CTA barrier m_running is the unit's maximum.  Each warp tests
//             its scores: keep iff s - m >= log2(tau) (no exp for the test); the
//             denominator l sums 2^(s - m) over every position; positions kept by any
//             head of the group are compacted (ballot + popcount) into the warp's
//             list, and the lists are concatenated in warp order into one CTA list.
//   V pass    16-row groups of the CTA list are dealt round-robin to the warps.  A warp
//             gathers only those kept V rows (cp.async 16-byte copies into its buffer,
//             three groups in flight), dequantizes them in registers and accumulates
//             p^T V on the tensor cores (head_dim x heads x positions).  Skipped
//             positions cost no HBM read, no dequant, no MMA.
//   output    The warps' accumulators are summed in shared memory; unnormalized o,
//             m (log2 units) and l of the unit go to the workspace and kvq_combine
//             merges the units of a sequence.
#include <mutex>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = 32 * kWarps;
constexpr int kLmax = KVQ_MAX_SPLIT_TOKENS;
constexpr int kMaxTiles = kLmax / kTile;
static_assert(kMaxTiles == kWarps, "one K tile per warp per unit");
constexpr int kWarpSlots = kTile;        // kept-list slots owned by one warp (its tile)
constexpr int kPktStride = kLmax + 8;    // halves per head row of the compacted weights
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
  static constexpr int CROW = kQ8 ? D : D / 2;          // code bytes per row
  static constexpr int NSC = kLut ? 1 : D / 32;          // fp16 per scale row
  static constexpr int SROW = 2 * NSC;                   // scale bytes per row
  static constexpr int RPW = 16 / SROW;                  // rows per 16-byte scale window
  static constexpr int NBLK = D / 32;
  static constexpr int KSTEPS = D / 16;
  static constexpr int STAGE_CODE = kTile * CROW;        // one K tile: codes ...
  static constexpr int STAGE_SC = kTile * SROW;          // ... then scales
  // XOR swizzle of 16-byte chunks within a code row: chunk ^= (row >> SWZ_SHIFT) & SWZ_MASK
  static constexpr int SWZ_SHIFT = CROW == 128 ? 0 : CROW == 64 ? 1 : 2;
  static constexpr int SWZ_MASK = CROW / 16 - 1;
  // V pass: thread (r, c) owns dims E*r .. E*r + E - 1
  static constexpr int E = D / 8;
  static constexpr int MT = D / 16;                      // m-tiles (16 dims each)
  static constexpr int RAWB = kQ8 ? E : E / 2;           // code bytes per position per thread
  static constexpr int NWORD = RAWB / 4;
  static constexpr int VSTRIDE = CROW + 16;              // staged row: codes + scale window
  static constexpr int NVS = 3;                          // V groups of 16 rows in flight per warp
  static constexpr int VGROUP = 16 * VSTRIDE;
  // one buffer per warp: its K tile, then its V groups
  static constexpr int WBUF = ((STAGE_CODE + STAGE_SC > NVS * VGROUP ? STAGE_CODE + STAGE_SC
                                                                      : NVS * VGROUP) + 127) / 128 * 128;
  static_assert(CROW % 16 == 0 && (CROW == 128 || CROW == 64 || CROW == 32), "row size");
};

template <int FMT, int D>
struct Layout {
  using C = Cfg<FMT, D>;
  static constexpr size_t wbuf = 0;                                           // [warps][WBUF]
  // reduction buffer float [8][NE][32]; before the epilogue it holds the per-lane score
  // slots (4 float4 per lane per warp)
  static constexpr size_t ORED = (size_t)8 * (D / 16) * 4 * 32 * 4 > (size_t)kWarps * 4 * 32 * 16
                                     ? (size_t)8 * (D / 16) * 4 * 32 * 4
                                     : (size_t)kWarps * 4 * 32 * 16;
  static constexpr size_t ored = wbuf + (size_t)kWarps * C::WBUF;
  static constexpr size_t pkt = ored + ORED;                                  // half [8][kPktStride]
  static constexpr size_t list = pkt + (size_t)8 * kPktStride * 2;            // u16 [kLmax]
  static constexpr size_t pktg = list + (size_t)kLmax * 2;                    // half [8][kPktStride]
  static constexpr size_t listg = pktg + (size_t)8 * kPktStride * 2;          // u16 [kLmax]
  static constexpr size_t q = listg + (size_t)kLmax * 2;                      // float [8][D]
  static constexpr size_t corr = q + (size_t)8 * D * 4;                       // float [8][NBLK]
  static constexpr size_t rows = corr + (size_t)8 * C::NBLK * 4;              // int [kMaxTiles]
  static constexpr size_t red = rows + kMaxTiles * 4;                         // float [2][warps][8]
  static constexpr size_t cnt = red + 2 * kWarps * 8 * 4;                     // int [2][warps]
  static constexpr size_t prefix = cnt + 2 * kWarps * 4;                      // int [MAX_BATCH + 1]
  static constexpr size_t total = prefix + (KVQ_MAX_BATCH + 1) * 4;
  static constexpr size_t alloc = total + 128;  // slack for aligning the base to 128
  static_assert(alloc <= 232448, "shared memory");
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
  if constexpr (!C::kLut) {
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

// Scale of a staged position (q8_0 / q4_0 block scale of this thread's dims, or the
// lut4 vector norm), read from the row's 16-byte scale window; 0 past the end so
// that stale rows contribute nothing.
template <int FMT, int D>
__device__ __forceinline__ __half v_scale(const uint8_t* grp, int slot, int n_valid, int blk,
                                          const uint16_t* list_grp) {
  using C = Cfg<FMT, D>;
  if (slot >= n_valid) return __ushort_as_half(0);
  const int tok = list_grp[slot];
  const int off = C::CROW + (tok & (C::RPW - 1)) * C::SROW + (C::kLut ? 0 : 2 * blk);
  return *reinterpret_cast<const __half*>(grp + slot * C::VSTRIDE + off);
}

// One group of 16 staged positions: acc[dims x heads] += v_hat^T p.
template <int FMT, int D>
__device__ __forceinline__ void v_group(const uint8_t* __restrict__ grp, const __half* __restrict__ prow,
                                        const uint16_t* __restrict__ list_grp, int n_valid, int r,
                                        int c, const Lut& lut, float (&acc)[Cfg<FMT, D>::MT][4]) {
  using C = Cfg<FMT, D>;
  const int blk = (C::E * r) / 32;
  const int sa = 2 * c, sc = sa + 8;
  const uint32_t b0 = lds32(prow + sa);
  const uint32_t b1 = lds32(prow + sc);
  const __half2 dab = __halves2half2(v_scale<FMT, D>(grp, sa, n_valid, blk, list_grp),
                                     v_scale<FMT, D>(grp, sa + 1, n_valid, blk, list_grp));
  const __half2 dcd = __halves2half2(v_scale<FMT, D>(grp, sc, n_valid, blk, list_grp),
                                     v_scale<FMT, D>(grp, sc + 1, n_valid, blk, list_grp));
  uint32_t wa[C::NWORD], wb[C::NWORD], wc[C::NWORD], wd[C::NWORD];
  const int boff = C::RAWB * r;
  v_raw<FMT, D>(grp + sa * C::VSTRIDE + boff, wa);
  v_raw<FMT, D>(grp + (sa + 1) * C::VSTRIDE + boff, wb);
  v_raw<FMT, D>(grp + sc * C::VSTRIDE + boff, wc);
  v_raw<FMT, D>(grp + (sc + 1) * C::VSTRIDE + boff, wd);
  uint32_t eab[C::E], ecd[C::E];
  v_dequant_pair<FMT, D>(wa, wb, lut, eab);
  v_dequant_pair<FMT, D>(wc, wd, lut, ecd);
#pragma unroll
  for (int e = 0; e < C::E; ++e) {
    eab[e] = h2_as_u32(__hmul2(u32_as_h2(eab[e]), dab));
    ecd[e] = h2_as_u32(__hmul2(u32_as_h2(ecd[e]), dcd));
  }
#pragma unroll
  for (int mt = 0; mt < C::MT; ++mt)
    mma16816(acc[mt], eab[2 * mt], eab[2 * mt + 1], ecd[2 * mt], ecd[2 * mt + 1], b0, b1);
}

// bit 4r set iff any of bits 4r .. 4r+3 of a ballot is set (one row per 4-lane group)
__device__ __forceinline__ uint32_t rows_of(uint32_t bal) {
  uint32_t x = bal | (bal >> 1);
  x |= x >> 2;
  return x & 0x11111111u;
}

// ------------------------------------------------------------------ the kernel
template <int FMT, int D>
__global__ void __launch_bounds__(kThreads, 1)
decode_kernel(const DecodeArgs a) {
  using C = Cfg<FMT, D>;
  using LY = Layout<FMT, D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((128 - (smem_u32(smem_raw) & 127)) & 127);
  float* ored = reinterpret_cast<float*>(smem + LY::ored);
  __half* pkt = reinterpret_cast<__half*>(smem + LY::pkt);
  uint16_t* list = reinterpret_cast<uint16_t*>(smem + LY::list);
  __half* pktg = reinterpret_cast<__half*>(smem + LY::pktg);        // CTA-wide compacted weights
  uint16_t* listg = reinterpret_cast<uint16_t*>(smem + LY::listg);  // CTA-wide kept list
  float* qs = reinterpret_cast<float*>(smem + LY::q);
  float* corr_s = reinterpret_cast<float*>(smem + LY::corr);
  int* item_rows = reinterpret_cast<int*>(smem + LY::rows);
  float* red_m = reinterpret_cast<float*>(smem + LY::red);
  float* red_l = red_m + kWarps * 8;
  int* cnt_skip = reinterpret_cast<int*>(smem + LY::cnt);
  int* cnt_kept = cnt_skip + kWarps;
  int* prefix = reinterpret_cast<int*>(smem + LY::prefix);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = lane >> 2, c = lane & 3;
  uint32_t* flags = reinterpret_cast<uint32_t*>(a.workspace);
  const int hkv = a.desc.num_kv_heads, G = a.group, P = a.desc.page_size, Ls = a.split_tokens;
  const int B = a.batch, Hq = a.num_q_heads;
  uint8_t* my_buf = smem + LY::wbuf + (size_t)warp * C::WBUF;

  // ---- work list: splits per sequence, exclusive prefix
  for (int b = tid; b < B; b += kThreads) {
    const int n = a.seq_lens[b];
    const int cap = min(a.max_seq_len, a.max_pages * P);
    if (n < 0 || n > cap) set_flag(flags, KVQ_FLAG_BAD_SEQLEN);
    const int nc = max(0, min(n, cap));
    prefix[b + 1] = (nc + Ls - 1) / Ls;
  }
  if (tid == 0) prefix[0] = 0;
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

  const float qk_scale = a.sm_scale * kLog2e;
  const float thr = a.tau > 0.f ? log2f(a.tau) : -INFINITY;  // keep iff s - m >= log2(tau)
  const __half* qg = static_cast<const __half*>(a.q);
  const uint8_t* kcodes = static_cast<const uint8_t*>(a.k_codes);
  const uint8_t* kscales = static_cast<const uint8_t*>(a.k_scales);
  const uint8_t* vcodes = static_cast<const uint8_t*>(a.v_codes);
  const uint8_t* vscales = static_cast<const uint8_t*>(a.v_scales);
  float* ws_o = reinterpret_cast<float*>(static_cast<uint8_t*>(a.workspace) + kWorkspaceHeader);
  const size_t n_part = (size_t)B * Hq * a.max_splits;
  float* ws_m = ws_o + n_part * D;
  float* ws_l = ws_m + n_part;
  const int wslot0 = warp * kWarpSlots;  // this warp's region of the kept list / weights
  const bool hl0 = 2 * c < G, hl1 = 2 * c + 1 < G;  // this lane's two heads exist

#pragma unroll 1
  for (int k = 0;; ++k) {
    const int it = blockIdx.x + k * gridDim.x;
    if (it >= total_items) break;
    const Item I = decode_item(a, prefix, it);
    const int ntiles = (I.n_tok + kTile - 1) / kTile;
    const bool has_tile = warp < ntiles;

    // ---- K fetch: this warp's tile (positions 64 w .. 64 w + 63 of the unit)
    if (has_tile) {
      const int tok0 = I.t0 + warp * kTile;
      const int lp = tok0 / P, off = tok0 - lp * P;  // tiles never straddle pages (P % 64 == 0)
      const int page = a.page_table ? a.page_table[(size_t)I.b * a.max_pages + lp]
                                    : I.b * a.max_pages + lp;
      const bool ok = page >= 0 && page < a.desc.num_pages;
      const int row0 = ok ? (page * hkv + I.kvh) * P + off : -1;
      if (lane == 0) {
        item_rows[warp] = row0;
        if (!ok) set_flag(flags, KVQ_FLAG_BAD_PAGE);
      }
      if (ok) {
        constexpr int CPR = C::CROW / 16;
        const uint8_t* src = kcodes + (size_t)row0 * C::CROW;
#pragma unroll
        for (int i = lane; i < kTile * CPR; i += 32) {
          const int row = i / CPR, cc = i - row * CPR;
          const int sc = cc ^ ((row >> C::SWZ_SHIFT) & C::SWZ_MASK);
          cp_async16(my_buf + row * C::CROW + (sc << 4), src + (size_t)i * 16);
        }
        const uint8_t* ssrc = kscales + (size_t)row0 * C::SROW;
#pragma unroll
        for (int i = lane; i < C::STAGE_SC / 16; i += 32)
          cp_async16(my_buf + C::STAGE_CODE + i * 16, ssrc + (size_t)i * 16);
      }
    }
    cp_async_commit();

    // ---- query group -> shared (fp32)
    {
      constexpr int kChunks = 8 * D / 8;  // 16-byte chunks of 8 heads x D fp16
      if (tid < kChunks) {
        const int h = tid / (D / 8), d0 = (tid - h * (D / 8)) * 8;
        uint4 raw = make_uint4(0, 0, 0, 0);
        if (h < G)
          raw = *reinterpret_cast<const uint4*>(qg + ((size_t)I.b * Hq + I.kvh * G + h) * D + d0);
        const __half2* hp = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __half22float2(hp[e]);
          qs[h * D + d0 + 2 * e] = f.x;
          qs[h * D + d0 + 2 * e + 1] = f.y;
        }
      }
    }
    __syncthreads();
    if (warp < 8) {
      const int h = warp;
      constexpr int K = D / 32;
      if constexpr (C::kLut) {
        // q' = c * H * (s .* q), butterflies in fp32; warp h rotates head h
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
      } else {
        // offset contribution per (head, block): sum_d q_d * (offset_d + 8) for q4_0
        // (offset 1024 on even dims, 64 on odd dims), sum_d q_d * 1152 for q8_0
#pragma unroll
        for (int m = 0; m < K; ++m) {
          const int d = 32 * m + lane;
          const float w = C::kQ8 ? 1152.f : ((d & 1) ? 72.f : 1032.f);
          float v = qs[h * D + d] * w;
#pragma unroll
          for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          if (lane == 0) corr_s[h * C::NBLK + m] = v;
        }
      }
    }
    __syncthreads();
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
    float corr[C::NBLK][2];
#pragma unroll
    for (int m = 0; m < C::NBLK; ++m) {
      corr[m][0] = C::kLut ? 0.f : corr_s[(2 * c) * C::NBLK + m];
      corr[m][1] = C::kLut ? 0.f : corr_s[(2 * c + 1) * C::NBLK + m];
    }

    // ---- K pass: the warp's tile, four 16-row jobs; scores to per-lane shared slots
    float4* sbuf = reinterpret_cast<float4*>(ored) + (size_t)warp * 4 * 32 + lane;
    float mx0 = -INFINITY, mx1 = -INFINITY;
    cp_async_wait<0>();
    __syncwarp();
    if (has_tile) {
#pragma unroll 1
      for (int mt = 0; mt < 4; ++mt) {
        const int row0 = 16 * mt + r;
        float s[4];
        k_job_scores<FMT, D>(my_buf, my_buf + C::STAGE_CODE, row0, qf, ql, corr, lut, c, s);
        const int p0 = warp * kTile + row0;
        const bool v0 = p0 < I.n_tok, v1 = p0 + 8 < I.n_tok;
        const float4 sv = make_float4(v0 ? s[0] * qk_scale : -INFINITY, v0 ? s[1] * qk_scale : -INFINITY,
                                      v1 ? s[2] * qk_scale : -INFINITY, v1 ? s[3] * qk_scale : -INFINITY);
        sbuf[mt * 32] = sv;
        mx0 = fmaxf(mx0, fmaxf(sv.x, sv.z));
        mx1 = fmaxf(mx1, fmaxf(sv.y, sv.w));
      }
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    if (r == 0) {
      red_m[warp * 8 + 2 * c] = mx0;
      red_m[warp * 8 + 2 * c + 1] = mx1;
    }
    __syncthreads();  // barrier 1: every warp's maxima are in shared memory

    // ---- weights, skip test, compaction (rows r, r+8 of each job; heads 2c, 2c+1)
    float mh0 = red_m[2 * c], mh1 = red_m[2 * c + 1];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) {
      mh0 = fmaxf(mh0, red_m[w * 8 + 2 * c]);
      mh1 = fmaxf(mh1, red_m[w * 8 + 2 * c + 1]);
    }
    float l0 = 0.f, l1 = 0.f;
    int nkept = 0, nskip = 0;
    const uint32_t below = (1u << (4 * r)) - 1u;
    if (has_tile) {
#pragma unroll 1
      for (int mt = 0; mt < 4; ++mt) {
        const float4 sv = sbuf[mt * 32];
        const int p0 = warp * kTile + 16 * mt + r;
        const bool va = p0 < I.n_tok, vb = p0 + 8 < I.n_tok;
        const bool la0 = va && hl0, la1 = va && hl1, lb0 = vb && hl0, lb1 = vb && hl1;
        const float da0 = sv.x - mh0, da1 = sv.y - mh1;
        const float db0 = sv.z - mh0, db1 = sv.w - mh1;
        const float ea0 = la0 ? ex2(da0) : 0.f, ea1 = la1 ? ex2(da1) : 0.f;
        const float eb0 = lb0 ? ex2(db0) : 0.f, eb1 = lb1 ? ex2(db1) : 0.f;
        l0 += ea0 + eb0;
        l1 += ea1 + eb1;
        const bool ka0 = la0 && da0 >= thr, ka1 = la1 && da1 >= thr;
        const bool kb0 = lb0 && db0 >= thr, kb1 = lb1 && db1 >= thr;
        nskip += (la0 && !ka0) + (la1 && !ka1) + (lb0 && !kb0) + (lb1 && !kb1);
        const uint32_t rows_a = rows_of(__ballot_sync(0xffffffffu, ka0 || ka1));
        const uint32_t rows_b = rows_of(__ballot_sync(0xffffffffu, kb0 || kb1));
        const int na = __popc(rows_a);
        if ((rows_a >> (4 * r)) & 1u) {
          const int slot = wslot0 + nkept + __popc(rows_a & below);
          if (c == 0) list[slot] = (uint16_t)p0;
          pkt[(2 * c) * kPktStride + slot] = __float2half_rn(ka0 ? ea0 * kPScale : 0.f);
          pkt[(2 * c + 1) * kPktStride + slot] = __float2half_rn(ka1 ? ea1 * kPScale : 0.f);
        }
        if ((rows_b >> (4 * r)) & 1u) {
          const int slot = wslot0 + nkept + na + __popc(rows_b & below);
          if (c == 0) list[slot] = (uint16_t)(p0 + 8);
          pkt[(2 * c) * kPktStride + slot] = __float2half_rn(kb0 ? eb0 * kPScale : 0.f);
          pkt[(2 * c + 1) * kPktStride + slot] = __float2half_rn(kb1 ? eb1 * kPScale : 0.f);
        }
        nkept += na + __popc(rows_b);
      }
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) nskip += __shfl_xor_sync(0xffffffffu, nskip, o);
    if (r == 0) {
      red_l[warp * 8 + 2 * c] = l0;
      red_l[warp * 8 + 2 * c + 1] = l1;
    }
    if (lane == 0) {
      cnt_skip[warp] = nskip;
      cnt_kept[warp] = nkept;
    }
    __syncthreads();  // barrier 2: every warp's kept count is known
    // ---- concatenate the warps' lists in warp order (deterministic) into the CTA list
    int gbase = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int n = cnt_kept[w];
      gbase += (w < warp) ? n : 0;
      total += n;
    }
    for (int i = lane; i < nkept; i += 32) {
      listg[gbase + i] = list[wslot0 + i];
#pragma unroll
      for (int h = 0; h < 8; ++h) pktg[h * kPktStride + gbase + i] = pkt[h * kPktStride + wslot0 + i];
    }
    if (warp == kWarps - 1) {  // zero the padding slots of the last partial group
      const int pad = ((total + 15) & ~15) - total;
      for (int i = lane; i < 8 * pad; i += 32)
        pktg[(i / pad) * kPktStride + total + (i % pad)] = __ushort_as_half(0);
    }
    __syncthreads();  // barrier 3: the CTA list is complete

    // ---- V pass: kept positions only, 16-row groups dealt round-robin to the warps
    float acc[C::MT][4];
#pragma unroll
    for (int mt = 0; mt < C::MT; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
    const int ngroups_all = (total + 15) >> 4;
    const int ngroups = ngroups_all > warp ? (ngroups_all - warp + kWarps - 1) / kWarps : 0;
    auto issue = [&](int gi) {  // this warp's gi-th group = CTA group warp + 16 gi
      uint8_t* grp = my_buf + (size_t)(gi % C::NVS) * C::VGROUP;
      const int s0 = 16 * (warp + kWarps * gi);
      constexpr int CPR = C::CROW / 16 + 1;  // code chunks + the scale window
#pragma unroll
      for (int i = lane; i < 16 * CPR; i += 32) {
        const int rl = i / CPR, cc = i - rl * CPR;
        const int slot = s0 + rl;
        if (slot < total) {
          const int tok = listg[slot];
          const int rb = item_rows[tok >> 6];
          if (rb >= 0) {
            const size_t row = (size_t)rb + (tok & 63);
            const uint8_t* src = cc < CPR - 1 ? vcodes + row * C::CROW + cc * 16
                                              : vscales + (row & ~(size_t)(C::RPW - 1)) * C::SROW;
            cp_async16(grp + rl * C::VSTRIDE + cc * 16, src);
          }
        }
      }
      cp_async_commit();
    };
#pragma unroll
    for (int i = 0; i < C::NVS; ++i) {
      if (i < ngroups) issue(i);
      else cp_async_commit();
    }
#pragma unroll 1
    for (int gi = 0; gi < ngroups; ++gi) {
      cp_async_wait<C::NVS - 1>();
      __syncwarp();
      const int s0 = 16 * (warp + kWarps * gi);
      v_group<FMT, D>(my_buf + (size_t)(gi % C::NVS) * C::VGROUP, pktg + r * kPktStride + s0,
                      listg + s0, min(16, total - s0), r, c, lut, acc);
      __syncwarp();
      if (gi + C::NVS < ngroups) issue(gi + C::NVS);
      else cp_async_commit();
    }
    cp_async_wait<0>();

    // ---- sum the warps' accumulators and write the unit
    constexpr int NE = C::MT * 4;  // accumulator registers per thread
    __syncthreads();  // barrier 4: every warp's V accumulation is done; score slots free
    if (warp >= 8) {
#pragma unroll
      for (int mt = 0; mt < C::MT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) ored[((warp - 8) * NE + mt * 4 + i) * 32 + lane] = acc[mt][i];
    }
    __syncthreads();  // barrier 5
    if (warp < 8) {
#pragma unroll
      for (int mt = 0; mt < C::MT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float* p = ored + (warp * NE + mt * 4 + i) * 32 + lane;
          *p = *p + acc[mt][i];
        }
    }
    __syncthreads();  // barrier 6
    {
      const size_t unit0 = ((size_t)I.b * Hq + (size_t)I.kvh * G) * a.max_splits + I.split;
      for (int q = tid; q < 32 * NE; q += kThreads) {
        const int ln = q & 31, e = q >> 5;
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) v += ored[(w * NE + e) * 32 + ln];
        const int mt = e >> 2, i = e & 3;
        const int rr = ln >> 2, cc = ln & 3;
        const int h = 2 * cc + (i & 1);
        const int dim = C::E * rr + 2 * mt + (i >> 1);
        if (h < G) ws_o[(unit0 + (size_t)h * a.max_splits) * D + dim] = v * kPUnscale;
      }
      if (tid < G) {
        float m = red_m[tid], l = red_l[tid];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) {
          m = fmaxf(m, red_m[w * 8 + tid]);
          l += red_l[w * 8 + tid];
        }
        const size_t u = unit0 + (size_t)tid * a.max_splits;
        ws_m[u] = m;
        ws_l[u] = l;
      }
      if (tid == 0 && a.stats) {
        int ns = 0, nk = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
          ns += cnt_skip[w];
          nk += cnt_kept[w];
        }
        atomicAdd(&a.stats[0], (unsigned long long)I.n_tok * G);
        atomicAdd(&a.stats[1], (unsigned long long)ns);
        atomicAdd(&a.stats[2], (unsigned long long)nk);
        atomicAdd(&a.stats[3], (unsigned long long)(I.n_tok - nk));
      }
    }
    __syncthreads();  // barrier 7: shared buffers free for the next unit
  }
}

// ------------------------------------------------------------------ host side
template <int FMT, int D>
int launch_decode_t(const DecodeArgs& a, cudaStream_t stream) {
  using LY = Layout<FMT, D>;
  auto kern = decode_kernel<FMT, D>;
  // The shared-memory opt-in is set once per device (so that later calls, including
  // ones made while a stream is being captured into a graph, issue no attribute call).
  static std::mutex mu;
  static uint64_t done_mask = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return KVQ_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!(done_mask >> dev & 1)) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)LY::alloc) != cudaSuccess)
        return KVQ_ERR_CUDA;
      done_mask |= 1ull << dev;
    }
  }
  // upper bound on work units: every sequence as long as max_seq_len
  const int64_t units = (int64_t)a.batch * a.desc.num_kv_heads * a.max_splits;
  const int grid = (int)std::min<int64_t>(units, a.num_sms);
  if (grid <= 0) return KVQ_OK;
  kern<<<grid, kThreads, LY::alloc, stream>>>(a);
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
