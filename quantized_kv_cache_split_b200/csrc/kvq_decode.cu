// Split-KV decode attention with sparse V dequantization (sm_100a).
//
// Method (tproger.ru, "Пропуск 90% работы по деквантизации ускорил
// декодирование LLM", section "Решение — не ускорять, а пропускать"): the
// softmax weights come from K before any V work, so V dequantization and
// accumulation are skipped for every position whose weight exp(s - m_running)
// is below tau.  Section "FAQ": K itself is always dequantized.
//
// Work unit: one split (<= 1024 positions = at most 16 tiles of 64) of one
// (sequence, KV head).  A thread-block cluster of CS CTAs (CS = 1, 2 or 4) takes CS
// consecutive splits of the same (sequence, KV head); clusters loop persistently
// over such groups.  Each CTA has 16 warps; warp w owns tile w of its split.
//   Q         Warp 0 builds the query fragments (lut4: rotates the query with
//             butterflies in registers and shuffles) while the K copies are in flight
//             and shares them through shared memory.
//   K fetch   The warp streams its tile's codes and block scales into its private
//             shared buffer with 16-byte cp.async copies, one copy group per 16-row
//             job (an XOR swizzle of the 16-byte chunks keeps the MMA fragment reads
//             free of bank conflicts).  With V fetched early (tau = 0, or when the
//             launch asks: the library's default except for nvfp4, since these steps
//             are bound by latency rather than bytes) it also copies its V tile at
//             once, when shared memory allows.
//   K pass    As each job's copies land, the warp scores its 16 positions x 8 query
//             heads on the tensor cores (mma m16n8k16: positions x heads x head_dim).
//             Codes enter the MMA as magic-number fp16 values (code + a fixed
//             offset); the offset's contribution, a per-(head, block) constant of the
//             query, is preloaded into the accumulator, and the block scale / vector
//             norm is applied to the fp32 score.  Scores stay in registers.
//   max       One CTA barrier gives the split's maximum per head; with the shared
//             maximum option, one cluster barrier and a read of the other CTAs'
//             maxima (distributed shared memory) give the cluster's; with the
//             sequence-wide option, a tagged exchange through the workspace gives the
//             maximum over every split of the (sequence, KV head).
//   weights   Each warp tests its scores: keep iff s - m >= log2(tau) (no exp needed
//             for the test); l sums 2^(s - m) over every position; positions kept by
//             any head of the group are compacted (ballot + popcount) into the warp's
//             own list.  No block-wide step.
//   V pass    Only the kept rows enter the contraction: p^T V on the tensor cores
//             (head_dim x heads x positions), the rows dequantized in registers.
//             Without the early copy the warp gathers just those rows (16-byte
//             cp.async copies of the codes plus a 16-byte window holding the row's
//             scales), so skipped positions cost no HBM read, no dequant and no MMA;
//             with it, the list addresses the kept rows inside the staged tile.  A
//             warp with nothing kept does nothing.
//   output    The warps' accumulators (only those of warps that kept something) are
//             summed through shared memory.  The CTAs of a cluster merge their (o, m,
//             l) through distributed shared memory into one partial per cluster.
//             When an output pointer is given the merge runs in this kernel: if every
//             unit has its own CTA, the splits of a (sequence, KV head) exchange their
//             (m, l) and each adds its normalized share into the output; otherwise
//             the last cluster to finish the pair (an arrival counter in the
//             workspace) merges the written partials by the log-sum-exp rule (lut4:
//             the output is rotated back), so no second kernel runs.
#include <mutex>

#include "kvq_decode_common.cuh"

namespace kvq {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = 32 * kWarps;
constexpr int kLmax = KVQ_MAX_SPLIT_TOKENS;
constexpr int kMaxTiles = kLmax / kTile;
static_assert(kMaxTiles == kWarps, "one K tile per warp per split");
constexpr int kPkStride = kTile + 8;     // halves per head row of a warp's compacted weights
constexpr int kMergeCap = 256;              // partials per (sequence, head) whose weights the merge keeps

template <int FMT, int D>
struct Layout {
  using C = Cfg<FMT, D>;
  static constexpr size_t kbuf = 0;                                            // [warps][KBUF]
  static constexpr size_t pk = kbuf + (size_t)kWarps * C::KBUF;               // half [warps][8][kPkStride]
  static constexpr size_t list = pk + (size_t)kWarps * 8 * kPkStride * 2;     // u8 [warps][64]
  static constexpr size_t red = list + (size_t)kWarps * kTile;                // float [2][warps][8]
  static constexpr size_t cnt = red + 2 * kWarps * 8 * 4;                     // int [2][warps]
  static constexpr size_t cmx = cnt + 2 * kWarps * 4;                         // float [3][8]
  static constexpr size_t mpart = cmx + 24 * 4;                               // float [8]
  static constexpr size_t lpart = mpart + 8 * 4;                              // float [8]
  static constexpr size_t octa = lpart + 8 * 4;                               // float [8][D]
  static constexpr size_t slen = octa + (size_t)8 * D * 4;                    // int [MAX_BATCH]
  static constexpr size_t misc = slen + KVQ_MAX_BATCH * 4;                     // int [4]
  static constexpr size_t mrg = misc + 16;                                     // float [2][8]
  static constexpr size_t scr = mrg + 64;                                      // float4 [warps][4][32] scores
  // query fragments shared by the warps: [words][32 lanes]
  static constexpr int kQfWords = 2 * C::KSTEPS + (C::kLut ? 2 * C::KSTEPS : 0) + 2 * C::NBLK;
  static constexpr size_t qfr = scr + (size_t)kWarps * 4 * 32 * 16;
  static constexpr size_t base_total = qfr + (size_t)kQfWords * 32 * 4;
  // the V tiles copied with K (tau = 0, or when the launch asks) when shared memory allows
  static constexpr size_t vtile = (base_total + 127) / 128 * 128;             // [warps][VT]
  static constexpr bool kPrefetchV = vtile + (size_t)kWarps * C::VT + 128 <= kSmemLimit;
  static constexpr size_t total = kPrefetchV ? vtile + (size_t)kWarps * C::VT : base_total;
  static constexpr size_t alloc = total + 128;  // slack for aligning the base to 128
  static_assert(alloc <= kSmemLimit, "shared memory");
  // cp.async destinations need 16-byte alignment; vector loads need 8 or 16
  static_assert(kbuf % 128 == 0 && C::KBUF % 128 == 0 && vtile % 128 == 0 && C::VT % 128 == 0,
                "staging buffers");
  static_assert(pk % 16 == 0 && red % 16 == 0 && octa % 16 == 0 && slen % 16 == 0 && scr % 16 == 0,
                "alignment");
  // the merges' scratch reuses the staging buffers
  static_assert((size_t)kWarps * C::KBUF >= (size_t)8 * kMergeCap * 4, "merge weights");
};


// ------------------------------------------------------------------ V groups
// Where the V rows of a group sit in the staging buffer: kVGathered: slot s holds the s-th
// kept row (codes) and the 16-byte window of the scales plane holding its scales;
// kVTile: slot s is row s of a staged 64-row tile; kVTileList: a staged tile whose kept
// rows are named by the warp's list (slot s is tile row list[s]; rows are masked into the
// tile, so a stale entry past the kept count still names a row of the tile).
enum VSrc { kVGathered = 0, kVTile = 1, kVTileList = 2 };

template <int SRC>
__device__ __forceinline__ int v_row(const uint8_t* list, int slot) {
  return SRC == kVTileList ? (list[slot] & (kTile - 1)) : slot;
}
// codes swizzled, then the scale rows (one copy group).
template <int FMT, int D>
__device__ __forceinline__ void copy_v_tile(uint8_t* dst, const uint8_t* vcodes, const uint8_t* vscales,
                                            size_t row0, int rows, int lane) {
  using C = Cfg<FMT, D>;
  constexpr int CPR = C::CROW / 16;
  const uint8_t* src = vcodes + row0 * C::CROW;
#pragma unroll 4
  for (int i = lane; i < rows * CPR; i += 32) {
    const int row = i / CPR, cc = i % CPR;
    cp_async16(dst + row * C::CROW + ((cc ^ swz<FMT, D>(row)) << 4), src + (size_t)row * C::CROW + cc * 16);
  }
  const uint8_t* ssrc = vscales + row0 * C::SROW;
  for (int i = lane; i < rows * C::SROW / 16; i += 32) cp_async16(dst + C::STAGE_CODE + i * 16, ssrc + i * 16);
  cp_async_commit();
}

// lut4 / nvfp4: one group of 16 staged V positions (slots s0 .. s0 + 15 of the staging
// buffer, placed as SRC says): acc[dims x heads] += v_hat^T p.  A gathered row's scales
// sit in its window at (trow & (RPW - 1)) * SROW (trow: the row's index in its tile;
// the list entries of the group).  Slots at or past n_valid (counted from s0) get scale
// 0, so whatever bytes they hold contribute nothing (every format decodes any bit pattern
// to a finite value).  Thread (r, c) owns dims E*r .. E*r + E - 1.
template <int FMT, int D, int SRC>
__device__ __forceinline__ void v_group(const uint8_t* __restrict__ buf, const __half* __restrict__ prow,
                                        const uint8_t* __restrict__ trow, int s0, int n_valid,
                                        int r, int c, const Lut& lut,
                                        float (&acc)[Cfg<FMT, D>::MT][4]) {
  using C = Cfg<FMT, D>;
  const int blk = (C::E * r) / 32;
  const int sa = 2 * c, sc = sa + 8;
  const uint32_t b0 = lds32(prow + sa);
  const uint32_t b1 = lds32(prow + sc);
  auto code = [&](int slot) -> const uint8_t* {
    const int row = SRC == kVTileList ? v_row<SRC>(trow, slot) : s0 + slot, o = C::RAWB * r;
    return buf + row * C::CROW + (((o >> 4) ^ swz<FMT, D>(row)) << 4) + (o & 15);
  };
  auto scale = [&](int slot) -> __half {
    if (slot >= n_valid) return __ushort_as_half(0);
    const uint8_t* srow =
        SRC == kVTile       ? buf + C::STAGE_CODE + (s0 + slot) * C::SROW
        : SRC == kVTileList ? buf + C::STAGE_CODE + v_row<SRC>(trow, slot) * C::SROW
                           : buf + C::GSC + (s0 + slot) * 16 + (trow[slot] & (C::RPW - 1)) * C::SROW;
    if constexpr (C::kNv)  // E4M3 block scale of this thread's dims times the vector scale
      return __float2half_rn(e4m3_float(srow[(C::E * r) / 16]) *
                             *reinterpret_cast<const float*>(srow + D / 16));
    return *reinterpret_cast<const __half*>(srow + (C::kLut ? 0 : 2 * blk));
  };
  const __half2 dab = __halves2half2(scale(sa), scale(sa + 1));
  const __half2 dcd = __halves2half2(scale(sc), scale(sc + 1));
  uint32_t wa[C::NWORD], wb[C::NWORD], wc[C::NWORD], wd[C::NWORD];
  v_raw<FMT, D>(code(sa), wa);
  v_raw<FMT, D>(code(sa + 1), wb);
  v_raw<FMT, D>(code(sc), wc);
  v_raw<FMT, D>(code(sc + 1), wd);
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
// q8_0 / q4_0 V pass.  Codes become fp16 by the magic-number bits (fp16 value = code +
// offset, exact) and one fp16 subtraction of the offset (exact: a small integer), read
// with transposing matrix loads so that one register already pairs two positions; the
// scale d of each (position, block) rides on the weights instead of the codes: B = p d'
// per block, with d' = d 2^-k, k >= 0 per block for the whole staged buffer, so that p d'
// (p stored as p 2^14) stays inside fp16; v_mag_finish undoes 2^-k.  The MMA pipe is the
// scarce unit here (mma.sync), so the offset is removed on the ALU rather than by an extra
// MMA.  Thread (r, c) ends up with, per m-tile mt and heads 2c, 2c + 1 (accumulator pairs
// 0, 1 and 2, 3):
//   q4_0: chunk b = block b, m-tile 2b + s: dims 32b + 4r + 2s (low nibble: 1024 + n,
//         minus 1032) and 32b + 4r + 2s + 1 (bits 4..7 in place: 64 + n, minus 72);
//   q8_0: chunk ch = dims 16ch .. 16ch + 15, m-tile ch: dims 16ch + 2r and 16ch + 2r + 1
//         ((byte ^ 0x80) | fp16 1024 = 1152 + code, minus 1152).
template <int FMT, int D>
__device__ __forceinline__ int v_dim(int r, int mt, int i) {
  using C = Cfg<FMT, D>;
  if constexpr (C::kQ4) return 32 * (mt >> 1) + 4 * r + 2 * (mt & 1) + (i >> 1);
  else if constexpr (C::kQ8) return 16 * mt + 2 * r + (i >> 1);
  else return C::E * r + 2 * mt + (i >> 1);
}

// The scale row of staged slot `slot` (a tile's scale rows, or the row's place in its
// gathered 16-byte window).
template <int FMT, int D, int SRC>
__device__ __forceinline__ uint8_t* v_scale_row(uint8_t* buf, const uint8_t* list, int slot) {
  using C = Cfg<FMT, D>;
  if constexpr (SRC == kVGathered) return buf + C::GSC + slot * 16 + (list[slot] & (C::RPW - 1)) * C::SROW;
  return buf + C::STAGE_CODE + v_row<SRC>(list, slot) * C::SROW;
}

// Per block, k = the smallest exponent >= 0 with d 2^-k < 2 for every staged slot
// 0 .. n - 1, and those scales multiplied by 2^-k in place (exact).  Warp-wide.
template <int FMT, int D, int SRC>
__device__ __forceinline__ void v_mag_normalize(uint8_t* buf, const uint8_t* list, int n, int lane,
                                                int (&k)[Cfg<FMT, D>::NBLK]) {
  using C = Cfg<FMT, D>;
  constexpr int NW = C::NBLK / 2;  // 32-bit words (two blocks' scales) per scale row
  uint32_t mx[NW];
#pragma unroll
  for (int w = 0; w < NW; ++w) mx[w] = 0u;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int slot = lane + 32 * h;
    if (slot < n) {
      const uint32_t* sr = reinterpret_cast<const uint32_t*>(v_scale_row<FMT, D, SRC>(buf, list, slot));
#pragma unroll
      for (int w = 0; w < NW; ++w)  // |d| (scales are >= 0 but may be -0)
        mx[w] = h2_as_u32(__hmax2(u32_as_h2(mx[w]), u32_as_h2(sr[w] & 0x7FFF7FFFu)));
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1)
#pragma unroll
    for (int w = 0; w < NW; ++w)
      mx[w] = h2_as_u32(__hmax2(u32_as_h2(mx[w]), u32_as_h2(__shfl_xor_sync(0xffffffffu, mx[w], o))));
  uint32_t f[NW];
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const int e0 = (mx[w] >> 10) & 31, e1 = (mx[w] >> 26) & 31;  // fp16 exponent fields
    k[2 * w] = min(14, max(0, e0 - 15));
    k[2 * w + 1] = min(14, max(0, e1 - 15));
    f[w] = ((uint32_t)(15 - k[2 * w]) << 10) | ((uint32_t)(15 - k[2 * w + 1]) << 26);  // 2^-k
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int slot = lane + 32 * h;
    if (slot < n) {
      uint32_t* sr = reinterpret_cast<uint32_t*>(v_scale_row<FMT, D, SRC>(buf, list, slot));
#pragma unroll
      for (int w = 0; w < NW; ++w) sr[w] = h2_as_u32(__hmul2(u32_as_h2(sr[w]), u32_as_h2(f[w])));
    }
  }
  __syncwarp();
}

// One group of 16 staged positions (slots s0 .. s0 + 15; slots at or past n_valid,
// counted from s0, get weight 0).
template <int FMT, int D, int SRC>
__device__ __forceinline__ void v_group_mag(uint8_t* __restrict__ buf, const __half* __restrict__ prow,
                                            const uint8_t* __restrict__ list, int s0, int n_valid,
                                            int lane, int r, int c, float (&acc)[Cfg<FMT, D>::MT][4]) {
  using C = Cfg<FMT, D>;
  constexpr int NCH = C::CROW / 16;  // 16-byte chunks per row
  constexpr int NW = C::NBLK / 2;
  // weights times scales: slots 2c, 2c + 1 (B rows k = 2c, 2c + 1) and 2c + 8, 2c + 9
  uint32_t ws[4][NW];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int slot = 2 * c + (q & 1) + 8 * (q >> 1);
    const uint32_t* sr = reinterpret_cast<const uint32_t*>(v_scale_row<FMT, D, SRC>(buf, list, s0 + slot));
#pragma unroll
    for (int w = 0; w < NW; ++w) ws[q][w] = slot < n_valid ? sr[w] : 0u;
  }
  const uint32_t p01 = lds32(prow + 2 * c), p89 = lds32(prow + 2 * c + 8);
  uint32_t b0[C::NBLK], b1[C::NBLK];
#pragma unroll
  for (int blk = 0; blk < C::NBLK; ++blk) {
    const uint32_t sel = (blk & 1) ? 0x7632u : 0x5410u;
    b0[blk] = h2_as_u32(__hmul2(u32_as_h2(p01), u32_as_h2(prmt(ws[0][blk >> 1], ws[1][blk >> 1], sel))));
    b1[blk] = h2_as_u32(__hmul2(u32_as_h2(p89), u32_as_h2(prmt(ws[2][blk >> 1], ws[3][blk >> 1], sel))));
  }
  auto sub = [](uint32_t x, uint32_t neg) { return h2_as_u32(__hadd2(u32_as_h2(x), u32_as_h2(neg))); };
  constexpr uint32_t kM1032 = 0xE408E408u, kM72 = 0xD480D480u, kM1152 = 0xE480E480u;  // fp16 pairs
  // codes, two chunks per matrix load: matrix i = (positions s0 + 8 (i & 1) .., chunk
  // cb + (i >> 1)), so R[j][h] = chunk cb + j, positions 2c, 2c + 1 (+ 8 h)
  const int mi = lane >> 3;
  const int row = v_row<SRC>(list, s0 + 8 * (mi & 1) + (lane & 7));
  const uint8_t* rp = buf + row * C::CROW;
  const int sw = swz<FMT, D>(row);
#pragma unroll
  for (int cb = 0; cb < NCH; cb += 2) {
    uint32_t R[2][2];
    ldsm_x4_trans(rp + (((cb + (mi >> 1)) ^ sw) << 4), R[0][0], R[0][1], R[1][0], R[1][1]);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int ch = cb + j;
      if constexpr (C::kQ4) {
        const uint32_t x0 = R[j][0], x1 = R[j][1], y0 = x0 >> 8, y1 = x1 >> 8;
        mma16816(acc[2 * ch], sub((x0 & 0x000F000Fu) | kMagic, kM1032), sub((x0 & 0x00F000F0u) | kMagic64, kM72),
                 sub((x1 & 0x000F000Fu) | kMagic, kM1032), sub((x1 & 0x00F000F0u) | kMagic64, kM72), b0[ch], b1[ch]);
        mma16816(acc[2 * ch + 1], sub((y0 & 0x000F000Fu) | kMagic, kM1032), sub((y0 & 0x00F000F0u) | kMagic64, kM72),
                 sub((y1 & 0x000F000Fu) | kMagic, kM1032), sub((y1 & 0x00F000F0u) | kMagic64, kM72), b0[ch], b1[ch]);
      } else {
        const uint32_t x0 = R[j][0] ^ 0x80808080u, x1 = R[j][1] ^ 0x80808080u;
        mma16816(acc[ch], sub(prmt(x0, 0x64646464u, 0x4240u), kM1152), sub(prmt(x0, 0x64646464u, 0x4341u), kM1152),
                 sub(prmt(x1, 0x64646464u, 0x4240u), kM1152), sub(prmt(x1, 0x64646464u, 0x4341u), kM1152),
                 b0[ch >> 1], b1[ch >> 1]);
      }
    }
  }
}

// acc *= 2^k, per block (undoes the scale normalization).
template <int FMT, int D>
__device__ __forceinline__ void v_mag_finish(float (&acc)[Cfg<FMT, D>::MT][4], const int (&k)[Cfg<FMT, D>::NBLK]) {
  using C = Cfg<FMT, D>;
#pragma unroll
  for (int mt = 0; mt < C::MT; ++mt) {
    const float f = __int_as_float((127 + k[mt >> 1]) << 23);
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[mt][i] *= f;
  }
}

// ------------------------------------------------------------------ unit schedule
// Units after the first round, for batches that fit one warp's ballot: the existing units
// (cu, b, kvh) (cu * span < len_b) whose place in the static list (cu-major, then b, then
// kvh) is `first` or later, in that order; CTA c takes the c-th, (c + ncl)-th, ... of them,
// so every CTA gets the same number of units (the static list, with its holes where
// sequences are shorter, gives some CTAs many more).  The cursor (lvl, base: the ranks
// before level lvl) only moves forward.  Warp-uniform; lens = clamped lengths.
struct UnitCursor {
  int lvl, base;
};

__device__ __forceinline__ bool next_dense_unit(int rank, const int* lens, int B, int hkv, int span,
                                                int levels, int first, int lane, UnitCursor& uc, int& cu,
                                                int& b, int& kvh) {
  const int per = B * hkv;
  const int l0 = first / per, s0 = first % per;  // where the remainder starts
  while (uc.lvl < levels) {
    const unsigned m = __ballot_sync(0xffffffffu, lane < B && lens[lane] > uc.lvl * span);
    unsigned mb = m;   // sequences whose every KV head counts at this level
    int part = 0, bs = 0, ks = 0;
    if (uc.lvl == l0) {  // the first level counts from static place s0 on
      bs = s0 / hkv;
      ks = s0 % hkv;
      part = ((m >> bs) & 1u) ? hkv - ks : 0;
      mb = m & ~((2u << bs) - 1u);
    }
    const int n = part + __popc(mb) * hkv;
    if (rank < uc.base + n) {
      int j = rank - uc.base;
      if (j < part) {
        b = bs;
        kvh = ks + j;
      } else {
        j -= part;
        b = (int)__fns(mb, 0, j / hkv + 1);
        kvh = j % hkv;
      }
      cu = uc.lvl;
      return true;
    }
    if (m == 0u) return false;  // no sequence reaches this level or any later one
    uc.base += n;
    ++uc.lvl;
  }
  return false;
}

// ------------------------------------------------------------------ the kernel
template <int FMT, int D>
__global__ void __launch_bounds__(kThreads, 1)
decode_kernel(const DecodeArgs a) {
  using C = Cfg<FMT, D>;
  using LY = Layout<FMT, D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((128 - (smem_u32(smem_raw) & 127)) & 127);
  float* red_m = reinterpret_cast<float*>(smem + LY::red);
  float* red_l = red_m + kWarps * 8;
  int* cnt_skip = reinterpret_cast<int*>(smem + LY::cnt);
  int* cnt_kept = cnt_skip + kWarps;
  // this CTA's maxima, the sequence's (log2), and this split's share of each head
  float* cmx = reinterpret_cast<float*>(smem + LY::cmx);
  float* mpart = reinterpret_cast<float*>(smem + LY::mpart);   // m of this CTA's partial
  float* lpart = reinterpret_cast<float*>(smem + LY::lpart);   // l of this CTA's partial
  float* octa = reinterpret_cast<float*>(smem + LY::octa);     // o of this CTA's partial [8][D]
  int* slen = reinterpret_cast<int*>(smem + LY::slen);         // clamped sequence lengths
  int* misc = reinterpret_cast<int*>(smem + LY::misc);
  float* mrg_m = reinterpret_cast<float*>(smem + LY::mrg);     // merge: per-head maximum ...
  float* mrg_d = mrg_m + 8;                                    // ... and denominator
  float* mrg_w = reinterpret_cast<float*>(smem + LY::kbuf);    // merge: weights [8][kMergeCap]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = lane >> 2, c = lane & 3;
  uint32_t* flags = reinterpret_cast<uint32_t*>(a.workspace);
  const int hkv = a.desc.num_kv_heads, G = a.group, P = a.desc.page_size, Ls = a.split_tokens;
  const int B = a.batch, Hq = a.num_q_heads, CS = a.cluster;
  const uint32_t rank = CS > 1 ? cluster_rank() : 0u;
  const int cid = CS > 1 ? (int)cluster_index() : (int)blockIdx.x;
  const int ncl = CS > 1 ? (int)cluster_count() : (int)gridDim.x;
  uint8_t* kbuf = smem + LY::kbuf + (size_t)warp * C::KBUF;
  uint8_t* vtile = smem + LY::vtile + (size_t)warp * C::VT;   // used only when kPrefetchV
  __half* pk_w = reinterpret_cast<__half*>(smem + LY::pk) + (size_t)warp * 8 * kPkStride;
  uint8_t* list_w = smem + LY::list + (size_t)warp * kTile;
  // Work units form a static list over (group of CS splits cu, sequence b, KV head),
  // cu-major, as if every sequence were max_seq_len long; a unit past its sequence's
  // end is skipped.  cu-major order puts the units that exist for every sequence first.
  const int NCU = a.units_per_seq;
  const int total = B * NCU * hkv;
  const int cap = min(a.max_seq_len, a.max_pages * P);  // positions that exist in memory

  // compacted weights of pad slots must be finite: start from zeros
  for (int i = lane; i < 8 * kPkStride / 2; i += 32) reinterpret_cast<uint32_t*>(pk_w)[i] = 0u;
  // Programmatic dependent launch: the next kernel on the stream may be scheduled now
  // (it waits for this grid to finish before reading anything), and this one reads no
  // input before the preceding grid has finished and its writes are visible.
  grid_dependents_launch();
  grid_dependency_wait();
  // Every CTA takes part in the launch count that tags the (m, l) exchange.  A CTA with
  // work has its last warp read the counter and the first 32 sequence lengths here, ahead
  // of the first copies (a load issued behind them waits for them), and store what it
  // read behind them.
  unsigned long long ep_raw = 0;
  int len_raw = 0;
  if (cid >= total) {
    if (tid == 0) epoch_advance(a.epoch);  // no work: only the count
  } else if (warp == kWarps - 1) {
    if (lane == 0) ep_raw = epoch_read(a.epoch);
    if (lane < B) len_raw = __ldg(a.seq_lens + lane);
  }

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
  } else if constexpr (C::kNv) {
    // E2M1 code -> fp16: 0, 0.5, 1, 1.5, 2, 3, 4, 6, then the same with the sign bit;
    // every low byte is zero
    const uint32_t hi[4] = {0x3E3C3800u, 0x46444240u, 0xBEBCB880u, 0xC6C4C2C0u};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      lut.lo[i] = 0u;
      lut.hi[i] = hi[i];
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) lut.lo[i] = lut.hi[i] = 0;
  }

  const float qk_scale = a.sm_scale * kLog2e;
  const float thr = a.tau > 0.f ? log2f(a.tau) : -INFINITY;  // keep iff s - m >= log2(tau)
  // V tiles copied with K (tau = 0: every row is kept; otherwise when the launch asks,
  // so that kept rows wait for no second DRAM round trip and skipped rows cost bytes only)
  const bool prefetch_v = LY::kPrefetchV && (!(a.tau > 0.f) || a.v_early);
  const __half* qg = static_cast<const __half*>(a.q);
  const uint8_t* kcodes = static_cast<const uint8_t*>(a.k_codes);
  const uint8_t* kscales = static_cast<const uint8_t*>(a.k_scales);
  const uint8_t* vcodes = static_cast<const uint8_t*>(a.v_codes);
  const uint8_t* vscales = static_cast<const uint8_t*>(a.v_scales);
  const bool hl0 = 2 * c < G, hl1 = 2 * c + 1 < G;  // this lane's two accumulator heads exist
  const uint32_t below = (1u << (4 * r)) - 1u;

  // after the first round, batches of up to 32 sequences take the existing units evenly
  const bool dense = B <= 32 && total > ncl;
  // Positions [seg0, seg0 + seg_len) of each split are this warp's: tile w for warp w.  A
  // split of kWarps - 2 tiles leaves two warps idle; for lut4 and nvfp4 its last two tiles
  // are then halved with them, so that each SM sub-partition (warp w runs on w % 4) holds
  // 3.5 tiles of the K and V passes instead of 4 on two of them and 3 on the others.
  // (Measured: this pays where the V pass dequantizes on the ALU; the q8_0 / q4_0 kernels,
  // whose V codes go to the MMA nearly as loaded, lose more to the extra live registers.)
  constexpr bool kHalfTiles = !C::kMag;
  const bool halves = kHalfTiles && Ls == (kWarps - 2) * kTile;
  int seg0 = warp * kTile, seg_len = kTile;
  if (halves && warp >= kWarps - 4) {
    seg_len = kTile / 2;
    if (warp >= kWarps - 2) seg0 = (warp - 2) * kTile + kTile / 2;
  }
  UnitCursor ucur{ncl / (B * hkv), 0};
#pragma unroll 1
  for (int k = 0;; ++k) {
    // ---- the cluster's (group of splits, sequence, KV head) and this CTA's split
    int kvh, b, cu;
    if (k > 0 && dense) {
      __syncthreads();  // the lengths in shared memory are visible (the first unit may have had no barrier)
      if (!next_dense_unit(cid + (k - 1) * ncl, slen, B, hkv, CS * Ls, NCU, ncl, lane, ucur, cu, b, kvh)) break;
    } else {
      const int it = cid + k * ncl;
      if (it >= total) break;
      kvh = it % hkv;
      const int bu = it / hkv;
      b = bu % B;
      cu = bu / B;
      if (k > 0) __syncthreads();  // as above
    }
    const int t0 = (cu * CS + (int)rank) * Ls;
    // The first unit reads its sequence length from global memory while its K copies
    // are already in flight (they cover what exists in memory, up to cap); later
    // units know the length before copying anything.
    int nb;
    if (k == 0) {
      nb = __ldg(a.seq_lens + b);  // in flight while the copies are issued
    } else {
      nb = slen[b];
      if (cu * CS * Ls >= nb) continue;  // no such unit (uniform over the cluster)
    }
    const int avail = k == 0 ? cap : nb;  // positions the copies may cover

    // ---- warp 0 loads the query words first, ahead of the copies in the load queue
    QRaw<D> qraw;
    if (warp == 0)
      load_query<FMT, D>(r < G ? qg + ((size_t)b * Hq + (size_t)kvh * G + r) * D : nullptr,
                         a.desc.signs, c, qraw);

    // ---- K fetch (and, when V is fetched early, the V tile): one copy group per 16-row job
    int row0 = -1;
    const int ncopy = min(seg_len, avail - t0 - seg0);
    if (ncopy > 0) {
      const int tok0 = t0 + seg0;
      const int lp = tok0 / P, off = tok0 - lp * P;  // tiles never straddle pages (P % 64 == 0)
      const int page = a.page_table ? __ldg(a.page_table + (size_t)b * a.max_pages + lp)
                                    : b * a.max_pages + lp;
      if (page >= 0 && page < a.desc.num_pages) {
        row0 = (page * hkv + kvh) * P + off;
        constexpr int CPR = C::CROW / 16;
        const uint8_t* src = kcodes + (size_t)row0 * C::CROW;
        const uint8_t* ssrc = kscales + (size_t)row0 * C::SROW;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (16 * j < seg_len) {  // a half tile copies two jobs; every warp commits four groups
#pragma unroll
            for (int i = lane; i < 16 * CPR; i += 32) {
              const int row = 16 * j + i / CPR, cc = i % CPR;
              const int sw = cc ^ ((row >> C::SWZ_SHIFT) & C::SWZ_MASK);
              cp_async16(kbuf + row * C::CROW + (sw << 4), src + (size_t)row * C::CROW + cc * 16);
            }
            if (lane < C::SROW)  // 16 rows of scales = SROW 16-byte chunks
              cp_async16(kbuf + C::STAGE_CODE + 16 * j * C::SROW + lane * 16,
                         ssrc + 16 * j * C::SROW + lane * 16);
          }
          cp_async_commit();
        }
        if (prefetch_v) copy_v_tile<FMT, D>(vtile, vcodes, vscales, (size_t)row0, seg_len, lane);
      }
    }
    if (k == 0) {
      nb = max(0, min(nb, cap));
      // this launch's exchange tag, and the clamped sequence lengths for later units and
      // the final zero fill, stored by the last warp (which builds no query fragments)
      // from what it read before the copies; visible after the next barrier
      if (warp == kWarps - 1) {
        if (lane == 0) {
          epoch_advance(a.epoch);
          misc[3] = (int)epoch_tag(ep_raw);  // read after the next barrier
        }
        for (int bb = lane; bb < B; bb += 32) {
          const int n = bb < 32 ? len_raw : a.seq_lens[bb];
          if (n < 0 || n > cap) set_flag(flags, KVQ_FLAG_BAD_SEQLEN);
          slen[bb] = max(0, min(n, cap));
        }
        // Every split adds its share into the output rows of its (sequence, KV head)
        // (single round only).  Split 0 clears them here, long before any share is
        // added, and raises the rows' flag with release semantics; whoever adds waits
        // for the flag with acquire semantics (a wait that is long over by then).
        if (a.out && a.group_merge && cu == 0 && nb > 0) {
          float4* orow = reinterpret_cast<float4*>(a.out + ((size_t)b * Hq + (size_t)kvh * G) * D);
          for (int i = lane; i < G * D / 4; i += 32) orow[i] = make_float4(0.f, 0.f, 0.f, 0.f);
          __syncwarp();
          if (lane == 0) flag_set_release(a.zflag + (size_t)b * hkv + kvh, epoch_tag(ep_raw));
        }
      }
    }
    const bool add_merge = a.out && a.group_merge;
    if (k == 0 && cu * CS * Ls >= nb) {  // a speculative unit past the sequence's end
      cp_async_wait<0>();
      continue;
    }
    const int n_tok = max(0, min(Ls, nb - t0));
    int nvalid = min(seg_len, n_tok - seg0);  // positions of this warp's tile
    if (nvalid > 0 && row0 < 0) {
      if (lane == 0) set_flag(flags, KVQ_FLAG_BAD_PAGE);
      nvalid = 0;
    }

    // ---- query fragments: warp 0 builds them once for the CTA while the copies are
    //      in flight; every warp then reads its lane's words
    uint32_t qf[C::KSTEPS][2], ql[C::KSTEPS][2];
    float corr[C::NBLK][2];
    uint32_t* qfr = reinterpret_cast<uint32_t*>(smem + LY::qfr);
    constexpr int kQl = 2 * C::KSTEPS, kCorr = C::kLut ? 4 * C::KSTEPS : 2 * C::KSTEPS;
    if (warp == 0) {
      build_query<FMT, D>(qraw, c, qf, ql, corr);
#pragma unroll
      for (int ks = 0; ks < C::KSTEPS; ++ks) {
        qfr[(2 * ks) * 32 + lane] = qf[ks][0];
        qfr[(2 * ks + 1) * 32 + lane] = qf[ks][1];
        if constexpr (C::kLut) {
          qfr[(kQl + 2 * ks) * 32 + lane] = ql[ks][0];
          qfr[(kQl + 2 * ks + 1) * 32 + lane] = ql[ks][1];
        }
      }
      if constexpr (!C::kLut) {
#pragma unroll
        for (int m = 0; m < C::NBLK; ++m) {
          qfr[(kCorr + 2 * m) * 32 + lane] = __float_as_uint(corr[m][0]);
          qfr[(kCorr + 2 * m + 1) * 32 + lane] = __float_as_uint(corr[m][1]);
        }
      }
    }
    __syncthreads();
#pragma unroll
    for (int ks = 0; ks < C::KSTEPS; ++ks) {
      qf[ks][0] = qfr[(2 * ks) * 32 + lane];
      qf[ks][1] = qfr[(2 * ks + 1) * 32 + lane];
      ql[ks][0] = C::kLut ? qfr[(kQl + 2 * ks) * 32 + lane] : 0u;
      ql[ks][1] = C::kLut ? qfr[(kQl + 2 * ks + 1) * 32 + lane] : 0u;
    }
#pragma unroll
    for (int m = 0; m < C::NBLK; ++m) {
      corr[m][0] = C::kLut ? 0.f : __uint_as_float(qfr[(kCorr + 2 * m) * 32 + lane]);
      corr[m][1] = C::kLut ? 0.f : __uint_as_float(qfr[(kCorr + 2 * m + 1) * 32 + lane]);
    }

    // ---- K pass: four 16-row jobs as their copies land; scores to this lane's slots,
    //      with the lane's largest and smallest valid score per head
    float4* scw = reinterpret_cast<float4*>(smem + LY::scr) + (size_t)warp * 4 * 32 + lane;
    float mx0 = -INFINITY, mx1 = -INFINITY;
    float mn0 = INFINITY, mn1 = INFINITY;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (16 * j >= nvalid) break;
      cp_async_wait_n(3 - j + (prefetch_v ? 1 : 0));
      __syncwarp();
      float s[4];
      k_job_scores<FMT, D>(kbuf, kbuf + C::STAGE_CODE, 16 * j + r, qf, ql, corr, lut, c, s);
      const bool v0 = 16 * j + r < nvalid, v1 = 16 * j + r + 8 < nvalid;
      const float4 sv = make_float4(v0 ? s[0] * qk_scale : -INFINITY, v0 ? s[1] * qk_scale : -INFINITY,
                                    v1 ? s[2] * qk_scale : -INFINITY, v1 ? s[3] * qk_scale : -INFINITY);
      scw[j * 32] = sv;
      mx0 = fmaxf(mx0, fmaxf(sv.x, sv.z));
      mx1 = fmaxf(mx1, fmaxf(sv.y, sv.w));
      mn0 = fminf(mn0, fminf(v0 ? sv.x : INFINITY, v1 ? sv.z : INFINITY));
      mn1 = fminf(mn1, fminf(v0 ? sv.y : INFINITY, v1 ? sv.w : INFINITY));
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
    __syncthreads();  // every warp's maxima are in shared memory
    if (tid < 8) {
      float m = red_m[tid];
#pragma unroll
      for (int w = 1; w < kWarps; ++w) m = fmaxf(m, red_m[w * 8 + tid]);
      cmx[tid] = m;
      if (tid == 0) {
        misc[0] = misc[1] = 1;  // exchanges not failed (yet)
        misc[2] = 0;            // warps done with their V pass (read after the next barrier)
      }
    }
    if (CS > 1) cluster_sync(); else __syncthreads();  // CTA maxima visible (cluster-wide)
    const size_t slot0 = ((size_t)b * Hq + (size_t)kvh * G) * a.max_splits + cu;  // head 0 of the group
    const uint32_t tag = (uint32_t)misc[3];
    if (a.global_max) {
      // every split publishes its maxima and its denominators relative to them; after one
      // barrier among the splits of this (sequence, KV head) each derives the final
      // maximum M and denominator L of every head (split 0 first clears the output rows
      // that the splits add their shares into)
      const int n = (nb + Ls - 1) / Ls;
      float lo0 = 0.f, lo1 = 0.f;
      const float c0 = cmx[2 * c], c1 = cmx[2 * c + 1];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (16 * j >= nvalid) break;
        const float4 sv = scw[j * 32];  // invalid rows hold -inf
        lo0 += ex2(sv.x - c0) + ex2(sv.z - c0);
        lo1 += ex2(sv.y - c1) + ex2(sv.w - c1);
      }
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        lo0 += __shfl_xor_sync(0xffffffffu, lo0, o);
        lo1 += __shfl_xor_sync(0xffffffffu, lo1, o);
      }
      if (r == 0) {
        red_l[warp * 8 + 2 * c] = lo0;
        red_l[warp * 8 + 2 * c + 1] = lo1;
      }
      __syncthreads();  // every warp's l is in shared memory
      if (tid < G) {
        float l = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) l += red_l[w * 8 + tid];
        xch_store(a.xch + slot0 + (size_t)tid * a.max_splits, tag, cmx[tid], l);
      }
      if (warp < G) {  // M and L of head `warp` over all splits, once every entry is in
        float M, L;
        const bool ok = xch_reduce<4>(a.xch + ((size_t)b * Hq + (size_t)kvh * G + warp) * a.max_splits,
                                      lane, 32, n, true, tag, M, L);
        if (ok) {
          xch_combine(M, L, 16);
          if (lane == 0) {
            cmx[8 + warp] = M;
            cmx[16 + warp] = 1.f / L;  // this split's share: 2^(M - M) / L
          }
        } else if (lane == 0) {
          set_flag(flags, KVQ_FLAG_TIMEOUT);
          misc[0] = misc[1] = 0;
        }
      }
      __syncthreads();
    }
    float mh0 = cmx[2 * c], mh1 = cmx[2 * c + 1];
    if (a.global_max && misc[1]) {
      mh0 = cmx[8 + 2 * c];
      mh1 = cmx[8 + 2 * c + 1];
    }
    if (CS > 1 && a.shared_max) {
      for (int rk = 0; rk < CS; ++rk) {
        if (rk == (int)rank) continue;
        mh0 = fmaxf(mh0, dsmem_ld(dsmem_addr(cmx + 2 * c, rk)));
        mh1 = fmaxf(mh1, dsmem_ld(dsmem_addr(cmx + 2 * c + 1, rk)));
      }
    }
    if (warp == 0 && r == 0) {
      mpart[2 * c] = mh0;
      mpart[2 * c + 1] = mh1;
    }

    // ---- skip test.  When every valid pair of the warp's tile is kept (the smallest
    //      scores pass), the V tile is copied at once and the weights go to row
    //      positions; otherwise kept positions are compacted into this warp's list (rows
    //      r, r + 8 of each job; heads 2c, 2c + 1).  Weights only for kept pairs.
    const bool all_kept = nvalid > 0 &&
                          __all_sync(0xffffffffu, (!hl0 || mn0 - mh0 >= thr) && (!hl1 || mn1 - mh1 >= thr));
    if (all_kept && !prefetch_v) {
      __syncwarp();  // every lane is done reading the K tile
      copy_v_tile<FMT, D>(kbuf, vcodes, vscales, (size_t)row0, seg_len, lane);
    }
    // the weights 2^(s - m) of every valid pair also give the denominator l
    int nkept = 0, nskip = 0;
    float l0 = 0.f, l1 = 0.f;
    if (all_kept) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (16 * j >= nvalid) break;
        const float4 sv = scw[j * 32];
        const int ra = 16 * j + r, rb = ra + 8;
        const bool va = ra < nvalid, vb = rb < nvalid;
        const float ea0 = va && hl0 ? ex2(sv.x - mh0) : 0.f, ea1 = va && hl1 ? ex2(sv.y - mh1) : 0.f;
        const float eb0 = vb && hl0 ? ex2(sv.z - mh0) : 0.f, eb1 = vb && hl1 ? ex2(sv.w - mh1) : 0.f;
        l0 += ea0 + eb0;
        l1 += ea1 + eb1;
        // two weights per conversion (the conversion pipe is the scarce unit here)
        const __half2 pa = __floats2half2_rn(ea0 * kPScale, ea1 * kPScale);
        const __half2 pb = __floats2half2_rn(eb0 * kPScale, eb1 * kPScale);
        pk_w[(2 * c) * kPkStride + ra] = __low2half(pa);
        pk_w[(2 * c + 1) * kPkStride + ra] = __high2half(pa);
        pk_w[(2 * c) * kPkStride + rb] = __low2half(pb);
        pk_w[(2 * c + 1) * kPkStride + rb] = __high2half(pb);
      }
      nkept = nvalid;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (!all_kept && 16 * j < nvalid) {
        const int ra = 16 * j + r, rb = ra + 8;
        const bool va = ra < nvalid, vb = rb < nvalid;
        const bool la0 = va && hl0, la1 = va && hl1, lb0 = vb && hl0, lb1 = vb && hl1;
        const float4 sv = scw[j * 32];
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
        const __half2 pa = __floats2half2_rn(ka0 ? ea0 * kPScale : 0.f, ka1 ? ea1 * kPScale : 0.f);
        const __half2 pb = __floats2half2_rn(kb0 ? eb0 * kPScale : 0.f, kb1 ? eb1 * kPScale : 0.f);
        if ((rows_a >> (4 * r)) & 1u) {
          const int slot = nkept + __popc(rows_a & below);
          if (c == 0) list_w[slot] = (uint8_t)ra;
          pk_w[(2 * c) * kPkStride + slot] = __low2half(pa);
          pk_w[(2 * c + 1) * kPkStride + slot] = __high2half(pa);
        }
        if ((rows_b >> (4 * r)) & 1u) {
          const int slot = nkept + na + __popc(rows_b & below);
          if (c == 0) list_w[slot] = (uint8_t)rb;
          pk_w[(2 * c) * kPkStride + slot] = __low2half(pb);
          pk_w[(2 * c + 1) * kPkStride + slot] = __high2half(pb);
        }
        nkept += na + __popc(rows_b);
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) nskip += __shfl_xor_sync(0xffffffffu, nskip, o);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
    if (r == 0) {
      red_l[warp * 8 + 2 * c] = l0;
      red_l[warp * 8 + 2 * c + 1] = l1;
    }
    if (lane == 0) {
      cnt_skip[warp] = nskip;
      cnt_kept[warp] = nkept;
    }
    __syncwarp();  // the warp's list and weights are complete

    // ---- additive in-kernel merge (every split on its own CTA): the split publishes its
    //      (m, l) and arrives at its (sequence, KV head) barrier now, so that the wait
    //      overlaps its V work; split 0 clears the output rows that the splits add into.
    //      (With the sequence-wide maximum this exchange already happened.)
    const int nsplit = (nb + Ls - 1) / Ls;
    if (add_merge && !a.global_max) {
      __syncthreads();  // every warp's l is in shared memory
      if (tid < G) {
        float l = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) l += red_l[w * 8 + tid];
        xch_store(a.xch + slot0 + (size_t)tid * a.max_splits, tag, mpart[tid], l);
      }
    }

    // ---- V pass: this warp's kept positions only
    if (nkept > 0) {
      float acc[C::MT][4];
#pragma unroll
      for (int mt = 0; mt < C::MT; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
      const int ng = (nkept + 15) >> 4;
      if (nkept == nvalid) {
        // every valid row is kept, so slot s is tile row s; without the prefetched tile,
        // one copy of the V tile into the (now free) K buffer
        uint8_t* vt = prefetch_v ? vtile : kbuf;
        if (!prefetch_v && !all_kept) {
          __syncwarp();  // every lane is done reading the K tile
          copy_v_tile<FMT, D>(kbuf, vcodes, vscales, (size_t)row0, seg_len, lane);
        }
        cp_async_wait<0>();
        __syncwarp();
        if constexpr (C::kMag) {
          int kx[C::NBLK];
          v_mag_normalize<FMT, D, kVTile>(vt, list_w, nkept, lane, kx);
#pragma unroll 2
          for (int g = 0; g < ng; ++g)
            v_group_mag<FMT, D, kVTile>(vt, pk_w + r * kPkStride + 16 * g, list_w, 16 * g,
                                       min(16, nkept - 16 * g), lane, r, c, acc);
          v_mag_finish<FMT, D>(acc, kx);
        } else {
#pragma unroll 2
          for (int g = 0; g < ng; ++g)
            v_group<FMT, D, kVTile>(vt, pk_w + r * kPkStride + 16 * g, nullptr, 16 * g,
                                   min(16, nkept - 16 * g), r, c, lut, acc);
        }
      } else if (prefetch_v) {
        // the tile is staged already: only its kept rows (the list) enter the contraction
        cp_async_wait<0>();
        __syncwarp();
        if constexpr (C::kMag) {
          int kx[C::NBLK];
          v_mag_normalize<FMT, D, kVTileList>(vtile, list_w, nkept, lane, kx);
#pragma unroll 2
          for (int g = 0; g < ng; ++g)
            v_group_mag<FMT, D, kVTileList>(vtile, pk_w + r * kPkStride + 16 * g, list_w, 16 * g,
                                           min(16, nkept - 16 * g), lane, r, c, acc);
          v_mag_finish<FMT, D>(acc, kx);
        } else {
#pragma unroll 2
          for (int g = 0; g < ng; ++g)
            v_group<FMT, D, kVTileList>(vtile, pk_w + r * kPkStride + 16 * g, list_w + 16 * g, 16 * g,
                                       min(16, nkept - 16 * g), r, c, lut, acc);
        }
      } else {
        // gather the kept rows into the (now free) K buffer: slot s gets its codes (chunk
        // swizzle of row s) and the 16-byte window of the scales plane holding its scales
        constexpr int CPR = C::CROW / 16;
        for (int i = lane; i < 16 * ng * (CPR + 1); i += 32) {
          const int sl = i / (CPR + 1), cc = i - sl * (CPR + 1);
          if (sl < nkept) {
            const size_t row = (size_t)row0 + list_w[sl];
            if (cc < CPR)
              cp_async16(kbuf + sl * C::CROW + ((cc ^ swz<FMT, D>(sl)) << 4), vcodes + row * C::CROW + cc * 16);
            else
              cp_async16(kbuf + C::GSC + sl * 16, vscales + (row & ~(size_t)(C::RPW - 1)) * C::SROW);
          }
        }
        cp_async_commit();
        cp_async_wait<0>();
        __syncwarp();
        if constexpr (C::kMag) {
          int kx[C::NBLK];
          v_mag_normalize<FMT, D, kVGathered>(kbuf, list_w, nkept, lane, kx);
#pragma unroll 2
          for (int g = 0; g < ng; ++g)
            v_group_mag<FMT, D, kVGathered>(kbuf, pk_w + r * kPkStride + 16 * g, list_w, 16 * g,
                                           min(16, nkept - 16 * g), lane, r, c, acc);
          v_mag_finish<FMT, D>(acc, kx);
        } else {
#pragma unroll 2
          for (int g = 0; g < ng; ++g)
            v_group<FMT, D, kVGathered>(kbuf, pk_w + r * kPkStride + 16 * g, list_w + 16 * g, 16 * g,
                                       min(16, nkept - 16 * g), r, c, lut, acc);
        }
      }
      __syncwarp();  // staged V fully read before the accumulators overwrite the buffer
      float* accw = reinterpret_cast<float*>(kbuf);
#pragma unroll
      for (int mt = 0; mt < C::MT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) accw[(mt * 4 + i) * 32 + lane] = acc[mt][i];
    }
    if (add_merge) {
      // One warp (the last when it has no tile, so it gets here right after the publish,
      // otherwise the first warp done with its V pass) waits, while the other warps are
      // still accumulating, for split 0's flag that the output rows are cleared (acquire:
      // the shares are added after it) and, without the sequence-wide maximum, for every
      // split of this (sequence, KV head) to publish, and computes this split's share of
      // each head, 2^(m_s - M) / L.
      int first = 0;
      if (!halves && n_tok <= (kWarps - 1) * kTile) {
        first = warp == kWarps - 1;
      } else {
        if (lane == 0) first = atomicAdd(&misc[2], 1) == 0;
        first = __shfl_sync(0xffffffffu, first, 0);
      }
      if (first) {
        // the cleared-rows flag (raised early) first, so that its round trip overlaps
        // the wait for the last split's (m, l) rather than following it
        bool ok = true;
        if (lane == 0) ok = flag_wait_acquire(a.zflag + (size_t)b * hkv + kvh, tag);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (ok && !a.global_max) {
          // lanes 4h .. 4h + 3 take head h, partials j, j + 4, ... (all loads of up to 64
          // partials in flight together), then combine across the four lanes
          const int h = lane >> 2, j = lane & 3;
          float M, L;
          ok = xch_reduce<16>(a.xch + ((size_t)b * Hq + (size_t)kvh * G + (h < G ? h : 0)) * a.max_splits,
                              j, 4, nsplit, h < G, tag, M, L);
          if (ok) {
            xch_combine(M, L, 2);
            if (j == 0 && h < G) cmx[16 + h] = ex2(mpart[h] - M) / L;
          }
        }
        if (lane == 0 && !ok) {
          set_flag(flags, KVQ_FLAG_TIMEOUT);
          misc[0] = 0;
        }
        __syncwarp();
      }
    }
    cp_async_wait<0>();  // nothing of this split stays in flight
    __syncthreads();     // every warp's accumulators, l and counts are in shared memory

    // ---- this CTA's partial: sum the accumulators of the warps that kept something.
    //      A lone CTA writes it straight to the workspace; a cluster merges first.
    //      Four consecutive entries per thread (one 16-byte load per warp), the warps
    //      in index order.
    uint32_t wk = 0;  // warps whose accumulators hold something
#pragma unroll
    for (int w = 0; w < kWarps; ++w) wk |= (cnt_kept[w] > 0 ? 1u : 0u) << w;
    for (int q4 = tid; q4 < 8 * C::NE; q4 += kThreads) {
      float v[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int w = 0; w < kWarps; ++w)
        if ((wk >> w) & 1u) {
          const float4 x = reinterpret_cast<const float4*>(smem + LY::kbuf + (size_t)w * C::KBUF)[q4];
          v[0] += x.x;
          v[1] += x.y;
          v[2] += x.z;
          v[3] += x.w;
        }
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int q = 4 * q4 + t;
        const int ln = q & 31, e = q >> 5;
        const int mt = e >> 2, i = e & 3;
        const int h = 2 * (ln & 3) + (i & 1);
        const int dim = v_dim<FMT, D>(ln >> 2, mt, i);
        if (h < G) {
          const float o = v[t] * kPUnscale;
          if (CS > 1 || add_merge) octa[h * D + dim] = o;
          else a.part_o[(slot0 + (size_t)h * a.max_splits) * D + dim] = o;
        }
      }
    }
    if (tid < G && !add_merge) {
      float l = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) l += red_l[w * 8 + tid];
      if (CS > 1) {
        lpart[tid] = l;
      } else {
        a.part_m[slot0 + (size_t)tid * a.max_splits] = mpart[tid];
        a.part_l[slot0 + (size_t)tid * a.max_splits] = l;
      }
    }
    if (tid == 32 && a.stats && n_tok > 0) {
      int ns = 0, nk = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        ns += cnt_skip[w];
        nk += cnt_kept[w];
      }
      atomicAdd(&a.stats[0], (unsigned long long)n_tok * G);
      atomicAdd(&a.stats[1], (unsigned long long)ns);
      atomicAdd(&a.stats[2], (unsigned long long)nk);
      atomicAdd(&a.stats[3], (unsigned long long)(n_tok - nk));
    }

    if (CS > 1) {
      // one partial per cluster: merge the CTAs' (o, m, l), each CTA a slice of dims
      cluster_sync();  // every CTA's partial is complete
      const int per = (G * D + CS - 1) / CS;
      for (int e = tid; e < per; e += kThreads) {
        const int idx = (int)rank * per + e;
        if (idx < G * D) {
          const int h = idx / D, d = idx - h * D;
          float mr[4], Mc = -INFINITY;
#pragma unroll
          for (int rk = 0; rk < 4; ++rk) {
            mr[rk] = rk < CS ? dsmem_ld(dsmem_addr(mpart + h, rk)) : -INFINITY;
            Mc = fmaxf(Mc, mr[rk]);
          }
          float o = 0.f;
#pragma unroll
          for (int rk = 0; rk < 4; ++rk)
            if (rk < CS && mr[rk] != -INFINITY) o += ex2(mr[rk] - Mc) * dsmem_ld(dsmem_addr(octa + idx, rk));
          a.part_o[(slot0 + (size_t)h * a.max_splits) * D + d] = o;
        }
      }
      if (rank == 0 && tid < G) {
        float mr[4], Mc = -INFINITY;
#pragma unroll
        for (int rk = 0; rk < 4; ++rk) {
          mr[rk] = rk < CS ? dsmem_ld(dsmem_addr(mpart + tid, rk)) : -INFINITY;
          Mc = fmaxf(Mc, mr[rk]);
        }
        float l = 0.f;
#pragma unroll
        for (int rk = 0; rk < 4; ++rk)
          if (rk < CS && mr[rk] != -INFINITY) l += ex2(mr[rk] - Mc) * dsmem_ld(dsmem_addr(lpart + tid, rk));
        a.part_m[slot0 + (size_t)tid * a.max_splits] = Mc;
        a.part_l[slot0 + (size_t)tid * a.max_splits] = l;
      }
      if (a.out) __threadfence();
      cluster_sync();  // no CTA reuses its shared partial before the others have read it
    } else if (a.out) {
      __syncthreads();  // the partial is written (the arrival below publishes it)
    }

    // ---- in-kernel merge.  When every split has its own CTA, each adds its share
    //      o_s 2^(m_s - M) / L (M, L over all splits, read once every split has
    //      published its (m, l)) into the output; otherwise the last cluster to finish
    //      the (sequence, KV head) merges the written partials by the log-sum-exp rule.
    if (add_merge) {
      __syncthreads();  // this CTA's o is in shared memory
      if (misc[0]) {
        if constexpr (C::kLut) {  // rotate the scaled rows back: s .* (c H (coef * o'))
          if (warp < G) {
            constexpr int K = D / 32;
            const float coef = cmx[16 + warp] * (D == 64 ? 0.125f : 0.08838834764831845f);
            float y[K];
#pragma unroll
            for (int kk = 0; kk < K; ++kk) y[kk] = octa[warp * D + 32 * kk + lane] * coef;
#pragma unroll
            for (int hb = 1; hb < 32; hb <<= 1) {
              const bool upper = (lane & hb) != 0;
#pragma unroll
              for (int kk = 0; kk < K; ++kk) {
                const float t = __shfl_xor_sync(0xffffffffu, y[kk], hb);
                y[kk] = upper ? (t - y[kk]) : (y[kk] + t);
              }
            }
#pragma unroll
            for (int hb = 1; hb < K; hb <<= 1)
#pragma unroll
              for (int kk = 0; kk < K; ++kk)
                if (!(kk & hb)) {
                  const float u = y[kk], v = y[kk + hb];
                  y[kk] = u + v;
                  y[kk + hb] = u - v;
                }
#pragma unroll
            for (int kk = 0; kk < K; ++kk)
              octa[warp * D + 32 * kk + lane] = y[kk] * (float)a.desc.signs[32 * kk + lane];
          }
          __syncthreads();
        }
        float* orow = a.out + ((size_t)b * Hq + (size_t)kvh * G) * D;
        for (int q4 = tid; q4 < G * D / 4; q4 += kThreads) {
          const int h = q4 / (D / 4);
          const float coef = C::kLut ? 1.f : cmx[16 + h];
          const float4 v = reinterpret_cast<const float4*>(octa)[q4];
          red_add_f32x4(orow + 4 * q4, make_float4(v.x * coef, v.y * coef, v.z * coef, v.w * coef));
        }
      }
    } else if (a.out && rank == 0) {
      const int ncu = ((nb + Ls - 1) / Ls + CS - 1) / CS;  // partials of sequence b
      if (tid == 0) {
        __threadfence();
        const int old = atomicAdd(&a.counters[(size_t)b * hkv + kvh], 1);
        misc[0] = old == ncu - 1;
      }
      __syncthreads();
      if (misc[0]) {
        __threadfence();
        const size_t u0 = ((size_t)b * Hq + (size_t)kvh * G) * a.max_splits;
        const bool keep_m = ncu <= kMergeCap;
        // Two threads per (head, 4 dims), each taking every other partial; the second
        // half hands its sum over in shared memory.  The partial outputs are requested
        // first so that they are in flight while the maxima are reduced.
        const int nq = G * (D / 4);
        const int half = tid >= nq ? 1 : 0;
        const int qq = tid - half * nq;
        const bool act = tid < 2 * nq;
        const int h = qq / (D / 4), d4 = qq - h * (D / 4);
        const size_t uh = u0 + (size_t)h * a.max_splits;
        constexpr int kBatch = C::kLut ? 12 : 20;  // partials per thread whose loads are in flight together
        float4 o4[kBatch];
#pragma unroll
        for (int t = 0; t < kBatch; ++t) {
          const int u = half + 2 * t;
          o4[t] = act && u < ncu ? __ldcg(reinterpret_cast<const float4*>(a.part_o + (uh + u) * D) + d4)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (warp < G) {  // head `warp`: maximum and denominator, 64 partials per round
          const size_t uw = u0 + (size_t)warp * a.max_splits;
          float M = -INFINITY, den = 0.f;
          for (int ub = 0; ub < ncu; ub += 64) {
            const int ua = ub + lane, uc = ub + 32 + lane;
            const float ma = ua < ncu ? __ldcg(a.part_m + uw + ua) : -INFINITY;
            const float mc = uc < ncu ? __ldcg(a.part_m + uw + uc) : -INFINITY;
            const float la = ua < ncu ? __ldcg(a.part_l + uw + ua) : 0.f;
            const float lc = uc < ncu ? __ldcg(a.part_l + uw + uc) : 0.f;
            if (keep_m) {
              if (ua < ncu) mrg_w[warp * kMergeCap + ua] = ma;
              if (uc < ncu) mrg_w[warp * kMergeCap + uc] = mc;
            }
            float bm = fmaxf(ma, mc);
#pragma unroll
            for (int o = 16; o; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
            const float nm = fmaxf(M, bm);
            float ds = (ma == -INFINITY ? 0.f : ex2(ma - nm) * la) + (mc == -INFINITY ? 0.f : ex2(mc - nm) * lc);
#pragma unroll
            for (int o = 16; o; o >>= 1) ds += __shfl_xor_sync(0xffffffffu, ds, o);
            den = (M == -INFINITY ? 0.f : den * ex2(M - nm)) + ds;
            M = nm;
          }
          if (lane == 0) {
            mrg_m[warp] = M;
            mrg_d[warp] = den;
          }
        }
        __syncthreads();
        float4 acc4 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (act) {
          const float Mh = mrg_m[h];
          auto weight = [&](int u) {
            return ex2((keep_m ? mrg_w[h * kMergeCap + u] : __ldcg(a.part_m + uh + u)) - Mh);
          };
#pragma unroll
          for (int t = 0; t < kBatch; ++t) {
            const int u = half + 2 * t;
            if (u < ncu) {
              const float w = weight(u);
              acc4.x = fmaf(w, o4[t].x, acc4.x);
              acc4.y = fmaf(w, o4[t].y, acc4.y);
              acc4.z = fmaf(w, o4[t].z, acc4.z);
              acc4.w = fmaf(w, o4[t].w, acc4.w);
            }
          }
          for (int u = half + 2 * kBatch; u < ncu; u += 2) {  // more partials than one batch
            const float w = weight(u);
            const float4 v4 = __ldcg(reinterpret_cast<const float4*>(a.part_o + (uh + u) * D) + d4);
            acc4.x = fmaf(w, v4.x, acc4.x);
            acc4.y = fmaf(w, v4.y, acc4.y);
            acc4.z = fmaf(w, v4.z, acc4.z);
            acc4.w = fmaf(w, v4.w, acc4.w);
          }
          if (half) reinterpret_cast<float4*>(octa)[qq] = acc4;
        }
        __syncthreads();
        if (act && !half) {
          const float4 o4 = reinterpret_cast<const float4*>(octa)[qq];
          const float inv = 1.f / mrg_d[h];
          const float4 v = make_float4((acc4.x + o4.x) * inv, (acc4.y + o4.y) * inv,
                                       (acc4.z + o4.z) * inv, (acc4.w + o4.w) * inv);
          if constexpr (C::kLut) reinterpret_cast<float4*>(octa)[qq] = v;
          else reinterpret_cast<float4*>(a.out + ((size_t)b * Hq + (size_t)kvh * G) * D)[qq] = v;
        }
        if constexpr (C::kLut) {
          __syncthreads();
          if (warp < G) {  // out = s .* (c H out'), one warp per head
            constexpr int K = D / 32;
            float y[K];
#pragma unroll
            for (int kk = 0; kk < K; ++kk) y[kk] = octa[warp * D + 32 * kk + lane];
#pragma unroll
            for (int hb = 1; hb < 32; hb <<= 1) {
              const bool upper = (lane & hb) != 0;
#pragma unroll
              for (int kk = 0; kk < K; ++kk) {
                const float t = __shfl_xor_sync(0xffffffffu, y[kk], hb);
                y[kk] = upper ? (t - y[kk]) : (y[kk] + t);
              }
            }
#pragma unroll
            for (int hb = 1; hb < K; hb <<= 1)
#pragma unroll
              for (int kk = 0; kk < K; ++kk)
                if (!(kk & hb)) {
                  const float u = y[kk], v = y[kk + hb];
                  y[kk] = u + v;
                  y[kk + hb] = u - v;
                }
            const float cs = D == 64 ? 0.125f : 0.08838834764831845f;
            float* dst = a.out + ((size_t)b * Hq + (size_t)kvh * G + warp) * D;
#pragma unroll
            for (int kk = 0; kk < K; ++kk)
              dst[32 * kk + lane] = y[kk] * cs * (float)a.desc.signs[32 * kk + lane];
          }
        }
        if (tid == 0) a.counters[(size_t)b * hkv + kvh] = 0;  // ready for the next call
      }
    }
  }

  // sequences with no positions get a zero output (they have no units)
  if (a.out && blockIdx.x == 0) {
    __syncthreads();  // the lengths in shared memory are visible
    for (int b = 0; b < B; ++b)
      if (slen[b] == 0)
        for (int i = tid; i < Hq * D; i += kThreads) a.out[(size_t)b * Hq * D + i] = 0.f;
  }
}

// ------------------------------------------------------------------ host side
std::mutex g_mu;

template <int FMT, int D>
int configure(int dev) {
  using LY = Layout<FMT, D>;
  static uint64_t done_mask = 0;  // guarded by g_mu
  if (!(done_mask >> dev & 1)) {
    auto kern = decode_kernel<FMT, D>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)LY::alloc) !=
        cudaSuccess)
      return KVQ_ERR_CUDA;
    done_mask |= 1ull << dev;
  }
  return KVQ_OK;
}

template <int FMT, int D>
int capacity_t(int cluster) {
  using LY = Layout<FMT, D>;
  static int cache[64][3] = {};  // [device][log2 cluster] = clusters + 1; guarded by g_mu
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  const int ci = cluster == 4 ? 2 : cluster == 2 ? 1 : 0;
  std::lock_guard<std::mutex> lock(g_mu);
  if (cache[dev][ci] == 0) {
    if (configure<FMT, D>(dev) != KVQ_OK) return 0;
    int n = 0;
    if (cluster == 1) {
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_kernel<FMT, D>, kThreads, LY::alloc) !=
          cudaSuccess)
        return 0;
      int sms = 0;
      if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
      n *= sms;
    } else {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = cluster;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(cluster * 64, 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = LY::alloc;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&n, decode_kernel<FMT, D>, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
      }
    }
    cache[dev][ci] = n + 1;
  }
  return cache[dev][ci] - 1;
}

template <int FMT, int D>
int launch_decode_t(const DecodeArgs& a, cudaStream_t stream) {
  using LY = Layout<FMT, D>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return KVQ_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (configure<FMT, D>(dev) != KVQ_OK) return KVQ_ERR_CUDA;
  }
  if (a.grid <= 0) return KVQ_OK;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[3];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = a.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(a.grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = LY::alloc;
  cfg.stream = stream;
  DecodeArgs b = a;
  // every unit with its own CTA (a single round): the in-kernel merge may use a barrier
  // among the CTAs of a (sequence, KV head), so all CTAs must be resident together
  b.group_merge = a.out && a.cluster == 1 && a.max_splits <= kMergeCap &&
                  (int64_t)a.batch * a.units_per_seq * a.desc.num_kv_heads <= a.grid;
  int na = 0;
  if (a.cluster > 1) attr[na++] = attr[0];
  const bool coop = b.group_merge || a.global_max;
  if (coop) {  // CTAs wait for one another: all resident together
    attr[na].id = cudaLaunchAttributeCooperative;
    attr[na].val.cooperative = 1;
    ++na;
  }
  // Programmatic dependent launch: this grid may be set up while the previous kernel on
  // the stream finishes (every CTA waits for that kernel before reading anything, so a
  // cooperative grid still has all its CTAs resident once it proceeds).
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  cfg.attrs = attr;
  cfg.numAttrs = na;
  cudaError_t e = cudaLaunchKernelEx(&cfg, decode_kernel<FMT, D>, b);
  if (e != cudaSuccess && coop) {  // a driver that does not take both: cooperative alone
    (void)cudaGetLastError();
    cfg.numAttrs = na - 1;
    e = cudaLaunchKernelEx(&cfg, decode_kernel<FMT, D>, b);
  }
  if (e != cudaSuccess) return KVQ_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

}  // namespace

namespace {
// The exchange's bounded waits against entries that never become this launch's: the
// (m, l) poll and the cleared-rows flag wait each give up after `limit` cycles and set
// KVQ_FLAG_TIMEOUT, as a decode that lost a split would.  The entries are four exchange
// entries and one flag word in the workspace header's spare bytes (64..143), read only.
__global__ void selftest_wait_kernel(uint8_t* ws, long long limit) {
  uint32_t* flags = reinterpret_cast<uint32_t*>(ws);
  const ulonglong2* e = reinterpret_cast<const ulonglong2*>(ws + 64);
  const unsigned long long* f = reinterpret_cast<const unsigned long long*>(ws + 128);
  const uint32_t never = 0xffffffffu;  // no launch reaches this tag
  float M, L;
  const bool ok1 = xch_reduce<4>(e, threadIdx.x & 31, 32, 4, true, never, M, L, limit);
  bool ok2 = true;
  if ((threadIdx.x & 31) == 0) ok2 = flag_wait_acquire(f, never, limit);
  if ((threadIdx.x & 31) == 0 && (!ok1 || !ok2)) set_flag(flags, KVQ_FLAG_TIMEOUT);
}
}  // namespace

int launch_selftest_wait(void* workspace, long long max_cycles, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(static_cast<uint8_t*>(workspace), max_cycles);
  return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

int launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  const int f = a.desc.fmt, d = a.desc.head_dim;
#define KVQ_CALL_LAUNCH(F, DD) launch_decode_t<F, DD>(a, stream)
  if (f == KVQ_FMT_Q8_0 && d == 128) return KVQ_CALL_LAUNCH(KVQ_FMT_Q8_0, 128);
  if (f == KVQ_FMT_Q8_0 && d == 64) return KVQ_CALL_LAUNCH(KVQ_FMT_Q8_0, 64);
  if (f == KVQ_FMT_Q4_0 && d == 128) return KVQ_CALL_LAUNCH(KVQ_FMT_Q4_0, 128);
  if (f == KVQ_FMT_Q4_0 && d == 64) return KVQ_CALL_LAUNCH(KVQ_FMT_Q4_0, 64);
  if (f == KVQ_FMT_LUT4 && d == 128) return KVQ_CALL_LAUNCH(KVQ_FMT_LUT4, 128);
  if (f == KVQ_FMT_NVFP4 && d == 64) return KVQ_CALL_LAUNCH(KVQ_FMT_NVFP4, 64);
  if (f == KVQ_FMT_NVFP4 && d == 128) return KVQ_CALL_LAUNCH(KVQ_FMT_NVFP4, 128);
  if (f == KVQ_FMT_LUT4 && d == 64) return KVQ_CALL_LAUNCH(KVQ_FMT_LUT4, 64);
#undef KVQ_CALL_LAUNCH
  return KVQ_ERR_UNSUPPORTED;
}

int decode_cluster_capacity(int f, int d, int cluster) {
  if (f == KVQ_FMT_Q8_0 && d == 128) return capacity_t<KVQ_FMT_Q8_0, 128>(cluster);
  if (f == KVQ_FMT_Q8_0 && d == 64) return capacity_t<KVQ_FMT_Q8_0, 64>(cluster);
  if (f == KVQ_FMT_Q4_0 && d == 128) return capacity_t<KVQ_FMT_Q4_0, 128>(cluster);
  if (f == KVQ_FMT_Q4_0 && d == 64) return capacity_t<KVQ_FMT_Q4_0, 64>(cluster);
  if (f == KVQ_FMT_LUT4 && d == 128) return capacity_t<KVQ_FMT_LUT4, 128>(cluster);
  if (f == KVQ_FMT_NVFP4 && d == 64) return capacity_t<KVQ_FMT_NVFP4, 64>(cluster);
  if (f == KVQ_FMT_NVFP4 && d == 128) return capacity_t<KVQ_FMT_NVFP4, 128>(cluster);
  if (f == KVQ_FMT_LUT4 && d == 64) return capacity_t<KVQ_FMT_LUT4, 64>(cluster);
  return 0;
}

}  // namespace kvq
