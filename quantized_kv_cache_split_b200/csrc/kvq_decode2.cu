// Split-KV decode attention with sparse V dequantization (sm_100a): the streaming kernel.
//
// Method (tproger.ru, "Пропуск 90% работы по деквантизации ускорил
// декодирование LLM", section "Решение — не ускорять, а пропускать"): the softmax
// weights come from K before any V work, so V dequantization and accumulation are
// skipped for every position whose weight exp(s - m_running) is below tau; section
// "FAQ": K itself is always dequantized.
//
// Work unit: one split (<= 1024 positions = 16 tiles of 64) of one (sequence, KV head).
// A CTA has one warp per tile of a split (4, 8 or 16 warps, so 4, 2 or 1 CTAs per SM);
// when there are more units than CTAs, the CTAs loop over the units.  Per unit:
//   copies    Lane 0 of warp w issues K tile w as one tensor copy (TMA, swizzled so that
//             the fragment loads are free of bank conflicts) and its scale rows as one
//             bulk copy, both completing on the warp's mbarrier.  V tiles copied whole go
//             into their own region when shared memory allows: right behind the K copy,
//             or, when every split has its own CTA and the split is long, after the K
//             pass, so that the launch's K copies have the memory system to themselves;
//             else into the K tile's place once its scores are taken.
//   query     Warp 0 builds the query fragments (lut4: the rotated query) for the CTA.
//   K pass    Each warp scores its tile on the tensor cores (mma.sync m16n8k16,
//             positions x heads x head_dim) once its copy lands, keeps the scores in
//             its shared-memory scratch, and folds them into its (max, denominator).
//   maximum   One CTA barrier; every warp reads the split's maximum per head (with the
//             cluster option, the maximum over a thread-block cluster of splits, through
//             distributed shared memory; with the sequence-wide option, the splits of the
//             (sequence, KV head) first exchange their (m, l) through tagged words).
//   weights   Each warp turns its scores into weights p = 2^(s - m), keeps a pair iff
//             s - m >= log2(tau), and turns the kept weights (fp16) into the B fragments
//             of its V pass (movmatrix); a 16-row group with no kept pair is skipped.
//   V pass    The tile's warp: per kept group, ldmatrix.trans of the V codes (magic-number
//             fp16 for q8_0 / q4_0, centroid or E2M1 lookups for lut4 / nvfp4) times the
//             group's weights on the tensor cores; skipped rows inside a kept group
//             contribute zero.  With V fetched after the test, the kept rows alone are
//             gathered first.
//   merge     When every unit has its own CTA, a poll warp publishes the split's (m, l)
//             right after the maximum and collects every split's during the V pass; the
//             CTA adds its normalized share into the output with vector atomics (lut4:
//             rotated back first) once split 0 has cleared the output rows.  Otherwise the
//             CTA writes its partial (o, m, l) and the combine kernel merges them.
// Every wait (mbarriers, exchange, flags) is bounded and reports KVQ_FLAG_TIMEOUT.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cfloat>
#include <mutex>

#include "kvq_decode2.h"
#include "kvq_decode_common.cuh"

namespace kvq {
namespace {

// NW warps per CTA (16, 8 or 4): warp w owns tile w of the unit, so a unit holds at most
// NW tiles, and 16 / NW CTAs share an SM (the register file holds 16 warps of 128).
constexpr int kMaxNW = 16;
constexpr int kPollSleepNs = 32;     // back-off between polls of the exchange
static_assert(kMaxNW * kTile == KVQ_MAX_SPLIT_TOKENS, "one tile per warp per split");

// ------------------------------------------------------------------ mbarriers, bulk copies
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
// True once the phase with the given parity has completed; a thread whose phase is not complete yet may be suspended (it takes no
// issue slots) until the phase completes or about `ns` nanoseconds have passed.
__device__ __forceinline__ bool mbar_try_suspend(uint64_t* bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}
constexpr uint32_t kSuspendNs = 1000000;  // one suspension at most (the loop bounds the wait)
// Wait for the phase with the given parity to complete; false after ~kWaitCycles.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_suspend(bar, parity, kSuspendNs)) return true;
  const long long t0 = clock64();
  while (!mbar_try_suspend(bar, parity, kSuspendNs))
    if (clock64() - t0 > kWaitCycles) return false;
  return true;
}

// Rows y .. y + 63 of a 2-D tensor map (x = 0) into shared memory (swizzled as the map says).
__device__ __forceinline__ void tma_rows(void* dst, const CUtensorMap* map, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
// A contiguous range (16-byte aligned, a multiple of 16 bytes) into shared memory.
__device__ __forceinline__ void bulk_copy(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// Generic-proxy accesses of shared memory before this point are ordered before later
// async-proxy (bulk copy) writes to it.
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ V groups
// The V pass of a warp covers its own tile, all of the head dimension, one group of 16
// staged rows (s0 .. s0 + 15, the first n_valid of them inside the sequence) at a time:
// acc[mt] (m16n8 tiles, rows = dims, cols = heads) += v_hat^T p.  The weights enter as
// B fragments kept in registers: p01 = (p of rows s0 + 2c, s0 + 2c + 1) and p89 = (rows
// s0 + 2c + 8, s0 + 2c + 9) for head r, as fp16 x 2^14, zero for skipped pairs.  Rows past
// n_valid get scale 0, so whatever bytes their slots hold contribute nothing (every
// format decodes any bit pattern to a finite value).  Output dim of tile mt, row r (row
// r + 8: that + 1):
//   q4_0: 32 (mt >> 1) + 4 r + 2 (mt & 1)     q8_0: 16 mt + 2 r     lut4 / nvfp4: E r + 2 mt
template <int FMT, int D>
__device__ __forceinline__ int out_dim(int r, int mt, int i) {
  using C = Cfg<FMT, D>;
  if constexpr (C::kQ4) return 32 * (mt >> 1) + 4 * r + 2 * (mt & 1) + (i >> 1);
  else if constexpr (C::kQ8) return 16 * mt + 2 * r + (i >> 1);
  else return C::E * r + 2 * mt + (i >> 1);
}

// q8_0 / q4_0: codes enter the MMA as magic-number fp16 with the offset removed by one
// exact fp16 subtraction; the block scale rides on the weights, B = p d' per block, with
// d' = d 2^-k[blk] (k >= 0 per block and tile, so that p 2^14 d' stays inside fp16; the
// tile's scale rows are rescaled in place by tile_mag_normalize and acc by mag_finish).
template <int FMT, int D>
__device__ __forceinline__ void vg_mag(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                                       int s0, int n_valid, uint32_t p01, uint32_t p89, int lane,
                                       float (&acc)[Cfg<FMT, D>::MT][4]) {
  using C = Cfg<FMT, D>;
  constexpr int NCH = C::CROW / 16;  // 16-byte chunks per row
  constexpr int NW = C::NBLK / 2;    // 32-bit scale words (two blocks each) per row
  const int c = lane & 3;
  uint32_t ws[4][NW];  // scale words of rows s0 + {2c, 2c + 1, 2c + 8, 2c + 9}
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int slot = 2 * c + (q & 1) + 8 * (q >> 1);
    const uint32_t* sr = reinterpret_cast<const uint32_t*>(scales + (s0 + slot) * C::SROW);
#pragma unroll
    for (int w = 0; w < NW; ++w) ws[q][w] = slot < n_valid ? sr[w] : 0u;
  }
  uint32_t b0[C::NBLK], b1[C::NBLK];
#pragma unroll
  for (int blk = 0; blk < C::NBLK; ++blk) {
    const uint32_t sel = (blk & 1) ? 0x7632u : 0x5410u;
    b0[blk] = h2_as_u32(__hmul2(u32_as_h2(p01), u32_as_h2(prmt(ws[0][blk >> 1], ws[1][blk >> 1], sel))));
    b1[blk] = h2_as_u32(__hmul2(u32_as_h2(p89), u32_as_h2(prmt(ws[2][blk >> 1], ws[3][blk >> 1], sel))));
  }
  auto sub = [](uint32_t x, uint32_t neg) { return h2_as_u32(__hadd2(u32_as_h2(x), u32_as_h2(neg))); };
  constexpr uint32_t kM1032 = 0xE408E408u, kM72 = 0xD480D480u, kM1152 = 0xE480E480u;  // fp16 pairs
  // two chunks per matrix load: matrix i = (rows s0 + 8 (i & 1) .., chunk cb + (i >> 1)),
  // so R[j][h] = chunk cb + j, rows 2c, 2c + 1 (+ 8 h)
  const int mi = lane >> 3;
  const int row = s0 + 8 * (mi & 1) + (lane & 7);
  const uint8_t* rp = codes + row * C::CROW;
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

// Per block, k = the smallest exponent >= 0 with d 2^-k < 2 over the tile's first n rows,
// and those scale rows multiplied by 2^-k in place (exact).  Warp-wide; every row is one
// lane's (rows lane and lane + 32).
template <int FMT, int D>
__device__ __forceinline__ void tile_mag_normalize(uint8_t* scales, int n, int lane, int (&k)[Cfg<FMT, D>::NBLK]) {
  using C = Cfg<FMT, D>;
  constexpr int NW = C::NBLK / 2;
  uint32_t mx[NW];
#pragma unroll
  for (int w = 0; w < NW; ++w) mx[w] = 0u;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int row = lane + 32 * h;
    if (row < n) {
      const uint32_t* sr = reinterpret_cast<const uint32_t*>(scales + row * C::SROW);
#pragma unroll
      for (int w = 0; w < NW; ++w)  // |d| (scales are >= 0 but may be -0)
        mx[w] = h2_as_u32(__hmax2(u32_as_h2(mx[w]), u32_as_h2(sr[w] & 0x7FFF7FFFu)));
    }
  }
#pragma unroll
  for (int b = 0; b < C::NBLK; ++b) k[b] = 0;
  // typical data: every |d| < 2 (fp16 exponent field < 16), nothing to rescale
  bool big = false;
#pragma unroll
  for (int w = 0; w < NW; ++w) big |= (mx[w] & 0x7C00u) >= 0x4000u || (mx[w] & 0x7C000000u) >= 0x40000000u;
  if (!__any_sync(0xffffffffu, big)) return;
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
    const int row = lane + 32 * h;
    if (row < n) {
      uint32_t* sr = reinterpret_cast<uint32_t*>(scales + row * C::SROW);
#pragma unroll
      for (int w = 0; w < NW; ++w) sr[w] = h2_as_u32(__hmul2(u32_as_h2(sr[w]), u32_as_h2(f[w])));
    }
  }
  __syncwarp();
}

// lut4 / nvfp4: thread (r, c) dequantizes dims E r .. E r + E - 1 of rows 2c, 2c + 1 and
// 2c + 8, 2c + 9 into fp16 pairs (centroid / E2M1 lookups) times the rows' scales; B = p.
template <int FMT, int D>
__device__ __forceinline__ void vg_lut(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                                       int s0, int n_valid, uint32_t p01, uint32_t p89, int lane, const Lut& lut,
                                       float (&acc)[Cfg<FMT, D>::MT][4]) {
  using C = Cfg<FMT, D>;
  const int r = lane >> 2, c = lane & 3;
  const int sa = 2 * c, sc = sa + 8;
  auto code = [&](int slot) -> const uint8_t* {
    const int row = s0 + slot, o = C::RAWB * r;
    return codes + row * C::CROW + (((o >> 4) ^ swz<FMT, D>(row)) << 4) + (o & 15);
  };
  auto scale = [&](int slot) -> __half {
    if (slot >= n_valid) return __ushort_as_half(0);
    const uint8_t* srow = scales + (s0 + slot) * C::SROW;
    if constexpr (C::kNv)  // E4M3 block scale of this thread's dims times the vector scale
      return __float2half_rn(e4m3_float(srow[(C::E * r) / 16]) * *reinterpret_cast<const float*>(srow + D / 16));
    return *reinterpret_cast<const __half*>(srow);
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
    mma16816(acc[mt], eab[2 * mt], eab[2 * mt + 1], ecd[2 * mt], ecd[2 * mt + 1], p01, p89);
}

// An 8x8 matrix of 16-bit elements held one row pair per lane (lane (r, c): row r,
// columns 2c, 2c + 1), transposed: lane (r, c) gets row 2c and 2c + 1 of column r.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// ------------------------------------------------------------------ exchange publication
// The split's (m, l) of every head (lane h holds head h) stored by lane 0, then its
// arrival on the (sequence, KV head)'s arrival word; returns (in lane 0) the count that
// word reaches once every split of the (sequence, KV head) has arrived.  Warp-uniform.
__device__ __forceinline__ unsigned long long publish_split(const DecodeArgs& a, size_t slot0, uint32_t tag,
                                                            float m, float l, int G, int lane, int pair,
                                                            bool first, int nsplit) {
  float mv[8], lv[8];
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    mv[h] = __shfl_sync(0xffffffffu, m, h);
    lv[h] = __shfl_sync(0xffffffffu, l, h);
  }
  unsigned long long target = 0;
  if (lane == 0) {
#pragma unroll
    for (int h = 0; h < 8; ++h)
      if (h < G) xch_store(a.xch + slot0 + (size_t)h * a.max_splits, tag, mv[h], lv[h]);
    target = arrive_add(a.arrive + pair, first, nsplit);
  }
  return target;
}
// Before polling the exchange words: lane 0 waits (briefly bounded) until every split of
// the (sequence, KV head) has arrived, so that the poll reads the entries about once instead
// of hammering them; the poll still checks every entry's tag and keeps the full bound.
constexpr long long kArriveWaitCycles = 1ll << 15;
__device__ __forceinline__ void arrivals_await(const DecodeArgs& a, int pair, unsigned long long target, int lane) {
  if (lane == 0) (void)arrivals_wait(a.arrive + pair, target, kArriveWaitCycles, kPollSleepNs);
  __syncwarp();
}

// ------------------------------------------------------------------ the kernel
template <int FMT, int D, int NW>
__global__ void __launch_bounds__(32 * NW, 16 / NW)
decode2_kernel(const __grid_constant__ Decode2Params pr, const __grid_constant__ CUtensorMap tmk,
               const __grid_constant__ CUtensorMap tmv) {
  using C = Cfg<FMT, D>;
  constexpr int kNW = NW;
  constexpr int kNT = 32 * NW;
  constexpr int kPollWarp = NW - 1;  // collects the exchange during the V pass
  const DecodeArgs& a = pr.a;
  constexpr int CODE = kTile * C::CROW; // code bytes of one staged tile
  constexpr int SC = kTile * C::SROW;   // scale bytes of one staged tile
  constexpr int kQfWords = 2 * C::KSTEPS + (C::kLut ? 2 * C::KSTEPS : 0) + 2 * C::NBLK;

  extern __shared__ __align__(1024) uint8_t smem2_raw[];
  __shared__ __align__(8) uint64_t kbar[kNW], vbar[kNW];
  __shared__ float red_m[kNW][8], red_l[kNW][8];
  __shared__ int cnt_skip[kNW], cnt_keep[kNW];
  __shared__ float mh_s[8], mc_s[8], share_s[8];  // split maximum, the one the skip test uses
  __shared__ float ls_s[8];                        // split denominator relative to mh_s
  __shared__ float mg_s[8];                        // sequence-wide maximum (that option)
  __shared__ int misc[4];  // 0: clamped length, 1: exchange ok, 2: tag, 3: warps holding accumulators
  __shared__ uint32_t qfr[kQfWords * 32];

  uint8_t* sm = smem2_raw + ((1024u - (smem_u32(smem2_raw) & 1023u)) & 1023u);
  uint8_t* kcode = sm + pr.off_kcode;
  uint8_t* kscale = sm + pr.off_kscale;
  uint8_t* vcode = sm + pr.off_vcode;    // == kcode when V goes into the K slots
  uint8_t* vscale = sm + pr.off_vscale;
  float* ostage = reinterpret_cast<float*>(sm + pr.off_ostage);  // [8][D] this unit's output rows
  float4* sscore = reinterpret_cast<float4*>(sm + pr.off_score);  // [warps][4 jobs][32 lanes] scores
  uint32_t* pword = reinterpret_cast<uint32_t*>(sm + pr.off_pword);  // [warps][4 groups][2][32] B fragments
  int* s_pre = reinterpret_cast<int*>(sm + pr.off_units);  // [batch + 1] units before sequence b

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = lane >> 2, c = lane & 3;
  uint32_t* flags = reinterpret_cast<uint32_t*>(a.workspace);
  const int hkv = a.desc.num_kv_heads, G = a.group, P = a.desc.page_size, Ls = a.split_tokens;
  const int B = a.batch, Hq = a.num_q_heads;
  const int NT = Ls / kTile;            // tiles per unit
  const int NCU = a.max_splits;
  // Thread-block clusters of CS consecutive splits of one (sequence, KV head) share one
  // running maximum (the skip test and the weights of every split of the group use the
  // maximum over the group's scores); CTA `rank` of the cluster takes split g CS + rank of
  // the group g it is on.  CS = 1: every split on its own.
  const int CS = a.cluster;
  const int rank = CS > 1 ? (int)cluster_rank() : 0;
  const int NG = (NCU + CS - 1) / CS;  // groups of splits per (sequence, KV head)
  const int total = B * NG * hkv;
  const int cap = min(a.max_seq_len, a.max_pages * P);
  const bool add_merge = a.out != nullptr && a.group_merge;
  const bool v_tma = pr.v_tma != 0;     // V tiles copied whole (with K, or right after it)
  const bool v_sep = pr.v_sep != 0;     // V tiles in their own region (copied with K)
  // ... after the K pass when the split is long (measured: short splits gain nothing)
  const bool v_late = v_sep && add_merge && NT >= 8;
  const float qk_scale = a.sm_scale * kLog2e;
  // keep iff s - m >= log2(tau); tau = 0 keeps every position in the sequence (a row
  // past the end holds s = -inf, below any finite threshold)
  const float thr = a.tau > 0.f ? log2f(a.tau) : -FLT_MAX;
  const bool hl0 = 2 * c < G, hl1 = 2 * c + 1 < G;

  // every warp's lane 0 initializes the warp's own barriers (it alone issues their copies;
  // the warp's lanes wait on them after a warp barrier), so no CTA barrier is needed here
  if (lane == 0) {
    mbar_init(&kbar[warp], 1);
    mbar_init(&vbar[warp], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  // Programmatic dependent launch: the next grid may be scheduled now; nothing is read
  // from global memory before the preceding grid has completed.
  grid_dependents_launch();
  grid_dependency_wait();
  unsigned long long ep_raw = 0;
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
      lut.lo[i] = lo;
      lut.hi[i] = hi;
    }
  } else if constexpr (C::kNv) {
    const uint32_t hi[4] = {0x3E3C3800u, 0x46444240u, 0xBEBCB880u, 0xC6C4C2C0u};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      lut.lo[i] = 0u;
      lut.hi[i] = hi[i];
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) lut.lo[i] = lut.hi[i] = 0u;
  }

  // Multi-round launches take only the units that exist (sequence-major: the splits of
  // sequence 0, then of sequence 1, ...; every KV head of a split in turn), so that every
  // CTA gets the same number of them; a single-round launch has one unit per CTA in the
  // static order (split-major) and a unit past its sequence's end exits at once.
  int total_units = total;
  if (pr.dense_units) {
    if (warp == 0) {
      int carry = 0;
      for (int b0 = 0; b0 < B; b0 += 32) {
        const int bb = b0 + lane;
        const int n = bb < B ? max(0, min(__ldg(a.seq_lens + bb), cap)) : 0;
        int v = (n + Ls - 1) / Ls * hkv;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, v, o);
          if (lane >= o) v += y;
        }
        if (bb < B) s_pre[bb + 1] = carry + v;
        carry += __shfl_sync(0xffffffffu, v, 31);
      }
      if (lane == 0) s_pre[0] = 0;
    }
    __syncthreads();
    total_units = s_pre[B];
  }

  const __half* qg = static_cast<const __half*>(a.q);
  const uint8_t* kscales_g = static_cast<const uint8_t*>(a.k_scales);
  const uint8_t* vcodes_g = static_cast<const uint8_t*>(a.v_codes);
  const uint8_t* vscales_g = static_cast<const uint8_t*>(a.v_scales);

  const int it0 = CS > 1 ? (int)blockIdx.x / CS : (int)blockIdx.x;
  const int it_step = CS > 1 ? (int)gridDim.x / CS : (int)gridDim.x;
#pragma unroll 1
  for (int it = it0, k = 0; it < total_units; it += it_step, ++k) {
    const uint32_t ph = (uint32_t)k & 1u;  // mbarrier phase of this unit
    int kvh, b, cu;
    if (pr.dense_units) {
      int lo = 0, hi = B;  // the sequence b with s_pre[b] <= it < s_pre[b + 1]
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_pre[mid] <= it) lo = mid;
        else hi = mid;
      }
      b = lo;
      const int rem = it - s_pre[b];
      cu = rem / hkv;
      kvh = rem - cu * hkv;
    } else {
      kvh = it % hkv;
      b = (it / hkv) % B;
      cu = (it / (hkv * B)) * CS + rank;
    }
    const int t0 = cu * Ls;
    const size_t slot0 = ((size_t)b * Hq + (size_t)kvh * G) * a.max_splits + cu;

    // ---- small loads first (a load issued behind the bulk copies waits for them): the
    //      query words (warp 0) and the sequence length (warp 1)
    QRaw<D> qraw;
    if (warp == 0)
      load_query<FMT, D>(r < G ? qg + ((size_t)b * Hq + (size_t)kvh * G + r) * D : nullptr, a.desc.signs, c,
                         qraw);
    int n_raw = 0;
    if (warp == 1 && lane == 0) {
      n_raw = __ldg(a.seq_lens + b);
      // every CTA takes part in the launch count that tags the exchange (its value is
      // stored before B0)
      if (k == 0) {
        ep_raw = epoch_read(a.epoch);
        epoch_advance(a.epoch);
      }
    }
    // ---- K copies: lane 0 of warp w issues tile w (positions that exist in memory; a
    //      tile past the sequence's end is copied speculatively and left unused)
    int row0 = -1;
    bool k_issued = false, v_issued = false;
    if (warp < NT) {
      if (lane == 0) {
        const int tok0 = t0 + warp * kTile;
        uint32_t kbytes = 0;
        if (tok0 < cap) {
          const int lp = tok0 / P, off = tok0 - lp * P;  // tiles never straddle pages (P % 64 == 0)
          const int page = a.page_table ? __ldg(a.page_table + (size_t)b * a.max_pages + lp)
                                        : b * a.max_pages + lp;
          if (page >= 0 && page < a.desc.num_pages) {  // else flagged below if it holds positions
            row0 = (page * hkv + kvh) * P + off;
            kbytes = CODE + SC;
          }
        }
        fence_proxy_async();
        mbar_expect_tx(&kbar[warp], kbytes);
        if (kbytes) {
          tma_rows(kcode + warp * CODE, &tmk, row0, &kbar[warp]);
          bulk_copy(kscale + warp * SC, kscales_g + (size_t)row0 * C::SROW, SC, &kbar[warp]);
        }
      }
      row0 = __shfl_sync(0xffffffffu, row0, 0);
      k_issued = row0 >= 0;
      // V tiles copied whole into their own region, CTAs looping over units or writing
      // partials: each V copy goes out right behind its K copy
      if (v_sep && !v_late) {
        if (lane == 0) {
          const uint32_t vbytes = k_issued ? CODE + SC : 0;
          mbar_expect_tx(&vbar[warp], vbytes);
          if (vbytes) {
            tma_rows(vcode + warp * CODE, &tmv, row0, &vbar[warp]);
            bulk_copy(vscale + warp * SC, vscales_g + (size_t)row0 * C::SROW, SC, &vbar[warp]);
          }
        }
        v_issued = k_issued;
      }
    }
    if (warp == 1 && lane == 0) {
      if (n_raw < 0 || n_raw > cap) set_flag(flags, KVQ_FLAG_BAD_SEQLEN);
      misc[0] = max(0, min(n_raw, cap));
      misc[1] = 1;
      misc[3] = 0;
      if (k == 0) misc[2] = (int)epoch_tag(ep_raw);
    }
    // ---- query fragments, built once for the CTA by warp 0
    if (warp == 0) {
      uint32_t qf[C::KSTEPS][2], ql[C::KSTEPS][2];
      float corr[C::NBLK][2];
      build_query<FMT, D>(qraw, c, qf, ql, corr);
#pragma unroll
      for (int ks = 0; ks < C::KSTEPS; ++ks) {
        qfr[(2 * ks) * 32 + lane] = qf[ks][0];
        qfr[(2 * ks + 1) * 32 + lane] = qf[ks][1];
        if constexpr (C::kLut) {
          qfr[(2 * C::KSTEPS + 2 * ks) * 32 + lane] = ql[ks][0];
          qfr[(2 * C::KSTEPS + 2 * ks + 1) * 32 + lane] = ql[ks][1];
        }
      }
      if constexpr (!C::kLut) {
#pragma unroll
        for (int m = 0; m < C::NBLK; ++m) {
          qfr[(2 * C::KSTEPS + 2 * m) * 32 + lane] = __float_as_uint(corr[m][0]);
          qfr[(2 * C::KSTEPS + 2 * m + 1) * 32 + lane] = __float_as_uint(corr[m][1]);
        }
      }
    }
    __syncthreads();  // B0: query fragments, length
    // ---- split 0 clears the output rows that the splits add their shares into and raises
    //      their flag with release semantics; whoever adds waits for it with acquire
    //      semantics (a wait that is long over by then)
    if (warp == 1 && add_merge && cu == 0) {
      float4* orow = reinterpret_cast<float4*>(a.out + ((size_t)b * Hq + (size_t)kvh * G) * D);
      for (int i = lane; i < G * D / 4; i += 32) orow[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      __syncwarp();
      if (lane == 0) flag_set_release(a.zflag + (size_t)b * hkv + kvh, (uint32_t)misc[2]);
    }
    const int nb = misc[0];
    const uint32_t tag = (uint32_t)misc[2];
    const int n_tok = max(0, min(Ls, nb - t0));
    const int nvalid = warp < NT ? max(0, min(kTile, n_tok - warp * kTile)) : 0;
    const bool has_tile = nvalid > 0 && k_issued;
    if (nvalid > 0 && !k_issued && lane == 0) set_flag(flags, KVQ_FLAG_BAD_PAGE);

    // ---- K pass (the four 16-row jobs in a loop, not unrolled: every warp runs this code
    //      once per unit, so its size is what the instruction cache sees); the scores go
    //      to the warp's scratch, invalid rows as -inf
    float4* scw = sscore + warp * 4 * 32 + lane;
    float mx0 = -INFINITY, mx1 = -INFINITY;
    bool k_waited = false;
    if (has_tile) {
      uint32_t qf[C::KSTEPS][2], ql[C::KSTEPS][2];
      float corr[C::NBLK][2];
#pragma unroll
      for (int ks = 0; ks < C::KSTEPS; ++ks) {
        qf[ks][0] = qfr[(2 * ks) * 32 + lane];
        qf[ks][1] = qfr[(2 * ks + 1) * 32 + lane];
        ql[ks][0] = C::kLut ? qfr[(2 * C::KSTEPS + 2 * ks) * 32 + lane] : 0u;
        ql[ks][1] = C::kLut ? qfr[(2 * C::KSTEPS + 2 * ks + 1) * 32 + lane] : 0u;
      }
#pragma unroll
      for (int m = 0; m < C::NBLK; ++m) {
        corr[m][0] = C::kLut ? 0.f : __uint_as_float(qfr[(2 * C::KSTEPS + 2 * m) * 32 + lane]);
        corr[m][1] = C::kLut ? 0.f : __uint_as_float(qfr[(2 * C::KSTEPS + 2 * m + 1) * 32 + lane]);
      }
      k_waited = true;
      if (!mbar_wait(&kbar[warp], ph)) {
        if (lane == 0) set_flag(flags, KVQ_FLAG_TIMEOUT);
        mbar_wait(&kbar[warp], ph);  // the copy must not be left in flight
      }
      const uint8_t* kc = kcode + warp * CODE;
      const uint8_t* ks_ = kscale + warp * SC;
#pragma unroll 1
      for (int j = 0; j < 4; ++j) {
        float4 sv = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        if (16 * j < nvalid) {
          float t[4];
          k_job_scores<FMT, D>(kc, ks_, 16 * j + r, qf, ql, corr, lut, c, t);
          const bool va = 16 * j + r < nvalid, vb = 16 * j + r + 8 < nvalid;
          sv = make_float4(va ? t[0] * qk_scale : -INFINITY, va ? t[1] * qk_scale : -INFINITY,
                           vb ? t[2] * qk_scale : -INFINITY, vb ? t[3] * qk_scale : -INFINITY);
          mx0 = fmaxf(mx0, fmaxf(sv.x, sv.z));
          mx1 = fmaxf(mx1, fmaxf(sv.y, sv.w));
        }
        scw[j * 32] = sv;
      }
    }
    if (k_issued && !k_waited) mbar_wait(&kbar[warp], ph);  // a speculative tile past the end
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    {
      // the tile's denominators relative to its own maxima (rows past the end hold -inf),
      // so that the split's (m, l) is known at the CTA barrier that follows
      float lw0 = 0.f, lw1 = 0.f;
      if (has_tile) {
#pragma unroll 1
        for (int j = 0; j < 4; ++j) {
          const float4 sv = scw[j * 32];
          lw0 += ex2(sv.x - mx0) + ex2(sv.z - mx0);
          lw1 += ex2(sv.y - mx1) + ex2(sv.w - mx1);
        }
      }
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        lw0 += __shfl_xor_sync(0xffffffffu, lw0, o);
        lw1 += __shfl_xor_sync(0xffffffffu, lw1, o);
      }
      if (r == 0) {
        red_m[warp][2 * c] = mx0;
        red_m[warp][2 * c + 1] = mx1;
        red_l[warp][2 * c] = lw0;
        red_l[warp][2 * c + 1] = lw1;
      }
    }
    // V into this warp's K slot right behind its K pass (V tiles copied whole but no
    // room for a separate region)
    if (v_tma && !v_sep && warp < NT) {
      __syncwarp();  // every lane is done reading the K tile
      if (lane == 0) {
        fence_proxy_async();
        const uint32_t vbytes = k_issued && nvalid > 0 ? CODE + SC : 0;
        mbar_expect_tx(&vbar[warp], vbytes);
        if (vbytes) {
          tma_rows(vcode + warp * CODE, &tmv, row0, &vbar[warp]);
          bulk_copy(vscale + warp * SC, vscales_g + (size_t)row0 * C::SROW, SC, &vbar[warp]);
        }
      }
      v_issued = k_issued && nvalid > 0;
    } else if (!v_sep && warp < NT && lane == 0) {
      mbar_expect_tx(&vbar[warp], 0);  // every barrier completes one phase per unit
    }
    __syncthreads();  // B1: every warp's maxima
    // V tiles copied whole into their own region, every split on its own CTA (the step is
    // one round of copies): the V copies go out once all K tiles of the CTA have landed, so
    // that the K copies of the launch have the memory system first
    if (v_sep && v_late && warp < NT) {
      if (lane == 0) {
        fence_proxy_async();
        mbar_expect_tx(&vbar[warp], has_tile ? CODE + SC : 0);
        if (has_tile) {
          tma_rows(vcode + warp * CODE, &tmv, row0, &vbar[warp]);
          bulk_copy(vscale + warp * SC, vscales_g + (size_t)row0 * C::SROW, SC, &vbar[warp]);
        }
      }
      v_issued = has_tile;
    }

    // ---- the split's maximum per head (log2 units); warp 0 and the poll warp also fold
    //      the tiles' denominators into the split's (lane h: head h)
    float mh0, mh1;
    float m_own = -INFINITY, l_own = 0.f;  // lanes < 8 of warp 0 and of the poll warp
    float m_use = -INFINITY;               // the maximum the weights use (lanes < 8)
    {
      // lane (head h = lane & 7, quarter q = lane >> 3) folds the tiles of warps q, q + 4,
      // ...; the quarters are combined by shuffles, so every lane holds head lane & 7
      const int hh = lane & 7, q = lane >> 3;
      float m = -INFINITY;
      for (int w = q; w < NT; w += 4) m = fmaxf(m, red_m[w][hh]);
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
      m_own = m;
      if (warp == 0 || warp == kPollWarp) {
        float l = 0.f;
        if (m > -INFINITY) {
          for (int w = q; w < NT; w += 4) {
            const float mw = red_m[w][hh];
            if (mw > -INFINITY) l = fmaf(red_l[w][hh], ex2(mw - m), l);
          }
        }
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        l_own = l;
      }
      mh0 = __shfl_sync(0xffffffffu, m, 2 * c);
      mh1 = __shfl_sync(0xffffffffu, m, 2 * c + 1);
      if (warp == 0 && lane < 8) {
        mh_s[lane] = m;
        ls_s[lane] = l_own;
      }
      if (CS > 1) {
        // the maximum over the cluster's splits: every CTA's maxima are written before the
        // cluster barrier, read from distributed shared memory after it; the arrive after
        // the reads lets each CTA know, at the end of the unit, that nobody reads its
        // maxima any more
        cluster_sync();
        for (int rk = 0; rk < CS; ++rk) {
          if (rk == rank) continue;
          mh0 = fmaxf(mh0, dsmem_ld(dsmem_addr(mh_s + 2 * c, rk)));
          mh1 = fmaxf(mh1, dsmem_ld(dsmem_addr(mh_s + 2 * c + 1, rk)));
          if (lane < 8) m = fmaxf(m, dsmem_ld(dsmem_addr(mh_s + lane, rk)));
        }
        cluster_arrive();
      }
      if (warp == 0 && lane < 8) mc_s[lane] = m;
      m_use = m;
    }
    if (a.global_max) {
      // every split publishes (m, l relative to m); the poll warp derives the final
      // maximum M and denominator L of every head; the weights below use M, and this
      // split's share of the output is 1 / L
      if (warp == kPollWarp && n_tok > 0) {
        const int nsplit = (nb + Ls - 1) / Ls;
        const unsigned long long target =
            publish_split(a, slot0, tag, m_own, l_own, G, lane, b * hkv + kvh, cu == 0, nsplit);
        const int h = lane >> 2, j = lane & 3;
        float M, L;
        arrivals_await(a, b * hkv + kvh, target, lane);
        bool ok = xch_reduce<16>(a.xch + ((size_t)b * Hq + (size_t)kvh * G + (h < G ? h : 0)) * a.max_splits,
                                 j, 4, nsplit, h < G, tag, M, L, kWaitCycles, kPollSleepNs);
        if (ok) {
          xch_combine(M, L, 2);
          if (j == 0 && h < G) {
            mg_s[h] = M;
            share_s[h] = 1.f / L;
          }
        } else if (lane == 0) {
          set_flag(flags, KVQ_FLAG_TIMEOUT);
          misc[1] = 0;
        }
      }
      __syncthreads();
      if (misc[1]) {
        mh0 = mg_s[2 * c < G ? 2 * c : 0];
        mh1 = mg_s[2 * c + 1 < G ? 2 * c + 1 : 0];
        if (warp == 0 && lane < G) mc_s[lane] = mg_s[lane];  // (read after the next CTA barrier)
      }
    }
    // In-kernel merge without the sequence-wide maximum: the poll warp publishes the
    // split's (m, l) at once (l relative to the maximum the weights use) and, after its own
    // tile if it has one, collects every split's while the others work; a warp without a
    // tile, if there is one besides, waits for split 0's cleared output rows meanwhile.
    const bool publish = add_merge && !a.global_max && n_tok > 0;
    const int zwarp = NT < kNW - 1 ? NT : kPollWarp;
    unsigned long long arrive_target = 0;  // (lane 0 of the poll warp)
    if (warp == kPollWarp && publish)
      arrive_target = publish_split(a, slot0, tag, m_use, l_own * ex2(m_own - m_use), G, lane, b * hkv + kvh,
                                    cu == 0, (nb + Ls - 1) / Ls);
    if (warp == zwarp && zwarp != kPollWarp && publish && lane == 0) {
      if (!flag_wait_acquire(a.zflag + (size_t)b * hkv + kvh, tag)) {
        set_flag(flags, KVQ_FLAG_TIMEOUT);
        misc[1] = 0;
      }
    }

    // a head past the group (G < 8) gets m = +inf: every one of its weights is 0 and none
    // of its positions is kept
    if (!hl0) mh0 = INFINITY;
    if (!hl1) mh1 = INFINITY;

    // ---- weights, skip test and V pass of this warp's own tile
    if (warp < NT) {
      int nskip = 0;
      uint32_t gk = 0;  // groups (16-row jobs) with a kept pair
      uint32_t* pww = pword + warp * 4 * 64 + lane;  // B fragments of the weights, per group
      unsigned long long rows = 0ull;
      const bool count = !v_tma || a.stats;  // the kept rows wanted (to gather them, or counted)
      if (has_tile) {
#pragma unroll 1
        for (int j = 0; j < 4; ++j) {
          // rows past the end hold s = -inf: weight 0, never kept
          const float4 sv = scw[j * 32];
          const float da0 = sv.x - mh0, da1 = sv.y - mh1;
          const float db0 = sv.z - mh0, db1 = sv.w - mh1;
          const float ea0 = ex2(da0), ea1 = ex2(da1), eb0 = ex2(db0), eb1 = ex2(db1);
          const bool ka0 = da0 >= thr, ka1 = da1 >= thr, kb0 = db0 >= thr, kb1 = db1 >= thr;
          // the kept weights as the V MMA's B fragments: rows 0-7 / 8-15 of the group,
          // transposed from (row r, heads 2c, 2c + 1) to (rows 2c, 2c + 1, head r)
          pww[j * 64] = movmatrix_trans(pack_h2(ka0 ? ea0 * kPScale : 0.f, ka1 ? ea1 * kPScale : 0.f));
          pww[j * 64 + 32] = movmatrix_trans(pack_h2(kb0 ? eb0 * kPScale : 0.f, kb1 ? eb1 * kPScale : 0.f));
          gk |= (__any_sync(0xffffffffu, ka0 || ka1 || kb0 || kb1) ? 1u : 0u) << j;
          if (count) {  // rows any head keeps (the rows to gather; V rows needed), skip count
            const bool va = 16 * j + r < nvalid, vb = 16 * j + r + 8 < nvalid;
            nskip += (va && hl0 && !ka0) + (va && hl1 && !ka1) + (vb && hl0 && !kb0) + (vb && hl1 && !kb1);
            const uint32_t rows_a = rows_of(__ballot_sync(0xffffffffu, ka0 || ka1));
            const uint32_t rows_b = rows_of(__ballot_sync(0xffffffffu, kb0 || kb1));
            const uint32_t mine =
                c == 0 ? ((((rows_a >> (4 * r)) & 1u) << r) | (((rows_b >> (4 * r)) & 1u) << (r + 8))) : 0u;
            rows |= (unsigned long long)__reduce_or_sync(0xffffffffu, mine) << (16 * j);
          }
        }
      }
      if (a.stats) {
#pragma unroll
        for (int o = 16; o; o >>= 1) nskip += __shfl_xor_sync(0xffffffffu, nskip, o);
        if (lane == 0) {
          cnt_skip[warp] = nskip;
          cnt_keep[warp] = __popcll(rows);
        }
      }

      uint8_t* vc = (v_sep ? vcode : kcode) + warp * CODE;
      uint8_t* vs = (v_sep ? vscale : kscale) + warp * SC;
      if (!v_tma && rows) {
        // gather the kept rows into this warp's (now free) K slot: codes with the tile's
        // chunk swizzle, and the rows' scales (lut4: the aligned pair holding the norm)
        const uint8_t* src = vcodes_g + (size_t)row0 * C::CROW;
        const uint8_t* ssrc = vscales_g + (size_t)row0 * C::SROW;
        constexpr int CPR = C::CROW / 16;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int i = lane + 32 * h;
          if ((rows >> i) & 1ull) {
#pragma unroll
            for (int cc = 0; cc < CPR; ++cc)
              cp_async16(vc + i * C::CROW + ((cc ^ swz<FMT, D>(i)) << 4), src + (size_t)i * C::CROW + cc * 16);
            if constexpr (C::SROW == 16) cp_async16(vs + i * 16, ssrc + (size_t)i * 16);
            else if constexpr (C::SROW == 8) cp_async8(vs + i * 8, ssrc + (size_t)i * 8);
            else if constexpr (C::SROW == 4) cp_async4(vs + i * 4, ssrc + (size_t)i * 4);
            else cp_async4(vs + (i & ~1) * 2, ssrc + (size_t)(i & ~1) * 2);  // 2-byte rows: the pair
            static_assert(C::SROW == 16 || C::SROW == 8 || C::SROW == 4 || C::SROW == 2, "scale row");
          }
        }
        cp_async_commit();
        cp_async_wait<0>();
        __syncwarp();
      }
      bool v_waited = false;
      if (gk) {
        if (v_tma) {
          v_waited = true;
          if (!mbar_wait(&vbar[warp], ph)) {
            if (lane == 0) set_flag(flags, KVQ_FLAG_TIMEOUT);
            mbar_wait(&vbar[warp], ph);  // the copy must not be left in flight
          }
        }
        float acc[C::MT][4];
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
        if constexpr (C::kMag) {
          int kx[C::NBLK];
          tile_mag_normalize<FMT, D>(vs, nvalid, lane, kx);
#pragma unroll 1
          for (int j = 0; j < 4; ++j)
            if ((gk >> j) & 1u)
              vg_mag<FMT, D>(vc, vs, 16 * j, min(16, nvalid - 16 * j), pww[j * 64], pww[j * 64 + 32], lane, acc);
#pragma unroll
          for (int mt = 0; mt < C::MT; ++mt) {
            const float f = __int_as_float((127 + kx[mt >> 1]) << 23) * kPUnscale;  // undo 2^-k, 2^14
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[mt][i] *= f;
          }
        } else {
#pragma unroll 1
          for (int j = 0; j < 4; ++j)
            if ((gk >> j) & 1u)
              vg_lut<FMT, D>(vc, vs, 16 * j, min(16, nvalid - 16 * j), pww[j * 64], pww[j * 64 + 32], lane, lut, acc);
#pragma unroll
          for (int mt = 0; mt < C::MT; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[mt][i] *= kPUnscale;
        }
        // the accumulators go to this warp's K code slot (its V data is read: same warp)
        __syncwarp();
        float* accw = reinterpret_cast<float*>(kcode + warp * CODE);
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt)
#pragma unroll
          for (int i = 0; i < 4; ++i) accw[(mt * 4 + i) * 32 + lane] = acc[mt][i];
        if (lane == 0) atomicOr(&misc[3], 1 << warp);
      }
      if (v_issued && !v_waited) mbar_wait(&vbar[warp], ph);  // no copy stays in flight
    }
    if (warp == kPollWarp && publish) {
      // wait for every split's (m, l) (and, with no other warp to do it, for split 0's
      // cleared output rows): this split's share of each head is 2^(m_s - M) / L
      bool ok = true;
      if (zwarp == kPollWarp && lane == 0) ok = flag_wait_acquire(a.zflag + (size_t)b * hkv + kvh, tag);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      const int h = lane >> 2, j = lane & 3;
      const float mine = __shfl_sync(0xffffffffu, m_use, h & 7);  // this split's maximum of head h
      if (ok) {
        const int nsplit = (nb + Ls - 1) / Ls;
        float M, L;
        arrivals_await(a, b * hkv + kvh, arrive_target, lane);
        ok = xch_reduce<16>(a.xch + ((size_t)b * Hq + (size_t)kvh * G + (h < G ? h : 0)) * a.max_splits, j, 4,
                            nsplit, h < G, tag, M, L, kWaitCycles, kPollSleepNs);
        if (ok) {
          xch_combine(M, L, 2);
          if (j == 0 && h < G) share_s[h] = ex2(mine - M) / L;
        }
      }
      if (lane == 0 && !ok) {
        set_flag(flags, KVQ_FLAG_TIMEOUT);
        misc[1] = 0;
      }
    } else if (warp == kPollWarp && add_merge && a.global_max && n_tok > 0 && lane == 0) {
      // the weights are final already; the output rows must be cleared before adding
      if (!flag_wait_acquire(a.zflag + (size_t)b * hkv + kvh, tag)) {
        set_flag(flags, KVQ_FLAG_TIMEOUT);
        misc[1] = 0;
      }
    }
    __syncthreads();  // B4: accumulators, denominators, shares

    // ---- this split's contribution: the warps' accumulators summed (four consecutive
    //      lanes' entries per thread), scaled by the share, staged as [head][dim]
    if (n_tok > 0) {
      if (!add_merge && tid < G) {
        // (the maximum the weights used, and the denominator relative to it)
        a.part_m[slot0 + (size_t)tid * a.max_splits] = mc_s[tid];
        a.part_l[slot0 + (size_t)tid * a.max_splits] = ls_s[tid] * ex2(mh_s[tid] - mc_s[tid]);
      }
      if (tid == 32 && a.stats) {
        int ns = 0, nk = 0;
        for (int w = 0; w < NT; ++w) {
          if (w * kTile < n_tok) {
            ns += cnt_skip[w];
            nk += cnt_keep[w];
          }
        }
        atomicAdd(&a.stats[0], (unsigned long long)n_tok * G);
        atomicAdd(&a.stats[1], (unsigned long long)ns);
        atomicAdd(&a.stats[2], (unsigned long long)nk);
        atomicAdd(&a.stats[3], (unsigned long long)(n_tok - nk));
      }
      const uint32_t wk = (uint32_t)misc[3];
      for (int q4 = tid; q4 < 8 * C::NE; q4 += kNT) {
        float v[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
        for (int w = 0; w < NT; ++w)
          if ((wk >> w) & 1u) {
            const float4 x = reinterpret_cast<const float4*>(kcode + w * CODE)[q4];
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
          ostage[h * D + out_dim<FMT, D>(ln >> 2, mt, i)] = add_merge && h < G ? v[t] * share_s[h] : v[t];
        }
      }
    }
    __syncthreads();
    if (n_tok > 0) {
      constexpr int Q4 = D / 4;
      if (add_merge) {
        if (misc[1]) {
          if constexpr (C::kLut) {
            // rotate back (R^T = diag(s) c H), one warp per head in turn, then add
#pragma unroll 1
            for (int hh = warp; hh < G; hh += kNW) {
              constexpr int K = D / 32;
              float y[K];
#pragma unroll
              for (int kk = 0; kk < K; ++kk) y[kk] = ostage[hh * D + 32 * kk + lane];
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
              float* dst = a.out + ((size_t)b * Hq + (size_t)kvh * G + hh) * D;
#pragma unroll
              for (int kk = 0; kk < K; ++kk)
                atomicAdd(dst + 32 * kk + lane, y[kk] * cs * (float)a.desc.signs[32 * kk + lane]);
            }
          } else {
            for (int e = tid; e < G * Q4; e += kNT)
              red_add_f32x4(a.out + ((size_t)b * Hq + (size_t)kvh * G) * D + 4 * e,
                            reinterpret_cast<const float4*>(ostage)[e]);
          }
        }
      } else {
        for (int e = tid; e < G * Q4; e += kNT) {
          const int h = e / Q4, d4 = e - h * Q4;
          reinterpret_cast<float4*>(a.part_o + (slot0 + (size_t)h * a.max_splits) * D)[d4] =
              reinterpret_cast<const float4*>(ostage)[e];
        }
      }
    }
    __syncthreads();  // B5: the unit's buffers are free
    if (CS > 1) cluster_wait();  // every CTA of the cluster is done reading this one's maxima
  }
}

// ------------------------------------------------------------------ host side
std::mutex g_mu2;

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// The codes plane as a 2-D tensor of `rows` rows of `crow` bytes; a box is one 64-row tile,
// swizzled in 16-byte chunks across the row (128-, 64- or 32-byte rows).
bool code_map(CUtensorMap* m, const void* base, uint64_t rows, int crow) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)crow, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)crow};
  cuuint32_t box[2] = {(cuuint32_t)crow, (cuuint32_t)kTile};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw = crow == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                : crow == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                             : CU_TENSOR_MAP_SWIZZLE_32B;
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr size_t kSmemSM = 233472;   // shared memory per SM (1 KB of it reserved per CTA)
constexpr size_t kStaticReserve = 8192;
// dynamic + static shared memory of one CTA when 16 / NW CTAs share an SM (a plan that
// does not fit is still launched, with fewer CTAs per SM: the capacity counts them)
constexpr size_t smem_budget(int nw) { return kSmemSM / (16 / nw) - 1024; }

template <int FMT, int D>
struct Plan {
  using C = Cfg<FMT, D>;
  static_assert(kTile * C::CROW >= C::NE * 32 * 4, "a warp's accumulators fit its K code slot");
  static constexpr size_t CODE = kTile * C::CROW, SC = kTile * C::SROW;
  // byte offsets for a unit of nt tiles; v_sep: V tiles get their own region
  static size_t layout(int nw, int nt, bool v_sep, Decode2Params* p) {
    auto up = [](size_t x, size_t m) { return (x + m - 1) / m * m; };
    size_t o = 0;
    p->off_kcode = (uint32_t)o;
    o += nt * CODE;
    p->off_kscale = (uint32_t)o;
    o = up(o + nt * SC, 1024);
    if (v_sep) {
      p->off_vcode = (uint32_t)o;
      o += nt * CODE;
      p->off_vscale = (uint32_t)o;
      o = up(o + nt * SC, 128);
    } else {
      p->off_vcode = p->off_kcode;
      p->off_vscale = p->off_kscale;
    }
    p->off_ostage = (uint32_t)o;
    o += (size_t)8 * D * 4;
    p->off_score = (uint32_t)o;  // per warp: 4 jobs x 32 lanes x float4
    o += (size_t)nw * 4 * 32 * 16;
    p->off_pword = (uint32_t)o;  // per warp: 4 groups x 2 x 32 lanes x u32
    o += (size_t)nw * 4 * 64 * 4;
    p->off_units = (uint32_t)o;  // prefix of the units per sequence
    o += (size_t)(KVQ_MAX_BATCH + 1) * 4;
    return o + 1024;  // slack for aligning the base to 1024
  }
};

template <int FMT, int D, int NW>
int configure2(int dev) {
  static uint64_t done_mask = 0;  // guarded by g_mu2
  if (!(done_mask >> dev & 1)) {
    if (cudaFuncSetAttribute(decode2_kernel<FMT, D, NW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(smem_budget(16) - kStaticReserve)) != cudaSuccess)
      return KVQ_ERR_CUDA;
    done_mask |= 1ull << dev;
  }
  return KVQ_OK;
}

// CTAs (CS = 1) or clusters of CS CTAs of the streaming kernel resident at once on the
// current device, cached per device and cluster size.
template <int FMT, int D, int NW>
int capacity2_t(int CS) {
  static int cache[64][4] = {};  // [device][log2 CS] = count + 1; guarded by g_mu2
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  const int ci = CS == 8 ? 3 : CS == 4 ? 2 : CS == 2 ? 1 : 0;
  std::lock_guard<std::mutex> lock(g_mu2);
  if (cache[dev][ci] == 0) {
    if (configure2<FMT, D, NW>(dev) != KVQ_OK) return 0;
    Decode2Params p{};
    const size_t bytes = Plan<FMT, D>::layout(NW, NW, false, &p);
    int n = 0;
    if (CS == 1) {
      int sms = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode2_kernel<FMT, D, NW>, 32 * NW, bytes) !=
              cudaSuccess ||
          cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
      n *= sms;
    } else {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = CS;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(CS * 64, 1, 1);
      cfg.blockDim = dim3(32 * NW, 1, 1);
      cfg.dynamicSmemBytes = bytes;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&n, decode2_kernel<FMT, D, NW>, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        n = 0;
      }
    }
    cache[dev][ci] = n + 1;
  }
  return cache[dev][ci] - 1;
}

template <int FMT, int D, int NW>
int launch2_t(const DecodeArgs& a, cudaStream_t stream) {
  using C = Cfg<FMT, D>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return KVQ_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lock(g_mu2);
    if (configure2<FMT, D, NW>(dev) != KVQ_OK) return KVQ_ERR_CUDA;
  }
  const int CS = a.cluster;
  const int cap = capacity2_t<FMT, D, NW>(CS);  // CTAs, or clusters of CS CTAs
  if (cap <= 0) return KVQ_ERR_CUDA;
  Decode2Params p{};
  p.a = a;
  const int nt = a.split_tokens / kTile;
  const int64_t groups = (int64_t)a.batch * a.desc.num_kv_heads * ((a.max_splits + CS - 1) / CS);
  p.a.grid = (int)std::min<int64_t>(groups, cap) * CS;
  if (p.a.grid <= 0) return KVQ_OK;
  // every group on its own CTAs at once: the splits exchange (m, l) and add their shares;
  // otherwise CTAs loop over the units (those that exist, when splits are independent)
  p.a.group_merge = a.out != nullptr && groups <= cap;
  p.dense_units = (CS == 1 && groups > cap) ? 1 : 0;
  if (a.global_max && groups > cap) return KVQ_ERR_UNSUPPORTED;
  // V tiles copied whole: tau = 0 (every row is needed) or when the launch asks; in their
  // own region when shared memory allows, else into the K slots right after the K pass
  const bool whole = !(a.tau > 0.f) || a.v_early;
  size_t bytes = Plan<FMT, D>::layout(NW, nt, whole, &p);
  p.v_sep = whole ? 1 : 0;
  if (bytes + kStaticReserve > smem_budget(NW)) {
    bytes = Plan<FMT, D>::layout(NW, nt, false, &p);
    p.v_sep = 0;
  }
  p.v_tma = whole ? 1 : 0;
  CUtensorMap tmk, tmv;
  const uint64_t rows = (uint64_t)a.desc.num_pages * a.desc.num_kv_heads * a.desc.page_size;
  if (!code_map(&tmk, a.k_codes, rows, C::CROW) || !code_map(&tmv, a.v_codes, rows, C::CROW))
    return KVQ_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[3];
  int na = 0;
  if (CS > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = CS;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  const bool coop = p.a.group_merge || a.global_max;
  if (coop) {  // CTAs wait for one another: all resident together
    attr[na].id = cudaLaunchAttributeCooperative;
    attr[na].val.cooperative = 1;
    ++na;
  }
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  cfg.gridDim = dim3(p.a.grid, 1, 1);
  cfg.blockDim = dim3(32 * NW, 1, 1);
  cfg.dynamicSmemBytes = bytes;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = na;
  cudaError_t e = cudaLaunchKernelEx(&cfg, decode2_kernel<FMT, D, NW>, p, tmk, tmv);
  if (e != cudaSuccess && coop) {  // a driver that does not take both: without PDL
    (void)cudaGetLastError();
    cfg.numAttrs = na - 1;
    e = cudaLaunchKernelEx(&cfg, decode2_kernel<FMT, D, NW>, p, tmk, tmv);
  }
  if (e != cudaSuccess) return KVQ_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

// Warps per CTA for a split of L positions: one tile per warp, the smallest CTA that
// holds the split.
int warps_for(int split_tokens) { return split_tokens <= 4 * kTile ? 4 : split_tokens <= 8 * kTile ? 8 : 16; }

template <int FMT, int D>
int launch_nw(const DecodeArgs& a, cudaStream_t stream) {
  const int nw = warps_for(a.split_tokens);
  if (nw == 4) return launch2_t<FMT, D, 4>(a, stream);
  if (nw == 8) return launch2_t<FMT, D, 8>(a, stream);
  return launch2_t<FMT, D, 16>(a, stream);
}

template <int FMT, int D>
int capacity_nw(int cluster, int split_tokens) {
  const int nw = warps_for(split_tokens);
  if (nw == 4) return capacity2_t<FMT, D, 4>(cluster);
  if (nw == 8) return capacity2_t<FMT, D, 8>(cluster);
  return capacity2_t<FMT, D, 16>(cluster);
}

}  // namespace

int launch_decode2(const DecodeArgs& a, cudaStream_t stream) {
  const int f = a.desc.fmt, d = a.desc.head_dim;
  if (f == KVQ_FMT_Q8_0 && d == 128) return launch_nw<KVQ_FMT_Q8_0, 128>(a, stream);
  if (f == KVQ_FMT_Q8_0 && d == 64) return launch_nw<KVQ_FMT_Q8_0, 64>(a, stream);
  if (f == KVQ_FMT_Q4_0 && d == 128) return launch_nw<KVQ_FMT_Q4_0, 128>(a, stream);
  if (f == KVQ_FMT_Q4_0 && d == 64) return launch_nw<KVQ_FMT_Q4_0, 64>(a, stream);
  if (f == KVQ_FMT_LUT4 && d == 128) return launch_nw<KVQ_FMT_LUT4, 128>(a, stream);
  if (f == KVQ_FMT_LUT4 && d == 64) return launch_nw<KVQ_FMT_LUT4, 64>(a, stream);
  if (f == KVQ_FMT_NVFP4 && d == 128) return launch_nw<KVQ_FMT_NVFP4, 128>(a, stream);
  if (f == KVQ_FMT_NVFP4 && d == 64) return launch_nw<KVQ_FMT_NVFP4, 64>(a, stream);
  return KVQ_ERR_UNSUPPORTED;
}

int decode2_capacity(int f, int d, int cluster, int split_tokens) {
  if (cluster != 1 && cluster != 2 && cluster != 4 && cluster != 8) return 0;
  if (f == KVQ_FMT_Q8_0 && d == 128) return capacity_nw<KVQ_FMT_Q8_0, 128>(cluster, split_tokens);
  if (f == KVQ_FMT_Q8_0 && d == 64) return capacity_nw<KVQ_FMT_Q8_0, 64>(cluster, split_tokens);
  if (f == KVQ_FMT_Q4_0 && d == 128) return capacity_nw<KVQ_FMT_Q4_0, 128>(cluster, split_tokens);
  if (f == KVQ_FMT_Q4_0 && d == 64) return capacity_nw<KVQ_FMT_Q4_0, 64>(cluster, split_tokens);
  if (f == KVQ_FMT_LUT4 && d == 128) return capacity_nw<KVQ_FMT_LUT4, 128>(cluster, split_tokens);
  if (f == KVQ_FMT_LUT4 && d == 64) return capacity_nw<KVQ_FMT_LUT4, 64>(cluster, split_tokens);
  if (f == KVQ_FMT_NVFP4 && d == 128) return capacity_nw<KVQ_FMT_NVFP4, 128>(cluster, split_tokens);
  if (f == KVQ_FMT_NVFP4 && d == 64) return capacity_nw<KVQ_FMT_NVFP4, 64>(cluster, split_tokens);
  return 0;
}

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

}  // namespace kvq
