// Device-side building blocks for sm_100a: cp.async copies, transposing matrix loads,
// the m16n8k16 f16 tensor-core MMA, cluster / DSMEM access, the tagged cross-CTA
// exchange, programmatic dependent launch, byte permutes.
#pragma once


#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

// Workspace header: word 0 holds the KVQ_FLAG_* bits.
constexpr size_t kWorkspaceHeader = 256;

// A bounded wait gives up after this many SM clock cycles (about 2 s at 1.9 GHz).
constexpr long long kWaitCycles = 4000000000LL;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void set_flag(uint32_t* flags, uint32_t bit) {
  if (flags) atomicOr(flags, bit);
}

// ------------------------------------------------------------------ cp.async gathers
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async8(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------------------------ tensor core
// D += A * B, m16n8k16, f16 inputs, f32 accumulators.
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Four 8x8 matrices of 16-bit elements from shared memory, transposed: lane l gives the
// address of row l % 8 of matrix l / 8; register i of lane (r = l / 4, c = l % 4) holds
// elements (row 2c, column r) and (row 2c + 1, column r) of matrix i (low half first).
__device__ __forceinline__ void ldsm_x4_trans(const void* p, uint32_t& d0, uint32_t& d1, uint32_t& d2,
                                              uint32_t& d3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(d0), "=r"(d1), "=r"(d2), "=r"(d3)
               : "r"(smem_u32(p))
               : "memory");
}

// ------------------------------------------------------------------ thread-block clusters
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_index() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_count() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// Every thread of every CTA of the cluster arrives (release) and waits (acquire).
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
// The two halves of cluster_sync: arrive (release; does not wait) and wait (acquire).
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory location in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t dsmem_addr(const void* local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(local)), "r"(rank));
  return r;
}
__device__ __forceinline__ float dsmem_ld(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// ------------------------------------------------------------------ tagged exchange
// The splits of one (sequence, KV head) publish their (m, l) to one another through
// 64-bit words that each carry a launch tag in the high half, so a reader needs no
// separate arrival counter: an entry is this launch's once its tag matches.  A 64-bit
// access is single-copy atomic, so value and tag are always seen together.
//
// The tag comes from a launch counter in the workspace header.  Every CTA reads it at
// its start and then adds its share of kEpochStep (CTA 0: kEpochStep - (grid - 1), the
// others 1), so each launch adds exactly kEpochStep; a CTA's read sees the previous
// launches' total plus less than kEpochStep of this launch's own adds, so
// read / kEpochStep is the same launch number e for every CTA, and the tag is e + 1.
constexpr int kEpochShift = 16;
constexpr unsigned long long kEpochStep = 1ull << kEpochShift;  // > any grid
constexpr size_t kEpochOffset = 8;                               // byte offset in the header

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void red_add_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("red.relaxed.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// One thread of every CTA: read the counter (epoch_read), then add this CTA's share
// (epoch_advance, after the read); the tag is epoch_tag of what was read.
__device__ __forceinline__ unsigned long long epoch_read(const unsigned long long* epoch) {
  return ld_relaxed_u64(epoch);
}
__device__ __forceinline__ void epoch_advance(unsigned long long* epoch) {
  red_add_u64(epoch, blockIdx.x == 0 ? kEpochStep - (gridDim.x - 1) : 1ull);
}
__device__ __forceinline__ uint32_t epoch_tag(unsigned long long read) {
  return (uint32_t)(read >> kEpochShift) + 1u;
}

// A flag word that holds the tag of the launch that last set it.  set: every write of
// the calling thread (and of the threads ordered before it by a barrier) made before it
// is visible to whoever reads the tag with flag_wait.
__device__ __forceinline__ void flag_set_release(unsigned long long* p, uint32_t tag) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"((unsigned long long)tag) : "memory");
}
// Wait (at most `limit` SM cycles) until the flag holds `tag`, with acquire semantics.
__device__ __forceinline__ bool flag_wait_acquire(const unsigned long long* p, uint32_t tag,
                                                  long long limit = kWaitCycles) {
  unsigned long long v;
  const long long t0 = clock64();
  for (;;) {
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    if ((uint32_t)v == tag) return true;
    if (clock64() - t0 > limit) return false;
    __nanosleep(32);
  }
}

// Arrival word of one (sequence, KV head): every launch adds exactly kArriveStep to it
// over the splits that publish (split 0: kArriveStep - (n - 1), the others 1), so a split
// that reads v before its own add knows that the word reaches (v / kArriveStep + 1) *
// kArriveStep once every split has arrived.  A relaxed add: the count is only a hint that
// the exchange entries are there (a reader still checks every entry's tag).
constexpr unsigned long long kArriveStep = 1ull << 16;  // > any number of splits
__device__ __forceinline__ unsigned long long arrive_add(unsigned long long* p, bool first, int n) {
  unsigned long long old;
  asm volatile("atom.relaxed.gpu.global.add.u64 %0, [%1], %2;"
               : "=l"(old)
               : "l"(p), "l"(first ? kArriveStep - (unsigned long long)(n - 1) : 1ull)
               : "memory");
  return (old / kArriveStep + 1) * kArriveStep;
}
// Wait (at most `limit` SM cycles) until the arrival word reaches `target`.
__device__ __forceinline__ bool arrivals_wait(const unsigned long long* p, unsigned long long target,
                                              long long limit, int sleep_ns) {
  const long long t0 = clock64();
  for (;;) {
    if (ld_relaxed_u64(p) >= target) return true;
    if (clock64() - t0 > limit) return false;
    __nanosleep(sleep_ns);
  }
}

__device__ __forceinline__ unsigned long long tag_word(uint32_t tag, float v) {
  return ((unsigned long long)tag << 32) | __float_as_uint(v);
}

// One entry: (m, l) of one head of one split, each word tagged.
__device__ __forceinline__ void xch_store(ulonglong2* p, uint32_t tag, float m, float l) {
  asm volatile("st.relaxed.gpu.global.v2.u64 [%0], {%1, %2};" ::"l"(p), "l"(tag_word(tag, m)),
               "l"(tag_word(tag, l))
               : "memory");
}

// Read an entry; false while it is not this launch's (tag mismatch in either word).
__device__ __forceinline__ bool xch_load(const ulonglong2* p, uint32_t tag, float& m, float& l) {
  unsigned long long a, b;
  asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
  m = __uint_as_float((uint32_t)a);
  l = __uint_as_float((uint32_t)b);
  return (uint32_t)(a >> 32) == tag && (uint32_t)(b >> 32) == tag;
}

// out[0..3] += v, one vector reduction in global memory (16-byte aligned address).
__device__ __forceinline__ void red_add_f32x4(float* out, float4 v) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(out), "f"(v.x), "f"(v.y),
               "f"(v.z), "f"(v.w)
               : "memory");
}

// ------------------------------------------------------------------ programmatic dependent launch
// Block until the grids this one depends on have completed and their memory is visible
// (a no-op when the launch has no programmatic dependency).
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
// Allow the dependent grid to be scheduled before this one completes.
__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------ bit tricks
// prmt in its default mode: selector nibble bit 3 replicates the sign of the chosen byte.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) {
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) {
  return *reinterpret_cast<__half2*>(&u);
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t lds32(const void* p) {
  return *reinterpret_cast<const uint32_t*>(p);
}
__device__ __forceinline__ uint32_t lds16(const void* p) {
  return *reinterpret_cast<const uint16_t*>(p);
}
__device__ __forceinline__ uint32_t lds8(const void* p) {
  return *reinterpret_cast<const uint8_t*>(p);
}

}  // namespace kvq
