// Internal interface of the streaming decode kernel (kvq_decode2.cu).
#pragma once

#include "kvq_internal.h"

namespace kvq {

// Launch parameters: the request (DecodeArgs) plus the shared-memory plan the host
// computed for it (byte offsets from the 1024-aligned base of dynamic shared memory).
struct Decode2Params {
  DecodeArgs a;
  uint32_t off_kcode, off_kscale;  // K tiles: codes (swizzled), scale rows
  uint32_t off_vcode, off_vscale;  // V tiles (== the K tiles' offsets when V reuses them)
  uint32_t off_ostage;             // one unit's output rows, fp32 [8 heads][head_dim]
  uint32_t off_score;              // per warp: the scores of its tile, [4 jobs][32 lanes] float4
  uint32_t off_pword;              // per warp: the weights' B fragments, [4 groups][2][32] u32
  uint32_t off_units;              // [batch + 1] prefix of the units per sequence
  int dense_units;                 // CTAs loop over the units that exist (more units than CTAs)
  int v_tma;                       // V tiles copied whole (else only the kept rows, gathered)
  int v_sep;                       // V tiles in their own region, copied together with K
};

// The streaming decode kernel for every format and head_dim (a.cluster > 1: clusters of
// that many splits share one running maximum); merges in-kernel when every group of splits
// has its own CTAs and `out` is given, else writes one partial per split (the caller then
// launches the combine kernel).  KVQ_ERR_UNSUPPORTED for the sequence-wide maximum when
// the units do not all fit at once.
int launch_decode2(const DecodeArgs& a, cudaStream_t stream);
// CTAs (cluster = 1) or clusters of `cluster` (2, 4 or 8) CTAs of the streaming kernel for
// splits of split_tokens positions resident at once on the current device (0 on error or
// if none fits).
int decode2_capacity(int fmt, int head_dim, int cluster, int split_tokens);

}  // namespace kvq
