"""Two-pass K filtering (tproger page, "FAQ": skipping K as well is left as future work):
how much a sound first pass over coarse K could prune, on the 32K and the 8-stream paged
q4_0 workloads.  Host only; the quantizers are the oracle's.

A first pass may skip a position's exact K work only if an upper bound on its score
proves the skip: ub(s_hj) < M_h + ln(tau) for the maximum M_h that the skip test uses
(here the final maximum of the whole sequence, the most favourable case).  K is read per
row, and one row serves every query head of the GQA group, so a row's bytes are saved
only when the bound holds for all heads of the group.

Bounds, with q4_0 x_i = (c_i - 8) d_b for element i of 32-element block b:
  (i)  scale only:   |q . k| <= sum_b |d_b| 8 sum_{i in b} |q_i|
  (ii) 2-bit coarse: the top two bits of each code, c ~ 4 (c >> 2) + 2, leave an error
       |c - c~| <= 2, so q . k <= q . k~ + sum_b 2 |d_b| sum_{i in b} |q_i|
These numbers back the decision not to build the coarse pass: (i) proves nothing, and
(ii) proves most pairs but few rows, so even a bit-sliced cache layout (the two high bits
of every code in one plane, read by the coarse pass, the two low bits in another, read
only for unpruned rows: 40 + 32 bytes per row instead of 72) would save under a tenth of
the K bytes, at the cost of a dependent pass in a latency-bound step.
"""
import math

import numpy as np
import pytest

import workloads as W
from oracle import quant as Q


def _prune_stats(name):
    wl = W.WORKLOADS[name]
    inp = W.generate(wl)
    G, D, Hkv = wl.group, wl.head_dim, wl.num_kv_heads
    sm = 1.0 / math.sqrt(D)
    thr = math.log(1e-6)
    offs = inp.seq_offsets()
    n = dict(pairs=0, rows=0, exact=0, p_scale=0, p_coarse=0, r_scale=0, r_coarse=0)
    dropped_l = 0.0
    for b in range(wl.batch):
        for h in range(Hkv):
            k = inp.k[offs[b]:offs[b + 1], h]
            q = inp.q[b, h * G:(h + 1) * G].astype(np.float64)
            codes, scales = Q.quantize_q4_0(k)
            s = (q @ Q.dequantize_q4_0(codes, scales).T) * sm           # exact scores [G, N]
            M = s.max(axis=1, keepdims=True)
            d = np.abs(scales.astype(np.float64))                       # [N, D/32]
            qa = np.abs(q).reshape(G, D // 32, 32).sum(-1)              # [G, D/32]
            per_block = (d @ qa.T).T * sm                               # [G, N]
            ub_scale = 8.0 * per_block
            c = codes.reshape(len(k), D).astype(np.int64)
            k_coarse = ((((c >> 2) << 2) + 2 - 8).astype(np.float64).reshape(len(k), D // 32, 32)
                        * scales.astype(np.float64)[..., None]).reshape(len(k), D)
            ub_coarse = (q @ k_coarse.T) * sm + 2.0 * per_block
            # the bounds are sound: never below the exact score
            assert np.all(ub_scale >= s - 1e-9) and np.all(ub_coarse >= s - 1e-9)
            ps, pc = ub_scale < M + thr, ub_coarse < M + thr
            n["pairs"] += s.size
            n["rows"] += s.shape[1]
            n["exact"] += int((s < M + thr).sum())
            n["p_scale"] += int(ps.sum())
            n["p_coarse"] += int(pc.sum())
            n["r_scale"] += int(ps.all(axis=0).sum())
            n["r_coarse"] += int(pc.all(axis=0).sum())
            e = np.exp(s - M)
            dropped_l = max(dropped_l, float(((e * pc).sum(1) / e.sum(1)).max()))
    return n, dropped_l


@pytest.mark.parametrize("name", ["gqa_32k_q4", "paged_b8_q4"])
def test_coarse_k_bounds_prune_pairs_but_few_rows(name):
    n, dropped_l = _prune_stats(name)
    exact = n["exact"] / n["pairs"]
    assert exact > 0.99                      # what the exact scores skip (sequence maximum)
    assert n["p_scale"] == 0                 # (i): the scale-only bound proves nothing
    assert n["r_scale"] == 0
    pairs_c, rows_c = n["p_coarse"] / n["pairs"], n["r_coarse"] / n["rows"]
    assert 0.6 < pairs_c < 0.8               # (ii) proves most (position, head) pairs ...
    assert rows_c < 0.2                      # ... but few whole rows of the 8-head group
    # K bytes per row under the bit-sliced layout (coarse plane 32 code bytes + 8 scale
    # bytes for every row, fine plane 32 bytes for the rows it cannot prune) against 72
    sliced = 40.0 + (1.0 - rows_c) * 32.0
    assert 1.0 - sliced / 72.0 < 0.1
    # dropping the pruned positions from the denominator would move l by at most this
    assert dropped_l < 1e-4
