"""Single-token decode attention, dense and sparse-V (oracle side; test infrastructure only).

All arithmetic in fp64 on the dequantized cache (``oracle.quant``).

Dense (the tau = 0 definition):
    s_j = (q . k_hat_j) * sm_scale,  w_j = exp(s_j - M) / sum_i exp(s_i - M),
    out = sum_j w_j v_hat_j.

Sparse V, schedule-exact (tproger page, section "Решение — не ускорять, а
пропускать": the softmax weights come from K before V is touched, and a
position whose weight is below the threshold has its V dequantization and
accumulation skipped entirely; section "FAQ": K is always processed).
The context of one (sequence, KV head) is cut into splits of ``split_len``
positions, [0, L), [L, 2L), ...; each split is one flash-decoding work unit:
    1. K pass: every K tile of the split is dequantized and scored, and folded
       into the running maximum m (so when V work starts, m is the maximum over
       the split's scores);
    2. weights p_j = exp(s_j - m); the denominator l = sum_j p_j runs over every
       position, skipped or not (only V work is skipped);
    3. V pass: position j contributes p_j v_hat_j iff p_j >= tau; otherwise its
       V is neither dequantized nor accumulated.
Optionally (``share`` > 1) the running maximum that decides the skips is the
one over a group of ``share`` consecutive splits of the same (sequence, KV head)
whose K passes have all finished before V work starts: every split of the group
uses m = max over the group's scores for its weights, its l and its skip test.
This is still a maximum over already-scored K, so m <= M and the skipped-mass
bound below holds unchanged.
Splits are merged by the log-sum-exp rule:
    M = max_s m_s,  out = sum_s e^{m_s - M} o_s / sum_s e^{m_s - M} l_s.
With tau = 0 every position is kept and the result equals dense attention.
The skip decision is a per (position, head) one; a V row is read when any head
of the query group keeps the position.

Query grouping (GQA): query head h reads KV head floor(h / G), G = Hq / Hkv.
"""
from __future__ import annotations

import numpy as np

from . import quant as Q


def scores(q: np.ndarray, k_hat: np.ndarray, sm_scale: float) -> np.ndarray:
    """q [G, D], k_hat [N, D] -> s [G, N] (fp64)."""
    return (np.asarray(q, dtype=np.float64) @ np.asarray(k_hat, dtype=np.float64).T) * sm_scale


def dense_attention(q, k_hat, v_hat, sm_scale):
    """Return (out [G, D], weights [G, N])."""
    s = scores(q, k_hat, sm_scale)
    if s.shape[1] == 0:
        return np.zeros((s.shape[0], np.asarray(v_hat).shape[-1])), s
    M = s.max(axis=1, keepdims=True)
    e = np.exp(s - M)
    w = e / e.sum(axis=1, keepdims=True)
    return w @ np.asarray(v_hat, dtype=np.float64), w


def split_bounds(n: int, split_len: int):
    return [(a, min(a + split_len, n)) for a in range(0, n, split_len)]


def combine(o: np.ndarray, m: np.ndarray, l: np.ndarray) -> np.ndarray:
    """Log-sum-exp merge.  o [S, G, D] (unnormalized), m [S, G], l [S, G] -> out [G, D]."""
    if o.shape[0] == 0:
        return np.zeros(o.shape[1:])
    M = m.max(axis=0)                           # [G]
    alpha = np.exp(m - M[None, :])              # [S, G]
    num = (alpha[:, :, None] * o).sum(axis=0)
    den = (alpha * l).sum(axis=0)
    return num / den[:, None]


def sparse_v_attention(q, k_hat, v_hat, sm_scale, tau, split_len, share=1):
    """Schedule-exact sparse-V attention for one (sequence, KV head) group.

    ``share``: number of consecutive splits whose K passes share one running
    maximum for the skip test (1 = each split uses its own).

    Returns a dict: out [G, D]; per-split o, m, l; keep [G, N] (bool);
    n_skipped (pairs); v_rows_read / v_rows_skipped (positions); skipped_mass [G]
    (final-normalized weight of the skipped pairs).
    """
    q = np.asarray(q, dtype=np.float64)
    k_hat = np.asarray(k_hat, dtype=np.float64)
    v_hat = np.asarray(v_hat, dtype=np.float64)
    G, D = q.shape
    N = k_hat.shape[0]
    keep = np.zeros((G, N), dtype=bool)
    s_all = np.zeros((G, N))
    os_, ms, ls = [], [], []
    bounds = split_bounds(N, split_len)
    group_max = []
    for g0 in range(0, len(bounds), share):
        a0, b0 = bounds[g0][0], bounds[min(g0 + share, len(bounds)) - 1][1]
        group_max.append(scores(q, k_hat[a0:b0], sm_scale).max(axis=1))
    for si, (a, b) in enumerate(bounds):
        # 1. K pass over the split: scores and the running maximum (over the
        #    split, or over its group of splits when they share it).
        s = scores(q, k_hat[a:b], sm_scale)
        m = group_max[si // share]
        # 2. weights relative to the running maximum; all of them enter l.
        p = np.exp(s - m[:, None])
        l = p.sum(axis=1)
        # 3. V pass: kept positions only.
        kp = p >= tau
        o = (p * kp) @ v_hat[a:b]
        keep[:, a:b] = kp
        s_all[:, a:b] = s
        os_.append(o)
        ms.append(m)
        ls.append(l)
    if N == 0:
        out = np.zeros((G, D))
        mass = np.zeros(G)
    else:
        o_arr, m_arr, l_arr = np.stack(os_), np.stack(ms), np.stack(ls)
        out = combine(o_arr, m_arr, l_arr)
        M = s_all.max(axis=1, keepdims=True)
        e = np.exp(s_all - M)
        mass = (e * ~keep).sum(axis=1) / e.sum(axis=1)
    rows_read = int(keep.any(axis=0).sum())
    return {
        "out": out,
        "o": os_, "m": ms, "l": ls,
        "keep": keep,
        "n_pairs": G * N,
        "n_skipped": int((~keep).sum()),
        "v_rows_read": rows_read,
        "v_rows_skipped": N - rows_read,
        "skipped_mass": mass,
    }


def decode_step(fmt, q16, k16, v16, seq_lens, num_kv_heads, sm_scale, tau, split_len,
                signs=None, codebook16=None, with_dense=True, groups=None, share=1):
    """Whole decode step on the logical (unpaged) cache.

    q16 [B, Hq, D] fp16; k16, v16 [T, Hkv, D] fp16 (sequences concatenated).
    The cache is quantized with the oracle's own quantizers and dequantized in
    fp64; for ``lut4`` attention runs in the rotated domain (the query is
    rotated with R = c H diag(s) in fp64) and the output is rotated back with R^T.

    ``groups``: optional list of (b, kv_head) to evaluate (others left as NaN).
    ``share``: splits per shared running maximum (see ``sparse_v_attention``).
    Returns dict with out_sparse [B, Hq, D], out_dense [B, Hq, D] (if asked),
    skipped_mass [B, Hq], vmax [B, Hkv] (max |v_hat|), and summed counters.
    """
    B, Hq, D = q16.shape
    Hkv = num_kv_heads
    G = Hq // Hkv
    offs = np.concatenate([[0], np.cumsum(seq_lens)]).astype(np.int64)
    out_s = np.full((B, Hq, D), np.nan)
    out_d = np.full((B, Hq, D), np.nan) if with_dense else None
    mass = np.full((B, Hq), np.nan)
    vmax = np.full((B, Hkv), np.nan)
    totals = dict(n_pairs=0, n_skipped=0, v_rows_read=0, v_rows_skipped=0)
    if groups is None:
        groups = [(b, h) for b in range(B) for h in range(Hkv)]
    for b, h in groups:
        ks = k16[offs[b]:offs[b + 1], h]
        vs = v16[offs[b]:offs[b + 1], h]
        kc, ksc = Q.quantize(fmt, ks, signs, codebook16)
        vc, vsc = Q.quantize(fmt, vs, signs, codebook16)
        k_hat = Q.dequantize(fmt, kc, ksc, codebook16)
        v_hat = Q.dequantize(fmt, vc, vsc, codebook16)
        qg = q16[b, h * G:(h + 1) * G].astype(np.float64)
        if fmt == "lut4":
            qg = Q.rotate_f64(qg, signs)
        r = sparse_v_attention(qg, k_hat, v_hat, sm_scale, tau, split_len, share)
        o = r["out"]
        if with_dense:
            od, _ = dense_attention(qg, k_hat, v_hat, sm_scale)
        if fmt == "lut4":
            o = Q.unrotate_f64(o, signs)
            if with_dense:
                od = Q.unrotate_f64(od, signs)
        out_s[b, h * G:(h + 1) * G] = o
        if with_dense:
            out_d[b, h * G:(h + 1) * G] = od
        mass[b, h * G:(h + 1) * G] = r["skipped_mass"]
        vmax[b, h] = np.abs(v_hat).max() if v_hat.size else 0.0
        for key in totals:
            totals[key] += r[key]
    res = dict(out_sparse=out_s, skipped_mass=mass, vmax=vmax, **totals)
    if with_dense:
        res["out_dense"] = out_d
    return res
