"""Pins for the oracle's attention (CPU only): brute force with plain loops,
closed-form special cases, the skipped-mass bound, split invariance, and the
rotation round trip of the LUT format."""
import math

import numpy as np
import pytest

from oracle import attention as A
from oracle import quant as Q
from oracle import codebook as CB
import workloads as W


def _rng(seed=0):
    return np.random.Generator(np.random.PCG64(seed))


def brute_force_attention(q, k, v, scale):
    """Plain Python loops, no numpy reductions."""
    G, D = len(q), len(q[0])
    N = len(k)
    out = []
    for g in range(G):
        s = []
        for j in range(N):
            acc = 0.0
            for d in range(D):
                acc += float(q[g][d]) * float(k[j][d])
            s.append(acc * scale)
        mx = max(s)
        e = [math.exp(x - mx) for x in s]
        tot = sum(e)
        row = []
        for d in range(D):
            row.append(sum(e[j] * float(v[j][d]) for j in range(N)) / tot)
        out.append(row)
    return np.array(out)


def test_dense_matches_brute_force():
    r = _rng(1)
    q = r.standard_normal((3, 8))
    k = r.standard_normal((11, 8)) * 2
    v = r.standard_normal((11, 8))
    out, w = A.dense_attention(q, k, v, 1 / math.sqrt(8))
    np.testing.assert_allclose(out, brute_force_attention(q, k, v, 1 / math.sqrt(8)), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=1e-14)


def test_special_cases():
    r = _rng(2)
    q = r.standard_normal((2, 16))
    v = r.standard_normal((1, 16))
    out, _ = A.dense_attention(q, r.standard_normal((1, 16)), v, 0.25)
    np.testing.assert_allclose(out, np.repeat(v, 2, axis=0), rtol=1e-15)     # single key
    k = np.repeat(r.standard_normal((1, 16)), 9, axis=0)
    v = r.standard_normal((9, 16))
    out, _ = A.dense_attention(q, k, v, 0.25)
    np.testing.assert_allclose(out, np.repeat(v.mean(0, keepdims=True), 2, 0), rtol=1e-13)  # equal keys


@pytest.mark.parametrize("split_len", [1, 3, 16, 64, 1000])
def test_sparse_tau0_equals_dense(split_len):
    r = _rng(3)
    q = r.standard_normal((4, 32))
    k = r.standard_normal((100, 32)) * 3
    v = r.standard_normal((100, 32))
    res = A.sparse_v_attention(q, k, v, 1 / math.sqrt(32), 0.0, split_len)
    dense, _ = A.dense_attention(q, k, v, 1 / math.sqrt(32))
    np.testing.assert_allclose(res["out"], dense, rtol=1e-12, atol=1e-14)
    assert res["n_skipped"] == 0 and res["v_rows_skipped"] == 0


@pytest.mark.parametrize("tau", [1e-6, 1e-4, 1e-2])
@pytest.mark.parametrize("split_len", [8, 37, 200])
def test_skipped_mass_bound_and_error_bound(tau, split_len):
    r = _rng(4)
    q = r.standard_normal((4, 32))
    k = r.standard_normal((300, 32)) * 4
    v = r.standard_normal((300, 32))
    res = A.sparse_v_attention(q, k, v, 1 / math.sqrt(32), tau, split_len)
    dense, w = A.dense_attention(q, k, v, 1 / math.sqrt(32))
    nskip_per_head = (~res["keep"]).sum(axis=1)
    assert (res["skipped_mass"] <= tau * nskip_per_head + 1e-15).all()
    # skipped mass is exactly the dense weight of the skipped pairs
    np.testing.assert_allclose(res["skipped_mass"], (w * ~res["keep"]).sum(1), rtol=1e-10, atol=1e-18)
    vmax = np.abs(v).max()
    err = np.abs(res["out"] - dense)
    assert (err <= res["skipped_mass"][:, None] * vmax * (1 + 1e-9) + 1e-14).all()
    assert res["n_skipped"] > 0


def test_tau_one_keeps_only_split_maxima():
    # closed form: with tau = 1 only p = 1 (the split maximum) survives
    r = _rng(5)
    q = r.standard_normal((2, 16))
    k = r.standard_normal((50, 16))
    v = r.standard_normal((50, 16))
    L = 12
    sc = 0.25
    res = A.sparse_v_attention(q, k, v, sc, 1.0, L)
    s = (q @ k.T) * sc
    for g in range(2):
        num = np.zeros(16)
        den = 0.0
        M = s[g].max()
        for a in range(0, 50, L):
            seg = s[g, a:a + L]
            j = a + int(np.argmax(seg))
            num += math.exp(seg.max() - M) * v[j]
            den += sum(math.exp(x - M) for x in seg)
        np.testing.assert_allclose(res["out"][g], num / den, rtol=1e-12)


def test_combine_identity_and_split_invariance():
    r = _rng(6)
    o = r.standard_normal((1, 3, 8))
    m = r.standard_normal((1, 3))
    l = r.random((1, 3)) + 0.5
    np.testing.assert_allclose(A.combine(o, m, l), o[0] / l[0][:, None], rtol=1e-15)
    # partial sums of one dense problem, merged, equal the dense result
    q = r.standard_normal((3, 8))
    k = r.standard_normal((40, 8))
    v = r.standard_normal((40, 8))
    parts = [(0, 7), (7, 8), (8, 40)]
    os_, ms, ls = [], [], []
    for a, b in parts:
        s = q @ k[a:b].T
        mm = s.max(1)
        p = np.exp(s - mm[:, None])
        os_.append(p @ v[a:b]); ms.append(mm); ls.append(p.sum(1))
    dense, _ = A.dense_attention(q, k, v, 1.0)
    np.testing.assert_allclose(A.combine(np.stack(os_), np.stack(ms), np.stack(ls)), dense, rtol=1e-12)


def test_lut4_rotated_domain_equals_unrotated():
    D = 64
    r = _rng(7)
    s = np.where(r.random(D) < 0.5, -1, 1).astype(np.int8)
    cb = CB.lloyd_max_f16(16, 1 / math.sqrt(D))
    q = r.standard_normal((4, D)).astype(np.float16)
    k = r.standard_normal((70, D)).astype(np.float16)
    v = r.standard_normal((70, D)).astype(np.float16)
    ki, kn = Q.quantize_lut4(k, s, cb)
    vi, vn = Q.quantize_lut4(v, s, cb)
    k_rot = Q.dequantize_lut4(ki, kn, cb)
    v_rot = Q.dequantize_lut4(vi, vn, cb)
    out_rot, _ = A.dense_attention(Q.rotate_f64(q.astype(np.float64), s), k_rot, v_rot, 1 / 8)
    out_rot = Q.unrotate_f64(out_rot, s)
    out_plain, _ = A.dense_attention(q.astype(np.float64), Q.unrotate_f64(k_rot, s),
                                     Q.unrotate_f64(v_rot, s), 1 / 8)
    np.testing.assert_allclose(out_rot, out_plain, rtol=1e-10, atol=1e-12)


def test_decode_step_gqa_grouping_and_paging_independence():
    wl = W.shrink(W.WORKLOADS["gqa_4k_q8"], [200, 70], n_planted=4).with_(page_size=64)
    inp = W.generate(wl)
    res = A.decode_step("q8_0", inp.q, inp.k, inp.v, inp.seq_lens, wl.num_kv_heads,
                        1 / math.sqrt(128), 1e-6, 64)
    G = wl.group
    offs = inp.seq_offsets()
    # brute force on one (b, h): query head 13 reads KV head 13 // G
    b, hq = 1, 13
    kc, ks = Q.quantize_q8_0(inp.k[offs[b]:offs[b + 1], hq // G])
    vc, vs = Q.quantize_q8_0(inp.v[offs[b]:offs[b + 1], hq // G])
    ref = brute_force_attention(inp.q[b, hq:hq + 1].astype(np.float64), Q.dequantize_q8_0(kc, ks),
                                Q.dequantize_q8_0(vc, vs), 1 / math.sqrt(128))
    np.testing.assert_allclose(res["out_dense"][b, hq], ref[0], rtol=1e-10, atol=1e-12)
    assert np.all(np.abs(res["out_sparse"] - res["out_dense"])
                  <= res["skipped_mass"][..., None] * np.repeat(res["vmax"], G, axis=1)[..., None] + 1e-12)


def test_planted_scores_concentrate_attention():
    # the workload recipe: planted keys dominate, most weights fall below 1e-6 at 32K
    wl = W.WORKLOADS["gqa_32k_q4"]
    inp = W.generate(wl)
    G = wl.group
    q = inp.q[0, :G].astype(np.float64)
    k = inp.k[:, 0].astype(np.float64)
    s = (q @ k.T) / math.sqrt(128)
    pos, a = inp.planted[0]
    np.testing.assert_allclose(s[:, pos], np.repeat(a[None], G, 0), rtol=2e-3)
    w = np.exp(s - s.max(1, keepdims=True))
    w /= w.sum(1, keepdims=True)
    assert (w < 1e-6).mean() > 0.9


@pytest.mark.parametrize("fmt", ["q8_0", "q4_0", "lut4"])
def test_decode_step_empty_and_single_position(fmt):
    wl = W.shrink(W.WORKLOADS["paged_b8_q4"].with_(fmt=fmt), [0, 1, 65], n_planted=1)
    inp = W.generate(wl)
    cb = CB.lloyd_max_f16(16, 1 / math.sqrt(128)) if fmt == "lut4" else None
    res = A.decode_step(fmt, inp.q, inp.k, inp.v, inp.seq_lens, wl.num_kv_heads,
                        1 / math.sqrt(128), 1e-6, 64, signs=inp.signs, codebook16=cb)
    assert np.all(res["out_sparse"][0] == 0) and np.all(res["out_dense"][0] == 0)
    # one position: the output is that position's dequantized V
    kc, ks = Q.quantize(fmt, inp.v[0:1, 0], inp.signs, cb)
    v1 = Q.dequantize(fmt, kc, ks, cb)
    if fmt == "lut4":
        v1 = Q.unrotate_f64(v1, inp.signs)
    np.testing.assert_allclose(res["out_sparse"][1, 0], v1[0], rtol=1e-12, atol=1e-12)


def _keep_brute_force(q, k, scale, tau, split_len, share):
    """Keep flags by plain loops: position j of split s is kept for head g iff
    exp(s_gj - m) >= tau, m the maximum over the splits of s's sharing group."""
    G, N = len(q), len(k)
    span = split_len * share
    keep = [[False] * N for _ in range(G)]
    for g in range(G):
        s = [sum(float(q[g][d]) * float(k[j][d]) for d in range(len(q[g]))) * scale for j in range(N)]
        for a in range(0, N, span):
            m = max(s[a:a + span])
            for j in range(a, min(a + span, N)):
                keep[g][j] = math.exp(s[j] - m) >= tau
    return np.array(keep)


@pytest.mark.parametrize("split_len,share", [(8, 1), (8, 3), (5, 4), (16, 100)])
def test_shared_running_max_keep_set_brute_force(split_len, share):
    r = _rng(11)
    q = r.standard_normal((3, 16))
    k = r.standard_normal((90, 16)) * 3
    k[[7, 41, 77]] = q.mean(0) * 6  # a few strong keys so groups differ
    v = r.standard_normal((90, 16))
    res = A.sparse_v_attention(q, k, v, 0.25, 1e-3, split_len, share)
    np.testing.assert_array_equal(res["keep"], _keep_brute_force(q, k, 0.25, 1e-3, split_len, share))
    dense, w = A.dense_attention(q, k, v, 0.25)
    np.testing.assert_allclose(res["skipped_mass"], (w * ~res["keep"]).sum(1), rtol=1e-10, atol=1e-18)
    assert (res["skipped_mass"] <= 1e-3 * (~res["keep"]).sum(1) + 1e-15).all()
    err = np.abs(res["out"] - dense)
    assert (err <= res["skipped_mass"][:, None] * np.abs(v).max() * (1 + 1e-9) + 1e-14).all()


def test_shared_running_max_special_cases():
    r = _rng(12)
    q = r.standard_normal((2, 16))
    k = r.standard_normal((70, 16)) * 3
    v = r.standard_normal((70, 16))
    dense, w = A.dense_attention(q, k, v, 0.25)
    # tau = 0 keeps everything whatever the sharing
    np.testing.assert_allclose(A.sparse_v_attention(q, k, v, 0.25, 0.0, 9, 4)["out"], dense,
                               rtol=1e-12, atol=1e-14)
    # one group covering every split: the skip test uses the final maximum M
    res = A.sparse_v_attention(q, k, v, 0.25, 1e-2, 9, 8)
    s = (q @ k.T) * 0.25
    np.testing.assert_array_equal(res["keep"], np.exp(s - s.max(1, keepdims=True)) >= 1e-2)
    # nested groups only raise the maximum, so they skip at least as much
    n1 = A.sparse_v_attention(q, k, v, 0.25, 1e-2, 9, 1)["n_skipped"]
    n2 = A.sparse_v_attention(q, k, v, 0.25, 1e-2, 9, 2)["n_skipped"]
    n4 = A.sparse_v_attention(q, k, v, 0.25, 1e-2, 9, 4)["n_skipped"]
    assert n1 <= n2 <= n4 <= res["n_skipped"]
