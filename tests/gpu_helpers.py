"""Drive the CUDA library and the oracle on the same generated workload."""
from __future__ import annotations

import math

import numpy as np
import torch

import workloads as W
from oracle import attention as OA
from oracle import codebook as OC
from oracle import quant as OQ

REL_TOL = 2e-3  # |out - oracle| <= REL_TOL * max|V_hat| (+ skipped mass * max|V_hat| vs dense)


def codebook_for(D: int) -> np.ndarray:
    return OC.lloyd_max_f16(16, 1.0 / math.sqrt(D))


def run_library(inp: W.Inputs, tau: float, split_tokens: int = 0, codebook16=None,
                max_scope: str = "split", fused: bool = True, v_fetch: str = "auto"):
    """One decode step through the C ABI.  ``fused``: the merge runs inside the decode
    kernel; otherwise kvq_combine runs it.  ``max_scope``: "split", "cluster" (the
    splits of a cluster share one running maximum; the oracle replays it with share =
    the cluster size) or "sequence" (share = every split).  ``v_fetch``: the V copy
    policy ("auto", "kept", "with_k"), which must not change the result."""
    import quantized_kv_cache_split_b200 as K
    wl = inp.wl
    D, Hkv = wl.head_dim, wl.num_kv_heads
    dev = torch.device("cuda")
    cb = sg = None
    if wl.fmt == "lut4":
        cb = torch.from_numpy(np.asarray(codebook16, dtype=np.float16).view(np.int16).copy())
        sg = torch.from_numpy(inp.signs)
    cache = K.QuantizedKVCache(wl.fmt, D, Hkv, inp.page_size, inp.num_pages, dev, cb, sg)
    if inp.k.shape[0]:
        cache.write(torch.from_numpy(inp.k).to(dev), torch.from_numpy(inp.v).to(dev),
                    torch.from_numpy(inp.slots).to(dev))
    q = torch.from_numpy(inp.q).to(dev)
    seq = torch.from_numpy(inp.seq_lens).to(dev)
    pt = None if inp.page_table is None else torch.from_numpy(inp.page_table).to(dev)
    stats = torch.zeros(4, dtype=torch.int64, device=dev)
    max_seq = int(max(inp.seq_lens.max(), 1))
    out = cache.attention(q, seq, max_seq, pt, inp.max_pages, tau=tau,
                          sm_scale=float(np.float32(1.0 / math.sqrt(D))),
                          split_tokens=split_tokens, stats=stats, max_scope=max_scope,
                          fused=fused, v_fetch=v_fetch)
    torch.cuda.synchronize()
    opts = {"split": 0, "cluster": K.KVQ_OPT_SHARED_MAX, "sequence": K.KVQ_OPT_GLOBAL_MAX}[max_scope]
    L = K.kvq_resolve_split(cache.desc, wl.batch, wl.num_q_heads, max_seq, split_tokens, opts)
    CS = K.kvq_resolve_cluster(cache.desc, wl.batch, wl.num_q_heads, max_seq, split_tokens, opts)
    flags = cache.device_flags()
    return dict(out=out.cpu().numpy().astype(np.float64), stats=stats.cpu().numpy(), split=L,
                cluster=CS, share={"split": 1, "cluster": CS, "sequence": 1 << 30}[max_scope],
                flags=flags, cache=cache)


def run_oracle(inp: W.Inputs, tau: float, split: int, codebook16=None, groups=None, share: int = 1):
    wl = inp.wl
    return OA.decode_step(wl.fmt, inp.q, inp.k, inp.v, inp.seq_lens, wl.num_kv_heads,
                          float(np.float32(1.0 / math.sqrt(wl.head_dim))), float(np.float32(tau)),
                          split, signs=inp.signs, codebook16=codebook16, groups=groups, share=share)


def check_parity(inp: W.Inputs, g: dict, o: dict, tau: float, groups=None):
    """The bar: |gpu - oracle_sparse| <= 2e-3 max|V|; |gpu - dense| <= (2e-3 + mass) max|V|;
    skip counts within 0.1% of the oracle's under the same split schedule."""
    wl = inp.wl
    G = wl.group
    vmax = np.repeat(o["vmax"], G, axis=1)[..., None]            # [B, Hq, 1]
    sel = np.ones(g["out"].shape[:2], dtype=bool)
    if groups is not None:
        sel[:] = False
        for b, h in groups:
            sel[b, h * G:(h + 1) * G] = True
    empty = inp.seq_lens == 0
    err_s = np.abs(g["out"] - np.nan_to_num(o["out_sparse"]))
    err_d = np.abs(g["out"] - np.nan_to_num(o["out_dense"]))
    bound_s = REL_TOL * np.nan_to_num(vmax) + 1e-12
    bound_d = (REL_TOL + np.nan_to_num(o["skipped_mass"])[..., None]) * np.nan_to_num(vmax) + 1e-12
    bad_s = (err_s > bound_s) & sel[..., None]
    bad_d = (err_d > bound_d) & sel[..., None]
    assert not bad_s.any(), (
        f"sparse parity: {bad_s.sum()} elements, max err/vmax "
        f"{np.max(err_s / np.maximum(vmax, 1e-30) * sel[..., None]):.3e}")
    assert not bad_d.any(), f"dense bound: {bad_d.sum()} elements"
    assert np.all(g["out"][empty] == 0)
    if groups is None:
        total = int(inp.seq_lens.sum())
        st = g["stats"]
        assert st[0] == total * wl.num_q_heads                     # every pair scored
        assert st[2] + st[3] == total * wl.num_kv_heads
        tol = max(1, int(math.ceil(1e-3 * o["n_skipped"])))
        assert abs(int(st[1]) - o["n_skipped"]) <= tol, (int(st[1]), o["n_skipped"])
        tol_r = max(1, int(math.ceil(1e-3 * o["v_rows_skipped"])))
        assert abs(int(st[3]) - o["v_rows_skipped"]) <= tol_r, (int(st[3]), o["v_rows_skipped"])
        if tau == 0.0:
            assert st[1] == 0 and st[3] == 0
    return dict(max_err_sparse=float(np.max(err_s / np.maximum(vmax, 1e-30) * sel[..., None])))
