"""GPU parity: the CUDA library (through the C ABI) against the fp64 oracle on
the same seeded inputs.  Quantized planes must match bit for bit; attention
outputs must satisfy the error bound of the method; skip counters must match
the oracle's under the same split schedule within 0.1%."""
import functools
import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

import workloads as W  # noqa: E402
from oracle import quant as OQ  # noqa: E402
from tests.gpu_helpers import check_parity, codebook_for, run_library, run_oracle  # noqa: E402


# ------------------------------------------------------------------ quantizers: bit-exact

def _special_vectors(rng, n, hkv, D):
    x = (rng.standard_normal((n, hkv, D)) * rng.choice([0.01, 1.0, 30.0], (n, hkv, 1))).astype(np.float16)
    x[0] = 0                                    # all-zero vector / blocks
    x[1, :, :] = 1.5                            # |x| ties everywhere
    x[1, :, 1::2] = -1.5
    x[2, :, :32] = np.float16(6e-5)             # subnormal-range values
    x[3, :, 5] = np.float16(-60000.0)           # one huge element
    x[4, :, :] = np.arange(D, dtype=np.float16) - D // 2
    return x


@pytest.mark.parametrize("fmt", ["q8_0", "q4_0", "lut4", "nvfp4"])
@pytest.mark.parametrize("D", [64, 128])
def test_quantize_bit_exact(fmt, D):
    import quantized_kv_cache_split_b200 as K
    rng = np.random.Generator(np.random.PCG64(77))
    hkv, P, npages, n = 2, 64, 6, 333
    x = _special_vectors(rng, n, hkv, D)
    slots = rng.permutation(npages * P)[:n].astype(np.int32)
    dev = torch.device("cuda")
    cb16 = codebook_for(D) if fmt == "lut4" else None
    signs = np.where(rng.random(D) < 0.5, -1, 1).astype(np.int8) if fmt == "lut4" else None
    cache = K.QuantizedKVCache(fmt, D, hkv, P, npages, dev,
                               None if cb16 is None else torch.from_numpy(cb16.view(np.int16).copy()),
                               None if signs is None else torch.from_numpy(signs))
    xt = torch.from_numpy(x).to(dev)
    cache.write(xt, xt, torch.from_numpy(slots).to(dev))
    torch.cuda.synchronize()
    codes = cache.k_codes.cpu().numpy()
    scales = cache.k_scales.cpu().numpy()
    page, off = slots // P, slots % P
    for h in range(hkv):
        got_c = codes[page, h, off]
        got_s = scales[page, h, off]
        c, s = OQ.quantize(fmt, x[:, h], signs, cb16)
        want_c = c.astype(np.int8).view(np.uint8) if fmt == "q8_0" else OQ.pack_nibbles(c)
        assert np.array_equal(got_c, want_c), f"codes differ at {np.argwhere(got_c != want_c)[:5]}"
        want_s = s if fmt == "nvfp4" else s.astype(np.float16).view(np.uint16)  # nvfp4: raw words
        assert np.array_equal(got_s.view(np.uint16), want_s), "scales"
    # the writer quantizes K and V in one launch (the second plane pair): same bytes
    assert np.array_equal(cache.v_codes.cpu().numpy(), codes)
    assert np.array_equal(cache.v_scales.cpu().numpy().view(np.uint16), scales.view(np.uint16))


# ------------------------------------------------------------------ attention parity

SMALL = [
    ("tiny_q8_d64", 1e-6, 0), ("tiny_q8_d64", 0.0, 0), ("tiny_q8_d64", 1e-6, 64),
    ("gqa_4k_q8", 1e-6, 0), ("gqa_4k_q8", 0.0, 0), ("gqa_4k_q8", 1e-6, 1024),
    ("lut_4k", 1e-6, 0), ("lut_4k", 0.0, 0),
]


@pytest.mark.parametrize("name,tau,split", SMALL)
def test_decode_parity_small(name, tau, split):
    wl = W.WORKLOADS[name]
    inp = W.generate(wl)
    cb = codebook_for(wl.head_dim) if wl.fmt == "lut4" else None
    g = run_library(inp, tau, split, cb)
    o = run_oracle(inp, tau, g["split"], cb)
    check_parity(inp, g, o, tau)
    assert g["flags"] == 0


@pytest.mark.parametrize("name,tau,split", [
    ("tiny_q8_d64", 1e-6, 64), ("gqa_4k_q8", 1e-6, 0), ("gqa_4k_q8", 1e-6, 256), ("lut_4k", 1e-6, 0),
    ("lut_4k", 1e-2, 128)])
def test_decode_parity_shared_max(name, tau, split):
    # the splits of a cluster share one running maximum for the skip test
    wl = W.WORKLOADS[name]
    inp = W.generate(wl)
    cb = codebook_for(wl.head_dim) if wl.fmt == "lut4" else None
    g = run_library(inp, tau, split, cb, max_scope="cluster")
    assert g["share"] > 1
    o = run_oracle(inp, tau, g["split"], cb, share=g["share"])
    check_parity(inp, g, o, tau)
    assert g["flags"] == 0


@pytest.mark.parametrize("name,tau,split", [
    ("tiny_q8_d64", 1e-6, 64), ("gqa_4k_q8", 1e-6, 0), ("lut_4k", 1e-6, 0), ("lut_4k", 1e-2, 512),
    ("gqa_4k_q8", 0.0, 256)])
def test_decode_parity_sequence_max(name, tau, split):
    # every split uses the maximum over all splits of its sequence (the final maximum)
    wl = W.WORKLOADS[name]
    inp = W.generate(wl)
    cb = codebook_for(wl.head_dim) if wl.fmt == "lut4" else None
    g = run_library(inp, tau, split, cb, max_scope="sequence")
    o = run_oracle(inp, tau, g["split"], cb, share=g["share"])
    check_parity(inp, g, o, tau)
    assert g["flags"] == 0


def test_sequence_max_rejects_requests_beyond_one_round():
    # more splits than CTAs that run at once: the maxima cannot be exchanged in one launch
    import quantized_kv_cache_split_b200 as K
    desc = K.make_desc("q8_0", 128, 8, 4096, 64)
    fake = 1 << 20  # never dereferenced: the call is refused before any launch
    st = K.kvq_decode_attn(desc, fake, 64, 32, fake, fake, fake, fake, None, 1, fake, 4096, 0.088,
                           1e-6, 64, fake, 1 << 40, options=K.KVQ_OPT_GLOBAL_MAX, check=False)
    assert st == K.KVQ_ERR_UNSUPPORTED


@pytest.mark.parametrize("name,tau", [("gqa_4k_q8", 1e-6), ("lut_4k", 0.0), ("tiny_q8_d64", 1e-6)])
def test_combine_kernel_matches_in_kernel_merge(name, tau):
    # kvq_combine over the workspace partials gives what the in-kernel merge gives
    wl = W.WORKLOADS[name]
    inp = W.generate(wl)
    cb = codebook_for(wl.head_dim) if wl.fmt == "lut4" else None
    g1 = run_library(inp, tau, 0, cb, fused=True)
    g2 = run_library(inp, tau, 0, cb, fused=False)
    o = run_oracle(inp, tau, g1["split"], cb)
    check_parity(inp, g2, o, tau)
    vmax = np.abs(inp.v.astype(np.float32)).max()
    assert np.max(np.abs(g1["out"] - g2["out"])) <= 1e-5 * vmax


@pytest.mark.parametrize("scope", ["split", "cluster"])
def test_in_kernel_merge_resets_its_counters(scope):
    # back-to-back multi-round calls on one workspace: each must merge exactly once (both
    # scopes merge with the combine kernel after the decode; the additive merge of a
    # single-round launch may change the last bits)
    import quantized_kv_cache_split_b200 as K
    wl = W.shrink(W.WORKLOADS["paged_b8_q4"], [3000, 64, 0, 1500, 777], n_planted=8)
    inp = W.generate(wl)
    g = run_library(inp, 1e-6, 128, max_scope=scope)
    cache = g["cache"]
    dev = torch.device("cuda")
    q = torch.from_numpy(inp.q).to(dev)
    seq = torch.from_numpy(inp.seq_lens).to(dev)
    pt = torch.from_numpy(inp.page_table).to(dev)
    outs = []
    for _ in range(3):
        o = torch.full((wl.batch, wl.num_q_heads, wl.head_dim), float("nan"), device=dev)
        cache.attention(q, seq, int(inp.seq_lens.max()), pt, inp.max_pages, tau=1e-6,
                        sm_scale=float(np.float32(1 / math.sqrt(128))), split_tokens=128, out=o,
                        max_scope=scope)
        outs.append(o.cpu().numpy())
    assert not np.isnan(outs[0]).any()
    vmax = float(np.abs(inp.v.astype(np.float32)).max())
    for o in outs[1:] + [g["out"].astype(np.float32)]:
        np.testing.assert_allclose(o, outs[0], rtol=0, atol=1e-5 * vmax)


def test_exchange_across_request_shapes_on_one_workspace():
    # The splits of a (sequence, KV head) find one another's (m, l) by a launch tag, not by
    # counters at shape-dependent places: requests of different batch sizes alternate on one
    # workspace with no re-init, and each must give what the full request gives for the
    # same sequences.  Every launch adds exactly 2^16 to the launch counter (header bytes
    # 8..15), whatever its grid.
    wl = W.shrink(W.WORKLOADS["paged_b8_q4"], [3000, 64, 0, 1500, 777], n_planted=8)
    inp = W.generate(wl)
    g = run_library(inp, 1e-6, 512)  # every split on its own CTA: the exchange path
    cache = g["cache"]
    dev = torch.device("cuda")
    q = torch.from_numpy(inp.q).to(dev)
    seq = torch.from_numpy(inp.seq_lens).to(dev)
    pt = torch.from_numpy(inp.page_table).to(dev)
    sel = torch.tensor([3, 0], device=dev)
    sm = float(np.float32(1 / math.sqrt(128)))
    vmax = float(np.abs(inp.v.astype(np.float32)).max())
    launches = 1  # run_library's call initialized the workspace and launched once
    for scope in ("split", "sequence", "split"):
        full = cache.attention(q, seq, 3000, pt, inp.max_pages, tau=1e-6, sm_scale=sm,
                               split_tokens=512, max_scope=scope)
        sub = cache.attention(q[sel].contiguous(), seq[sel].contiguous(), 3000, pt[sel].contiguous(),
                              inp.max_pages, tau=1e-6, sm_scale=sm, split_tokens=512, max_scope=scope)
        launches += 2
        np.testing.assert_allclose(sub.cpu().numpy(), full[sel].cpu().numpy(), rtol=0, atol=1e-5 * vmax)
        if scope == "split":
            np.testing.assert_allclose(full.cpu().numpy(), g["out"], rtol=0, atol=1e-5 * vmax)
    assert cache.device_flags() == 0
    header = cache._ws[:16].cpu().numpy()
    assert int(header[8:16].view(np.uint64)[0]) == launches * (1 << 16)


@pytest.mark.parametrize("fmt,tau", [("q4_0", 1e-6), ("q8_0", 0.0)])
def test_decode_parity_many_sequences(fmt, tau):
    # 40 sequences (more than one warp ballot): after the first round the units follow
    # the static list; 64-position splits make several rounds on any device
    rng = np.random.Generator(np.random.PCG64(4040))
    lens = [int(x) for x in rng.integers(0, 600, size=40)]
    lens[3], lens[17] = 0, 1
    wl = W.shrink(W.WORKLOADS["paged_b8_q4"].with_(fmt=fmt), lens, n_planted=4)
    inp = W.generate(wl)
    g = run_library(inp, tau, 64)
    o = run_oracle(inp, tau, g["split"])
    check_parity(inp, g, o, tau)
    assert g["flags"] == 0


def test_bounded_waits_give_up_and_leave_the_context_usable():
    # The exchange poll and the flag wait of the decode kernel, run against entries that
    # never become ready with a 2M-cycle bound: KVQ_FLAG_TIMEOUT, no hang, and the next
    # decode on a fresh workspace is correct.
    import quantized_kv_cache_split_b200 as K
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    K.kvq_workspace_init(ws, ws.numel())
    K.kvq_selftest_wait(ws, ws.numel(), 2_000_000)
    assert K.kvq_read_device_flags(ws) & K.KVQ_FLAG_TIMEOUT
    wl = W.WORKLOADS["tiny_q8_d64"]
    inp = W.generate(wl)
    g = run_library(inp, 1e-6, 64)
    check_parity(inp, g, run_oracle(inp, 1e-6, g["split"]), 1e-6)
    assert g["flags"] == 0


RAGGED_LENS = [1000, 70, 1, 0, 2049, 64, 130, 3001]


@pytest.mark.parametrize("fmt", ["q8_0", "q4_0", "lut4", "nvfp4"])
@pytest.mark.parametrize("tau,split,scope", [(0.0, 128, "split"), (1e-6, 0, "split"), (1e-4, 192, "split"),
                                             (1e-6, 1024, "split"), (1e-6, 128, "cluster"),
                                             (1e-6, 0, "sequence"), (1e-6, 896, "split"), (0.0, 896, "split")])
def test_decode_parity_paged_ragged(fmt, tau, split, scope):
    # split 896 = 14 tiles: the last two tiles are halved between four warps
    base = W.WORKLOADS["paged_b8_q4"].with_(fmt=fmt)
    wl = W.shrink(base, RAGGED_LENS, n_planted=8)
    inp = W.generate(wl)
    cb = codebook_for(wl.head_dim) if fmt == "lut4" else None
    g = run_library(inp, tau, split, cb, max_scope=scope)
    o = run_oracle(inp, tau, g["split"], cb, share=g["share"])
    check_parity(inp, g, o, tau)
    assert g["flags"] == 0


@pytest.mark.parametrize("fmt", ["q8_0", "q4_0", "lut4", "nvfp4"])
@pytest.mark.parametrize("v_fetch", ["kept", "with_k"])
@pytest.mark.parametrize("tau,split,scope", [(1e-6, 0, "split"), (1e-4, 128, "split"), (1e-6, 0, "sequence"),
                                             (1e-2, 64, "cluster")])
def test_decode_parity_v_fetch_policies(fmt, v_fetch, tau, split, scope):
    # V rows copied after the skip test (kept rows only) or together with K (skipped
    # rows left out of the contraction): the same result, the same skip counts, in
    # single-round (split 0) and multi-round (split 128, 64) launches
    base = W.WORKLOADS["paged_b8_q4"].with_(fmt=fmt)
    wl = W.shrink(base, RAGGED_LENS, n_planted=8)
    inp = W.generate(wl)
    cb = codebook_for(wl.head_dim) if fmt == "lut4" else None
    g = run_library(inp, tau, split, cb, max_scope=scope, v_fetch=v_fetch)
    o = run_oracle(inp, tau, g["split"], cb, share=g["share"])
    check_parity(inp, g, o, tau)
    assert g["flags"] == 0


@pytest.mark.parametrize("fmt", ["q8_0", "q4_0", "lut4", "nvfp4"])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (4, 2), (8, 1)])
def test_decode_parity_head_dim_64_and_groups(fmt, hq, hkv):
    wl = W.WORKLOADS["tiny_q8_d64"].with_(fmt=fmt, num_q_heads=hq, num_kv_heads=hkv,
                                          seq_lens=(777, 300), batch=2, n_planted=6)
    inp = W.generate(wl)
    cb = codebook_for(64) if fmt == "lut4" else None
    # the library's V fetch, both explicit policies (tau > 0), and dense
    for tau, split, v_fetch in [(1e-6, 0, "auto"), (1e-6, 0, "kept"), (1e-4, 128, "with_k"), (0.0, 64, "auto")]:
        g = run_library(inp, tau, split, cb, v_fetch=v_fetch)
        o = run_oracle(inp, tau, g["split"], cb)
        check_parity(inp, g, o, tau)


# ------------------------------------------------------------------ full sizes

@pytest.mark.parametrize("name", ["gqa_32k_q4", "lut_32k", "nvfp4_32k"])
@pytest.mark.parametrize("tau,scope", [(1e-6, "split"), (0.0, "split"), (1e-6, "cluster"),
                                       (1e-6, "sequence")])
def test_decode_parity_full_32k(name, tau, scope):
    wl = W.WORKLOADS[name]
    inp = W.generate(wl)
    cb = codebook_for(wl.head_dim) if wl.fmt == "lut4" else None
    g = run_library(inp, tau, 0, cb, max_scope=scope)
    o = run_oracle(inp, tau, g["split"], cb, share=g["share"])
    check_parity(inp, g, o, tau)
    if tau > 0:
        # the workload's point: most weights are skipped
        assert g["stats"][1] > 0.5 * g["stats"][0]


@pytest.mark.parametrize("v_fetch,scope", [("kept", "split"), ("kept", "sequence"), ("with_k", "cluster")])
def test_decode_parity_full_32k_v_fetch(v_fetch, scope):
    # the single-round 32K launch copies V with K by default: the other policy too
    wl = W.WORKLOADS["gqa_32k_q4"]
    inp = W.generate(wl)
    g = run_library(inp, 1e-6, 0, None, max_scope=scope, v_fetch=v_fetch)
    o = run_oracle(inp, 1e-6, g["split"], None, share=g["share"])
    check_parity(inp, g, o, 1e-6)


@functools.lru_cache(maxsize=2)
def _paged_inputs(name):
    return W.generate(W.WORKLOADS[name])


@pytest.mark.parametrize("name", ["paged_b8_q4", "paged_b8_q8"])
@pytest.mark.parametrize("tau", [0.0, 1e-6, 1e-4])
def test_decode_parity_full_paged(name, tau):
    # The 8-stream paged configuration at full size (245,760 positions, 3840 pages) over its
    # tau sweep: every output element of all 32 (sequence, KV head) groups against the
    # oracle, and the skip counters (pairs and V rows) within 0.1% of the oracle's under the
    # same split schedule.
    wl = W.WORKLOADS[name]
    inp = _paged_inputs(name)
    g = run_library(inp, tau, 0)
    o = run_oracle(inp, tau, g["split"])
    check_parity(inp, g, o, tau)
    assert g["flags"] == 0
    if tau > 0:
        assert g["stats"][1] > 0.3 * g["stats"][0]


# ------------------------------------------------------------------ device-side fault reporting

def test_bad_page_index_is_flagged_not_faulted():
    import quantized_kv_cache_split_b200 as K
    wl = W.shrink(W.WORKLOADS["paged_b8_q8"], [200, 100], n_planted=2)
    inp = W.generate(wl)
    inp.page_table[1, 0] = inp.num_pages + 5          # out of range: must not be read
    g = run_library(inp, 1e-6, 0)
    assert g["flags"] & K.KVQ_FLAG_BAD_PAGE


def test_bad_seq_len_is_flagged_and_clamped():
    import quantized_kv_cache_split_b200 as K
    wl = W.shrink(W.WORKLOADS["gqa_4k_q8"], [300], n_planted=2)
    inp = W.generate(wl)
    dev = torch.device("cuda")
    cache = K.QuantizedKVCache("q8_0", 128, 8, inp.page_size, inp.num_pages, dev)
    cache.write(torch.from_numpy(inp.k).to(dev), torch.from_numpy(inp.v).to(dev),
                torch.from_numpy(inp.slots).to(dev))
    seq = torch.tensor([300 + 5000], dtype=torch.int32, device=dev)   # beyond max_seq_len
    cache.attention(torch.from_numpy(inp.q).to(dev), seq, 300, None, 1, tau=1e-6)
    assert cache.device_flags() & K.KVQ_FLAG_BAD_SEQLEN
