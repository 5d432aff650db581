"""kvq_decode_attn_noalloc through the C ABI: against the fp64 oracle and against the
regular entry point (kvq_decode_attn with a caller-provided workspace).

Callers that cannot allocate device memory while decoding (a serving runtime that
plans all of its buffers up front, or code confined to a fixed memory pool) use
kvq_decode_attn_noalloc, which keeps the split partials in a static array owned by
the library.  Two calls in a row, on different problems, must each give the oracle's
result within the parity tolerance, and the regular path's result within it too, so
stale scratch contents from the first call cannot leak into the second.  Faults the
kernel detects must reach the caller through kvq_noalloc_read_flags, and a request
too large for the scratch must be refused before anything is launched.  This file is
collected last on purpose.
"""
import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

import workloads as W  # noqa: E402
from tests.gpu_helpers import REL_TOL, check_parity, run_oracle  # noqa: E402


def _setup(wl):
    import quantized_kv_cache_split_b200 as K
    inp = W.generate(wl)
    dev = torch.device("cuda")
    cache = K.QuantizedKVCache(wl.fmt, wl.head_dim, wl.num_kv_heads, inp.page_size, inp.num_pages,
                               dev)
    cache.write(torch.from_numpy(inp.k).to(dev), torch.from_numpy(inp.v).to(dev),
                torch.from_numpy(inp.slots).to(dev))
    args = dict(q=torch.from_numpy(inp.q).to(dev), seq=torch.from_numpy(inp.seq_lens).to(dev),
                pt=None if inp.page_table is None else torch.from_numpy(inp.page_table).to(dev),
                max_seq=int(inp.seq_lens.max()))
    return inp, cache, args


def test_noalloc_matches_oracle_and_workspace_path_on_two_calls():
    import quantized_kv_cache_split_b200 as K
    problems = [
        W.WORKLOADS["gqa_32k_q4"],
        W.shrink(W.WORKLOADS["paged_b8_q8"], [3000, 64, 0, 1500, 777], n_planted=8),
    ]
    for wl in problems:
        inp, cache, a = _setup(wl)
        D, B, Hq = wl.head_dim, wl.batch, wl.num_q_heads
        sm = float(np.float32(1.0 / math.sqrt(D)))
        st_ref = torch.zeros(4, dtype=torch.int64, device="cuda")
        ref = cache.attention(a["q"], a["seq"], a["max_seq"], a["pt"], inp.max_pages, tau=1e-6,
                              sm_scale=sm, stats=st_ref)
        out = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
        st = torch.zeros(4, dtype=torch.int64, device="cuda")
        K.kvq_decode_attn_noalloc(cache.desc, a["q"], B, Hq, cache.k_codes, cache.k_scales,
                                  cache.v_codes, cache.v_scales, a["pt"], inp.max_pages, a["seq"],
                                  a["max_seq"], sm, 1e-6, 0, out, stats=st)
        torch.cuda.synchronize()
        assert not torch.isnan(out).any()
        assert K.kvq_noalloc_read_flags() == 0
        # against the oracle, under the schedule the library resolved for this request
        L = K.kvq_resolve_split(cache.desc, B, Hq, a["max_seq"], 0)
        g = dict(out=out.cpu().numpy().astype(np.float64), stats=st.cpu().numpy())
        check_parity(inp, g, run_oracle(inp, 1e-6, L), 1e-6)
        # against the regular entry point
        vmax = float(np.abs(inp.v.astype(np.float32)).max())
        err = (out - ref).abs().max().item()
        assert err <= REL_TOL * vmax, (wl.name, err)
        assert torch.equal(st, st_ref)


def test_noalloc_reports_device_faults():
    # a sequence length beyond what its pages hold is clamped and flagged by the kernel;
    # the flag reaches the caller through the scratch's flag word, and the next clean
    # call clears it
    import quantized_kv_cache_split_b200 as K
    wl = W.shrink(W.WORKLOADS["gqa_4k_q8"], [300], n_planted=2)
    inp, cache, a = _setup(wl)
    sm = float(np.float32(1.0 / math.sqrt(128)))
    out = torch.empty((1, 32, 128), dtype=torch.float32, device="cuda")
    bad_seq = torch.tensor([inp.page_size + 64], dtype=torch.int32, device="cuda")
    K.kvq_decode_attn_noalloc(cache.desc, a["q"], 1, 32, cache.k_codes, cache.k_scales,
                              cache.v_codes, cache.v_scales, None, 1, bad_seq, inp.page_size + 64,
                              sm, 1e-6, 0, out)
    assert K.kvq_noalloc_read_flags() & K.KVQ_FLAG_BAD_SEQLEN
    K.kvq_decode_attn_noalloc(cache.desc, a["q"], 1, 32, cache.k_codes, cache.k_scales,
                              cache.v_codes, cache.v_scales, None, 1, a["seq"], a["max_seq"],
                              sm, 1e-6, 0, out)
    assert K.kvq_noalloc_read_flags() == 0


def test_noalloc_rejects_requests_beyond_its_scratch():
    # 32 query heads x 512 splits of 64 positions need ~8.8 MB of partials, above the 8 MiB
    # scratch.  Every pointer is a real device buffer of the request's size, so even a call
    # that got past the check would read valid memory; the output must stay untouched.
    import quantized_kv_cache_split_b200 as K
    n, Hkv, Hq, D = 32768, 4, 32, 128
    dev = torch.device("cuda")
    cache = K.QuantizedKVCache("q8_0", D, Hkv, n, 1, dev)
    q = torch.zeros((1, Hq, D), dtype=torch.float16, device=dev)
    seq = torch.tensor([n], dtype=torch.int32, device=dev)
    out = torch.full((1, Hq, D), 7.0, dtype=torch.float32, device=dev)
    L = K.kvq_resolve_split(cache.desc, 1, Hq, n, 64)
    assert K.kvq_workspace_size(1, Hq, D, n, L) > K.KVQ_NOALLOC_SCRATCH_BYTES
    st = K.kvq_decode_attn_noalloc(cache.desc, q, 1, Hq, cache.k_codes, cache.k_scales,
                                   cache.v_codes, cache.v_scales, None, 1, seq, n,
                                   1.0 / math.sqrt(D), 1e-6, 64, out, check=False)
    assert st == K.KVQ_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())
