"""kvq_decode_attn_noalloc against the regular workspace path, through the C ABI.

Callers that cannot allocate device memory while decoding (a serving runtime that
plans all of its buffers up front, or code confined to a fixed memory pool) use
kvq_decode_attn_noalloc, which keeps the split partials in a static array owned by
the library.  Two calls in a row, on different problems, must give the same output
as kvq_decode_attn + kvq_combine with a caller-provided workspace (so stale scratch
contents from the first call cannot leak into the second), within the tolerance the
parity tests use.  This file is collected last on purpose.
"""
import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

import workloads as W  # noqa: E402
from tests.gpu_helpers import REL_TOL  # noqa: E402


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


def test_noalloc_matches_workspace_path_on_two_calls():
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
        vmax = float(np.abs(inp.v.astype(np.float32)).max())
        err = (out - ref).abs().max().item()
        assert err <= REL_TOL * vmax, (wl.name, err)
        assert torch.equal(st, st_ref)
        assert not torch.isnan(out).any()


def test_noalloc_rejects_requests_beyond_its_scratch():
    import quantized_kv_cache_split_b200 as K
    desc = K.make_desc("q8_0", 128, 8, 64, 1 << 16)
    # 256 sequences x 64 heads x 1024 splits of partials is far above the static scratch
    st = K.kvq_decode_attn_noalloc(desc, 1 << 20, 256, 64, 1 << 20, 1 << 20, 1 << 20, 1 << 20,
                                   1 << 20, 1024, 1 << 20, 65536, 0.088, 1e-6, 64, 1 << 20,
                                   check=False)
    assert st == K.KVQ_ERR_WORKSPACE
