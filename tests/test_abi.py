"""Host-only checks of the C-ABI library: it loads, exports every symbol the
header declares, validates arguments before launching anything, and its host
codebook routine agrees with the oracle.  No compute call needs a GPU here."""
import ctypes
import math
import os
import re

import numpy as np
import pytest

import quantized_kv_cache_split_b200 as K
from quantized_kv_cache_split_b200 import _binding as kb
from oracle import codebook as CB

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvq.h")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = header_functions()
    assert len(names) >= 10
    lib = ctypes.CDLL(kb.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_binding_wraps_every_declared_function():
    for n in header_functions():
        assert hasattr(K, n), n


def test_row_sizes():
    assert K.kvq_code_row_bytes("q8_0", 128) == 128
    assert K.kvq_code_row_bytes("q4_0", 128) == 64
    assert K.kvq_code_row_bytes("lut4", 64) == 32
    assert K.kvq_scale_row_count("q8_0", 128) == 4
    assert K.kvq_scale_row_count("lut4", 128) == 1
    assert K.kvq_code_row_bytes("nvfp4", 128) == 64
    # nvfp4 scale rows: D/16 E4M3 bytes + fp32 vector scale, padded to 8 bytes (fp16 slots)
    assert K.kvq_scale_row_count("nvfp4", 128) == 8 and K.kvq_scale_row_count("nvfp4", 64) == 4
    assert K.kvq_code_row_bytes("q8_0", 96) == 0


@pytest.mark.parametrize("D", [64, 128])
def test_library_codebook_equals_oracle(D):
    lib_cb = K.kvq_lloyd_max_codebook(16, 1 / math.sqrt(D))
    ora_cb = CB.lloyd_max_f16(16, 1 / math.sqrt(D))
    assert (lib_cb.view(np.uint16) == ora_cb.view(np.uint16)).all()


def test_status_strings():
    assert K.kvq_status_string(0) == "ok"
    assert "workspace" in K.kvq_status_string(K.KVQ_ERR_WORKSPACE)


FAKE = 1 << 20  # aligned dummy device pointer: never dereferenced on these paths


def _desc(**kw):
    a = dict(fmt="q8_0", head_dim=128, num_kv_heads=4, page_size=64, num_pages=8)
    a.update(kw)
    return K.make_desc(a["fmt"], a["head_dim"], a["num_kv_heads"], a["page_size"], a["num_pages"],
                       a.get("codebook"), a.get("signs"))


def test_split_resolution_and_workspace_size():
    d = _desc()
    assert K.kvq_resolve_split(d, 1, 32, 4096, 100) == 128
    assert K.kvq_resolve_split(d, 1, 32, 4096, 5000) == K.KVQ_MAX_SPLIT_TOKENS
    assert K.kvq_resolve_split(d, 1, 32, 4096, 1) == 64
    ws = K.kvq_workspace_size(2, 32, 128, 1000, 128)
    # header, cleared-rows flags and exchange arrival words (u64 each) per (sequence,
    # head) rounded to 256, then per partial the tagged (m, l) exchange entry and (o, m, l)
    assert ws == 256 + 1024 + 2 * 32 * 8 * (16 + (128 + 2) * 4)
    assert K.kvq_workspace_size(3, 32, 128, 1000, 128) == 256 + 1536 + 3 * 32 * 8 * (16 + (128 + 2) * 4)


@pytest.mark.parametrize("kw,code", [
    (dict(fmt=7), K.KVQ_ERR_UNSUPPORTED),
    (dict(head_dim=96), K.KVQ_ERR_UNSUPPORTED),
    (dict(page_size=48), K.KVQ_ERR_UNSUPPORTED),
    (dict(num_kv_heads=0), K.KVQ_ERR_INVALID_ARG),
    (dict(fmt="lut4"), K.KVQ_ERR_INVALID_ARG),       # no codebook / signs
])
def test_quantize_rejects_bad_descriptors(kw, code):
    d = _desc(**kw) if "fmt" not in kw or isinstance(kw["fmt"], str) else K.KvqCacheDesc(
        kw["fmt"], 128, 4, 64, 8, None, None)
    assert K.kvq_quantize(d, FAKE, 4, None, FAKE, FAKE, 0, check=False) == code


def test_quantize_rejects_bad_pointers():
    d = _desc()
    assert K.kvq_quantize(d, None, 4, None, FAKE, FAKE, stream=0, check=False) == K.KVQ_ERR_INVALID_ARG
    assert K.kvq_quantize(d, FAKE, 4, None, FAKE + 8, FAKE, 0, check=False) == K.KVQ_ERR_INVALID_ARG
    assert K.kvq_quantize(d, FAKE, -1, None, FAKE, FAKE, stream=0, check=False) == K.KVQ_ERR_INVALID_ARG
    assert K.kvq_quantize(d, FAKE, 0, None, FAKE, FAKE, stream=0, check=False) == K.KVQ_OK
    # more tokens than the cache holds, with identity slots
    assert K.kvq_quantize(d, FAKE, 8 * 64 + 1, None, FAKE, FAKE, stream=0, check=False) == K.KVQ_ERR_INVALID_ARG


def test_quantize_kv_rejects_bad_pointers():
    # the K + V append: the checks of two kvq_quantize calls, before any launch
    d = _desc()
    q = lambda *a: K.kvq_quantize_kv(d, *a, stream=0, check=False)  # noqa: E731
    assert q(FAKE, None, 4, None, FAKE, FAKE, FAKE, FAKE) == K.KVQ_ERR_INVALID_ARG
    assert q(None, FAKE, 4, None, FAKE, FAKE, FAKE, FAKE) == K.KVQ_ERR_INVALID_ARG
    assert q(FAKE, FAKE, 4, None, FAKE, FAKE, FAKE + 8, FAKE) == K.KVQ_ERR_INVALID_ARG
    assert q(FAKE, FAKE + 1, 4, None, FAKE, FAKE, FAKE, FAKE) == K.KVQ_ERR_INVALID_ARG
    assert q(FAKE, FAKE, -1, None, FAKE, FAKE, FAKE, FAKE) == K.KVQ_ERR_INVALID_ARG
    assert q(FAKE, FAKE, 0, None, FAKE, FAKE, FAKE, FAKE) == K.KVQ_OK
    assert q(FAKE, FAKE, 8 * 64 + 1, None, FAKE, FAKE, FAKE, FAKE) == K.KVQ_ERR_INVALID_ARG
    assert K.kvq_quantize_kv(K.KvqCacheDesc(7, 128, 4, 64, 8, None, None),
                             FAKE, FAKE, 4, None, FAKE, FAKE, FAKE, FAKE, 0, check=False) == K.KVQ_ERR_UNSUPPORTED


def test_selftest_wait_rejects_bad_arguments():
    assert K.kvq_selftest_wait(None, 256, 1000, 0, check=False) == K.KVQ_ERR_INVALID_ARG
    assert K.kvq_selftest_wait(FAKE, 256, 0, 0, check=False) == K.KVQ_ERR_INVALID_ARG
    assert K.kvq_selftest_wait(FAKE + 8, 256, 1000, 0, check=False) == K.KVQ_ERR_INVALID_ARG
    assert K.kvq_selftest_wait(FAKE, 255, 1000, 0, check=False) == K.KVQ_ERR_WORKSPACE


def _decode(d, **kw):
    a = dict(q=FAKE, batch=1, num_q_heads=32, k_codes=FAKE, k_scales=FAKE, v_codes=FAKE,
             v_scales=FAKE, page_table=None, max_pages=1, seq_lens=FAKE, max_seq_len=256,
             sm_scale=0.088, tau=1e-6, split_tokens=64, workspace=FAKE, workspace_bytes=1 << 30,
             stats=None, out=None, options=0, stream=0)
    a.update(kw)
    return K.kvq_decode_attn(d, check=False, **a)


@pytest.mark.parametrize("kw,code", [
    (dict(num_q_heads=30), K.KVQ_ERR_INVALID_ARG),      # not a multiple of num_kv_heads
    (dict(num_q_heads=64), K.KVQ_ERR_UNSUPPORTED),      # group 16 > 8
    (dict(tau=-1.0), K.KVQ_ERR_INVALID_ARG),
    (dict(tau=float("nan")), K.KVQ_ERR_INVALID_ARG),
    (dict(q=None), K.KVQ_ERR_INVALID_ARG),
    (dict(seq_lens=None), K.KVQ_ERR_INVALID_ARG),
    (dict(v_codes=FAKE + 4), K.KVQ_ERR_INVALID_ARG),    # not 16-byte aligned
    (dict(workspace_bytes=100), K.KVQ_ERR_WORKSPACE),
    (dict(batch=K.KVQ_MAX_BATCH + 1, max_pages=1), K.KVQ_ERR_UNSUPPORTED),
    (dict(batch=9, max_pages=1), K.KVQ_ERR_INVALID_ARG),  # identity pages beyond num_pages
    (dict(batch=0), K.KVQ_OK),
    (dict(options=16), K.KVQ_ERR_INVALID_ARG),          # unknown option bit
    (dict(options=3), K.KVQ_ERR_INVALID_ARG),           # two maximum scopes at once
    (dict(options=12), K.KVQ_ERR_INVALID_ARG),          # two V fetch policies at once
    (dict(q=FAKE + 8), K.KVQ_ERR_INVALID_ARG),          # query not 16-byte aligned
    (dict(out=FAKE + 2), K.KVQ_ERR_INVALID_ARG),        # output not 4-byte aligned
    (dict(workspace=FAKE + 8), K.KVQ_ERR_INVALID_ARG),  # workspace not 16-byte aligned
])
def test_decode_rejects_bad_arguments(kw, code):
    assert _decode(_desc(), **kw) == code


def test_combine_rejects_bad_arguments():
    d = _desc()
    assert K.kvq_combine(d, None, 1, 32, 256, 64, FAKE, FAKE, stream=0, check=False) == K.KVQ_ERR_INVALID_ARG
    assert K.kvq_combine(d, FAKE, 1, 32, 256, 64, FAKE, None, stream=0, check=False) == K.KVQ_ERR_INVALID_ARG
    assert K.kvq_combine(d, FAKE, 0, 32, 256, 64, FAKE, FAKE, stream=0, check=False) == K.KVQ_OK


def test_product_code_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "quantized_kv_cache_split_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle", text, re.M), f
                assert "oracle/" not in text, f


def test_cache_attention_rejects_unknown_scope_and_fetch_policy():
    # checked before any device call: a CPU-resident cache is enough
    import torch
    cache = K.QuantizedKVCache("q4_0", 128, 4, 64, 2, "cpu")
    q = torch.zeros((1, 32, 128), dtype=torch.float16)
    lens = torch.zeros(1, dtype=torch.int32)
    with pytest.raises(ValueError, match="max_scope"):
        cache.attention(q, lens, 64, max_scope="global")
    with pytest.raises(ValueError, match="v_fetch"):
        cache.attention(q, lens, 64, v_fetch="all")
