"""ctypes binding of libkvq (include/kvq.h).  Argument marshalling only: every
step of the computation runs in the CUDA library; this module turns torch
tensors into device pointers and status codes into exceptions.

The library must exist (built in-tree by ``quantized_kv_cache_split_b200.build``);
there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkvq.so")

KVQ_OK = 0
KVQ_ERR_INVALID_ARG = -1
KVQ_ERR_UNSUPPORTED = -2
KVQ_ERR_CUDA = -3
KVQ_ERR_WORKSPACE = -4
KVQ_ERR_DEVICE = -5

KVQ_FMT_Q8_0 = 0
KVQ_FMT_Q4_0 = 1
KVQ_FMT_LUT4 = 2
KVQ_FMT_NVFP4 = 3
FORMATS = {"q8_0": KVQ_FMT_Q8_0, "q4_0": KVQ_FMT_Q4_0, "lut4": KVQ_FMT_LUT4, "nvfp4": KVQ_FMT_NVFP4}

KVQ_OPT_SHARED_MAX = 1
KVQ_OPT_GLOBAL_MAX = 2
KVQ_OPT_V_KEPT_ONLY = 4
KVQ_OPT_V_WITH_K = 8

KVQ_FLAG_BAD_PAGE = 1
KVQ_FLAG_BAD_SEQLEN = 2
KVQ_FLAG_TIMEOUT = 4

KVQ_MAX_GROUP = 8
KVQ_MAX_SPLIT_TOKENS = 1024
KVQ_MAX_BATCH = 1024
KVQ_MAX_SPLITS = 4096
KVQ_NOALLOC_SCRATCH_BYTES = 8 << 20


class KvqCacheDesc(ctypes.Structure):
    _fields_ = [
        ("fmt", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
        ("codebook", ctypes.c_void_p),
        ("signs", ctypes.c_void_p),
    ]


class KvqError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status} ({kvq_status_string(status)})")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python quantized_kv_cache_split_b200/build.py` "
            "(the CUDA library is required; there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, SZ, F32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_float
    U32 = ctypes.c_uint32
    D = ctypes.POINTER(KvqCacheDesc)
    sig = {
        "kvq_code_row_bytes": (SZ, [I32, I32]),
        "kvq_scale_row_count": (SZ, [I32, I32]),
        "kvq_quantize": (ctypes.c_int, [D, P, I32, P, P, P, P]),
        "kvq_quantize_kv": (ctypes.c_int, [D, P, P, I32, P, P, P, P, P, P]),
        "kvq_resolve_split": (I32, [D, I32, I32, I32, I32, U32]),
        "kvq_resolve_cluster": (I32, [D, I32, I32, I32, I32, U32]),
        "kvq_workspace_size": (SZ, [I32, I32, I32, I32, I32]),
        "kvq_workspace_init": (ctypes.c_int, [P, SZ, P]),
        "kvq_read_device_flags": (ctypes.c_int, [P, ctypes.POINTER(ctypes.c_uint32), P]),
        "kvq_selftest_wait": (ctypes.c_int, [P, ctypes.c_size_t, ctypes.c_longlong, P]),
        "kvq_decode_attn": (ctypes.c_int, [D, P, I32, I32, P, P, P, P, P, I32, P, I32, F32, F32,
                                           I32, U32, P, SZ, P, P, P]),
        "kvq_combine": (ctypes.c_int, [D, P, I32, I32, I32, I32, U32, P, P, P]),
        "kvq_decode_attn_noalloc": (ctypes.c_int, [D, P, I32, I32, P, P, P, P, P, I32, P, I32, F32,
                                                   F32, I32, U32, P, P, P]),
        "kvq_noalloc_read_flags": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32), P]),
        "kvq_lloyd_max_codebook": (ctypes.c_int, [I32, ctypes.c_double,
                                                  ctypes.POINTER(ctypes.c_uint16)]),
        "kvq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


_lib = _load()


def lib():
    return _lib


# ------------------------------------------------------------------ marshalling helpers

def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, st: int):
    if st != KVQ_OK:
        raise KvqError(fn, st)


def make_desc(fmt, head_dim: int, num_kv_heads: int, page_size: int, num_pages: int,
              codebook=None, signs=None) -> KvqCacheDesc:
    f = FORMATS[fmt] if isinstance(fmt, str) else int(fmt)
    return KvqCacheDesc(f, head_dim, num_kv_heads, page_size, num_pages,
                        _ptr(codebook), _ptr(signs))


# ------------------------------------------------------------------ the C calls, same names

def kvq_status_string(status: int) -> str:
    return _lib.kvq_status_string(int(status)).decode()


def kvq_code_row_bytes(fmt, head_dim: int) -> int:
    return _lib.kvq_code_row_bytes(FORMATS.get(fmt, fmt) if isinstance(fmt, str) else fmt, head_dim)


def kvq_scale_row_count(fmt, head_dim: int) -> int:
    return _lib.kvq_scale_row_count(FORMATS.get(fmt, fmt) if isinstance(fmt, str) else fmt, head_dim)


def kvq_quantize(desc: KvqCacheDesc, x, n_tokens: int, slots, codes, scales, stream=None,
                 check: bool = True) -> int:
    st = _lib.kvq_quantize(ctypes.byref(desc), _ptr(x), int(n_tokens), _ptr(slots), _ptr(codes),
                           _ptr(scales), _stream(stream))
    if check:
        _check("kvq_quantize", st)
    return st


def kvq_quantize_kv(desc: KvqCacheDesc, k, v, n_tokens: int, slots, k_codes, k_scales, v_codes,
                    v_scales, stream=None, check: bool = True) -> int:
    st = _lib.kvq_quantize_kv(ctypes.byref(desc), _ptr(k), _ptr(v), int(n_tokens), _ptr(slots),
                              _ptr(k_codes), _ptr(k_scales), _ptr(v_codes), _ptr(v_scales),
                              _stream(stream))
    if check:
        _check("kvq_quantize_kv", st)
    return st


def kvq_resolve_split(desc: KvqCacheDesc, batch: int, num_q_heads: int, max_seq_len: int,
                      split_tokens: int = 0, options: int = 0, check: bool = True) -> int:
    v = _lib.kvq_resolve_split(ctypes.byref(desc), batch, num_q_heads, max_seq_len, split_tokens,
                               int(options))
    if check and v < 0:
        raise KvqError("kvq_resolve_split", v)
    return v


def kvq_resolve_cluster(desc: KvqCacheDesc, batch: int, num_q_heads: int, max_seq_len: int,
                        split_tokens: int = 0, options: int = 0, check: bool = True) -> int:
    v = _lib.kvq_resolve_cluster(ctypes.byref(desc), batch, num_q_heads, max_seq_len, split_tokens,
                                 int(options))
    if check and v < 0:
        raise KvqError("kvq_resolve_cluster", v)
    return v


def kvq_workspace_size(batch: int, num_q_heads: int, head_dim: int, max_seq_len: int,
                       split_tokens: int) -> int:
    return _lib.kvq_workspace_size(batch, num_q_heads, head_dim, max_seq_len, split_tokens)


def kvq_workspace_init(workspace, nbytes: int, stream=None):
    _check("kvq_workspace_init", _lib.kvq_workspace_init(_ptr(workspace), nbytes, _stream(stream)))


def kvq_read_device_flags(workspace, stream=None) -> int:
    out = ctypes.c_uint32(0)
    _check("kvq_read_device_flags",
           _lib.kvq_read_device_flags(_ptr(workspace), ctypes.byref(out), _stream(stream)))
    return out.value


def kvq_selftest_wait(workspace, workspace_bytes: int, max_cycles: int, stream=None,
                      check: bool = True) -> int:
    st = _lib.kvq_selftest_wait(_ptr(workspace), int(workspace_bytes), int(max_cycles), _stream(stream))
    if check:
        _check("kvq_selftest_wait", st)
    return st


def kvq_decode_attn(desc: KvqCacheDesc, q, batch: int, num_q_heads: int, k_codes, k_scales,
                    v_codes, v_scales, page_table, max_pages: int, seq_lens, max_seq_len: int,
                    sm_scale: float, tau: float, split_tokens: int, workspace, workspace_bytes: int,
                    stats=None, out=None, options: int = 0, stream=None, check: bool = True) -> int:
    st = _lib.kvq_decode_attn(ctypes.byref(desc), _ptr(q), batch, num_q_heads, _ptr(k_codes),
                              _ptr(k_scales), _ptr(v_codes), _ptr(v_scales), _ptr(page_table),
                              max_pages, _ptr(seq_lens), max_seq_len, float(sm_scale), float(tau),
                              split_tokens, int(options), _ptr(workspace), workspace_bytes,
                              _ptr(stats), _ptr(out), _stream(stream))
    if check:
        _check("kvq_decode_attn", st)
    return st


def kvq_combine(desc: KvqCacheDesc, workspace, batch: int, num_q_heads: int, max_seq_len: int,
                split_tokens: int, seq_lens, out, options: int = 0, stream=None,
                check: bool = True) -> int:
    st = _lib.kvq_combine(ctypes.byref(desc), _ptr(workspace), batch, num_q_heads, max_seq_len,
                          split_tokens, int(options), _ptr(seq_lens), _ptr(out), _stream(stream))
    if check:
        _check("kvq_combine", st)
    return st


def kvq_lloyd_max_codebook(levels: int = 16, sigma: float = 1.0) -> np.ndarray:
    buf = (ctypes.c_uint16 * levels)()
    _check("kvq_lloyd_max_codebook", _lib.kvq_lloyd_max_codebook(levels, float(sigma), buf))
    return np.frombuffer(bytes(buf), dtype=np.float16).copy()


def kvq_decode_attn_noalloc(desc: KvqCacheDesc, q, batch: int, num_q_heads: int, k_codes,
                            k_scales, v_codes, v_scales, page_table, max_pages: int, seq_lens,
                            max_seq_len: int, sm_scale: float, tau: float, split_tokens: int, out,
                            stats=None, options: int = 0, stream=None, check: bool = True) -> int:
    """Decode + merge using the library's static scratch (no device allocation)."""
    st = _lib.kvq_decode_attn_noalloc(ctypes.byref(desc), _ptr(q), batch, num_q_heads,
                                      _ptr(k_codes), _ptr(k_scales), _ptr(v_codes), _ptr(v_scales),
                                      _ptr(page_table), max_pages, _ptr(seq_lens), max_seq_len,
                                      float(sm_scale), float(tau), split_tokens, int(options),
                                      _ptr(stats), _ptr(out), _stream(stream))
    if check:
        _check("kvq_decode_attn_noalloc", st)
    return st


def kvq_noalloc_read_flags(stream=None) -> int:
    """KVQ_FLAG_* bits of the last kvq_decode_attn_noalloc call on the current device."""
    flags = ctypes.c_uint32(0)
    _check("kvq_noalloc_read_flags", _lib.kvq_noalloc_read_flags(ctypes.byref(flags), _stream(stream)))
    return int(flags.value)
