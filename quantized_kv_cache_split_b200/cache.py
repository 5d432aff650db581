"""A paged, block-quantized KV cache on one GPU, driven through libkvq.

PyTorch supplies device memory and the stream; every computation (quantizing
appended K/V, split-KV decode attention with sparse V, the log-sum-exp merge)
is a libkvq call.
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np
import torch

from . import _binding as kb


class QuantizedKVCache:
    """K and V planes of one attention layer.

    Layout (per plane pair): codes uint8 [num_pages, num_kv_heads, page_size, row_bytes],
    scales fp16 [num_pages, num_kv_heads, page_size, scale_count].  A contiguous
    cache is page_size = capacity with one page per sequence.
    """

    def __init__(self, fmt: str, head_dim: int, num_kv_heads: int, page_size: int, num_pages: int,
                 device="cuda", codebook: Optional[torch.Tensor] = None,
                 signs: Optional[torch.Tensor] = None):
        self.fmt = fmt
        self.head_dim = head_dim
        self.num_kv_heads = num_kv_heads
        self.page_size = page_size
        self.num_pages = num_pages
        self.device = torch.device(device)
        row = kb.kvq_code_row_bytes(fmt, head_dim)
        nsc = kb.kvq_scale_row_count(fmt, head_dim)
        if row == 0 or nsc == 0:
            raise kb.KvqError("QuantizedKVCache", kb.KVQ_ERR_UNSUPPORTED)
        shape = (num_pages, num_kv_heads, page_size)
        self.k_codes = torch.zeros(shape + (row,), dtype=torch.uint8, device=self.device)
        self.v_codes = torch.zeros_like(self.k_codes)
        self.k_scales = torch.zeros(shape + (nsc,), dtype=torch.float16, device=self.device)
        self.v_scales = torch.zeros_like(self.k_scales)
        self.codebook = None
        self.signs = None
        if fmt == "lut4":
            if codebook is None:
                cb = kb.kvq_lloyd_max_codebook(16, 1.0 / math.sqrt(head_dim))
                codebook = torch.from_numpy(cb.view(np.int16).copy())
            self.codebook = codebook.to(self.device).contiguous()
            if signs is None:
                raise ValueError("lut4 needs the rotation signs")
            self.signs = signs.to(device=self.device, dtype=torch.int8).contiguous()
        self.desc = kb.make_desc(fmt, head_dim, num_kv_heads, page_size, num_pages,
                                 self.codebook, self.signs)
        self._ws = None

    # ---------------------------------------------------------------- writes
    def write(self, k: torch.Tensor, v: torch.Tensor, slots: Optional[torch.Tensor] = None,
              stream=None):
        """Quantize fp16 K/V [n_tokens, num_kv_heads, head_dim] into physical ``slots``."""
        n = k.shape[0]
        kb.kvq_quantize_kv(self.desc, k, v, n, slots, self.k_codes, self.k_scales, self.v_codes,
                           self.v_scales, stream)

    # ---------------------------------------------------------------- decode
    def workspace(self, batch: int, num_q_heads: int, max_seq_len: int, split_tokens: int,
                  options: int = 0):
        L = kb.kvq_resolve_split(self.desc, batch, num_q_heads, max_seq_len, split_tokens, options)
        nbytes = kb.kvq_workspace_size(batch, num_q_heads, self.head_dim, max_seq_len, L)
        if self._ws is None or self._ws.numel() < nbytes:
            self._ws = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
            kb.kvq_workspace_init(self._ws, self._ws.numel())  # once; any later shape reuses it
        return self._ws, nbytes, L

    def attention(self, q: torch.Tensor, seq_lens: torch.Tensor, max_seq_len: int,
                  page_table: Optional[torch.Tensor] = None, max_pages: int = 1,
                  tau: float = 1e-6, sm_scale: Optional[float] = None, split_tokens: int = 0,
                  out: Optional[torch.Tensor] = None, stats: Optional[torch.Tensor] = None,
                  max_scope: str = "split", fused: bool = True, v_fetch: str = "auto",
                  stream=None) -> torch.Tensor:
        """Decode attention of q [batch, num_q_heads, head_dim] (fp16) -> fp32 output.

        ``fused``: merge the split partials inside the decode kernel (one launch);
        otherwise kvq_combine merges them in a second launch.  ``max_scope``: the running
        maximum the skip test uses: "split" (each split's own), "cluster" (shared by the
        splits of a thread-block cluster) or "sequence" (over all splits of the
        sequence and KV head).  ``v_fetch``: how V rows reach the SM when tau > 0:
        "kept" (only the kept rows, after the skip test), "with_k" (every V tile with its
        K tile; skipped rows are left out of the contraction only) or "auto" (with_k);
        the result is the same."""
        scopes = {"split": 0, "cluster": kb.KVQ_OPT_SHARED_MAX, "sequence": kb.KVQ_OPT_GLOBAL_MAX}
        fetches = {"auto": 0, "kept": kb.KVQ_OPT_V_KEPT_ONLY, "with_k": kb.KVQ_OPT_V_WITH_K}
        if max_scope not in scopes:
            raise ValueError(f"max_scope must be one of {sorted(scopes)}, not {max_scope!r}")
        if v_fetch not in fetches:
            raise ValueError(f"v_fetch must be one of {sorted(fetches)}, not {v_fetch!r}")
        B, Hq, D = q.shape
        if sm_scale is None:
            sm_scale = 1.0 / math.sqrt(D)
        opts = scopes[max_scope]
        ws, nbytes, L = self.workspace(B, Hq, max_seq_len, split_tokens, opts)
        opts |= fetches[v_fetch]
        if out is None:
            out = torch.empty((B, Hq, D), dtype=torch.float32, device=self.device)
        kb.kvq_decode_attn(self.desc, q, B, Hq, self.k_codes, self.k_scales, self.v_codes,
                           self.v_scales, page_table, max_pages, seq_lens, max_seq_len, sm_scale,
                           tau, L, ws, nbytes, stats, out if fused else None, opts, stream)
        if not fused:
            kb.kvq_combine(self.desc, ws, B, Hq, max_seq_len, L, seq_lens, out, opts, stream)
        return out

    def device_flags(self) -> int:
        return 0 if self._ws is None else kb.kvq_read_device_flags(self._ws)
