"""Seeded synthetic inputs for single-token decode attention over a quantized KV cache.

This module only draws random numbers and lays them out.  It holds none of the
method's arithmetic (no quantizer, no softmax, no rotation), so both the fp64
oracle and the CUDA library can be fed from it without sharing code.

Recipe (every workload):
  * numpy ``Generator(PCG64(seed))``; Q, K, V ~ N(0, 1) drawn in float32 and
    rounded to float16 (round-to-nearest-even).
  * "Planted" keys make attention concentrate the way long-context attention
    does in practice: for each (sequence, KV head), ``n_planted`` positions are
    drawn uniformly without replacement, a target score ``a ~ U(lo, hi)`` is
    drawn per position, and the key there is replaced by the minimum-norm
    vector that gives every query head of the group that scaled score:
    ``k = Qg^T (Qg Qg^T)^-1 (a sqrt(D) 1)`` with ``Qg`` the group's G query
    rows, so ``q_h . k / sqrt(D) = a`` for each head h of the group (before
    fp16 rounding and quantization).  With G = 1 this is
    ``a sqrt(D) q / |q|^2``.  V is left unplanted.
  * LUT workloads also draw ``D`` random signs (+1/-1) from ``seed + 1``.
  * Paged workloads place each sequence's 64-token pages at a seeded random
    permutation of the physical pages.

Layouts returned (all numpy):
  q          [B, Hq, D]            float16
  k, v       [T, Hkv, D]           float16, T = sum of seq_lens, sequences
                                    concatenated in batch order
  slots      [T]                   int32, physical token slot of each row
                                    (slot = page * page_size + offset)
  page_table [B, max_pages]        int32, -1 where unused (None if contiguous)
  seq_lens   [B]                   int32
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np

FMT_Q8_0 = "q8_0"
FMT_Q4_0 = "q4_0"
FMT_LUT4 = "lut4"
FMT_NVFP4 = "nvfp4"


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    seq_lens: tuple
    n_planted: int
    planted_lo: float
    planted_hi: float
    fmt: str
    taus: tuple
    seed: int
    page_size: Optional[int] = None  # None: one contiguous region per sequence

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seq_lens))

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


_PAGED_LENS = (8192, 16384, 32768, 65536, 65536, 32768, 16384, 8192)

WORKLOADS = {
    # 4 query heads on 1 KV head, head_dim 64, 256 positions, q8_0.
    "tiny_q8_d64": Workload("tiny_q8_d64", 1, 4, 1, 64, (256,), 8, 8.0, 12.0,
                            FMT_Q8_0, (1e-6, 0.0), 1001),
    # GQA 32/8, head_dim 128, 4K context, q8_0.
    "gqa_4k_q8": Workload("gqa_4k_q8", 1, 32, 8, 128, (4096,), 32, 6.0, 14.0,
                          FMT_Q8_0, (0.0, 1e-6), 1002),
    # GQA 32/4, head_dim 128, 32K context, q4_0 (the headline decode case).
    "gqa_32k_q4": Workload("gqa_32k_q4", 1, 32, 4, 128, (32768,), 64, 10.0, 20.0,
                           FMT_Q4_0, (0.0, 1e-6), 1003),
    # Rotated 4-bit LUT codebook at the 4K shape and at the 32K shape.
    "lut_4k": Workload("lut_4k", 1, 32, 8, 128, (4096,), 32, 6.0, 14.0,
                       FMT_LUT4, (0.0, 1e-6), 1004),
    "lut_32k": Workload("lut_32k", 1, 32, 4, 128, (32768,), 64, 10.0, 20.0,
                        FMT_LUT4, (0.0, 1e-6), 1014),
    # NVFP4 (E2M1 + E4M3 block scales) at the 32K GQA-8 shape.
    "nvfp4_32k": Workload("nvfp4_32k", 1, 32, 4, 128, (32768,), 64, 10.0, 20.0,
                          FMT_NVFP4, (0.0, 1e-6), 1023),
    # 8 concurrent streams, paged 64-token pages, mixed context lengths.
    "paged_b8_q8": Workload("paged_b8_q8", 8, 32, 4, 128, _PAGED_LENS, 64, 10.0, 20.0,
                            FMT_Q8_0, (0.0, 1e-6, 1e-4), 1005, page_size=64),
    "paged_b8_q4": Workload("paged_b8_q4", 8, 32, 4, 128, _PAGED_LENS, 64, 10.0, 20.0,
                            FMT_Q4_0, (0.0, 1e-6, 1e-4), 1015, page_size=64),
}


def round_up(x: int, m: int) -> int:
    return (x + m - 1) // m * m


@dataclasses.dataclass
class Inputs:
    wl: Workload
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    slots: np.ndarray
    page_table: Optional[np.ndarray]
    seq_lens: np.ndarray
    page_size: int
    num_pages: int
    max_pages: int
    planted: list          # per (b, kvh): (positions, target scores)
    signs: Optional[np.ndarray]

    def seq_offsets(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.seq_lens)]).astype(np.int64)


def _to_f16(x: np.ndarray) -> np.ndarray:
    """IEEE fp32 -> fp16, round to nearest even (torch's vectorised cast when torch is
    importable, else numpy's; both are the same IEEE conversion, bit for bit)."""
    try:
        import torch
    except ImportError:  # pragma: no cover - torch is always present in this project
        return x.astype(np.float16)
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.float16).numpy()


def _normal_f16(rng: np.random.Generator, shape) -> np.ndarray:
    return _to_f16(rng.standard_normal(shape, dtype=np.float32))


def generate(wl: Workload, seed: Optional[int] = None) -> Inputs:
    """Draw one workload.  Same (workload, seed) -> bit-identical arrays."""
    seed = wl.seed if seed is None else seed
    rng = np.random.Generator(np.random.PCG64(seed))
    B, Hq, Hkv, D, G = wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.group
    lens = np.asarray(wl.seq_lens, dtype=np.int32)
    T = int(lens.sum())

    q = _normal_f16(rng, (B, Hq, D))
    k = _normal_f16(rng, (T, Hkv, D))
    v = _normal_f16(rng, (T, Hkv, D))

    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    planted = []
    for b in range(B):
        for h in range(Hkv):
            n = int(lens[b])
            npl = min(wl.n_planted, n)
            pos = np.sort(rng.choice(n, size=npl, replace=False))
            a = rng.uniform(wl.planted_lo, wl.planted_hi, size=npl)
            Qg = q[b, h * G:(h + 1) * G].astype(np.float64)
            direction = Qg.T @ np.linalg.solve(Qg @ Qg.T, np.ones(G))
            keys = (a[:, None] * math.sqrt(D)) * direction[None, :]
            k[offs[b] + pos, h, :] = keys.astype(np.float16)
            planted.append((pos, a))

    if wl.page_size is None:
        # One region per sequence, capacity rounded up to 64 tokens.
        cap = round_up(int(lens.max()), 64)
        page_size, num_pages, max_pages = cap, B, 1
        page_table = None
        slots = np.concatenate([b * cap + np.arange(lens[b]) for b in range(B)])
    else:
        page_size = wl.page_size
        pages_per_seq = [(int(n) + page_size - 1) // page_size for n in lens]
        num_pages = int(sum(pages_per_seq))
        max_pages = int(max(pages_per_seq))
        perm = rng.permutation(num_pages).astype(np.int32)
        page_table = np.full((B, max_pages), -1, dtype=np.int32)
        cursor = 0
        slot_list = []
        for b in range(B):
            npg = pages_per_seq[b]
            page_table[b, :npg] = perm[cursor:cursor + npg]
            cursor += npg
            t = np.arange(lens[b])
            slot_list.append(page_table[b, t // page_size].astype(np.int64) * page_size
                             + t % page_size)
        slots = np.concatenate(slot_list)

    signs = None
    if wl.fmt == FMT_LUT4:
        srng = np.random.Generator(np.random.PCG64(seed + 1))
        signs = np.where(srng.random(D) < 0.5, -1, 1).astype(np.int8)

    return Inputs(wl=wl, q=q, k=k, v=v, slots=slots.astype(np.int32),
                  page_table=page_table, seq_lens=lens, page_size=page_size,
                  num_pages=num_pages, max_pages=max_pages, planted=planted,
                  signs=signs)


def shrink(wl: Workload, seq_lens: Sequence[int], n_planted: Optional[int] = None) -> Workload:
    """Same recipe at other context lengths (parity cases the oracle finishes fast)."""
    return wl.with_(name=f"{wl.name}_x{len(seq_lens)}", batch=len(seq_lens),
                    seq_lens=tuple(int(s) for s in seq_lens),
                    n_planted=wl.n_planted if n_planted is None else n_planted)
