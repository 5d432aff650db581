"""The roofline numerator of bench.py: the algorithmic HBM bytes of one decode step,
checked against the byte counts written out by hand for the 32K and paged workloads
(host only; no GPU)."""
from types import SimpleNamespace

import numpy as np

import bench
import workloads as W


def _rep(name, page_table):
    wl = W.WORKLOADS[name]
    inp = SimpleNamespace(seq_lens=np.asarray(wl.seq_lens, dtype=np.int64),
                          page_table=page_table, page_size=64)
    return SimpleNamespace(wl=wl, inp=inp)


def test_32k_q4_sparse_bytes():
    # K: 32768 positions x 4 KV heads x (64 code bytes + 4 fp16 scales); kept V rows at the
    # same 72 bytes; Q fp16; (m, l) of 37 splits x 4 KV heads x 8 heads, written and read;
    # the fp32 output.  No page table (contiguous cache).
    rep = _rep("gqa_32k_q4", None)
    k = 32768 * 4 * 72
    v = 54994 * 72
    q = 32 * 128 * 2
    part = 2 * (37 * 4) * 8 * 2 * 4
    out = 32 * 128 * 4
    assert bench.algorithmic_bytes(rep, 54994, 37 * 4, with_o=False) == k + v + q + part + out == 13440272


def test_32k_q4_dense_bytes_count_every_v_row():
    rep = _rep("gqa_32k_q4", None)
    assert bench.algorithmic_bytes(rep, 131072, 148, with_o=False) == 2 * 32768 * 4 * 72 + 8192 + 18944 + 16384


def test_paged_bytes_include_page_table_and_o_partials():
    # 8 streams {8,16,32,64,64,32,16,8}K at 64-token pages: 3840 page-table entries; with the
    # combine kernel the partials carry o (head_dim floats) as well as (m, l).
    rep = _rep("paged_b8_q4", np.zeros((8, 1024), dtype=np.int32))
    n = 245760
    splits = sum(-(-int(s) // 1024) for s in W.WORKLOADS["paged_b8_q4"].seq_lens)  # 240
    k = n * 4 * 72
    v = 466267 * 72
    q = 8 * 32 * 128 * 2
    pt = 3840 * 4
    part = 2 * (splits * 4) * 8 * (128 + 2) * 4
    out = 8 * 32 * 128 * 4
    got = bench.algorithmic_bytes(rep, 466267, splits * 4, with_o=True)
    assert got == k + v + q + pt + part + out == 112549272


def test_timed_region_is_one_graph_of_exactly_the_timed_steps():
    # whatever --steps is (here fewer steps than cache copies, and a warm-up that is not a
    # multiple of anything), the warm-up and the timed region are each ONE capture: steps
    # 0 .. W-1 and W .. W+K-1
    calls = []

    def fake_capture(fn, n_steps, start):
        calls.append((n_steps, start))
        return ("graph", n_steps, start)

    g = bench.StepGraphs(lambda i: None, steps=20, warmup=5, capture_fn=fake_capture,
                         upload_fn=lambda graph: True)
    assert calls == [(5, 0), (20, 5)]
    assert g.warm == ("graph", 5, 0) and g.timed == ("graph", 20, 5)


def test_cpu_oracle_group_runs_on_the_host():
    # the CPU baseline's unit of work (one (sequence, KV head) group of the oracle, truncated)
    dt = bench._oracle_group(("tiny_q8_d64", 0, 0, 128, 64, 1e-6))
    assert dt > 0.0
