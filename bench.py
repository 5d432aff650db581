"""Benchmark: single-token decode attention over a block-quantized KV cache with
sparse V dequantization, on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload gqa_32k_q4] [--tau 1e-6] [--headline-only]

One step = the whole decode-attention hot path for one decode token of every
sequence in the workload: one kvq_decode_attn call (K tiles -> scores -> running
maximum -> skip decision -> V of the kept rows -> merge of the splits into the
output).  Inputs are resident in HBM; the cache is replicated into enough copies
that successive steps rotate through more than 3x the L2 size, so every step
reads HBM.  The W warm-up steps and the K timed steps are each captured as one
CUDA graph; the timed region is one replay, bracketed by CUDA events.  Prints one
JSON line: the headline workload (every variant of the skip test and V fetch, the
two-launch path, the end-to-end path through the Python API with host buffers),
then, unless --headline-only, a table of every workload (dense and sparse at each
of its tau values).

--impl reference times the fp64 CPU oracle (the only reference available for
this method) on bounded samples of the same workload.
Multi-GPU (torchrun): every rank runs an independent replica (no collective on
the data path; weak scaling); timings are reduced with MAX over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "decode-attn µs/token & achieved KV HBM GB/s at 32K ctx, sparse-V vs dense"
UNIT = "us/token"
L2_BYTES = 126 * 1024 * 1024
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "decode_traffic.json")
DECODE_SRC = os.path.join(ROOT, "quantized_kv_cache_split_b200", "csrc", "kvq_decode2.cu")


# ------------------------------------------------------------------ distributed plumbing

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    import torch.distributed as td
    if world > 1 and not td.is_initialized():
        import datetime
        td.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return td


def reduce_max(value: float, world: int, device="cpu") -> float:
    """MAX over ranks of a per-rank float (timings)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as td
    t = torch.tensor([value], dtype=torch.float64, device=device)
    td.all_reduce(t, op=td.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as td
        td.barrier()


# ------------------------------------------------------------------ clocks (NVML, sampled during timing)

_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
            0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
            0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, cuda_index: int):
        self.ok = False
        self.samples = []
        self.reasons = 0
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            props = torch.cuda.get_device_properties(cuda_index)
            try:
                bus = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(cuda_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            f = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
            self._reason_fn = f
            self.ok = True
        except Exception as e:  # pragma: no cover - no NVML here
            self.err = str(e)

    def _sample(self):
        self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
        self.reasons |= int(self._reason_fn(self.h))

    def start(self):
        if not self.ok:
            return
        self._stop = False
        self._sample()

        def run():
            while not self._stop:
                self._sample()
                time.sleep(0.001)
        self.t = threading.Thread(target=run, daemon=True)
        self.t.start()

    def stop(self):
        if not self.ok:
            return
        self._stop = True
        self.t.join()
        self._sample()

    def report(self):
        if not self.ok or not self.samples:
            return None
        names = [n for b, n in _REASONS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": float(self.max_mhz),
                "reasons": names, "samples": len(self.samples)}


# ------------------------------------------------------------------ GPU arm

def traffic_from_profile(unit_key: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current source."""
    try:
        prof = json.load(open(PROFILE_TRAFFIC))
        src_hash = hashlib.sha256(open(DECODE_SRC, "rb").read()).hexdigest()[:16]
        if prof.get("source_sha256_16") != src_hash:
            return None
        ent = prof["launches"].get(unit_key)
        return None if ent is None else float(ent["dram_bytes_per_launch"])
    except Exception:
        return None


def measured_peaks():
    try:
        p = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class Replicas:
    """R copies of the quantized cache so that successive steps miss in L2."""

    def __init__(self, wl: W.Workload, inp: W.Inputs, device, min_bytes: int, split_tokens: int = 0):
        import torch
        import quantized_kv_cache_split_b200 as K
        self.wl, self.inp = wl, inp
        D = wl.head_dim
        cb = sg = None
        if wl.fmt == "lut4":
            cb = torch.from_numpy(K.kvq_lloyd_max_codebook(16, 1.0 / math.sqrt(D)).view(np.int16).copy())
            sg = torch.from_numpy(inp.signs)
        first = K.QuantizedKVCache(wl.fmt, D, wl.num_kv_heads, inp.page_size, inp.num_pages,
                                   device, cb, sg)
        first.write(torch.from_numpy(inp.k).to(device), torch.from_numpy(inp.v).to(device),
                    torch.from_numpy(inp.slots).to(device))
        plane_bytes = sum(t.numel() * t.element_size()
                          for t in (first.k_codes, first.k_scales, first.v_codes, first.v_scales))
        self.plane_bytes = plane_bytes
        # rotate over enough copies to exceed 3x L2, at most 512 (a tiny cache cannot reach
        # it with any sensible number of copies: it is then timed with its copies in L2,
        # which the config's "l2" field says)
        self.R = max(2, min(512, math.ceil(min_bytes / plane_bytes)))
        self.l2_cold = self.R * plane_bytes >= min_bytes
        self.caches = [first]
        for _ in range(self.R - 1):
            c = K.QuantizedKVCache(wl.fmt, D, wl.num_kv_heads, inp.page_size, inp.num_pages,
                                   device, first.codebook, first.signs)
            for dst, src in ((c.k_codes, first.k_codes), (c.k_scales, first.k_scales),
                             (c.v_codes, first.v_codes), (c.v_scales, first.v_scales)):
                dst.copy_(src)
            self.caches.append(c)
        self.q = torch.from_numpy(inp.q).to(device)
        self.seq = torch.from_numpy(inp.seq_lens).to(device)
        self.pt = None if inp.page_table is None else torch.from_numpy(inp.page_table).to(device)
        self.max_seq = int(inp.seq_lens.max())
        self.B, self.Hq, self.D = wl.batch, wl.num_q_heads, D
        # the schedule: L positions per split; the shared-maximum option runs clusters of
        # CS splits (its own L and CS)
        self.L = K.kvq_resolve_split(first.desc, self.B, self.Hq, self.max_seq, split_tokens)
        self.L_sh = K.kvq_resolve_split(first.desc, self.B, self.Hq, self.max_seq, 0,
                                        K.KVQ_OPT_SHARED_MAX)
        self.CS_sh = K.kvq_resolve_cluster(first.desc, self.B, self.Hq, self.max_seq, 0,
                                           K.KVQ_OPT_SHARED_MAX)
        self.ws_bytes = max(K.kvq_workspace_size(self.B, self.Hq, D, self.max_seq, L)
                            for L in (self.L, self.L_sh))
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=device)
        K.kvq_workspace_init(self.ws, self.ws_bytes)
        self.out = torch.empty((self.B, self.Hq, D), dtype=torch.float32, device=device)
        self.sm = float(np.float32(1.0 / math.sqrt(D)))

    def decode(self, i, tau, stats=None, scope="split", fused=True, v_opt=0):
        """One decode step on cache copy i % R; ``fused``: the merge runs in the same
        kernel and writes ``self.out``; ``scope``: the running maximum of the skip test
        ("split", "cluster" or "sequence"); ``v_opt``: a V fetch option bit (0: the
        library's choice)."""
        import quantized_kv_cache_split_b200 as K
        c = self.caches[i % self.R]
        opts = {"split": 0, "cluster": K.KVQ_OPT_SHARED_MAX, "sequence": K.KVQ_OPT_GLOBAL_MAX}[scope] | v_opt
        K.kvq_decode_attn(c.desc, self.q, self.B, self.Hq, c.k_codes, c.k_scales, c.v_codes,
                          c.v_scales, self.pt, self.inp.max_pages, self.seq, self.max_seq, self.sm,
                          tau, self.L_sh if scope == "cluster" else self.L, self.ws, self.ws_bytes,
                          stats, self.out if fused else None, opts)

    def combine(self, i):
        import quantized_kv_cache_split_b200 as K
        c = self.caches[i % self.R]
        K.kvq_combine(c.desc, self.ws, self.B, self.Hq, self.max_seq, self.L, self.seq, self.out)


def capture(fn, n_steps, start):
    """One CUDA graph holding steps start .. start + n_steps - 1 of ``fn`` (each step
    launched once before the capture, so host-side first-call paths are warm)."""
    import torch
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for i in range(n_steps):
            fn(start + i)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        for i in range(n_steps):
            fn(start + i)
    return g


def upload_graph(g) -> bool:
    """Upload an instantiated graph to the device ahead of its first replay (cuGraphUpload),
    so that the first, timed replay does not include the upload.  False if the driver
    call is unavailable."""
    import ctypes
    import torch
    try:
        cu = ctypes.CDLL("libcuda.so.1")
        cu.cuGraphUpload.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
        cu.cuGraphUpload.restype = ctypes.c_int
        st = cu.cuGraphUpload(ctypes.c_void_p(g.raw_cuda_graph_exec()),
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        torch.cuda.synchronize()
        return st == 0
    except Exception:
        return False


class StepGraphs:
    """The warm-up steps 0 .. warmup - 1 and the timed steps warmup .. warmup + steps - 1
    of ``fn`` (step i works on cache copy i % R inside ``fn``), each captured as ONE
    graph, so the timed region is a single replay of exactly ``steps`` launches of the
    hot path whatever ``steps`` is.  The timed graph is uploaded to the device before it
    is first replayed."""

    def __init__(self, fn, steps, warmup, capture_fn=capture, upload_fn=upload_graph):
        self.steps, self.warmup = steps, warmup
        self.warm = capture_fn(fn, warmup, 0)
        self.timed = capture_fn(fn, steps, warmup)
        self.uploaded = upload_fn(self.timed)


def prewarm(fn, seconds: float = 0.3, n_steps: int = 50):
    """Untimed: replay a graph of ``n_steps`` steps of ``fn`` for about ``seconds``, so that
    the first timed variant does not meet a GPU still leaving its idle clocks (measured:
    without it the first variant of a run came out ~1 us per step slower than the same
    variant timed later in the run)."""
    import torch
    g = capture(fn, n_steps, 0)
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        g.replay()
        torch.cuda.synchronize()
    del g


def time_steps(graphs: StepGraphs, world, sampler=None):
    """Replay the warm-up graph, then time one replay of the timed graph with CUDA
    events on the current stream (barrier and synchronize on both sides); ms."""
    import torch
    graphs.warm.replay()
    torch.cuda.synchronize()
    barrier(world)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if sampler:
        sampler.start()
    # the device first spins ~1 ms, so that the timed region starts with the graph already
    # queued behind the start event: host-side delays (the sampler thread's NVML calls, the
    # replay call itself) then never appear as idle time between the events
    torch.cuda._sleep(2_000_000)
    start.record()
    graphs.timed.replay()
    end.record()
    torch.cuda.synchronize()
    if sampler:
        sampler.stop()
    barrier(world)
    return start.elapsed_time(end)


def algorithmic_bytes(rep: Replicas, v_rows_read: int, n_partials: int, with_o: bool):
    """HBM bytes one decode step must move: every K row, the kept V rows, Q, the page
    table, the partials (one per cluster of splits, written once and read once by the
    merge: (m, l) only when each split adds its share into the output itself, also o
    when a last cluster or the combine kernel merges) and the output."""
    import quantized_kv_cache_split_b200 as K
    wl = rep.wl
    row = K.kvq_code_row_bytes(wl.fmt, wl.head_dim) + 2 * K.kvq_scale_row_count(wl.fmt, wl.head_dim)
    tokens = int(rep.inp.seq_lens.sum())
    k_bytes = tokens * wl.num_kv_heads * row
    v_bytes = v_rows_read * row
    q_bytes = wl.batch * wl.num_q_heads * wl.head_dim * 2
    pt_bytes = 0 if rep.inp.page_table is None else sum(
        (int(n) + rep.inp.page_size - 1) // rep.inp.page_size for n in rep.inp.seq_lens) * 4
    part_bytes = 2 * n_partials * wl.group * ((wl.head_dim if with_o else 0) + 2) * 4
    out_bytes = wl.batch * wl.num_q_heads * wl.head_dim * 4
    return k_bytes + v_bytes + q_bytes + pt_bytes + part_bytes + out_bytes


def _round(d):
    return {k: (round(v, 6) if isinstance(v, float) else v) for k, v in d.items()}


def n_partials(wl, inp, L, CS):
    return sum(wl.num_kv_heads * (((int(n) + L - 1) // L + CS - 1) // CS) for n in inp.seq_lens)


def measure_variant(rep, args, world, device, tau, scope, v_opt, hbm_peak, sampler=None,
                    traffic_key=None):
    """Counters of one launch, then the timed graph of args.steps launches; one dict per
    variant (absent keys: the variant is unsupported for this request)."""
    import torch
    import quantized_kv_cache_split_b200 as K
    wl, inp = rep.wl, rep.inp
    st = torch.zeros(4, dtype=torch.int64, device=device)
    try:
        rep.decode(0, tau, st, scope=scope, v_opt=v_opt)
        torch.cuda.synchronize()
    except K.KvqError as e:  # e.g. the sequence-wide maximum needs every split on its own CTA
        return {"tau": tau, "max_scope": scope, "unavailable": str(e)}
    st = [int(x) for x in st.cpu()]
    graphs = StepGraphs(lambda i: rep.decode(i, tau, scope=scope, v_opt=v_opt), args.steps,
                        args.warmup)
    ms = reduce_max(time_steps(graphs, world, sampler), world, device)
    del graphs
    launches = decode_launches_per_call(rep, device)
    abytes = algorithmic_bytes(rep, st[2], n_partials(wl, inp, rep.L_sh, rep.CS_sh) if scope == "cluster"
                               else n_partials(wl, inp, rep.L, 1),
                               with_o=scope == "cluster" or launches == 2)
    us_step = ms * 1e3 / args.steps
    achieved = abytes / (us_step * 1e-6) / 1e9
    return dict(tau=tau, max_scope=scope,
                v_fetch={0: "auto", K.KVQ_OPT_V_KEPT_ONLY: "kept_only", K.KVQ_OPT_V_WITH_K: "with_k"}[v_opt],
                ms_per_step=ms / args.steps, us_per_token=us_step / (wl.batch * world),
                us_per_step=us_step, tokens_per_s=wl.batch * world / (us_step * 1e-6),
                algorithmic_bytes=abytes, achieved_gbs=achieved, frac=achieved / hbm_peak,
                skipped_pair_frac=st[1] / max(st[0], 1), v_rows_read=st[2], v_rows_skipped=st[3],
                launches_per_step=launches,
                traffic=traffic_from_profile(traffic_key) if traffic_key else None)


def workload_table(args, world, device, name, hbm_peak):
    """Dense and sparse (every tau of the workload), with the library's default V fetch,
    plus the sequence-wide maximum and the two V fetch policies at args.tau."""
    import torch
    import quantized_kv_cache_split_b200 as K
    wl = W.WORKLOADS[name]
    inp = W.generate(wl)
    rep = Replicas(wl, inp, device, 3 * L2_BYTES, 0)
    res = {"config": {"batch": wl.batch, "num_q_heads": wl.num_q_heads, "num_kv_heads": wl.num_kv_heads,
                      "head_dim": wl.head_dim, "context": list(wl.seq_lens) if wl.batch > 1 else wl.seq_lens[0],
                      "cache_format": wl.fmt, "split_tokens": rep.L, "copies": rep.R,
                      "l2_cold": rep.l2_cold}}
    taus = sorted(set(wl.taus) | {0.0, args.tau})
    for tau in taus:
        tag = "dense" if tau == 0.0 else f"sparse_tau_{tau:g}"
        res[tag] = _round(measure_variant(rep, args, world, device, tau, "split", 0, hbm_peak))
    for tag, scope, v_opt in (("sparse_sequence_max", "sequence", 0),
                              ("sparse_v_kept_only", "split", K.KVQ_OPT_V_KEPT_ONLY),
                              ("sparse_v_with_k", "split", K.KVQ_OPT_V_WITH_K)):
        res[tag] = _round(measure_variant(rep, args, world, device, args.tau, scope, v_opt, hbm_peak))
    sp, de = res.get(f"sparse_tau_{args.tau:g}", {}), res["dense"]
    if "us_per_step" in sp and "us_per_step" in de:
        res["sparse_speedup_vs_dense"] = round(de["us_per_step"] / sp["us_per_step"], 4)
    del rep
    torch.cuda.empty_cache()
    return res


def gpu_arm(args, world, rank, local):
    import torch
    import quantized_kv_cache_split_b200 as K
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")
    wl = W.WORKLOADS[args.workload]
    inp = W.generate(wl)
    rep = Replicas(wl, inp, device, 3 * L2_BYTES, args.split_tokens)
    hbm_peak, peak_kind = measured_peaks()
    sampler = ClockSampler(local)
    # the headline leaves the V fetch to the library; the other variants are context
    variants = (("sparse", args.tau, "split", 0), ("dense", 0.0, "split", 0),
                ("sparse_v_kept_only", args.tau, "split", K.KVQ_OPT_V_KEPT_ONLY),
                ("sparse_v_with_k", args.tau, "split", K.KVQ_OPT_V_WITH_K),
                ("sparse_cluster_max", args.tau, "cluster", 0), ("sparse_sequence_max", args.tau, "sequence", 0),
                ("sparse_sequence_max_v_kept_only", args.tau, "sequence", K.KVQ_OPT_V_KEPT_ONLY))
    if not args.cluster_variant:
        variants = tuple(v for v in variants if v[2] != "cluster")
    prewarm(lambda i: rep.decode(i, args.tau))
    res = {}
    for tag, tau, scope, v_opt in variants:
        res[tag] = measure_variant(rep, args, world, device, tau, scope, v_opt, hbm_peak,
                                   sampler if tag == "sparse" else None,
                                   traffic_key=f"{args.workload}:{tag}")
    # the two-launch path (partials, then kvq_combine) for comparison
    two = StepGraphs(lambda i: (rep.decode(i, args.tau, fused=False), rep.combine(i)), args.steps, args.warmup)
    ms_two = reduce_max(time_steps(two, world), world, device)
    del two
    e2e = None if args.skip_e2e else e2e_arm(args, rep, wl, inp, device, world)
    sp = res["sparse"]
    launches = decode_launches_per_call(rep, device)
    line = {
        "metric": METRIC, "value": round(sp["us_per_token"], 4), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(sp["ms_per_step"], 6),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic",
        "config": {"workload": args.workload, "batch": wl.batch, "num_q_heads": wl.num_q_heads,
                   "num_kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim,
                   "context": list(wl.seq_lens) if wl.batch > 1 else wl.seq_lens[0],
                   "cache_format": wl.fmt, "tau": args.tau, "split_tokens": rep.L,
                   "v_fetch": V_FETCH_DEFAULT,
                   "cluster_max_schedule": {"split_tokens": rep.L_sh, "splits_per_cluster": rep.CS_sh},
                   "l2": (f"inputs rotate over {rep.R} cache copies "
                          f"({rep.R * rep.plane_bytes / 2**20:.0f} MiB > 3x L2)" if rep.l2_cold else
                          f"inputs rotate over {rep.R} cache copies "
                          f"({rep.R * rep.plane_bytes / 2**20:.1f} MiB < L2: timed with the cache in L2)"),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "timing": (f"warm-up and timed steps each one CUDA graph ({args.warmup} and "
                              f"{args.steps} kvq_decode_attn calls), CUDA events around one replay"),
                   "step": ("one kvq_decode_attn call: "
                            + ("one launch, merge in the kernel" if launches == 1
                               else "decode launch + combine launch"))},
        "roofline": {"bound": "hbm", "achieved": round(sp["achieved_gbs"], 1),
                     "peak": hbm_peak, "unit": "GB/s", "frac": round(sp["frac"], 4),
                     "traffic": sp["traffic"], "peak_kind": peak_kind,
                     "kernel": f"decode kernel <{wl.fmt},{wl.head_dim}>",
                     "algorithmic_bytes_per_launch": sp["algorithmic_bytes"],
                     "us_per_launch": round(sp["us_per_step"] / launches, 3)},
        "e2e": e2e,
        "gpu_launches": args.steps * launches,
        **{tag: _round(v) for tag, v in res.items()},
        "two_launch_us_per_token": round(ms_two * 1e3 / args.steps / (wl.batch * world), 4),
        "clocks": sampler.report(),
    }
    head_L = rep.L
    del rep
    torch.cuda.empty_cache()
    if args.all_workloads:
        line["workloads"] = {name: workload_table(args, world, device, name, hbm_peak)
                             for name in W.WORKLOADS}
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        line["cpu_baseline"] = cpu_baseline(wl, inp, head_L, args.tau, budget_s=args.cpu_seconds)
    if world > 1:
        import torch.distributed as td
        td.barrier()
        td.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


V_FETCH_DEFAULT = "library's choice (kvq.h: KVQ_OPT_V_KEPT_ONLY / KVQ_OPT_V_WITH_K)"


def decode_launches_per_call(rep, device):
    """Kernels one kvq_decode_attn call with an output launches: the decode kernel, plus the
    combine kernel when the request has more (split, sequence, KV head) units than CTAs
    that run at once (one per SM), as the library decides."""
    import torch
    units = rep.wl.batch * rep.wl.num_kv_heads * -(-max(rep.max_seq, 1) // rep.L)
    return 1 if units <= torch.cuda.get_device_properties(device).multi_processor_count else 2


def e2e_arm(args, rep, wl, inp, device, world):
    """Same metric through the public API with host buffers: every step copies the new
    token's q, k, v (one packed pinned host buffer) to the device, appends k/v to the
    cache (kvq_quantize_kv), runs the decode (with its in-kernel merge) and reads the
    output back to pinned host memory.  The step is captured once per cache copy as a
    CUDA graph of those public-API calls (how a serving loop issues it) and replayed;
    the eager form (every call from Python each step) is reported beside it, and the
    dense (tau = 0) path is timed the same way."""
    import torch
    B, Hq, Hkv, D = wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.head_dim
    nq, nkv = B * Hq * D, B * Hkv * D
    h_in = torch.cat([torch.from_numpy(inp.q).reshape(-1),
                      torch.from_numpy(inp.k[-B:]).reshape(-1),     # the newest position of each sequence
                      torch.from_numpy(inp.v[-B:]).reshape(-1)]).pin_memory()
    last = torch.from_numpy(np.array([int(inp.slots[int(o) - 1]) for o in inp.seq_offsets()[1:]],
                                     dtype=np.int32)).to(device)
    h_out = torch.empty((B, Hq, D), dtype=torch.float32).pin_memory()
    d_in = torch.empty_like(h_in, device=device)
    d_q = d_in[:nq].view(B, Hq, D)
    d_k = d_in[nq:nq + nkv].view(B, Hkv, D)
    d_v = d_in[nq + nkv:].view(B, Hkv, D)
    out = torch.empty((B, Hq, D), dtype=torch.float32, device=device)

    def make_step(tau):
        def step(i):
            c = rep.caches[i % rep.R]
            d_in.copy_(h_in, non_blocking=True)
            c.write(d_k, d_v, last)
            c.attention(d_q, rep.seq, rep.max_seq, rep.pt, inp.max_pages, tau=tau,
                        sm_scale=rep.sm, split_tokens=rep.L, out=out)
            h_out.copy_(out, non_blocking=True)
        return step

    def timed(run):
        for i in range(args.warmup):
            run(i)
        torch.cuda.synchronize()
        barrier(world)
        t0 = time.perf_counter()
        for i in range(args.steps):
            run(args.warmup + i)
        torch.cuda.synchronize()
        return reduce_max(time.perf_counter() - t0, world, device)

    per = lambda e: round(e * 1e6 / args.steps / (B * world), 3)  # noqa: E731
    res = {}
    for tag, tau in (("", args.tau), ("dense_", 0.0)):
        step = make_step(tau)
        el_eager = timed(step)
        R = min(rep.R, args.steps + args.warmup)  # one graph per cache copy the steps use
        graphs = [capture(step, 1, i) for i in range(R)]
        el = timed(lambda i: graphs[i % R].replay())
        del graphs
        res[tag + "value"] = per(el)
        res[tag + "eager_value"] = per(el_eager)
    bi = h_in.numel() * 2
    bo = h_out.numel() * 4
    return {"value": res["value"], "unit": UNIT,
            "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo,
            "how": "public API per step: H2D(q, k, v) + QuantizedKVCache.write + .attention + "
                   "D2H(out), captured as one CUDA graph per cache copy and replayed (host-timed)",
            "eager_value": res["eager_value"],
            "dense_value": res["dense_value"], "dense_eager_value": res["dense_eager_value"],
            "gpu_launches_per_step": 1 + decode_launches_per_call(rep, device)}


# ------------------------------------------------------------------ CPU oracle (baseline / reference arm)

def _oracle_group(task):
    """One (sequence, KV head) group of the oracle's sparse-V decode step, truncated to
    n_pos positions; runs in a worker process (spawned) or inline.  Returns seconds."""
    name, b, h, n_pos, split, tau = task
    from threadpoolctl import threadpool_limits
    from oracle import attention as OA
    from oracle import codebook as OC
    wl = W.WORKLOADS[name]
    inp = W.generate(wl) if _GEN.get(name) is None else _GEN[name]
    _GEN[name] = inp
    cb = OC.lloyd_max_f16(16, 1.0 / math.sqrt(wl.head_dim)) if wl.fmt == "lut4" else None
    off = int(inp.seq_offsets()[b])
    n = min(n_pos, int(inp.seq_lens[b]))
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        OA.decode_step(wl.fmt, inp.q[b:b + 1], inp.k[off:off + n], inp.v[off:off + n],
                       np.array([n], dtype=np.int32), wl.num_kv_heads, 1.0 / math.sqrt(wl.head_dim),
                       tau, split, signs=inp.signs, codebook16=cb, with_dense=False, groups=[(0, h)])
        return time.perf_counter() - t0


_GEN = {}


def _pool(n):
    import multiprocessing as mp
    return mp.get_context("spawn").Pool(n)


def oracle_all_cores(wl, inp, split, tau, n_pos, pool, workers):
    """Wall time of the oracle over every (sequence, KV head) group (each truncated to
    n_pos positions), the groups spread over ``workers`` spawned processes; returns
    (seconds, fraction of the workload's positions x KV heads covered)."""
    tasks = [(wl.name, b, h, n_pos, split, tau) for b in range(wl.batch) for h in range(wl.num_kv_heads)]
    t0 = time.perf_counter()
    pool.map(_oracle_group, tasks, chunksize=1)
    dt = time.perf_counter() - t0
    covered = sum(min(n_pos, int(n)) for n in inp.seq_lens) * wl.num_kv_heads
    return dt, covered / (int(inp.seq_lens.sum()) * wl.num_kv_heads)


def cpu_baseline(wl, inp, split, tau, budget_s=15.0):
    """The fp64 oracle as it stands on the host cores: one core (one group, repeated for
    about half the budget) and all cores (every group in parallel over spawned workers)."""
    _GEN[wl.name] = inp
    n_pos = int(inp.seq_lens[0])
    times = []
    t_end = time.perf_counter() + budget_s / 2
    while time.perf_counter() < t_end or not times:
        times.append(_oracle_group((wl.name, 0, 0, n_pos, split, tau)))
    frac1 = min(n_pos, int(inp.seq_lens[0])) / (int(inp.seq_lens.sum()) * wl.num_kv_heads)
    us_1 = statistics.median(times) / frac1 * 1e6 / wl.batch
    cores = len(os.sched_getaffinity(0))
    groups = wl.batch * wl.num_kv_heads
    workers = max(1, min(cores, groups))
    all_cores = None
    try:
        with _pool(workers) as pool:
            pool.map(_oracle_group, [(wl.name, 0, 0, 64, split, tau)] * workers)  # start-up, not timed
            reps = []
            t_end = time.perf_counter() + budget_s / 2
            while time.perf_counter() < t_end or not reps:
                dt, fr = oracle_all_cores(wl, inp, split, tau, n_pos, pool, workers)
                reps.append(dt / fr)
        all_cores = {"value": round(statistics.median(reps) * 1e6 / wl.batch, 1), "unit": UNIT,
                     "cores": workers, "host_cores": cores,
                     "sample": f"every (sequence, KV head) group ({groups}) truncated to {n_pos} positions, "
                               f"{len(reps)} runs over {workers} spawned worker processes, scaled to the workload"}
    except Exception as e:  # pragma: no cover - a host without process support
        all_cores = {"unavailable": str(e)}
    return {"value": round(us_1, 1), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"fp64 numpy oracle (quantize + dequant + schedule-exact sparse-V attention) "
                      f"on 1 of {wl.num_kv_heads} KV heads x {n_pos} positions, {len(times)} runs, "
                      f"scaled to the whole workload",
            "all_cores": all_cores}


def reference_arm(args, world, rank):
    if rank != 0:
        return
    wl = W.WORKLOADS[args.workload]
    inp = W.generate(wl)
    _GEN[wl.name] = inp
    split = 896
    cores = len(os.sched_getaffinity(0))
    workers = max(1, min(cores, wl.batch * wl.num_kv_heads))
    with _pool(workers) as pool:
        # size one step so that warmup + steps finish in about args.ref_budget seconds
        pilot = 1024
        dt, fr = oracle_all_cores(wl, inp, split, args.tau, pilot, pool, workers)
        per_pos = dt / pilot
        n_pos = int(args.ref_budget / max(args.steps + args.warmup, 1) / max(per_pos, 1e-9))
        n_pos = max(64, min(n_pos, int(inp.seq_lens.max())))
        for _ in range(args.warmup):
            oracle_all_cores(wl, inp, split, args.tau, n_pos, pool, workers)
        t = []
        frac = None
        for _ in range(args.steps):
            dt, frac = oracle_all_cores(wl, inp, split, args.tau, n_pos, pool, workers)
            t.append(dt)
    us_step = sum(t) / len(t) / frac * 1e6
    value = us_step / wl.batch
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(us_step / 1e3, 3), "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "cache_format": wl.fmt, "tau": args.tau,
                       "split_tokens": split},
            "cpu_baseline": {"value": round(value, 1), "unit": UNIT, "cores": workers, "kind": "oracle",
                             "sample": f"each step: fp64 oracle on every (sequence, KV head) group truncated "
                                       f"to {n_pos} positions over {workers} spawned workers "
                                       f"({cores} host cores), scaled to the whole workload"},
            "e2e": {"value": round(value, 1), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="gqa_32k_q4", choices=sorted(W.WORKLOADS))
    ap.add_argument("--tau", type=float, default=1e-6)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-budget", type=float, default=120.0)
    ap.add_argument("--skip-e2e", action="store_true", help="(profiling runs) skip the e2e leg")
    ap.add_argument("--split-tokens", type=int, default=0,
                    help="positions per split (0: the library's choice, kvq_resolve_split)")
    ap.add_argument("--headline-only", dest="all_workloads", action="store_false",
                    help="(profiling runs) skip the per-workload table of every configuration")
    ap.add_argument("--no-cluster", dest="cluster_variant", action="store_false",
                    help="(profiling runs) skip the cluster-shared-maximum variant, whose "
                         "cooperative cluster launch ncu's injection does not run")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_env()
    if args.impl == "reference":
        reference_arm(args, world, rank)
        return
    gpu_arm(args, world, rank, local)


if __name__ == "__main__":
    main()
