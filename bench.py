#!/usr/bin/env python
"""Benchmark of one DELTA decode step (every layer of the stack) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config 2]

Default workload: the Qwen-7B-shaped stack in bf16 (28 layers: 0-1 full, delta-layers 2
and 14, 24 sparse; 28 query / 4 KV heads, head_dim 128; batch 1, context 8192, 16-token
pages; budget 1024 tokens + 16-token sink + 256-token recency window), synthetic inputs with
32 planted salient keys per (layer, KV head).  A step is one decode step: kv_append, then
full, delta or sparse attention, for each of the 28 layers, captured as one CUDA graph.

Timing: W untimed replays, then K timed replays, L2 flushed (a 2x L2-sized write) before every
replay outside the events; CUDA events on the replay stream; max over ranks.  Prints one JSON
line.  With --gpus N > 1 (torchrun) every rank runs an independent replica (the path does
not shard across GPUs) and the reported time is the slowest rank's.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "us_per_decode_step_layer_stack"
UNIT = "us/step"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="budget of the oracle sample")
    ap.add_argument("--print-source-hash", action="store_true", help="print the kernel-source hash and exit")
    ap.add_argument("--drift-checks", type=int, default=10, help="oracle selection checks along a trajectory")
    ap.add_argument("--reduce", choices=["sum", "max"], default="sum",
                    help="head aggregation of the page score: sum (default) or the page's max rule")
    ap.add_argument("--delta-sweep", type=str, default="",
                    help="comma list of delta-layer counts: time the step for each (spread placement)")
    return ap.parse_args()


# ---------------------------------------------------------------------------- helpers
def kernel_source_hash() -> str:
    """sha256 over the CUDA sources of the library (identifies the kernels a profile was taken on)."""
    import hashlib
    d = os.path.join(ROOT, "long_context_layer_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(os.listdir(d)):
        if f.endswith((".cu", ".cuh", ".h")):
            h.update(f.encode())
            with open(os.path.join(d, f), "rb") as fh:
                h.update(fh.read())
    return h.hexdigest()


def profiled_traffic(workload: str, kind: str = "full_layer"):
    """DRAM bytes per launch of the decode kernel in a full or sparse layer, from the committed ncu
    summary of this workload, or None when the kernels changed since that capture."""
    path = os.path.join(ROOT, "profiles", f"decode_{kind}_{workload}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    fields = {}
    for line in text.splitlines():
        if ":" in line and line.strip().startswith("- "):
            k, v = line.strip()[2:].split(":", 1)
            fields[k.strip()] = v.strip().strip("`")
    if fields.get("kernel_sources_sha256") != kernel_source_hash():
        return None
    try:
        return int(fields["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        mhz, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(mhz)}


def dist_init():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1:
        import torch.distributed as dist
        from datetime import timedelta
        # NCCL on GPUs; the CPU tests of the multi-rank path run the same code over gloo
        dist.init_process_group(os.environ.get("DELTA_DIST_BACKEND", "nccl"), timeout=timedelta(seconds=120))
        return dist, int(os.environ.get("RANK", "0")), ws, int(os.environ.get("LOCAL_RANK", "0"))
    return None, 0, 1, 0


def max_over_ranks(dist, x: float, device) -> float:
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist, device):
    import torch
    if dist is not None:
        if device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()
    if device.type == "cuda":
        torch.cuda.synchronize(device)


# ---------------------------------------------------------------------------- accounting
def attended_tokens(cfg, case):
    """(delta_stack_tokens, full_stack_tokens) attended per step, summed over layers and sequences.

    Sparse layers attend the tokens of the selected pages: every sink/recency page plus k
    candidate pages, the last page partial (computed from the selection rule's page counts).
    """
    P = cfg.page_size
    kinds = cfg.layer_kinds()
    full_tok = 0
    sparse_tok = 0
    for n in case.n.tolist():
        N = -(-n // P)
        sinkP = -(-min(cfg.sink_tokens, n) // P)
        recStart = max(n - cfg.recency_tokens, 0) // P if cfg.recency_tokens > 0 else N
        forced = set(range(sinkP)) | set(range(recStart, N))
        cand = N - len(forced)
        pages = len(forced) + min(cfg.budget_pages, cand)
        tail_missing = (N * P - n) if (N - 1) in forced or cand <= cfg.budget_pages else 0
        sparse_tok += pages * P - tail_missing
        full_tok += n
    n_sparse = kinds.count("sparse")
    n_dense = len(kinds) - n_sparse
    return n_dense * full_tok + n_sparse * sparse_tok, len(kinds) * full_tok, full_tok, sparse_tok


# ---------------------------------------------------------------------------- reference arm
class OracleSample:
    """The fp64 oracle on one full, one delta and one sparse layer of sequence 0 (inputs
    generated once, outside any timing); a step estimate scales them to the whole stack."""

    def __init__(self, cfg, case):
        import numpy as np
        from oracle import delta_oracle as O
        from synth import rng
        self.cfg, self.O = cfg, O
        kinds = cfg.layer_kinds()
        self.kinds = kinds
        self.l_delta = kinds.index("delta")
        self.l_full = kinds.index("full") if "full" in kinds else self.l_delta
        self.l_sparse = kinds.index("sparse")
        b = 0
        self.n = int(case.n[b])

        def kv(l):
            K = np.stack([case.kv_logical(rng.T_K, l, b, g) for g in range(cfg.num_kv_heads)]).astype(np.float64)
            V = np.stack([case.kv_logical(rng.T_V, l, b, g) for g in range(cfg.num_kv_heads)]).astype(np.float64)
            return K, V

        self.data = {l: (case.q(l)[b].astype(np.float64),) + kv(l) for l in (self.l_full, self.l_delta, self.l_sparse)}
        self.sel = self._select(self.data[self.l_delta])

    def _select(self, qkv):
        c, O = self.cfg, self.O
        _, p = O.full_attention(*qkv)
        return O.select_pages(O.page_scores(p, c.page_size), self.n, c.page_size, c.budget_pages, c.sink_tokens,
                              c.recency_tokens)

    def layer_us(self, min_seconds: float = 0.0, max_reps: int = 200) -> dict:
        """Wall-clock microseconds per layer of each kind for one sequence."""
        O, c = self.O, self.cfg
        fns = {"full": lambda: O.full_attention(*self.data[self.l_full]),
               "delta": lambda: self._select(self.data[self.l_delta]),
               "sparse": lambda: O.sparse_attention(*self.data[self.l_sparse], self.sel, c.page_size)}
        out = {}
        for name, fn in fns.items():
            k, t0 = 0, time.perf_counter()
            while True:
                fn()
                k += 1
                el = time.perf_counter() - t0
                if el >= min_seconds / 3 or k >= max_reps:
                    break
            out[name] = el / k * 1e6
        return out

    def step_us(self, times: dict) -> tuple:
        """(delta-stack us per step, full-stack us per step) for the whole batch."""
        n_kind = {k: self.kinds.count(k) for k in ("full", "delta", "sparse")}
        delta_us = self.cfg.batch * sum(n_kind[k] * times[k] for k in times)
        full_us = self.cfg.batch * len(self.kinds) * times["full"]
        return delta_us, full_us


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info] or [1])
    except Exception:
        return os.cpu_count() or 1


def run_reference(args):
    dist, rank, world, local = dist_init()
    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return
    from synth import configs as C
    from synth.case import Case
    cfg = C.CONFIGS[args.config]
    case = Case(cfg)
    sample = OracleSample(cfg, case)
    per_step = []
    desc = None
    for i in range(args.warmup + args.steps):
        times = sample.layer_us(max_reps=1)
        d_us, _ = sample.step_us(times)
        if i >= args.warmup:
            per_step.append(d_us)
        desc = times
    value = statistics.mean(per_step)
    cores = blas_threads()
    sample = (f"fp64 numpy oracle, sequence 0, one full / delta / sparse layer per step "
              f"({', '.join(f'{k} {v:.0f} us' for k, v in desc.items())}), scaled to {cfg.num_layers} layers "
              f"x batch {cfg.batch}")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(value / 1000, 6),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "batch": cfg.batch, "context": int(case.n.max()), "layers": cfg.num_layers},
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


# ---------------------------------------------------------------------------- drifting trajectory
def run_trajectory(args, cfg):
    """The drifting workload: one CUDA graph per decode step replayed along the trajectory, the
    cache growing one token per step and the planted keys moving every `drift_every` steps.
    Reports per-step latency and, on sampled steps, the rate at which the GPU selection of
    sequence 0 at the first delta-layer matches the fp64 oracle's."""
    import numpy as np
    import torch
    from long_context_layer_b200.stack import DeltaStack
    from synth.trajectory import Trajectory

    dist, rank, world, local = dist_init()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    tr = Trajectory(cfg, device=device)
    dc = tr.dc
    stack = DeltaStack(cfg.layer_kinds(), cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, dc.dtype, dc.indptr,
                       dc.indices, dc.kv_len, tr.case0.max_pages_per_seq, dc.num_phys_pages, cfg.budget_pages,
                       cfg.sink_tokens, cfg.recency_tokens)
    tr.prepare(0)
    g = stack.capture(dc.q, dc.k_new, dc.v_new, dc.k_pools, dc.v_pools, dc.out)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=device)
    flush_rd = torch.ones(max(2 * l2, 256 << 20) // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)
    steps = min(args.steps, cfg.steps)
    check_every = max(steps // max(args.drift_checks, 1), 1)
    checks = set(range(0, steps, check_every)) if args.drift_checks > 0 else set()
    lat, matched, checked = [], 0, 0
    ld = cfg.layer_kinds().index("delta")
    for step in range(steps):
        tr.prepare(step)
        for _ in range(args.warmup if step == 0 else 0):
            g.replay()
        flush.fill_(1)
        flush_rd.sum()
        barrier(dist, device)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        g.replay()
        s1.record(stream)
        s1.synchronize()
        lat.append(s0.elapsed_time(s1) * 1000.0)
        if rank == 0 and step in checks:
            from oracle import delta_oracle as O
            from synth import rng
            case = tr.case_at(step)
            n = int(case.n[0])
            K = np.stack([case.kv_logical(rng.T_K, ld, 0, h) for h in range(cfg.num_kv_heads)]).astype(np.float64)
            V = np.stack([case.kv_logical(rng.T_V, ld, 0, h) for h in range(cfg.num_kv_heads)]).astype(np.float64)
            _, p = O.full_attention(case.q(ld)[0].astype(np.float64), K, V)
            ref = O.select_pages(O.page_scores(p, cfg.page_size), n, cfg.page_size, cfg.budget_pages,
                                 cfg.sink_tokens, cfg.recency_tokens)
            matched += int(stack.selection(stack.delta_layers.index(ld))[0] == ref)
            checked += 1
    per = np.array(lat)
    us = max_over_ranks(dist, float(per.mean()), device)
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(us, 3), "unit": UNIT, "n_gpus": world, "steps": steps,
            "warmup": args.warmup, "ms_per_step": round(us / 1000, 6), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
            "config": {"workload": cfg.name, "layers": cfg.num_layers, "delta_layers": list(cfg.delta_layers),
                       "q_heads": cfg.num_q_heads, "kv_heads": cfg.num_kv_heads, "head_dim": cfg.head_dim,
                       "batch": cfg.batch, "start_context": int(tr.case0.n.max()), "drift_every": cfg.drift_every,
                       "drift_shift": cfg.drift_shift, "budget_tokens": cfg.budget_tokens,
                       "l2": "flushed before every timed replay (2xL2 write, then 2xL2 read)"},
            "trajectory": {"per_step_us": {"mean": round(float(per.mean()), 3),
                                           "median": round(float(np.median(per)), 3),
                                           "p99": round(float(np.percentile(per, 99)), 3),
                                           "first": round(float(per[0]), 3), "last": round(float(per[-1]), 3)},
                           "selection_match_rate": (round(matched / checked, 4) if checked else None),
                           "selection_checks": checked,
                           "selection_check": "sequence 0, first delta-layer, exact match with the fp64 oracle"},
            "gpu_launches": stack.launches_per_step() * steps,
        }
        print(json.dumps(line), flush=True)
    del g
    stack.graph = None
    if dist is not None:
        dist.destroy_process_group()


# ---------------------------------------------------------------------------- our arm
def run_ours(args):
    import torch
    from long_context_layer_b200 import _native as NAT
    from long_context_layer_b200.stack import DeltaStack
    from synth import configs as C
    from synth.case import Case
    from synth.gpu import DeviceCase

    dist, rank, world, local = dist_init()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    cfg = C.CONFIGS[args.config]
    case = Case(cfg)
    dc = DeviceCase(case, device=device, prefill="append")
    kinds = cfg.layer_kinds()
    reduce = NAT.DELTA_HEAD_MAX if args.reduce == "max" else NAT.DELTA_HEAD_SUM
    mk = lambda kk: DeltaStack(kk, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, dc.dtype, dc.indptr, dc.indices,
                               dc.kv_len, case.max_pages_per_seq, dc.num_phys_pages, cfg.budget_pages,
                               cfg.sink_tokens, cfg.recency_tokens, reduce=reduce)
    delta_stack = mk(kinds)
    full_stack = mk(["full"] * cfg.num_layers)
    args_step = (dc.q, dc.k_new, dc.v_new, dc.k_pools, dc.v_pools, dc.out)
    g_delta = delta_stack.capture(*args_step)
    g_full = full_stack.capture(*args_step)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=device)
    flush_rd = torch.ones(max(2 * l2, 256 << 20) // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)

    def flush_l2():
        # write a buffer twice the size of L2, then read another one, so no dirty lines of the
        # flush are left to be written back inside the timed region
        flush.fill_(1)
        flush_rd.sum()

    def timed(replay, k, warm):
        for _ in range(warm):
            flush_l2()
            replay()
        barrier(dist, device)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(k)]
        for s, e in ev:
            flush_l2()
            s.record(stream)
            replay()
            e.record(stream)
        barrier(dist, device)
        return [s.elapsed_time(e) * 1000.0 for s, e in ev]   # us

    sampler = ClockSampler(device.index if not os.environ.get("CUDA_VISIBLE_DEVICES") else
                           int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[device.index]))
    sampler.start()
    time.sleep(0.3)
    t_delta = timed(g_delta.replay, args.steps, args.warmup)
    clocks = sampler.stop()
    t_full = timed(g_full.replay, max(args.steps // 2, 3), 3)
    us_delta = max_over_ranks(dist, statistics.mean(t_delta), device)
    us_full = max_over_ranks(dist, statistics.mean(t_full), device)

    # -- dominant kernel: the decode kernel of a full layer, timed alone (one launch per call)
    st = stream.cuda_stream
    d0 = delta_stack
    layer0 = 0

    def full_call():
        NAT.full_attn(d0.desc, d0.pt, dc.q[layer0], dc.k_pools[layer0], dc.v_pools[layer0], dc.out[layer0],
                      d0.workspace, d0.ws_bytes, st)

    t_kernel = timed(full_call, max(args.steps, 20), 3)
    us_kernel = max_over_ranks(dist, statistics.mean(t_kernel), device)

    # -- per-call breakdown (each call timed alone, L2 flushed before it)
    lk = kinds.index("delta")
    ls = kinds.index("sparse")
    di = d0.delta_layers.index(lk)

    def append_call():
        NAT.kv_append(d0.desc, d0.pt, dc.k_new[0], dc.v_new[0], dc.k_pools[0], dc.v_pools[0], st)

    def select_call():
        NAT.select_attn(d0.desc, d0.pt, d0.sp, dc.q[lk], dc.k_pools[lk], dc.v_pools[lk], dc.out[lk], d0.sel_cnt[di],
                        d0.sel_pages[di], d0.sel_stride, None, d0.workspace, d0.ws_bytes, st)

    def sparse_call():
        NAT.sparse_attn(d0.desc, d0.pt, d0.sel_cnt[di], d0.sel_pages[di], d0.sel_stride, dc.q[ls], dc.k_pools[ls],
                        dc.v_pools[ls], dc.out[ls], d0.workspace, d0.ws_bytes, st)

    # -- the sparse-layer decode (24 of the 28 launches of a step): L launches of it in one graph,
    #    all on the delta-layer's selection, timed like the steps; per-launch average.  As in the
    #    step, every launch after the first uses the settled entry (its predecessor is sparse).
    lay = list(range(cfg.num_layers))
    sg = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(device)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for l in lay:   # warm outside capture (per-device kernel attributes)
            NAT.sparse_attn(d0.desc, d0.pt, d0.sel_cnt[di], d0.sel_pages[di], d0.sel_stride, dc.q[l], dc.k_pools[l],
                            dc.v_pools[l], dc.out[l], d0.workspace, d0.ws_bytes, side.cuda_stream)
    stream.wait_stream(side)
    with torch.cuda.graph(sg):
        cs = torch.cuda.current_stream(device).cuda_stream
        for l in lay:
            fn = NAT.sparse_attn if l == 0 else NAT.sparse_attn_settled
            fn(d0.desc, d0.pt, d0.sel_cnt[di], d0.sel_pages[di], d0.sel_stride, dc.q[l], dc.k_pools[l],
               dc.v_pools[l], dc.out[l], d0.workspace, d0.ws_bytes, cs)
    t_sparse = timed(sg.replay, max(args.steps // 2, 10), 3)
    us_sparse_launch = max_over_ranks(dist, statistics.mean(t_sparse), device) / len(lay)
    del sg

    n_b = max(args.steps // 2, 10)
    breakdown = {name: round(max_over_ranks(dist, statistics.mean(timed(fn, n_b, 3)), device), 3)
                 for name, fn in (("kv_append", append_call), ("full_attn", full_call),
                                  ("select_attn", select_call), ("sparse_attn", sparse_call))}
    e = 2 if cfg.dtype == "bf16" else 4
    kv_bytes = int(case.n.sum()) * 2 * cfg.num_kv_heads * cfg.head_dim * e
    qo_bytes = 2 * cfg.batch * cfg.num_q_heads * cfg.head_dim * e
    alg_bytes = kv_bytes + qo_bytes
    peak, peak_kind = load_peaks()
    # The full-attention stack is one graph of L launches of this same decode kernel (plus one
    # append launch), timed with CUDA events: its per-launch average is the kernel's duration in
    # steady state (the append is charged to it, which only lowers the figure).  The single call
    # timed above also carries a launch latency no graph pays; it is reported alongside.
    us_launch = us_full / cfg.num_layers
    achieved = alg_bytes / (us_launch * 1e-6) / 1e9
    achieved_single = alg_bytes / (us_kernel * 1e-6) / 1e9
    # sparse layers: the tokens of the selected pages of every sequence
    _, _, _, sparse_tok = attended_tokens(cfg, case)
    alg_sparse = sparse_tok * 2 * cfg.num_kv_heads * cfg.head_dim * e + qo_bytes
    achieved_sparse = alg_sparse / (us_sparse_launch * 1e-6) / 1e9
    n_sparse = kinds.count("sparse")

    # -- end to end through the public API: every step the step's inputs (q, k_new, v_new) come
    #    from one pinned host staging buffer in one copy, the step runs (the same calls, captured in
    #    a graph over views of the device staging buffer) and every layer's output goes back to
    #    pinned host memory
    nq, nk = dc.q.numel(), dc.k_new.numel()
    in_h = torch.cat([dc.q.reshape(-1), dc.k_new.reshape(-1), dc.v_new.reshape(-1)]).cpu().pin_memory()
    in_d = torch.empty_like(in_h, device=device)
    in_d.copy_(in_h)
    q_v = in_d[:nq].view_as(dc.q)
    kn_v = in_d[nq:nq + nk].view_as(dc.k_new)
    vn_v = in_d[nq + nk:].view_as(dc.v_new)
    out_h = torch.empty_like(dc.out, device="cpu").pin_memory()
    e2e_stack = mk(kinds)
    g_e2e = e2e_stack.capture(q_v, kn_v, vn_v, dc.k_pools, dc.v_pools, dc.out)

    def e2e_step():
        in_d.copy_(in_h, non_blocking=True)
        g_e2e.replay()
        out_h.copy_(dc.out, non_blocking=True)

    t_e2e = timed(e2e_step, args.steps, 3)
    us_e2e = max_over_ranks(dist, statistics.mean(t_e2e), device)
    h2d = in_h.numel() * e
    d2h = out_h.numel() * e
    del g_e2e
    e2e_stack.graph = None

    tok_delta, tok_full, _, _ = attended_tokens(cfg, case)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sample = OracleSample(cfg, case)
        times = sample.layer_us(min_seconds=args.cpu_seconds)
        d_us, f_us = sample.step_us(times)
        cpu = {"value": round(d_us, 1), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": ("fp64 numpy oracle on the host cores, sequence 0, one full / delta / sparse layer "
                          f"repeated for ~{args.cpu_seconds:.0f} s ({', '.join(f'{k} {v:.0f} us' for k, v in times.items())}), "
                          f"scaled to the {cfg.num_layers}-layer step x batch {cfg.batch}"),
               "full_stack_value": round(f_us, 1)}
    launches = delta_stack.launches_per_step() * args.steps
    if rank == 0:
        line = {
            # whole job: N replicas each finish a decode step in us_delta (slowest rank), so the job
            # spends us_delta / N per decode step; ms_per_step is one step iteration of the job
            "metric": METRIC, "value": round(us_delta / world, 3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(us_delta / 1000, 6),
            "replica_step_us": round(us_delta, 3), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
            "config": {"workload": cfg.name, "layers": cfg.num_layers, "delta_layers": list(cfg.delta_layers),
                       "q_heads": cfg.num_q_heads, "kv_heads": cfg.num_kv_heads, "head_dim": cfg.head_dim,
                       "batch": cfg.batch, "context": int(case.n.max()), "page_size": cfg.page_size,
                       "budget_tokens": cfg.budget_tokens, "sink_tokens": cfg.sink_tokens,
                       "recency_tokens": cfg.recency_tokens, "l2": "flushed before every timed replay (2xL2 write, then 2xL2 read)",
                       "parallelism": f"replicas x{world}", "score": f"head {args.reduce}"},
            "full_stack_us": round(us_full, 3),
            "speedup_vs_full_stack": round(us_full / us_delta, 3),
            "attended_token_reduction": round(tok_full / tok_delta, 3),
            # the kernel that dominates the step: the decode kernel of the sparse layers
            "roofline": {"kernel": "decode_mma_kernel, sparse layer (selected pages, split-KV, cluster merge)",
                         "bound": "hbm", "achieved": round(achieved_sparse, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved_sparse / peak, 4), "peak_source": peak_kind,
                         "alg_bytes_per_launch": alg_sparse, "us_per_launch": round(us_sparse_launch, 3),
                         "launches_per_step": n_sparse,
                         "share_of_step": round(n_sparse * us_sparse_launch / us_delta, 3),
                         "timing": ("graph of L sparse launches on the delta-layer's selection (all but the first "
                                    "through the settled entry, as in the step) / L, CUDA events, L2 flushed"),
                         "traffic": profiled_traffic(cfg.name, "sparse_layer")},
            "roofline_full_layer": {"kernel": "decode_mma_kernel, full layer (split-KV, cluster merge)", "bound": "hbm",
                                    "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                                    "frac": round(achieved / peak, 4), "peak_source": peak_kind,
                                    "alg_bytes_per_launch": alg_bytes, "us_per_launch": round(us_launch, 3),
                                    "launches_per_step": len(kinds) - n_sparse,
                                    "timing": "full-attention stack graph (L launches + 1 append) / L, CUDA events, L2 flushed",
                                    "single_call_us": round(us_kernel, 3),
                                    "single_call_frac": round(achieved_single / peak, 4),
                                    "traffic": profiled_traffic(cfg.name, "full_layer")},
            "breakdown_us_per_call": breakdown,
            "e2e": {"value": round(us_e2e / world, 3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches,
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    # release graphs before tearing down the process group
    del g_delta, g_full
    delta_stack.graph = None
    full_stack.graph = None
    if dist is not None:
        dist.destroy_process_group()


# ---------------------------------------------------------------------------- delta-layer sweep
def delta_placement(num_layers: int, m: int) -> list:
    """m delta-layers, the first at layer 2 (the page's rule) and the rest spread evenly to the end."""
    span = num_layers - 2
    return sorted({2 + (i * span) // m for i in range(m)})


def run_delta_sweep(args, cfg, counts):
    """Decode-step time against the number of delta-layers on one workload (one JSON line)."""
    import torch
    from long_context_layer_b200.stack import DeltaStack
    from synth.case import Case
    from synth.gpu import DeviceCase

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    case = Case(cfg)
    dc = DeviceCase(case, device=device, prefill="append")
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=device)
    flush_rd = torch.ones(max(2 * l2, 256 << 20) // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)
    args_step = (dc.q, dc.k_new, dc.v_new, dc.k_pools, dc.v_pools, dc.out)

    def time_kinds(kinds):
        st = DeltaStack(kinds, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, dc.dtype, dc.indptr, dc.indices,
                        dc.kv_len, case.max_pages_per_seq, dc.num_phys_pages, cfg.budget_pages, cfg.sink_tokens,
                        cfg.recency_tokens)
        g = st.capture(*args_step)
        ts = []
        for i in range(args.warmup + args.steps):
            flush.fill_(1)
            flush_rd.sum()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            g.replay()
            e1.record(stream)
            e1.synchronize()
            if i >= args.warmup:
                ts.append(e0.elapsed_time(e1) * 1000.0)
        del g
        st.graph = None
        return statistics.median(ts)

    points = []
    L = cfg.num_layers
    full_us = time_kinds(["full"] * L)
    for m in counts:
        m = max(1, min(m, L - 2))
        dl = delta_placement(L, m)
        c2 = cfg.with_(delta_layers=tuple(dl))
        tok_delta, tok_full, _, _ = attended_tokens(c2, case)
        us = time_kinds(c2.layer_kinds())
        points.append({"delta_layers": dl, "count": len(dl), "us_per_step": round(us, 3),
                       "speedup_vs_full_stack": round(full_us / us, 3),
                       "attended_token_reduction": round(tok_full / tok_delta, 3)})
    print(json.dumps({"metric": "us_per_decode_step_vs_delta_layer_count", "unit": "us/step",
                      "config": {"workload": cfg.name, "layers": L, "batch": cfg.batch,
                                 "context": int(case.n.max())},
                      "full_stack_us": round(full_us, 3), "steps": args.steps, "warmup": args.warmup,
                      "points": points}), flush=True)


def main():
    args = parse()
    if args.print_source_hash:
        print(kernel_source_hash())
        return
    if args.impl == "reference":
        run_reference(args)
        return
    from synth import configs as C
    cfg = C.CONFIGS[args.config]
    if args.delta_sweep:
        run_delta_sweep(args, cfg, [int(x) for x in args.delta_sweep.split(",")])
    elif cfg.steps > 1:
        run_trajectory(args, cfg)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
