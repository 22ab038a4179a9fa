#!/usr/bin/env python
"""Benchmark of the DELTA decode attention stack on B200: one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config 5]

Default workload: the largest one that fits one GPU, the drifting decode trajectory
(drift-48l-b16-16k-bf16): 48 layers (0-1 full, delta-layers 2, 6 and 42, 43 sparse), 40 query /
8 KV heads, head_dim 128, batch 16, 16385-token start context growing one token per step for
1000 steps, 16-token pages, budget 2048 tokens + 16-token sink + 512-token recency window, 32
planted salient keys per (layer, sequence, KV head) that move by 256 tokens every 100 steps
(about 52 GB of KV cache).  A step is one decode step: the kv_append of every layer, then full,
delta or sparse attention for each of the 48 layers, replayed as one CUDA graph.

Timing: every step of the trajectory runs; K of them (all by default), evenly spread, are timed
with CUDA events on the replay stream, L2 flushed before each timed replay (outside the
events); W untimed replays of the first step come first.  The value is the mean time of a timed
step (with --gpus N, N independent replicas: the slowest replica's mean).  The same line carries
the kernel rooflines, the same build's all-full stack, the attended-token reduction, an
end-to-end time through the public API with host buffers, the fp64 oracle timed on the host
cores, and (on rank 0) the oracle's verdict on every delta-layer selection of every sequence at
the sampled steps.  --config 1..4 time one decode step of the other workloads instead.
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
L2_NOTE = "flushed before every timed replay (2xL2 write, then 2xL2 read), outside the events"


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (trajectory default: every step; single-step workloads: 200)")
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="budget of the oracle sample")
    ap.add_argument("--checks", type=int, default=-1,
                    help="trajectory steps whose delta-layer selections (every sequence) the oracle checks: "
                         "-1 every step at a drift boundary (0, 99, 100, ..., last), 0 none, m the first m of those")
    ap.add_argument("--oracle-procs", type=int, default=0, help="oracle worker processes (0: every host core)")
    ap.add_argument("--check-every-step", action="store_true",
                    help="trajectory: also check every step's delta-layer selections against the oracle "
                         "(minutes of host CPU after the timed loop)")
    ap.add_argument("--no-extra", action="store_true", help="skip the summaries of the 64k and 8k workloads")
    ap.add_argument("--print-source-hash", action="store_true", help="print the kernel-source hash and exit")
    ap.add_argument("--reduce", choices=["sum", "max"], default="sum",
                    help="head aggregation of the page score: sum (default) or the page's max rule")
    ap.add_argument("--delta-sweep", type=str, default="",
                    help="comma list of delta-layer counts: time the step for each (spread placement)")
    ap.add_argument("--layers", type=int, default=0,
                    help="keep only the first N layers of the workload (same shapes; for profiler captures)")
    ap.add_argument("--profile-run", action="store_true",
                    help="replay the decode step W + K times and exit without timing (for an ncu capture)")
    return ap.parse_args(argv)


def workload(args):
    """The selected workload, truncated to its first --layers layers when asked."""
    from synth import configs as C
    cfg = C.CONFIGS[args.config]
    if args.layers and args.layers < cfg.num_layers:
        dl = tuple(l for l in cfg.delta_layers if l < args.layers)
        if not dl:
            raise SystemExit("--layers must keep at least one delta-layer")
        cfg = cfg.with_(name=f"{cfg.name}-first{args.layers}", num_layers=args.layers, delta_layers=dl)
    return cfg


def run_profile(args):
    """Replay one decode step (the trajectory's first) W + K times: a short, fixed launch sequence for
    a profiler (per step: the append, then one attention launch per layer)."""
    import torch
    from synth.case import Case
    from synth.gpu import DeviceCase
    cfg = workload(args)
    if cfg.steps > 1:
        cfg = cfg.with_(steps=1, drift_every=0)
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    case = Case(cfg)
    dc = DeviceCase(case, device=device, prefill="append")
    st = make_stacks(cfg, case, dc, args.reduce)(cfg.layer_kinds())
    for _ in range(args.warmup + (args.steps or 3)):
        st.step(dc.q, dc.k_new, dc.v_new, dc.k_pools, dc.v_pools, dc.out)
    torch.cuda.synchronize()
    print(f"profile run: {cfg.name}, {args.warmup + (args.steps or 3)} steps of {st.launches_per_step()} launches "
          f"({', '.join(cfg.layer_kinds())})", flush=True)


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


def profiled_traffic(workload: str, kind: str):
    """(DRAM bytes per launch, summary file) of the decode kernel of a full, delta or sparse layer
    from the committed ncu summary of this workload, or (None, why) when there is none or the
    kernels changed since that capture."""
    name = f"decode_{kind}_{workload}.md"
    path = os.path.join(ROOT, "profiles", name)
    try:
        text = open(path).read()
    except OSError:
        return None, "no ncu summary for this workload"
    fields = {}
    for line in text.splitlines():
        if ":" in line and line.strip().startswith("- "):
            k, v = line.strip()[2:].split(":", 1)
            fields[k.strip()] = v.strip().strip("`")
    if fields.get("kernel_sources_sha256") != kernel_source_hash():
        return None, f"profiles/{name} was taken on other kernel sources"
    try:
        return int(fields["traffic_bytes_per_launch"]), f"profiles/{name}"
    except (KeyError, ValueError):
        return None, f"profiles/{name} has no traffic figure"


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


def gpu_index(device) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        try:
            return int(vis.split(",")[device.index])
        except (ValueError, IndexError):
            return device.index
    return device.index


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


def config_dict(cfg, reduce: str = "sum", world: int = 1) -> dict:
    """The workload, as both arms of the benchmark report it."""
    d = {"workload": cfg.name, "layers": cfg.num_layers, "delta_layers": list(cfg.delta_layers),
         "q_heads": cfg.num_q_heads, "kv_heads": cfg.num_kv_heads, "head_dim": cfg.head_dim, "batch": cfg.batch,
         "page_size": cfg.page_size, "budget_tokens": cfg.budget_tokens, "sink_tokens": cfg.sink_tokens,
         "recency_tokens": cfg.recency_tokens, "score": f"head {reduce}", "parallelism": f"replicas x{world}",
         "l2": L2_NOTE}
    if cfg.context_list:
        d["context"] = list(cfg.context_list)
    elif cfg.context:
        d["context"] = cfg.context
    else:
        d["context_range"] = list(cfg.context_range)
    if cfg.steps > 1:
        d.update({"trajectory_steps": cfg.steps, "drift_every": cfg.drift_every, "drift_shift": cfg.drift_shift})
    return d


# ---------------------------------------------------------------------------- accounting
def attended_tokens(cfg, case):
    """(delta_stack_tokens, full_stack_tokens, full_tokens_per_layer, sparse_tokens_per_layer) attended per
    step, summed over layers and sequences.

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


def delta_page_term_bytes(cfg, case) -> int:
    """Bytes a delta-layer moves for its page scores beyond attention: each (head, page) log-sum-exp
    and each (KV head, page) score share, written once and read once, plus the selection."""
    pages = sum(-(-int(n) // cfg.page_size) for n in case.n.tolist())
    sel = cfg.batch * (cfg.budget_pages + 40) * 4
    return pages * (cfg.num_q_heads + cfg.num_kv_heads) * 4 * 2 + sel


# ---------------------------------------------------------------------------- the oracle leg
class OracleSample:
    """The fp64 oracle (test infrastructure: only this leg of the benchmark runs it) on one full,
    one delta and one sparse layer of sequence 0, inputs generated once outside any timing; a
    step estimate scales them to the whole stack and batch."""

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

    def layer_us(self, min_seconds: float) -> dict:
        """Wall-clock microseconds per layer of each kind for one sequence (each kind repeated for
        about a third of min_seconds, at least twice, the first call not timed)."""
        O, c = self.O, self.cfg
        fns = {"full": lambda: O.full_attention(*self.data[self.l_full]),
               "delta": lambda: self._select(self.data[self.l_delta]),
               "sparse": lambda: O.sparse_attention(*self.data[self.l_sparse], self.sel, c.page_size)}
        out = {}
        for name, fn in fns.items():
            fn()
            k, t0 = 0, time.perf_counter()
            while True:
                fn()
                k += 1
                el = time.perf_counter() - t0
                if k >= 2 and el >= min_seconds / 3:
                    break
            out[name] = el / k * 1e6
        return out

    def step_us(self, times: dict) -> tuple:
        """(delta-stack us per step, full-stack us per step) for the whole batch."""
        n_kind = {k: self.kinds.count(k) for k in ("full", "delta", "sparse")}
        delta_us = self.cfg.batch * sum(n_kind[k] * times[k] for k in times)
        full_us = self.cfg.batch * len(self.kinds) * times["full"]
        return delta_us, full_us

    def describe(self, times: dict, seconds: float) -> str:
        c = self.cfg
        return (f"fp64 numpy oracle on the host cores, sequence 0 of {c.name}: one full / delta / sparse layer, each "
                f"repeated for ~{seconds / 3:.1f} s ({', '.join(f'{k} {v:.0f} us' for k, v in times.items())}), "
                f"scaled to the {c.num_layers}-layer step x batch {c.batch}")


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info] or [1])
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline_leg(cfg, case, seconds: float) -> dict:
    sample = OracleSample(cfg, case)
    times = sample.layer_us(min_seconds=seconds)
    d_us, f_us = sample.step_us(times)
    return {"value": round(d_us, 1), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": sample.describe(times, seconds), "full_stack_value": round(f_us, 1)}


def run_reference(args):
    """The reference arm: the fp64 oracle as it stands, timed on the host cores on a bounded sample of
    each step (rank 0 only)."""
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
    K = args.steps if args.steps else 20
    per_step_s = max(0.3, min(args.cpu_seconds / max(K + args.warmup, 1), 3.0))
    per_step, desc = [], None
    for i in range(args.warmup + K):
        times = sample.layer_us(min_seconds=per_step_s)
        d_us, _ = sample.step_us(times)
        if i >= args.warmup:
            per_step.append(d_us)
        desc = times
    value = statistics.mean(per_step)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": args.gpus,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(value / 1000, 6), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(cfg, args.reduce, world),
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": sample.describe(desc, per_step_s)},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


# ---------------------------------------------------------------------------- GPU measurement
class Gpu:
    """L2 flush buffers and event timing on the current stream of one device."""

    def __init__(self, device, dist=None):
        import torch
        self.torch = torch
        self.device, self.dist = device, dist
        l2 = torch.cuda.get_device_properties(device).L2_cache_size
        self.flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=device)
        self.flush_rd = torch.ones(max(2 * l2, 256 << 20) // 4, dtype=torch.float32, device=device)
        self.stream = torch.cuda.current_stream(device)

    def flush_l2(self):
        # write a buffer twice the size of L2, then read another one, so no dirty lines of the flush
        # are left to be written back inside the timed region
        self.flush.fill_(1)
        self.flush_rd.sum()

    def timed(self, replay, k: int, warm: int) -> list:
        torch = self.torch
        for _ in range(warm):
            self.flush_l2()
            replay()
        barrier(self.dist, self.device)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(k)]
        for s, e in ev:
            self.flush_l2()
            s.record(self.stream)
            replay()
            e.record(self.stream)
        barrier(self.dist, self.device)
        return [s.elapsed_time(e) * 1000.0 for s, e in ev]   # us

    def mean_us(self, replay, k: int, warm: int = 3) -> float:
        return max_over_ranks(self.dist, statistics.mean(self.timed(replay, k, warm)), self.device)


def make_stacks(cfg, case, dc, reduce):
    from long_context_layer_b200 import _native as NAT
    from long_context_layer_b200.stack import DeltaStack
    red = NAT.DELTA_HEAD_MAX if reduce == "max" else NAT.DELTA_HEAD_SUM
    mk = lambda kk: DeltaStack(kk, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, dc.dtype, dc.indptr, dc.indices,
                               dc.kv_len, case.max_pages_per_seq, dc.num_phys_pages, cfg.budget_pages,
                               cfg.sink_tokens, cfg.recency_tokens, reduce=red)
    return mk


def kernel_measurements(gpu, cfg, case, dc, d0, us_full_stack: float, k: int, with_breakdown: bool = True) -> dict:
    """Rooflines of the three decode kernels of a step and a per-call breakdown.

    Each kernel runs L times in one CUDA graph (the layers' own q and pools), timed like the steps;
    the per-launch average is its steady-state duration.  Sparse layers run on the first
    delta-layer's selection, all but the first launch through the settled entry, as in a step;
    the full-layer figure comes from the all-full stack graph (L launches + 1 append, the append
    charged to the kernel).  Algorithmic bytes: the attended tokens' K and V of every sequence,
    plus q and o (delta-layers also their page-score terms).
    """
    import torch
    from long_context_layer_b200 import _native as NAT
    st = gpu.stream.cuda_stream
    kinds = cfg.layer_kinds()
    L = cfg.num_layers
    lk = kinds.index("delta")
    ls = kinds.index("sparse")
    di = d0.delta_layers.index(lk)
    e = 2 if cfg.dtype == "bf16" else 4
    kvtok = 2 * cfg.num_kv_heads * cfg.head_dim * e
    qo = 2 * cfg.batch * cfg.num_q_heads * cfg.head_dim * e
    _, _, full_tok, sparse_tok = attended_tokens(cfg, case)
    peak, peak_kind = load_peaks()

    def graph_of(calls):
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(gpu.device)
        side.wait_stream(gpu.stream)
        with torch.cuda.stream(side):
            calls(side.cuda_stream)   # warm outside capture (per-device kernel attributes)
        gpu.stream.wait_stream(side)
        with torch.cuda.graph(g):
            calls(torch.cuda.current_stream(gpu.device).cuda_stream)
        return g

    def sparse_calls(s):
        for l in range(L):
            fn = NAT.sparse_attn if l == 0 else NAT.sparse_attn_settled
            fn(d0.desc, d0.pt, d0.sel_cnt[di], d0.sel_pages[di], d0.sel_stride, dc.q[l], dc.k_pools[l],
               dc.v_pools[l], dc.out[l], d0.workspace, d0.ws_bytes, s)

    def delta_calls(s):
        for l in range(L):
            NAT.select_attn(d0.desc, d0.pt, d0.sp, dc.q[l], dc.k_pools[l], dc.v_pools[l], dc.out[l], d0.sel_cnt[di],
                            d0.sel_pages[di], d0.sel_stride, None, d0.workspace, d0.ws_bytes, s)
        # leave the first delta-layer's own selection in place for the sparse launches
        NAT.select_attn(d0.desc, d0.pt, d0.sp, dc.q[lk], dc.k_pools[lk], dc.v_pools[lk], dc.out[lk], d0.sel_cnt[di],
                        d0.sel_pages[di], d0.sel_stride, None, d0.workspace, d0.ws_bytes, s)

    g_delta = graph_of(delta_calls)
    us_delta_launch = gpu.mean_us(g_delta.replay, k) / (L + 1)
    g_sparse = graph_of(sparse_calls)
    us_sparse_launch = gpu.mean_us(g_sparse.replay, k) / L
    del g_delta, g_sparse

    def roof(kernel, alg, us, launches, timing, kind):
        traffic, source = profiled_traffic(cfg.name, kind)
        achieved = alg / (us * 1e-6) / 1e9
        return {"kernel": kernel, "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "peak_source": peak_kind, "alg_bytes_per_launch": int(alg),
                "us_per_launch": round(us, 3), "launches_per_step": launches, "timing": timing,
                "traffic": traffic, "traffic_source": source}

    n_sparse = kinds.count("sparse")
    n_delta = kinds.count("delta")
    out = {
        "roofline": roof("decode_mma_kernel, sparse layer (selected pages, split-KV, cluster merge)",
                         sparse_tok * kvtok + qo, us_sparse_launch, n_sparse,
                         "graph of L sparse launches on a delta-layer's selection (all but the first through the "
                         "settled entry, as in the step) / L, CUDA events, L2 flushed", "sparse_layer"),
        "roofline_full_layer": roof("decode_mma_kernel, full layer (split-KV, cluster merge)",
                                    full_tok * kvtok + qo, us_full_stack / L, L - n_sparse - n_delta,
                                    "all-full stack graph (L launches + 1 append) / L, CUDA events, L2 flushed",
                                    "full_layer"),
        "roofline_delta_layer": roof("decode_mma_kernel, delta layer (full attention + page scores + selection in "
                                     "the last CTA of each sequence)",
                                     full_tok * kvtok + qo + delta_page_term_bytes(cfg, case), us_delta_launch,
                                     n_delta, "graph of L + 1 delta-layer launches / (L + 1), CUDA events, L2 flushed",
                                     "delta_layer"),
    }
    if cfg.dtype != "bf16":
        for key in out:
            out[key]["kernel"] = out[key]["kernel"].replace("decode_mma_kernel", "decode_kernel (fp32)")
    if with_breakdown:
        def append_call():
            NAT.kv_append(d0.desc, d0.pt, dc.k_new[0], dc.v_new[0], dc.k_pools[0], dc.v_pools[0], st)

        def full_call():
            NAT.full_attn(d0.desc, d0.pt, dc.q[0], dc.k_pools[0], dc.v_pools[0], dc.out[0], d0.workspace,
                          d0.ws_bytes, st)

        def select_call():
            NAT.select_attn(d0.desc, d0.pt, d0.sp, dc.q[lk], dc.k_pools[lk], dc.v_pools[lk], dc.out[lk],
                            d0.sel_cnt[di], d0.sel_pages[di], d0.sel_stride, None, d0.workspace, d0.ws_bytes, st)

        def sparse_call():
            NAT.sparse_attn(d0.desc, d0.pt, d0.sel_cnt[di], d0.sel_pages[di], d0.sel_stride, dc.q[ls],
                            dc.k_pools[ls], dc.v_pools[ls], dc.out[ls], d0.workspace, d0.ws_bytes, st)

        out["breakdown_us_per_call"] = {
            name: round(gpu.mean_us(fn, k), 3)
            for name, fn in (("kv_append", append_call), ("full_attn", full_call), ("select_attn", select_call),
                             ("sparse_attn", sparse_call))}
        out["breakdown_note"] = "each call launched alone from the host, L2 flushed before it (includes launch latency)"
    out["roofline"]["share_of_step"] = None
    return out


def e2e_measure(gpu, cfg, dc, mk, k: int) -> dict:
    """End to end through the public API with host buffers (DeltaStack.step_host): every step the
    appended tokens and every layer's q go from pinned host memory to the device (q layer by layer
    on a copy stream, overlapping the earlier layers' attention), the step runs, and each layer's
    output returns to pinned host memory as soon as its kernel is done; one CUDA graph per step."""
    import torch
    q_h, kn_h, vn_h = (x.cpu().pin_memory() for x in (dc.q, dc.k_new, dc.v_new))
    out_h = torch.empty_like(dc.out, device="cpu").pin_memory()
    q_d, kn_d, vn_d = (torch.empty_like(x) for x in (dc.q, dc.k_new, dc.v_new))
    stack = mk(cfg.layer_kinds())
    host_args = (q_h, kn_h, vn_h, dc.k_pools, dc.v_pools, out_h, q_d, kn_d, vn_d, dc.out)
    stack.step_host(*host_args)   # outside capture: per-device kernel attributes, copy streams
    torch.cuda.synchronize(gpu.device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        stack.step_host(*host_args)
    us = gpu.mean_us(g.replay, k)
    e = q_h.element_size()
    del g
    return {"value": round(us, 3), "unit": UNIT, "h2d_bytes_per_step": (q_h.numel() + kn_h.numel() + vn_h.numel()) * e,
            "d2h_bytes_per_step": out_h.numel() * e,
            "how": "DeltaStack.step_host in one CUDA graph: pinned host k_new/v_new, then each layer's q, to the "
                   "device on a copy stream; each layer's output to pinned host as its kernel ends; CUDA events "
                   "around the replay"}


def run_static(args, cfg, dist, rank, world, device, headline: bool = True) -> dict:
    """One decode step of a single-step workload: the DELTA stack, the all-full stack, the kernel
    rooflines, a per-call breakdown, e2e and the oracle on the host cores."""
    import torch
    from synth.case import Case
    from synth.gpu import DeviceCase
    case = Case(cfg)
    dc = DeviceCase(case, device=device, prefill="append")
    mk = make_stacks(cfg, case, dc, args.reduce)
    delta_stack = mk(cfg.layer_kinds())
    full_stack = mk(["full"] * cfg.num_layers)
    step_args = (dc.q, dc.k_new, dc.v_new, dc.k_pools, dc.v_pools, dc.out)
    g_delta = delta_stack.capture(*step_args)
    g_full = full_stack.capture(*step_args)
    gpu = Gpu(device, dist)
    K = args.steps if args.steps else 200
    k2 = max(min(K, 100), 10)
    sampler = ClockSampler(gpu_index(device))
    sampler.start()
    time.sleep(0.3)
    t_delta = gpu.timed(g_delta.replay, K, args.warmup)
    clocks = sampler.stop()
    us_delta = max_over_ranks(dist, statistics.mean(t_delta), device)
    us_full = gpu.mean_us(g_full.replay, k2)
    km = kernel_measurements(gpu, cfg, case, dc, delta_stack, us_full, k2, with_breakdown=headline)
    n_sparse = cfg.layer_kinds().count("sparse")
    km["roofline"]["share_of_step"] = round(n_sparse * km["roofline"]["us_per_launch"] / us_delta, 3)
    tok_delta, tok_full, _, _ = attended_tokens(cfg, case)
    res = {"us_per_step": round(us_delta, 3), "full_stack_us": round(us_full, 3),
           "speedup_vs_full_stack": round(us_full / us_delta, 3),
           "attended_token_reduction": round(tok_full / tok_delta, 3)}
    res.update(km)
    if headline:
        res["e2e"] = e2e_measure(gpu, cfg, dc, mk, K)
        res["clocks"] = clocks
        res["gpu_launches"] = delta_stack.launches_per_step() * K
        res["cpu_baseline"] = (cpu_baseline_leg(cfg, case, args.cpu_seconds)
                               if rank == 0 and world == 1 and not args.no_cpu_baseline else None)
        res["planted_logit_boost"] = planted_logit_boost(cfg, case, sorted(cfg.delta_layers))
    del g_delta, g_full
    delta_stack.graph = None
    full_stack.graph = None
    del dc
    torch.cuda.empty_cache()
    return res


def check_points(cfg, m: int) -> list:
    """Trajectory steps the oracle checks: the first step, both sides of every drift boundary, the last."""
    T = cfg.steps
    pts = {0, T - 1}
    if cfg.drift_every:
        for s in range(cfg.drift_every, T, cfg.drift_every):
            pts.update((s - 1, s))
    pts = sorted(pts)
    return pts if m < 0 else pts[:m]


def planted_logit_boost(cfg, case, layers, sample: int = 256) -> dict | None:
    """The synthetic workload's planted-key strength, measured on its stored values: the mean rise of
    the scaled logit q_h . k / sqrt(D) that planting gives a key (planted row against the same
    position's unplanted generator row, over the G query heads of its KV head), and the standard
    deviation of the unplanted logits (the first `sample` positions), for the given layers."""
    import numpy as np
    from synth import rng
    if cfg.planted == 0 or not layers:
        return None
    G, D = cfg.group, cfg.head_dim
    sc = 1.0 / np.sqrt(D)
    rises, spread = [], []
    for l in layers:
        q = case.q(l).astype(np.float64)
        for b in range(cfg.batch):
            for g in range(cfg.num_kv_heads):
                qg = q[b, g * G:(g + 1) * G]
                pos, rows = case.planted_rows(l, b, g)
                if pos.size:
                    base = case.kv_base(rng.T_K, l, b, g, pos).astype(np.float64)
                    rises.append(((rows.astype(np.float64) - base) @ qg.T * sc).ravel())
                ref = case.kv_base(rng.T_K, l, b, g, np.arange(min(sample, int(case.n[b])))).astype(np.float64)
                spread.append((ref @ qg.T * sc).std(axis=0))
    return {"mean_rise_nats": round(float(np.concatenate(rises).mean()), 3) if rises else None,
            "unplanted_logit_std": round(float(np.concatenate(spread).mean()), 3),
            "layers": list(layers)}


def selection_quality(cfg, case, layers, cnt, pages) -> dict:
    """How the GPU's selections behave along the trajectory: the fraction of each step's selected
    pages that the previous step also selected (per delta-layer and sequence), and the fraction of
    the planted keys' pages that the selection in force covers, for every layer it serves (the
    delta-layer itself and the sparse layers after it).  cnt [T, n_delta, B], pages [T, n_delta, B, stride]."""
    import numpy as np
    T, nd, B, stride = pages.shape
    P, de = cfg.page_size, cfg.drift_every or T
    mask = np.zeros((T, nd, B, case.max_pages_per_seq), dtype=bool)
    t, i, b, s = np.nonzero(np.arange(stride)[None, None, None, :] < cnt[..., None])
    mask[t, i, b, np.clip(pages[t, i, b, s], 0, case.max_pages_per_seq - 1)] = True
    res = {}
    if T > 1:
        ov = (mask[1:] & mask[:-1]).sum(-1) / np.maximum(mask[1:].sum(-1), 1)   # [T-1, nd, B]
        moved = np.array([(k + 1) % de == 0 for k in range(T - 1)])
        res["step_overlap"] = {"mean": round(float(ov.mean()), 4), "min": round(float(ov.min()), 4),
                               "mean_at_drift_steps": round(float(ov[moved].mean()), 4) if moved.any() else None,
                               "mean_other_steps": round(float(ov[~moved].mean()), 4)}
    served = [range(l, layers[k + 1] if k + 1 < nd else cfg.num_layers) for k, l in enumerate(layers)]
    rec_all, rec_delta, rec_first = [], [], []
    for t0 in range(0, T, de):
        t1 = min(t0 + de, T)
        for k in range(nd):
            for l in served[k]:
                for bb in range(B):
                    pos = [case.planted_positions(l, bb, g, t0) for g in range(cfg.num_kv_heads)]
                    pp = np.unique(np.concatenate(pos) // P) if pos else np.zeros(0, dtype=np.int64)
                    if len(pp) == 0:
                        continue
                    r = mask[t0:t1, k, bb][:, pp].mean(axis=1)   # per step
                    rec_all.append(r)
                    if l == layers[k]:
                        rec_delta.append(r)
                    rec_first.append(r[:1])
    if rec_all:
        res["planted_page_recall"] = {
            "served_layers_mean": round(float(np.concatenate(rec_all).mean()), 4),
            "served_layers_min": round(float(np.concatenate(rec_all).min()), 4),
            "delta_layers_mean": round(float(np.concatenate(rec_delta).mean()), 4),
            "first_step_after_each_drift_mean": round(float(np.concatenate(rec_first).mean()), 4)}
    res["how"] = ("every step's selections copied to pinned host memory after the step (outside the timed "
                  "region); overlap = |sel_t & sel_t-1| / |sel_t|; recall = share of the pages holding a "
                  "layer's planted keys (all KV heads) inside the selection that layer uses")
    return res


def run_trajectory(args, cfg, dist, rank, world, device) -> dict:
    """The drifting trajectory: every decode step replays one CUDA graph; between steps (untimed)
    the cache grows by one token per sequence and, every drift_every steps, the planted keys move."""
    import numpy as np
    import torch
    from synth.trajectory import Trajectory

    T = cfg.steps
    K = min(args.steps, T) if args.steps else T
    timed_steps = sorted({int(round(i * (T - 1) / max(K - 1, 1))) for i in range(K)}) if K > 1 else [0]
    checks = check_points(cfg, args.checks) if rank == 0 else []
    every_step = rank == 0 and args.check_every_step and bool(cfg.delta_layers)
    pool = None
    if checks or every_step:
        from oracle.parallel import OraclePool
        pool = OraclePool(args.oracle_procs or None)   # spawn-started: safe after CUDA init

    tr = Trajectory(cfg, device=device)
    dc = tr.dc
    case0 = tr.case0
    mk = make_stacks(cfg, case0, dc, args.reduce)
    stack = mk(cfg.layer_kinds())
    full_stack = mk(["full"] * cfg.num_layers)
    tr.prepare(0)
    step_args = (dc.q, dc.k_new, dc.v_new, dc.k_pools, dc.v_pools, dc.out)
    g = stack.capture(*step_args)
    g_full = full_stack.capture(*step_args)
    gpu = Gpu(device, dist)
    k2 = max(min(K, 50), 10)

    # ---- at the first step (appending the same token again changes nothing): DELTA vs all-full
    #      stack, kernel rooflines, per-call breakdown, end to end through the public API
    us_delta0 = gpu.mean_us(g.replay, k2)
    us_full0 = gpu.mean_us(g_full.replay, k2)
    km = kernel_measurements(gpu, cfg, case0, dc, stack, us_full0, k2)
    e2e = e2e_measure(gpu, cfg, dc, mk, k2)
    del g_full
    full_stack.graph = None

    # ---- the trajectory (the headline)
    sampler = ClockSampler(gpu_index(device))
    sampler.start()
    time.sleep(0.3)
    for _ in range(args.warmup):
        gpu.flush_l2()
        g.replay()
    barrier(dist, device)
    timed = set(timed_steps)
    events, pending, gpu_sel, gpu_out = [], [], {}, {}
    ld = stack.delta_layers
    hist_cnt = torch.empty((T, len(ld), cfg.batch), dtype=torch.int32, pin_memory=True)
    hist_pages = torch.empty((T, len(ld), cfg.batch, stack.sel_stride), dtype=torch.int32, pin_memory=True)
    for step in range(T):
        tr.prepare(step)
        if step in timed:
            gpu.flush_l2()
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record(gpu.stream)
            g.replay()
            s1.record(gpu.stream)
            events.append((s0, s1))
        else:
            g.replay()
        hist_cnt[step].copy_(stack.sel_cnt, non_blocking=True)    # after the step's end event
        hist_pages[step].copy_(stack.sel_pages, non_blocking=True)
        if step in checks:   # copies only: the oracle runs after the timed loop (host cores stay free)
            cnt = stack.sel_cnt.cpu().numpy()
            pages = stack.sel_pages.cpu().numpy()
            outs = dc.out[ld].float().cpu().numpy()
            for i, l in enumerate(ld):
                for b in range(cfg.batch):
                    gpu_sel[(step, l, b)] = pages[i, b, :cnt[i, b]].tolist()
                    gpu_out[(step, l, b)] = outs[i, b]
    barrier(dist, device)
    clocks = sampler.stop()
    if checks:
        pending.append(pool.submit([(cfg, step, "delta", l, b) for step in checks for l in ld
                                    for b in range(cfg.batch)]))
    lat = np.array([s.elapsed_time(e) * 1000.0 for s, e in events])
    us = max_over_ranks(dist, float(lat.mean()), device)

    # ---- the oracle's verdict on the sampled steps
    check = None
    if pending:
        from oracle.checks import selection_ok
        ok = exact = total = 0
        worst_abs = worst_rel = 0.0
        for res in pending:
            for job, (o_ref, S) in res.get():
                _, step, _, l, b = job
                n = int(cfg.contexts(step)[b])
                good, ex, _ = selection_ok(gpu_sel[(step, l, b)], S, n, cfg.budget_pages, cfg.sink_tokens,
                                           cfg.recency_tokens, cfg.page_size)
                ok += int(good)
                exact += int(ex)
                total += 1
                o = gpu_out[(step, l, b)].astype(np.float64)
                worst_abs = max(worst_abs, float(np.abs(o - o_ref).max()))
                worst_rel = max(worst_rel, float(np.linalg.norm(o - o_ref) / max(np.linalg.norm(o_ref), 1e-30)))
        check = {"selection_match_rate": round(ok / total, 4), "selections_checked": total,
                 "selections_exact": exact, "steps_checked": checks,
                 "rule": "every delta-layer x every sequence at each checked step; a match is the oracle's set, "
                         "pages swapped only inside a band of scores within 1e-4 relative plus 2^-50 absolute "
                         "of the k-th",
                 "delta_output_max_abs_err": round(worst_abs, 6), "delta_output_max_rel_l2": round(worst_rel, 6)}
    every = None
    if every_step:
        from oracle.checks import selection_ok
        t_chk = time.time()
        de = cfg.drift_every or T
        jobs = [(cfg, min(t0 + de, T) - 1, "delta_block", l, b, list(range(t0, min(t0 + de, T))))
                for t0 in range(0, T, de) for l in ld for b in range(cfg.batch)]
        ok = exact = total = 0
        bad = []
        for job, scores in pool.imap(jobs):
            _, _, _, l, b, steps = job
            i = ld.index(l)
            for t, S in zip(steps, scores):
                n = int(cfg.contexts(t)[b])
                sel = hist_pages[t, i, b, :int(hist_cnt[t, i, b])].tolist()
                good, ex, _ = selection_ok(sel, S, n, cfg.budget_pages, cfg.sink_tokens, cfg.recency_tokens,
                                           cfg.page_size)
                ok += int(good)
                exact += int(ex)
                total += 1
                if not good and len(bad) < 8:
                    bad.append({"step": t, "layer": l, "b": b})
        every = {"selection_match_rate": round(ok / max(total, 1), 4), "selections_checked": total,
                 "selections_exact": exact, "steps": T, "mismatches": bad,
                 "host_seconds": round(time.time() - t_chk, 1)}
    if pool is not None:
        pool.close()

    quality = selection_quality(cfg, case0, ld, hist_cnt.numpy(), hist_pages.numpy()) if ld else None
    tok = [attended_tokens(cfg, tr.case_at(s)) for s in (0, T - 1)]
    n_sparse = cfg.layer_kinds().count("sparse")
    km["roofline"]["share_of_step"] = round(n_sparse * km["roofline"]["us_per_launch"] / us_delta0, 3)
    res = {
        "us_per_step": round(us, 3),
        "trajectory": {"per_step_us": {"mean": round(float(lat.mean()), 3), "median": round(float(np.median(lat)), 3),
                                       "p99": round(float(np.percentile(lat, 99)), 3),
                                       "first": round(float(lat[0]), 3), "last": round(float(lat[-1]), 3)},
                       "timed_steps": len(timed_steps), "steps_run": T, "oracle_check": check,
                       "selection_quality": quality, "every_step_check": every,
                       "planted_logit_boost": planted_logit_boost(cfg, case0, ld)},
        "step0_us": round(us_delta0, 3), "full_stack_us": round(us_full0, 3),
        "speedup_vs_full_stack": round(us_full0 / us_delta0, 3),
        "attended_token_reduction": round(statistics.mean(t[1] / t[0] for t in tok), 3),
        "speedup_note": "DELTA and all-full stacks both timed at the trajectory's first step",
    }
    res.update(km)
    res["e2e"] = e2e
    res["clocks"] = clocks
    res["gpu_launches"] = stack.launches_per_step() * len(timed_steps)
    res["cpu_baseline"] = (cpu_baseline_leg(cfg, case0, args.cpu_seconds)
                           if rank == 0 and world == 1 and not args.no_cpu_baseline else None)
    del g
    stack.graph = None
    del tr, dc
    torch.cuda.empty_cache()
    return res


def run_ours(args):
    import torch
    from synth import configs as C
    dist, rank, world, local = dist_init()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    cfg = workload(args)
    if cfg.steps > 1:
        r = run_trajectory(args, cfg, dist, rank, world, device)
        K = r["trajectory"]["timed_steps"]
    else:
        r = run_static(args, cfg, dist, rank, world, device)
        K = args.steps if args.steps else 200
    also = {}
    if not args.no_extra and world == 1 and args.config == 5:
        ea = parse(["--steps", "20", "--warmup", "3", "--reduce", args.reduce])
        for c in (C.LLAMA8B_64K, C.QWEN7B_8K):
            x = run_static(ea, c, dist, rank, world, device, headline=False)
            also[c.name] = {key: x[key] for key in ("us_per_step", "full_stack_us", "speedup_vs_full_stack",
                                                    "attended_token_reduction")}
            for key in ("roofline", "roofline_full_layer", "roofline_delta_layer"):
                also[c.name][key] = {f: x[key][f] for f in ("frac", "achieved", "us_per_launch", "alg_bytes_per_launch")}
    us = r.pop("us_per_step")
    if rank == 0:
        line = {"metric": METRIC, "value": us, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
                "ms_per_step": round(us / 1000, 6), "higher_is_better": False, "scaling": "weak",
                "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
                "config": config_dict(cfg, args.reduce, world)}
        line.update(r)
        if also:
            line["also"] = also
        print(json.dumps(line), flush=True)
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
    from synth.case import Case
    from synth.gpu import DeviceCase

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    case = Case(cfg)
    dc = DeviceCase(case, device=device, prefill="append")
    gpu = Gpu(device)
    step_args = (dc.q, dc.k_new, dc.v_new, dc.k_pools, dc.v_pools, dc.out)
    mk = make_stacks(cfg, case, dc, args.reduce)
    K = args.steps if args.steps else 50

    def time_kinds(kinds):
        st = mk(kinds)
        g = st.capture(*step_args)
        ts = gpu.timed(g.replay, K, args.warmup)
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
                      "kernel_sources_sha256": kernel_source_hash(),
                      "full_stack_us": round(full_us, 3), "steps": K, "warmup": args.warmup,
                      "points": points}), flush=True)


def main():
    args = parse()
    if args.print_source_hash:
        print(kernel_source_hash())
        return
    if args.impl == "reference":
        run_reference(args)
        return
    if args.profile_run:
        run_profile(args)
    elif args.delta_sweep:
        run_delta_sweep(args, workload(args), [int(x) for x in args.delta_sweep.split(",")])
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
