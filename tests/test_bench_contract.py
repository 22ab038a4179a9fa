"""Host-side checks of bench.py: the reference arm's JSON line and the attended-token accounting
that the roofline's algorithmic bytes are built from (no GPU needed)."""
import json
import os
import subprocess
import sys

import numpy as np

from oracle import delta_oracle as O
from synth import configs as C
from synth.case import Case

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "1",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["higher_is_better"] is False and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"] == C.TINY.name


def test_attended_tokens_match_the_oracle_selection():
    # the sparse-layer token count the roofline uses equals the tokens of the oracle's selection
    import bench
    for cfg in (C.TINY, C.QWEN7B_8K.with_(context=8192 - 5)):
        case = Case(cfg)
        delta_tok, full_tok_stack, full_tok, sparse_tok = bench.attended_tokens(cfg, case)
        n = int(case.n[0])
        S = np.zeros(-(-n // 16))   # scores do not change the count: ties keep k candidates
        sel = O.select_pages(S, n, 16, cfg.budget_pages, cfg.sink_tokens, cfg.recency_tokens)
        assert sparse_tok == len(O.page_tokens(sel, n, 16))
        assert full_tok == n
        kinds = cfg.layer_kinds()
        assert full_tok_stack == len(kinds) * n
        assert delta_tok == kinds.count("sparse") * sparse_tok + (len(kinds) - kinds.count("sparse")) * n


def test_sweep_placement_spreads_delta_layers_from_layer_2():
    import bench
    for L in (28, 32, 48):
        for m in range(1, L - 1):
            pl = bench.delta_placement(L, m)
            assert pl[0] == 2 and len(pl) == m and pl == sorted(set(pl)) and pl[-1] < L
        assert bench.delta_placement(L, L - 2) == list(range(2, L))   # every layer from 2: the full stack


def test_both_arms_report_the_same_config_dict():
    import bench
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "1",
                        "--steps", "2", "--warmup", "1", "--cpu-seconds", "1"], capture_output=True, text=True,
                       timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads([l for l in r.stdout.splitlines() if l.strip().startswith("{")][0])
    # the GPU arm prints bench.config_dict(cfg, reduce, world) for the same workload
    assert d["config"] == json.loads(json.dumps(bench.config_dict(C.TINY, "sum", 1)))
    assert d["steps"] == 2 and d["warmup"] == 1


def test_trajectory_check_points_straddle_every_drift_boundary():
    import bench
    pts = bench.check_points(C.DRIFT_48L, -1)
    assert pts[0] == 0 and pts[-1] == 999 and len(pts) == 20   # 0, 99, 100, ..., 899, 900, 999
    for s in range(100, 1000, 100):
        assert s - 1 in pts and s in pts
    assert bench.check_points(C.DRIFT_48L, 3) == [0, 99, 100]
    assert bench.check_points(C.DRIFT_48L, 0) == []


def test_selection_quality_overlap_and_planted_recall():
    import dataclasses
    import bench
    cfg = dataclasses.replace(C.DRIFT_48L, batch=2, num_layers=8, steps=6, drift_every=3)
    case = Case(cfg, step=0)
    layers = [2, 5]
    T, nd, B, N = cfg.steps, len(layers), cfg.batch, case.max_pages_per_seq
    stride = N
    # every page selected at every step: overlap 1, recall 1
    cnt = np.full((T, nd, B), N, dtype=np.int32)
    pages = np.broadcast_to(np.arange(N, dtype=np.int32), (T, nd, B, N)).copy()
    q = bench.selection_quality(cfg, case, layers, cnt, pages)
    assert q["step_overlap"]["mean"] == 1.0 and q["planted_page_recall"]["served_layers_mean"] == 1.0
    # only the sink page: planted keys lie past the sink tokens, so recall is 0
    cnt1 = np.ones((T, nd, B), dtype=np.int32)
    pages1 = np.zeros((T, nd, B, stride), dtype=np.int32)
    q = bench.selection_quality(cfg, case, layers, cnt1, pages1)
    assert q["planted_page_recall"]["served_layers_mean"] == 0.0 and q["step_overlap"]["min"] == 1.0
    # exactly the delta-layer's own planted pages at each step: its recall is 1; the selection
    # changes at the drift step (3), where the overlap drops
    cnt2 = np.zeros((T, nd, B), dtype=np.int32)
    pages2 = np.zeros((T, nd, B, stride), dtype=np.int32)
    for t in range(T):
        for k, l in enumerate(layers):
            for b in range(B):
                pos = np.concatenate([case.planted_positions(l, b, g, t) for g in range(cfg.num_kv_heads)])
                pp = np.unique(pos // cfg.page_size)
                cnt2[t, k, b] = len(pp)
                pages2[t, k, b, :len(pp)] = pp
    q = bench.selection_quality(cfg, case, layers, cnt2, pages2)
    r = q["planted_page_recall"]
    assert r["delta_layers_mean"] == 1.0 and 0.0 < r["served_layers_mean"] < 1.0
    ov = q["step_overlap"]
    assert ov["mean_other_steps"] == 1.0 and ov["mean_at_drift_steps"] < 1.0


def test_planted_logit_boost_reports_the_rise_of_planted_keys():
    import bench
    cfg = C.QWEN7B_8K.with_(num_layers=4, delta_layers=(2,))
    q = bench.planted_logit_boost(cfg, Case(cfg), [2])
    # k <- 0.5 k + 3 q_hat with q_hat the unit mean of the group's queries: about 3 |q| cos / sqrt(D)
    assert 0.8 < q["mean_rise_nats"] < 1.6
    assert 0.9 < q["unplanted_logit_std"] < 1.1
    assert bench.planted_logit_boost(C.TINY, Case(C.TINY), [1]) is None   # nothing planted
