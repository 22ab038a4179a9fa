"""GPU parity at the full sizes of the two largest workloads, checked by the fp64 oracle on every
host core (a spawn-started pool, so it is safe after CUDA initialisation).

* The drifting 48-layer trajectory (batch 16, 16385-token start, delta-layers 2, 6, 42): steps 0
  to 100 run as in the benchmark (one token appended per step, the planted keys moved at step
  100).  At steps 0 and 100 every delta-layer selection of every sequence is checked, and the
  outputs of layers 0, 2, 3, 6, 7, 42, 43 and 47 of three sequences.
* The Llama-3-8B-shaped 64k stack (batch 4, delta-layers 2, 12, 22): every delta-layer selection
  of every sequence and the outputs of layers 0, 2, 3, 12, 13, 22 and 31 of sequences 0 and 3.

Sparse layers are checked against the oracle's attention over the pages the GPU selected (the
selection itself is checked against the oracle's separately).
"""
import gc

import numpy as np
import pytest
import torch

from oracle.checks import selection_ok
from oracle.parallel import OraclePool
from synth import configs as C
from tests.helpers import assert_close

pytestmark = pytest.mark.gpu


def governing_delta(kinds, layer):
    return max(l for l in range(layer + 1) if kinds[l] == C.DELTA)


def jobs_for(cfg, step, gpu_sel, out_layers, out_seqs):
    """Oracle jobs: every delta-layer of every sequence, and the sampled outputs."""
    kinds = cfg.layer_kinds()
    jobs = [(cfg, step, "delta", l, b) for l in cfg.delta_layers for b in range(cfg.batch)]
    for b in out_seqs:
        for l in out_layers:
            if kinds[l] == C.FULL:
                jobs.append((cfg, step, "full", l, b))
            elif kinds[l] == C.SPARSE:
                jobs.append((cfg, step, "sparse", l, b, tuple(gpu_sel[(governing_delta(kinds, l), b)])))
    return jobs


def snapshot(stack, dc):
    cnt = stack.sel_cnt.cpu().numpy()
    pages = stack.sel_pages.cpu().numpy()
    sel = {(l, b): pages[i, b, :cnt[i, b]].tolist() for i, l in enumerate(stack.delta_layers)
           for b in range(cnt.shape[1])}
    return sel, dc.out.float().cpu().numpy()


def verify(cfg, step, results, sel, out, out_seqs):
    exact = 0
    for job, res in results:
        kind, l, b = job[2], job[3], job[4]
        if kind == "delta":
            o_ref, S = res
            n = int(cfg.contexts(step)[b])
            ok, ex, _ = selection_ok(sel[(l, b)], S, n, cfg.budget_pages, cfg.sink_tokens, cfg.recency_tokens)
            assert ok, f"{cfg.name} step {step}: delta-layer {l} sequence {b} selection differs from the oracle"
            exact += ex
            if b in out_seqs:
                assert_close(out[l, b], o_ref, cfg.dtype, f"{cfg.name} step {step} delta l={l} b={b}")
        else:
            assert_close(out[l, b], res, cfg.dtype, f"{cfg.name} step {step} {kind} l={l} b={b}")
    return exact


def test_drift_trajectory_full_size_steps_0_and_100():
    from long_context_layer_b200.stack import DeltaStack
    from synth.trajectory import Trajectory
    cfg = C.DRIFT_48L
    out_layers, out_seqs = (0, 2, 3, 6, 7, 42, 43, 47), (0, 7, 15)
    with OraclePool() as pool:
        tr = Trajectory(cfg)
        dc = tr.dc
        st = DeltaStack(cfg.layer_kinds(), cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, dc.dtype, dc.indptr,
                        dc.indices, dc.kv_len, tr.case0.max_pages_per_seq, dc.num_phys_pages, cfg.budget_pages,
                        cfg.sink_tokens, cfg.recency_tokens)
        pending = []
        for step in range(101):
            tr.prepare(step)
            st.step(dc.q, dc.k_new, dc.v_new, dc.k_pools, dc.v_pools, dc.out)
            if step in (0, 100):
                sel, out = snapshot(st, dc)
                pending.append((step, sel, out, pool.submit(jobs_for(cfg, step, sel, out_layers, out_seqs))))
        from long_context_layer_b200 import read_device_error
        assert read_device_error(st.workspace, torch.cuda.current_stream().cuda_stream) == (0, 0)
        del tr, dc, st
        gc.collect()
        torch.cuda.empty_cache()
        total_exact = 0
        for step, sel, out, res in pending:
            total_exact += verify(cfg, step, res.get(), sel, out, out_seqs)
    # near-ties are rare: almost every selection is the oracle's set exactly
    assert total_exact >= 2 * 3 * cfg.batch - 2


def test_llama_64k_full_size_every_delta_selection():
    from long_context_layer_b200.stack import DeltaStack
    from synth.case import Case
    from synth.gpu import DeviceCase
    cfg = C.LLAMA8B_64K
    out_layers, out_seqs = (0, 2, 3, 12, 13, 22, 31), (0, 3)
    with OraclePool() as pool:
        case = Case(cfg)
        dc = DeviceCase(case, prefill="append")
        st = DeltaStack(cfg.layer_kinds(), cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, dc.dtype, dc.indptr,
                        dc.indices, dc.kv_len, case.max_pages_per_seq, dc.num_phys_pages, cfg.budget_pages,
                        cfg.sink_tokens, cfg.recency_tokens)
        st.step(dc.q, dc.k_new, dc.v_new, dc.k_pools, dc.v_pools, dc.out)
        sel, out = snapshot(st, dc)
        res = pool.submit(jobs_for(cfg, 0, sel, out_layers, out_seqs))
        del dc, st
        gc.collect()
        torch.cuda.empty_cache()
        exact = verify(cfg, 0, res.get(), sel, out, out_seqs)
    assert exact >= 3 * cfg.batch - 1
