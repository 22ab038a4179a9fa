"""GPU parity along a drifting decode trajectory: the cache grows by one token per step and the
planted salient keys move every `drift_every` steps; outputs and selections are checked against
the fp64 oracle before and after each move."""
import numpy as np
import pytest
import torch

from oracle import delta_oracle as O
from synth import configs as C
from tests.helpers import assert_close, oracle_kv, selection_ok

pytestmark = pytest.mark.gpu

# The drifting workload's shape (40 query / 8 KV heads, D = 128, bf16, delta-layers as the
# 48-layer list) at a reduced length: 8 layers, 2 sequences, 2049-token start, 300 steps.
SMALL_DRIFT = C.DRIFT_48L.with_(name="drift-small", cfg_id=95, num_layers=8, delta_layers=(2, 6), batch=2,
                                context=2049, steps=300, drift_every=100, drift_shift=64, budget_tokens=256,
                                recency_tokens=128)


def test_drift_trajectory_matches_oracle_across_moves():
    from long_context_layer_b200.stack import DeltaStack
    from synth.trajectory import Trajectory
    cfg = SMALL_DRIFT
    tr = Trajectory(cfg)
    dc = tr.dc
    st = DeltaStack(cfg.layer_kinds(), cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, dc.dtype, dc.indptr,
                    dc.indices, dc.kv_len, tr.case0.max_pages_per_seq, dc.num_phys_pages, cfg.budget_pages,
                    cfg.sink_tokens, cfg.recency_tokens)
    checks = {0, 99, 100, 199, 200, 299}
    matched, total = 0, 0
    for step in range(cfg.steps):
        tr.prepare(step)
        st.step(dc.q, dc.k_new, dc.v_new, dc.k_pools, dc.v_pools, dc.out)
        if step not in checks:
            continue
        torch.cuda.synchronize()
        case = tr.case_at(step)
        out = dc.out.float().cpu().numpy()
        kinds = cfg.layer_kinds()
        for b in range(cfg.batch):
            n = int(case.n[b])
            assert n == cfg.context + step
            sel = None
            for l, kind in enumerate(kinds):
                K, V = oracle_kv(case, l, b)
                q = case.q(l)[b].astype(np.float64)
                if kind == C.SPARSE:
                    assert_close(out[l, b], O.sparse_attention(q, K, V, sel, 16), "bf16", f"step {step} l={l}")
                    continue
                o, p = O.full_attention(q, K, V)
                assert_close(out[l, b], o, "bf16", f"step {step} l={l} b={b}")
                if kind == C.DELTA:
                    S = O.page_scores(p, 16)
                    gsel = st.selection(st.delta_layers.index(l))[b]
                    ok, exact, ref = selection_ok(gsel, S, n, cfg.budget_pages, cfg.sink_tokens, cfg.recency_tokens)
                    assert ok, f"step {step} layer {l} b={b}"
                    matched += exact
                    total += 1
                    sel = gsel
    assert total == len(checks) * cfg.batch * len(cfg.delta_layers)
    assert matched >= total - 1
