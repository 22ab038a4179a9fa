"""The oracle pool's jobs against direct oracle calls (CPU, small drifting workload)."""
import numpy as np
import pytest

from oracle import delta_oracle as O
from oracle import parallel as PP
from synth import configs as C
from synth.case import Case

# a small drifting stack: 3 layers, 2 sequences of ~200 tokens, the planted keys move every 4 steps
SMALL = C.DRIFT_48L.with_(name="drift-small", num_layers=3, delta_layers=(1,), num_q_heads=4, num_kv_heads=2,
                          head_dim=64, batch=2, context=200, budget_tokens=32, recency_tokens=32, planted=4,
                          steps=12, drift_every=4, drift_shift=16)


def direct_scores(step, layer, b):
    case = Case(SMALL, step=step)
    K, V = PP._kv(case, layer, b)
    _, p = O.full_attention(case.q(layer)[b].astype(np.float64), K, V)
    return O.page_scores(p, SMALL.page_size)


def test_delta_block_equals_per_step_delta_jobs():
    steps = [4, 5, 6, 7]
    job, out = PP.run_job((SMALL, 7, "delta_block", 1, 1, steps))
    assert len(out) == len(steps)
    for t, S in zip(steps, out):
        _, (o, S_ref) = PP.run_job((SMALL, t, "delta", 1, 1))
        np.testing.assert_array_equal(S, S_ref)
        np.testing.assert_array_equal(S, direct_scores(t, 1, 1))
        assert len(S) == O.num_pages(int(SMALL.contexts(t)[1]), SMALL.page_size)


def test_delta_block_rejects_steps_of_another_block():
    with pytest.raises(ValueError):
        PP.run_job((SMALL, 7, "delta_block", 1, 0, [3, 7]))    # step 3 is in the previous block
    with pytest.raises(ValueError):
        PP.run_job((SMALL, 6, "delta_block", 1, 0, [6, 7]))    # after the job's own step
