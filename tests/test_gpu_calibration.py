"""GPU parity of the delta-layer calibration metric (1 - cos between consecutive layers' page
scores) and of the placement it leads to, against the fp64 oracle."""
import numpy as np
import pytest
import torch

from oracle import delta_oracle as O
from synth import configs as C
from synth.case import Case
from tests.helpers import oracle_kv

pytestmark = pytest.mark.gpu

CASES = [
    C.TINY.with_(name="calib-f32", cfg_id=96, num_layers=7, context=0, context_list=(1000, 333), batch=2,
                 planted=8),
    C.QWEN7B_8K.with_(name="calib-bf16", cfg_id=97, num_layers=8, batch=2, context=0, context_list=(3000, 1201)),
]


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_calibration_shifts_match_oracle(cfg):
    from long_context_layer_b200.stack import DeltaStack, choose_delta_layers
    from synth.gpu import DeviceCase
    case = Case(cfg)
    dc = DeviceCase(case, prefill="all")
    st = DeltaStack(cfg.layer_kinds(), cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, dc.dtype, dc.indptr,
                    dc.indices, dc.kv_len, case.max_pages_per_seq, dc.num_phys_pages, cfg.budget_pages,
                    cfg.sink_tokens, cfg.recency_tokens)
    shift = st.calibration_shifts(dc.q, dc.k_pools, dc.v_pools, dc.out).cpu().numpy()
    ref = np.zeros((cfg.num_layers, cfg.batch))
    for b in range(cfg.batch):
        prev = None
        for l in range(1, cfg.num_layers):
            K, V = oracle_kv(case, l, b)
            _, p = O.full_attention(case.q(l)[b].astype(np.float64), K, V)
            S = O.page_scores(p, 16)
            if prev is not None:
                ref[l, b] = O.layer_shift(prev, S)
            prev = S
    np.testing.assert_allclose(shift, ref, atol=2e-5, rtol=0)
    assert (ref[2:] > 0).all()
    mean_gpu, mean_ref = shift.mean(1), ref.mean(1)
    for count in (2, 3):
        assert choose_delta_layers(mean_gpu, count) == O.choose_delta_layers(mean_ref, count)


def test_layer_shift_zero_vector_and_empty_sequence():
    from long_context_layer_b200 import _native as N
    dev = torch.device("cuda")
    kv_len = torch.tensor([40, 0, 17], dtype=torch.int32, device=dev)
    indptr = torch.tensor([0, 3, 3, 5], dtype=torch.int32, device=dev)
    indices = torch.arange(5, dtype=torch.int32, device=dev)
    pt = N.DeltaPageTable(indptr.data_ptr(), indices.data_ptr(), kv_len.data_ptr(), 3, 3)
    a = torch.zeros(3, 3, device=dev)
    b = torch.zeros(3, 3, device=dev)
    a[0] = torch.tensor([1.0, 2.0, 2.0]); b[0] = torch.tensor([2.0, 4.0, 4.0])   # parallel: shift 0
    a[2, :2] = torch.tensor([1.0, 0.0]); b[2, :2] = torch.tensor([0.0, 3.0])     # orthogonal: shift 1
    a[2, 2] = 5.0; b[2, 2] = 7.0                                                  # past the sequence's 2 pages
    out = torch.full((3,), -1.0, device=dev)
    N.layer_shift(pt, a, b, out, torch.cuda.current_stream().cuda_stream)
    got = out.cpu().numpy()
    ref = [O.layer_shift([1, 2, 2], [2, 4, 4]), O.layer_shift([], []), O.layer_shift([1, 0], [0, 3])]
    np.testing.assert_allclose(got, ref, atol=1e-6)
