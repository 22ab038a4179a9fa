"""GPU parity of whole decode steps (every layer of a stack) against the fp64 oracle."""
import numpy as np
import pytest
import torch

from oracle import delta_oracle as O
from synth import configs as C
from synth.case import Case
from tests.helpers import assert_close, oracle_kv, selection_ok

pytestmark = pytest.mark.gpu


def build(cfg, layers=None, keep_scores=True):
    from long_context_layer_b200.stack import DeltaStack
    from synth.gpu import DeviceCase
    case = Case(cfg)
    dc = DeviceCase(case, layers=layers, prefill="append")
    stack = DeltaStack(cfg.layer_kinds(), cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, dc.dtype, dc.indptr,
                       dc.indices, dc.kv_len, case.max_pages_per_seq, dc.num_phys_pages, cfg.budget_pages,
                       cfg.sink_tokens, cfg.recency_tokens, keep_scores=keep_scores)
    return case, dc, stack


def run(stack, dc):
    stack.step(dc.q, dc.k_new, dc.v_new, dc.k_pools, dc.v_pools, dc.out)
    torch.cuda.synchronize()


def check_stack_against_oracle(cfg, case, dc, stack, layers=None, batch=None):
    """Compare outputs of the given layers (default all) and every delta-layer's selection."""
    out = dc.out.float().cpu().numpy()
    kinds = cfg.layer_kinds()
    batch = range(cfg.batch) if batch is None else batch
    n_exact = 0
    for b in batch:
        n = int(case.n[b])
        sel = None
        for l, kind in enumerate(kinds):
            want = layers is None or l in layers
            if kind == C.SPARSE and not want:
                continue
            K, V = oracle_kv(case, l, b)
            q = case.q(l)[b].astype(np.float64)
            if kind == C.SPARSE:
                assert_close(out[l, b], O.sparse_attention(q, K, V, sel, 16), cfg.dtype, f"sparse l={l} b={b}")
                continue
            o, p = O.full_attention(q, K, V)
            if want:
                assert_close(out[l, b], o, cfg.dtype, f"{kind} l={l} b={b}")
            if kind == C.DELTA:
                S = O.page_scores(p, 16)
                d = stack.delta_layers.index(l)
                gsel = stack.selection(d)[b]
                ok, exact, ref = selection_ok(gsel, S, n, cfg.budget_pages, cfg.sink_tokens, cfg.recency_tokens)
                assert ok, f"selection l={l} b={b}"
                n_exact += exact
                sel = gsel          # sparse layers are checked against the selection the GPU used
    return n_exact


def test_tiny_stack_matches_oracle():
    cfg = C.TINY
    case, dc, stack = build(cfg)
    run(stack, dc)
    assert check_stack_against_oracle(cfg, case, dc, stack) == 1
    from long_context_layer_b200 import read_device_error
    assert read_device_error(stack.workspace, torch.cuda.current_stream().cuda_stream) == (0, 0)


def test_qwen7b_8k_stack_matches_oracle():
    cfg = C.QWEN7B_8K
    case, dc, stack = build(cfg)
    run(stack, dc)
    check_stack_against_oracle(cfg, case, dc, stack)


def test_graph_replay_is_bit_identical_and_deterministic():
    cfg = C.QWEN7B_8K
    case, dc, stack = build(cfg)
    run(stack, dc)
    ref_out = dc.out.clone()
    ref_sel = stack.sel_pages.clone(), stack.sel_cnt.clone()
    g = stack.capture(dc.q, dc.k_new, dc.v_new, dc.k_pools, dc.v_pools, dc.out)
    for _ in range(20):
        dc.out.zero_()
        stack.sel_pages.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(dc.out, ref_out)
        assert torch.equal(stack.sel_pages, ref_sel[0]) and torch.equal(stack.sel_cnt, ref_sel[1])


def test_sparse_layers_read_only_selected_tokens():
    # Budget covering every page: the sparse layers must reproduce full attention.
    cfg = C.TINY.with_(budget_tokens=1024 * 2)
    case, dc, stack = build(cfg)
    run(stack, dc)
    out = dc.out.float().cpu().numpy()
    for l in (2, 3):
        K, V = oracle_kv(case, l, 0)
        assert_close(out[l, 0], O.full_attention(case.q(l)[0].astype(np.float64), K, V)[0], "f32", f"l={l}")


@pytest.mark.parametrize("cfg,layers,batch", [
    (C.QWEN7B_B8_VAR, [0, 2, 3, 13, 14, 27], [0, 5]),
    (C.LLAMA8B_64K, [2, 3, 12, 31], [1]),
])
def test_full_size_workload_sampled(cfg, layers, batch):
    case, dc, stack = build(cfg, keep_scores=False)
    run(stack, dc)
    # every delta-layer's selection is checked for the sampled sequences, outputs of the sampled layers
    check_stack_against_oracle(cfg, case, dc, stack, layers=layers, batch=batch)


@pytest.mark.parametrize("cfg", [C.TINY, C.QWEN7B_8K])
def test_step_host_matches_the_device_step(cfg):
    # the host-buffer step (per-layer uploads and downloads on copy streams) runs the same kernels on
    # the same values: the same bits as the device-buffer step, eagerly and replayed from a graph
    case, dc, stack = build(cfg)
    run(stack, dc)
    ref = dc.out.clone()
    ref_sel = stack.sel_pages.clone()
    q_h, kn_h, vn_h = (x.cpu().pin_memory() for x in (dc.q, dc.k_new, dc.v_new))
    out_h = torch.full(tuple(dc.out.shape), float("nan"), dtype=dc.out.dtype).pin_memory()
    q_d, kn_d, vn_d = (torch.zeros_like(x) for x in (dc.q, dc.k_new, dc.v_new))
    args = (q_h, kn_h, vn_h, dc.k_pools, dc.v_pools, out_h, q_d, kn_d, vn_d, dc.out)
    dc.out.zero_()
    stack.step_host(*args)
    torch.cuda.synchronize()
    assert torch.equal(out_h, ref.cpu())
    assert torch.equal(stack.sel_pages, ref_sel)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        stack.step_host(*args)
    for _ in range(3):
        out_h.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out_h, ref.cpu())
