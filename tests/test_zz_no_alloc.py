"""The allocation-free full-attention entry point (collected last on purpose).

delta_full_attn_noalloc serves callers that cannot allocate device memory (graph-captured
code, real-time loops, frameworks that own every allocation): it uses a fixed scratch array
inside the library instead of a caller workspace.  Its output must match delta_full_attn's,
call after call, even though every call reuses the same scratch.
"""
import numpy as np
import pytest
import torch

from oracle import delta_oracle as O
from synth import configs as C
from synth.case import Case
from tests.helpers import assert_close, oracle_kv

pytestmark = pytest.mark.gpu


def test_noalloc_full_attn_matches_workspace_call_twice():
    import long_context_layer_b200 as L
    from synth.gpu import DeviceCase
    cfg = C.TINY.with_(name="noalloc", cfg_id=91, dtype="bf16", num_layers=1, delta_layers=(0,), num_q_heads=28,
                       num_kv_heads=4, head_dim=128, batch=3, context=0, context_list=(8192, 333, 1),
                       planted=32, budget_tokens=1024, sink_tokens=16, recency_tokens=256)
    dc = DeviceCase(Case(cfg), prefill="all")
    desc = L.DeltaDesc(cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, 16, L.DELTA_BF16, 0.0, dc.num_phys_pages)
    pt = L.DeltaPageTable(dc.indptr.data_ptr(), dc.indices.data_ptr(), dc.kv_len.data_ptr(), cfg.batch,
                          dc.case.max_pages_per_seq)
    st = torch.cuda.current_stream().cuda_stream
    nb = L.workspace_size(desc, cfg.batch, dc.case.max_pages_per_seq)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    L.workspace_init(ws, nb, st)
    ref = torch.empty_like(dc.out[0])
    L.full_attn(desc, pt, dc.q[0], dc.k_pools[0], dc.v_pools[0], ref, ws, nb, st)
    ref_np = ref.float().cpu().numpy()
    outs = []
    for _ in range(2):
        o = torch.full_like(dc.out[0], float("nan"))
        L.full_attn_noalloc(desc, pt, dc.q[0], dc.k_pools[0], dc.v_pools[0], o, st)
        outs.append(o.float().cpu().numpy())
    for o in outs:
        assert np.isfinite(o).all()
        for b in range(cfg.batch):
            assert_close(o[b], ref_np[b], "bf16", f"noalloc b={b}")
    assert np.array_equal(outs[0], outs[1])
    # and against the fp64 oracle directly
    for b in range(cfg.batch):
        K, V = oracle_kv(dc.case, 0, b)
        assert_close(outs[1][b], O.full_attention(dc.case.q(0)[b].astype(np.float64), K, V)[0], "bf16",
                     f"noalloc vs oracle b={b}")


def test_noalloc_skips_a_corrupt_page_id():
    # A page id outside the pool is skipped (never read), as on the workspace path; the call returns
    # normally and the sequences whose pages are valid still get their exact outputs.  (The device
    # flag that the workspace path raises stays in the library's scratch and is not reported.)
    import long_context_layer_b200 as L
    from synth.gpu import DeviceCase
    cfg = C.TINY.with_(name="noalloc-bad", cfg_id=92, dtype="bf16", num_layers=1, delta_layers=(0,), num_q_heads=8,
                       num_kv_heads=2, head_dim=128, batch=3, context=0, context_list=(700, 300, 1000), planted=0)
    dc = DeviceCase(Case(cfg), prefill="all")
    desc = L.DeltaDesc(8, 2, 128, 16, L.DELTA_BF16, 0.0, dc.num_phys_pages)
    bad = dc.indices.clone()
    bad[int(dc.case.page_indptr[1]) + 4] = dc.num_phys_pages + 1000      # sequence 1, logical page 4
    pt = L.DeltaPageTable(dc.indptr.data_ptr(), bad.data_ptr(), dc.kv_len.data_ptr(), 3, dc.case.max_pages_per_seq)
    st = torch.cuda.current_stream().cuda_stream
    nb = L.workspace_size(desc, 3, dc.case.max_pages_per_seq)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    L.workspace_init(ws, nb, st)
    ref = torch.empty_like(dc.out[0])
    L.full_attn(desc, pt, dc.q[0], dc.k_pools[0], dc.v_pools[0], ref, ws, nb, st)
    status, flags = L.read_device_error(ws, st)
    assert status == L._native.DELTA_ERR_BOUNDS and flags & 1
    o = torch.full_like(dc.out[0], float("nan"))
    assert L.full_attn_noalloc(desc, pt, dc.q[0], dc.k_pools[0], dc.v_pools[0], o, st) == 0
    torch.cuda.synchronize()
    got, want = o.float().cpu().numpy(), ref.float().cpu().numpy()
    assert np.isfinite(got).all()
    assert np.array_equal(got, want)          # same kernel, same plan: the same bits, bad page included
    for b in (0, 2):
        K, V = oracle_kv(dc.case, 0, b)
        assert_close(got[b], O.full_attention(dc.case.q(0)[b].astype(np.float64), K, V)[0], "bf16", f"b={b}")


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import long_context_layer_b200 as L
    desc = L.DeltaDesc(64, 8, 128, 16, L.DELTA_BF16, 0.0, 1 << 20)
    need = L.workspace_size(desc, 64, 32768)
    assert need > 8 << 20
    fake = 1 << 40   # never dereferenced: the size check comes first
    pt = L.DeltaPageTable(fake, fake, fake, 64, 32768)
    assert L.full_attn_noalloc(desc, pt, fake, fake, fake, fake, 0, check=False) == L._native.DELTA_ERR_UNSUPPORTED
