"""The allocation-free full-attention entry point (collected last on purpose).

delta_full_attn_noalloc serves callers that cannot allocate device memory (graph-captured
code, real-time loops, frameworks that own every allocation): it uses a fixed scratch array
inside the library instead of a caller workspace.  Its output must match delta_full_attn's,
call after call, even though every call reuses the same scratch.
"""
import numpy as np
import pytest
import torch

from synth import configs as C
from synth.case import Case
from tests.helpers import assert_close

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


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import long_context_layer_b200 as L
    desc = L.DeltaDesc(64, 8, 128, 16, L.DELTA_BF16, 0.0, 1 << 20)
    need = L.workspace_size(desc, 64, 32768)
    assert need > 8 << 20
    fake = 1 << 40   # never dereferenced: the size check comes first
    pt = L.DeltaPageTable(fake, fake, fake, 64, 32768)
    assert L.full_attn_noalloc(desc, pt, fake, fake, fake, fake, 0, check=False) == L._native.DELTA_ERR_UNSUPPORTED
