"""GPU parity of each C-ABI call against the fp64 oracle (element by element).

Inputs come only from the seeded generator (host values for the oracle, the bit-identical
device fill for the kernels); expected values only from ``oracle/``.
"""
import numpy as np
import pytest
import torch

from oracle import delta_oracle as O
from synth import configs as C
from synth import rng
from synth.case import Case
from tests.helpers import assert_close, oracle_kv, selection_ok

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    import long_context_layer_b200 as lib
    return lib


_ID = [100]


def make_cfg(G, Hkv, D, dtype, contexts, layers=1, delta=(0,), budget_pages=8, sink=16, rec=64, planted=0,
             extra_pool=0):
    _ID[0] += 1
    return C.TINY.with_(name=f"t{_ID[0]}", cfg_id=_ID[0], dtype=dtype, num_layers=layers, delta_layers=delta,
                        num_q_heads=G * Hkv, num_kv_heads=Hkv, head_dim=D, batch=len(contexts), context=0,
                        context_list=tuple(contexts), budget_tokens=budget_pages * 16, sink_tokens=sink,
                        recency_tokens=rec, planted=planted,
                        pool_pages_per_layer=(sum(-(-n // 16) for n in contexts) + extra_pool) if extra_pool else 0)


def device_case(cfg, prefill="all"):
    from synth.gpu import DeviceCase
    return DeviceCase(Case(cfg), prefill=prefill)


def stream():
    return torch.cuda.current_stream().cuda_stream


def make_desc(L, cfg, dc):
    return L.DeltaDesc(cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, 16,
                       L.DELTA_BF16 if cfg.dtype == "bf16" else L.DELTA_F32, 0.0, dc.num_phys_pages)


def make_pt(L, dc):
    return L.DeltaPageTable(dc.indptr.data_ptr(), dc.indices.data_ptr(), dc.kv_len.data_ptr(), dc.cfg.batch,
                            dc.case.max_pages_per_seq)


def workspace(L, desc, dc):
    nb = L.workspace_size(desc, dc.cfg.batch, dc.case.max_pages_per_seq)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    L.workspace_init(ws, nb, stream())
    return ws, nb


def ok_flags(L, ws):
    s, flags = L.read_device_error(ws, stream())
    assert s == 0 and flags == 0, f"device error flags {flags}"


# ----------------------------------------------------------------- generator fill
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_device_fill_matches_host_generator(dtype):
    cfg = make_cfg(4, 2, 128, dtype, [100, 37], planted=0)
    dc = device_case(cfg)
    case = dc.case
    for b in range(2):
        for g in range(2):
            for t, pool in ((rng.T_K, dc.k_pools[0]), (rng.T_V, dc.v_pools[0])):
                host = case.kv_logical(t, 0, b, g)
                dev = np.stack([dc.pool_row(0, t, b, g, pos).float().cpu().numpy() for pos in range(host.shape[0])])
                assert np.array_equal(dev.view(np.uint32), host.view(np.uint32))


# ----------------------------------------------------------------- full attention
FULL_CASES = [
    (8, 1, 64, "f32", [1024]),
    (1, 2, 64, "f32", [1, 15, 16, 17]),
    (3, 3, 128, "f32", [50, 2000]),
    (8, 1, 128, "f32", [777]),
    (4, 2, 128, "bf16", [100, 1000]),
    (5, 2, 128, "bf16", [4097, 33]),
    (7, 4, 128, "bf16", [8192]),
    (7, 1, 64, "bf16", [300]),
    (2, 2, 64, "bf16", [16, 32]),
    (6, 1, 128, "bf16", [513]),
    (8, 8, 128, "bf16", [2500, 1, 64]),
    # few units and long contexts: each unit's splits form several clusters, whose partials meet in
    # the workspace (the last CTA of each (sequence, KV head) merges them)
    (4, 2, 128, "bf16", [150000, 9000]),
    (2, 1, 64, "f32", [100000]),
]


@pytest.mark.parametrize("G,Hkv,D,dtype,ctx", FULL_CASES)
def test_full_attn_matches_oracle(L, G, Hkv, D, dtype, ctx):
    cfg = make_cfg(G, Hkv, D, dtype, ctx, extra_pool=7)
    dc = device_case(cfg)
    desc, pt = make_desc(L, cfg, dc), make_pt(L, dc)
    ws, nb = workspace(L, desc, dc)
    L.full_attn(desc, pt, dc.q[0], dc.k_pools[0], dc.v_pools[0], dc.out[0], ws, nb, stream())
    out = dc.out[0].float().cpu().numpy()
    ok_flags(L, ws)
    for b, n in enumerate(ctx):
        K, V = oracle_kv(dc.case, 0, b)
        ref, _ = O.full_attention(dc.case.q(0)[b].astype(np.float64), K, V)
        assert_close(out[b], ref, dtype, f"b={b} n={n}")


@pytest.mark.parametrize("dtype,D", [("f32", 64), ("bf16", 128), ("bf16", 64)])
def test_unwritten_slots_holding_nan_do_not_leak(L, dtype, D):
    # the last page of each sequence is partial; its unwritten slots hold NaN
    from synth.gpu import DeviceCase
    cfg = make_cfg(7, 2, D, dtype, [33, 1000, 17])
    case = Case(cfg)
    dc = DeviceCase(case, prefill="all", garbage=float("nan"))
    desc, pt = make_desc(L, cfg, dc), make_pt(L, dc)
    ws, nb = workspace(L, desc, dc)
    L.full_attn(desc, pt, dc.q[0], dc.k_pools[0], dc.v_pools[0], dc.out[0], ws, nb, stream())
    out = dc.out[0].float().cpu().numpy()
    assert np.isfinite(out).all()
    for b in range(3):
        K, V = oracle_kv(case, 0, b)
        assert_close(out[b], O.full_attention(case.q(0)[b].astype(np.float64), K, V)[0], dtype, f"b={b}")


def test_empty_sequence_gives_zero_output(L):
    cfg = make_cfg(4, 1, 64, "f32", [0, 20])
    cfg = cfg.with_(context_list=(0, 20))
    from synth.gpu import DeviceCase
    case = Case(cfg)
    dc = DeviceCase(case, prefill="all")
    desc, pt = make_desc(L, cfg, dc), make_pt(L, dc)
    ws, nb = workspace(L, desc, dc)
    dc.out.fill_(7.0)
    L.full_attn(desc, pt, dc.q[0], dc.k_pools[0], dc.v_pools[0], dc.out[0], ws, nb, stream())
    out = dc.out[0].cpu().numpy()
    assert np.all(out[0] == 0)
    K, V = oracle_kv(case, 0, 1)
    assert_close(out[1], O.full_attention(case.q(0)[1].astype(np.float64), K, V)[0], "f32")


# ----------------------------------------------------------------- delta-layer
SELECT_CASES = [
    # G, Hkv, D, dtype, contexts, budget, sink, rec, planted
    (8, 1, 64, "f32", [1024], 8, 16, 64, 0),
    (7, 4, 128, "bf16", [8192], 64, 16, 256, 32),
    (4, 2, 128, "bf16", [3000, 1500, 17], 16, 16, 100, 32),
    (5, 1, 64, "f32", [400], 100, 16, 64, 0),       # budget above the candidates: all pages
    (5, 1, 64, "f32", [400], 0, 0, 0, 0),           # nothing selected
    (2, 2, 128, "bf16", [700], 1, 0, 0, 8),         # k = 1, no sink, no recency
    (8, 1, 128, "f32", [16], 4, 16, 64, 0),         # one-page context
    # 16 units (a mid-size batch: 8-warp CTAs, 64 columns, 96 KB of stages): 23,750 pages per sequence
    # are more order keys than the selecting CTA's idle shared memory holds (about 22,300), so the
    # selection keeps them in the workspace, one row per sequence
    (2, 8, 64, "bf16", [380000, 240000], 300, 16, 512, 32),
    # 28,125 pages of one sequence in one 16-CTA cluster: close to the longest list the selection
    # accepts (32,768 pages); order keys in the workspace
    (8, 1, 64, "bf16", [450000], 300, 16, 512, 32),
    # 48 sequences x 8 KV heads = 384 units, more than one wave of CTAs: tickets across waves
    (4, 8, 128, "bf16", [100 + 61 * i for i in range(48)], 16, 16, 64, 8),
]


MAX_CASES = [
    (8, 1, 64, "f32", [1024], 8, 16, 64, 0),
    (7, 4, 128, "bf16", [8192], 64, 16, 256, 32),
    (4, 2, 128, "bf16", [3000, 1500, 17], 16, 16, 100, 32),
    (1, 1, 128, "bf16", [777], 5, 16, 32, 8),          # one query head: MAX equals SUM
]


@pytest.mark.parametrize("mode,G,Hkv,D,dtype,ctx,k,sink,rec,planted",
                         [("sum",) + c for c in SELECT_CASES] + [("max",) + c for c in MAX_CASES])
def test_select_attn_matches_oracle(L, mode, G, Hkv, D, dtype, ctx, k, sink, rec, planted):
    cfg = make_cfg(G, Hkv, D, dtype, ctx, budget_pages=k, sink=sink, rec=rec, planted=planted)
    dc = device_case(cfg)
    desc, pt = make_desc(L, cfg, dc), make_pt(L, dc)
    reduce = L.DELTA_HEAD_MAX if mode == "max" else L.DELTA_HEAD_SUM
    nb = L.workspace_size_reduce(desc, cfg.batch, dc.case.max_pages_per_seq, reduce)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    L.workspace_init(ws, nb, stream())
    sp = L.DeltaSelectParams(k, sink, rec, reduce)
    stride = L.sel_capacity(sp) + 3
    B, maxp = cfg.batch, dc.case.max_pages_per_seq
    sel_cnt = torch.full((B,), -1, dtype=torch.int32, device="cuda")
    sel_pages = torch.full((B, stride), -1, dtype=torch.int32, device="cuda")
    scores = torch.zeros((B, maxp), dtype=torch.float32, device="cuda")
    L.select_attn(desc, pt, sp, dc.q[0], dc.k_pools[0], dc.v_pools[0], dc.out[0], sel_cnt, sel_pages, stride,
                  scores, ws, nb, stream())
    out = dc.out[0].float().cpu().numpy()
    cnt, pages, sc = sel_cnt.cpu().numpy(), sel_pages.cpu().numpy(), scores.cpu().numpy()
    ok_flags(L, ws)
    for b, n in enumerate(ctx):
        K, V = oracle_kv(dc.case, 0, b)
        ref, p = O.full_attention(dc.case.q(0)[b].astype(np.float64), K, V)
        assert_close(out[b], ref, dtype, f"o b={b}")
        S = O.page_scores(p, 16, O.HEAD_MAX if mode == "max" else O.HEAD_SUM)
        np.testing.assert_allclose(sc[b, :len(S)], S, rtol=2e-5 if mode == "sum" else 1e-4,
                                   atol=1e-6 * cfg.num_q_heads)
        gsel = pages[b, :cnt[b]].tolist()
        ok, exact, ref_sel = selection_ok(gsel, S, n, k, sink, rec)
        assert ok, f"b={b}: gpu {gsel} vs oracle {ref_sel}"


@pytest.mark.parametrize("n,k,hkv", [(16384 + 5, 700, 4), (3000 + 5, 40, 4), (40000 + 7, 900, 1)])
def test_select_exact_ties(L, n, k, hkv):
    # Identical keys give identical page scores: the selection must take the lowest-index
    # candidates.  Every candidate has the same order key, so the threshold search ends in its
    # first pass on a one-value bucket and the compaction takes the first k equal pages; each
    # thread of the selecting CTA owns a run of pages, so the taken range crosses run boundaries.
    cfg = make_cfg(8, hkv, 128, "bf16", [n], budget_pages=k, sink=16, rec=256)
    dc = device_case(cfg)
    dc.k_pools[0].fill_(1.0)
    desc, pt = make_desc(L, cfg, dc), make_pt(L, dc)
    ws, nb = workspace(L, desc, dc)
    sp = L.DeltaSelectParams(k, 16, 256, L.DELTA_HEAD_SUM)
    stride = L.sel_capacity(sp)
    maxp = dc.case.max_pages_per_seq
    sel_cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    sel_pages = torch.full((1, stride), -1, dtype=torch.int32, device="cuda")
    scores = torch.zeros((1, maxp), dtype=torch.float32, device="cuda")
    L.select_attn(desc, pt, sp, dc.q[0], dc.k_pools[0], dc.v_pools[0], dc.out[0], sel_cnt, sel_pages, stride,
                  scores, ws, nb, stream())
    ok_flags(L, ws)
    K = np.ones((hkv, n, 128))
    V = oracle_kv(dc.case, 0, 0)[1]
    ref, p = O.full_attention(dc.case.q(0)[0].astype(np.float64), K, V)
    assert_close(dc.out[0].float().cpu().numpy()[0], ref, "bf16", "o")
    S = O.page_scores(p, 16)
    np.testing.assert_allclose(scores.cpu().numpy()[0, :len(S)], S, rtol=2e-5)
    got = sel_pages.cpu().numpy()[0, :int(sel_cnt.item())].tolist()
    assert got == O.select_pages(S, n, 16, k, 16, 256)
    assert got[:k + 1] == list(range(k + 1))


# ----------------------------------------------------------------- large-magnitude logits
@pytest.mark.parametrize("dtype,D,G,Hkv,ctx", [("bf16", 128, 7, 4, [8192, 300]), ("f32", 64, 8, 1, [1024]),
                                               ("bf16", 128, 5, 8, [2048])])
def test_large_logits_match_oracle(L, dtype, D, G, Hkv, ctx):
    # q scaled by 8 (exact in both storage types): logits of about 8 standard deviations, so the
    # softmax is dominated by a few tokens per head; full, delta and sparse layers against the oracle
    cfg = make_cfg(G, Hkv, D, dtype, ctx, budget_pages=16, sink=16, rec=64, planted=8)
    dc = device_case(cfg)
    dc.q.mul_(8.0)
    desc, pt = make_desc(L, cfg, dc), make_pt(L, dc)
    ws, nb = workspace(L, desc, dc)
    sp = L.DeltaSelectParams(16, 16, 64, L.DELTA_HEAD_SUM)
    stride = L.sel_capacity(sp)
    B, maxp = cfg.batch, dc.case.max_pages_per_seq
    sel_cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
    sel_pages = torch.zeros((B, stride), dtype=torch.int32, device="cuda")
    scores = torch.zeros((B, maxp), dtype=torch.float32, device="cuda")
    full = torch.empty_like(dc.out[0])
    sparse = torch.empty_like(dc.out[0])
    L.full_attn(desc, pt, dc.q[0], dc.k_pools[0], dc.v_pools[0], full, ws, nb, stream())
    L.select_attn(desc, pt, sp, dc.q[0], dc.k_pools[0], dc.v_pools[0], dc.out[0], sel_cnt, sel_pages, stride,
                  scores, ws, nb, stream())
    L.sparse_attn(desc, pt, sel_cnt, sel_pages, stride, dc.q[0], dc.k_pools[0], dc.v_pools[0], sparse, ws, nb,
                  stream())
    ok_flags(L, ws)
    f, o, sp_o = full.float().cpu().numpy(), dc.out[0].float().cpu().numpy(), sparse.float().cpu().numpy()
    cnt, pages, sc = sel_cnt.cpu().numpy(), sel_pages.cpu().numpy(), scores.cpu().numpy()
    for b, n in enumerate(ctx):
        K, V = oracle_kv(dc.case, 0, b)
        q = dc.case.q(0)[b].astype(np.float64) * 8.0
        ref, p = O.full_attention(q, K, V)
        assert_close(f[b], ref, dtype, f"full b={b}")
        assert_close(o[b], ref, dtype, f"delta b={b}")
        S = O.page_scores(p, 16)
        np.testing.assert_allclose(sc[b, :len(S)], S, rtol=2e-5, atol=1e-6 * cfg.num_q_heads)
        gsel = pages[b, :cnt[b]].tolist()
        ok, _, ref_sel = selection_ok(gsel, S, n, 16, 16, 64)
        assert ok, f"b={b}: gpu {gsel} vs oracle {ref_sel}"
        assert_close(sp_o[b], O.sparse_attention(q, K, V, gsel, 16), dtype, f"sparse b={b}")


# ----------------------------------------------------------------- sparse attention
@pytest.mark.parametrize("G,Hkv,D,dtype,ctx", [
    (8, 1, 64, "f32", [1024]), (7, 4, 128, "bf16", [8192, 333]), (5, 2, 128, "bf16", [1000]),
    (1, 1, 64, "f32", [45]), (4, 8, 128, "bf16", [6000, 17, 900])])
def test_sparse_attn_matches_oracle(L, G, Hkv, D, dtype, ctx):
    cfg = make_cfg(G, Hkv, D, dtype, ctx)
    dc = device_case(cfg)
    desc, pt = make_desc(L, cfg, dc), make_pt(L, dc)
    ws, nb = workspace(L, desc, dc)
    r = np.random.default_rng(len(ctx) * 100 + G)
    stride = 90
    sels = []
    for n in ctx:
        N = -(-n // 16)
        m = min(N, int(r.integers(1, stride)))
        sel = sorted(r.choice(N, size=m, replace=False).tolist())
        if N - 1 not in sel:
            sel[-1] = N - 1                      # always include the (possibly partial) last page
            sel = sorted(set(sel))
        sels.append(sel)
    sel_pages = torch.zeros((len(ctx), stride), dtype=torch.int32)
    for b, s in enumerate(sels):
        sel_pages[b, :len(s)] = torch.tensor(s)
    sel_cnt = torch.tensor([len(s) for s in sels], dtype=torch.int32).cuda()
    sel_pages = sel_pages.cuda()
    L.sparse_attn(desc, pt, sel_cnt, sel_pages, stride, dc.q[0], dc.k_pools[0], dc.v_pools[0], dc.out[0], ws, nb,
                  stream())
    out = dc.out[0].float().cpu().numpy()
    ok_flags(L, ws)
    for b, n in enumerate(ctx):
        K, V = oracle_kv(dc.case, 0, b)
        ref = O.sparse_attention(dc.case.q(0)[b].astype(np.float64), K, V, sels[b], 16)
        assert_close(out[b], ref, dtype, f"sparse b={b}")
    # the settled entry (selection read before the wait) gives the same bits; here the previous
    # kernel of the stream is the sparse call above, so the statement it relies on holds
    first = dc.out[0].clone()
    dc.out[0].zero_()
    L.sparse_attn_settled(desc, pt, sel_cnt, sel_pages, stride, dc.q[0], dc.k_pools[0], dc.v_pools[0], dc.out[0],
                          ws, nb, stream())
    ok_flags(L, ws)
    assert torch.equal(dc.out[0], first)


def test_sparse_with_every_page_equals_full(L):
    cfg = make_cfg(7, 4, 128, "bf16", [5000, 1234])
    dc = device_case(cfg)
    desc, pt = make_desc(L, cfg, dc), make_pt(L, dc)
    ws, nb = workspace(L, desc, dc)
    maxp = dc.case.max_pages_per_seq
    sel_pages = torch.arange(maxp, dtype=torch.int32).repeat(2, 1).cuda()
    sel_cnt = torch.tensor([-(-5000 // 16), -(-1234 // 16)], dtype=torch.int32).cuda()
    full = torch.empty_like(dc.out[0])
    L.full_attn(desc, pt, dc.q[0], dc.k_pools[0], dc.v_pools[0], full, ws, nb, stream())
    L.sparse_attn(desc, pt, sel_cnt, sel_pages, maxp, dc.q[0], dc.k_pools[0], dc.v_pools[0], dc.out[0], ws, nb,
                  stream())
    a, b = full.float().cpu().numpy(), dc.out[0].float().cpu().numpy()
    assert np.abs(a - b).max() <= 1e-2


# ----------------------------------------------------------------- kv append
@pytest.mark.parametrize("dtype,D", [("f32", 64), ("bf16", 128)])
def test_kv_append_writes_exactly_one_slot(L, dtype, D):
    cfg = make_cfg(4, 2, D, dtype, [33, 16, 1, 100], extra_pool=5)
    dc = device_case(cfg, prefill="append")
    desc, pt = make_desc(L, cfg, dc), make_pt(L, dc)
    bits = torch.int16 if dtype == "bf16" else torch.int32           # compare bytes: garbage may hold NaNs
    before_k, before_v = dc.k_pools[0].view(bits).clone(), dc.v_pools[0].view(bits).clone()
    L.kv_append(desc, pt, dc.k_new[0], dc.v_new[0], dc.k_pools[0], dc.v_pools[0], stream())
    torch.cuda.synchronize()
    changed = (dc.k_pools[0].view(bits) != before_k).any(-1) | (dc.v_pools[0].view(bits) != before_v).any(-1)
    for b, n in enumerate(cfg.context_list):
        for g in range(2):
            for t, new in ((rng.T_K, dc.k_new[0]), (rng.T_V, dc.v_new[0])):
                row = dc.pool_row(0, t, b, g, n - 1)
                assert torch.equal(row, new[b, g])
                host = dc.case.kv_logical(t, 0, b, g)[n - 1]
                assert np.array_equal(row.float().cpu().numpy(), host)
    # everything else untouched (only slots that held different bytes can show up as changed)
    allowed = set()
    for b, n in enumerate(cfg.context_list):
        phys = dc.case.page_indices[dc.case.page_indptr[b] + (n - 1) // 16]
        for g in range(2):
            allowed.add((int(phys), g, (n - 1) % 16))
    idx = {tuple(x) for x in changed.nonzero().cpu().tolist()}
    assert idx <= allowed


def test_kv_append_layers_matches_per_layer_append(L):
    cfg = make_cfg(5, 2, 128, "bf16", [33, 16, 1, 100], layers=3, delta=(0,), extra_pool=5)
    a = device_case(cfg, prefill="append")
    b = device_case(cfg, prefill="append")
    desc, pt = make_desc(L, cfg, a), make_pt(L, a)
    for l in range(3):
        L.kv_append(desc, pt, a.k_new[l], a.v_new[l], a.k_pools[l], a.v_pools[l], stream())
    pt_b = make_pt(L, b)
    L.kv_append_layers(desc, pt_b, b.k_new, b.v_new, b.k_pools, b.v_pools, stream())
    torch.cuda.synchronize()
    for l in range(3):
        for pa, pb in ((a.k_pools[l], b.k_pools[l]), (a.v_pools[l], b.v_pools[l])):
            for bb, n in enumerate(cfg.context_list):
                for g in range(2):
                    phys = a.case.page_indices[a.case.page_indptr[bb] + (n - 1) // 16]
                    assert torch.equal(pa[phys, g, (n - 1) % 16], pb[phys, g, (n - 1) % 16])
                    assert torch.equal(pb[phys, g, (n - 1) % 16], b.k_new[l][bb, g] if pa is a.k_pools[l] else
                                       b.v_new[l][bb, g])


# ----------------------------------------------------------------- device-side checks
def test_corrupt_page_id_is_flagged_not_trapped(L):
    cfg = make_cfg(4, 1, 64, "f32", [300])
    dc = device_case(cfg)
    desc, pt = make_desc(L, cfg, dc), make_pt(L, dc)
    ws, nb = workspace(L, desc, dc)
    bad = dc.indices.clone()
    bad[3] = dc.num_phys_pages + 5
    pt_bad = L.DeltaPageTable(dc.indptr.data_ptr(), bad.data_ptr(), dc.kv_len.data_ptr(), 1,
                              dc.case.max_pages_per_seq)
    L.full_attn(desc, pt_bad, dc.q[0], dc.k_pools[0], dc.v_pools[0], dc.out[0], ws, nb, stream())
    s, flags = L.read_device_error(ws, stream())
    assert s == 5 and flags & 1
    # the flag is cleared by the read; a clean call reports nothing
    L.full_attn(desc, pt, dc.q[0], dc.k_pools[0], dc.v_pools[0], dc.out[0], ws, nb, stream())
    assert L.read_device_error(ws, stream()) == (0, 0)


def test_kv_len_beyond_pages_and_bad_selection_are_flagged(L):
    cfg = make_cfg(4, 1, 64, "f32", [300])
    dc = device_case(cfg)
    desc = make_desc(L, cfg, dc)
    nb = L.workspace_size(desc, 1, dc.case.max_pages_per_seq + 4)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    L.workspace_init(ws, nb, stream())
    long_len = torch.tensor([300 + 64], dtype=torch.int32, device="cuda")
    pt_bad = L.DeltaPageTable(dc.indptr.data_ptr(), dc.indices.data_ptr(), long_len.data_ptr(), 1,
                              dc.case.max_pages_per_seq + 4)
    L.full_attn(desc, pt_bad, dc.q[0], dc.k_pools[0], dc.v_pools[0], dc.out[0], ws, nb, stream())
    s, flags = L.read_device_error(ws, stream())
    assert s == 5 and flags & 2
    pt = make_pt(L, dc)
    sel_pages = torch.tensor([[0, 5, 400]], dtype=torch.int32, device="cuda")
    sel_cnt = torch.tensor([3], dtype=torch.int32, device="cuda")
    L.sparse_attn(desc, pt, sel_cnt, sel_pages, 3, dc.q[0], dc.k_pools[0], dc.v_pools[0], dc.out[0], ws, nb,
                  stream())
    s, flags = L.read_device_error(ws, stream())
    assert s == 5 and flags & 4
    L.sparse_attn_settled(desc, pt, sel_cnt, sel_pages, 3, dc.q[0], dc.k_pools[0], dc.v_pools[0], dc.out[0], ws,
                          nb, stream())
    s, flags = L.read_device_error(ws, stream())
    assert s == 5 and flags & 4


def test_settled_sparse_flags_a_bad_selection_bf16(L):
    # the tensor-core kernel reads a settled selection before its wait: bad entries are still
    # skipped and flagged
    cfg = make_cfg(7, 2, 128, "bf16", [700])
    dc = device_case(cfg)
    desc, pt = make_desc(L, cfg, dc), make_pt(L, dc)
    ws, nb = workspace(L, desc, dc)
    sel_pages = torch.tensor([[0, 7, 9999, 43]], dtype=torch.int32, device="cuda")
    sel_cnt = torch.tensor([4], dtype=torch.int32, device="cuda")
    L.sparse_attn_settled(desc, pt, sel_cnt, sel_pages, 4, dc.q[0], dc.k_pools[0], dc.v_pools[0], dc.out[0], ws,
                          nb, stream())
    s, flags = L.read_device_error(ws, stream())
    assert s == 5 and flags & 4
    K, V = oracle_kv(dc.case, 0, 0)
    ref = O.sparse_attention(dc.case.q(0)[0].astype(np.float64), K, V, [0, 7, 43], 16)
    assert_close(dc.out[0].float().cpu().numpy()[0], ref, "bf16", "settled, bad entry skipped")
