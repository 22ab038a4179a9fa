"""Pins of the fp64 oracle against things other than itself.

Closed forms, invariants the method's definition fixes, brute force on tiny
inputs and independent library routines (torch CPU fp64 attention, a stable
torch sort).  The planted-mistake tests at the end check that a plausible
error in the oracle trips at least one of these pins.
"""
import itertools
import math

import numpy as np
import pytest
import torch

from oracle import delta_oracle as O

RNG = np.random.default_rng(1234)


def rand(*shape):
    return RNG.standard_normal(shape)


# ----------------------------------------------------------------- dense attention
def test_identical_keys_give_mean_of_values():
    n, D = 37, 64
    k = rand(D)
    K = np.tile(k, (n, 1))
    V = rand(n, D)
    o, p = O.softmax_attention(rand(3, D), K, V, 1 / 8)
    np.testing.assert_allclose(o, np.tile(V.mean(0), (3, 1)), atol=1e-12)
    np.testing.assert_allclose(p, 1.0 / n, atol=1e-15)


def test_zero_query_gives_mean_of_values():
    K, V = rand(50, 32), rand(50, 32)
    o, _ = O.softmax_attention(np.zeros((2, 32)), K, V, 0.3)
    np.testing.assert_allclose(o[0], V.mean(0), atol=1e-12)


def test_single_token_gives_its_value():
    K, V = rand(1, 128), rand(1, 128)
    o, p = O.softmax_attention(rand(7, 128), K, V, 1 / math.sqrt(128))
    np.testing.assert_allclose(o, np.tile(V[0], (7, 1)), atol=1e-14)
    assert np.all(p == 1.0)


def test_one_hot_huge_logit_selects_that_value():
    n, D = 40, 16
    K = rand(n, D) * 1e-3
    q = np.zeros((1, D)); q[0, 0] = 1.0
    K[23, 0] = 1e4
    V = rand(n, D)
    o, p = O.softmax_attention(q, K, V, 1.0)
    np.testing.assert_allclose(o[0], V[23], atol=1e-12)
    assert p[0, 23] > 1 - 1e-12


def test_rows_sum_to_one():
    _, p = O.full_attention(rand(8, 64), rand(2, 300, 64), rand(2, 300, 64))
    np.testing.assert_allclose(p.sum(1), 1.0, atol=1e-12)
    assert np.all(p >= 0)


@pytest.mark.parametrize("Hq,Hkv,n,D", [(8, 1, 1024, 64), (28, 4, 333, 128), (5, 5, 17, 64), (40, 8, 65, 128)])
def test_full_attention_matches_torch_sdpa(Hq, Hkv, n, D):
    q, K, V = rand(Hq, D), rand(Hkv, n, D), rand(Hkv, n, D)
    o, _ = O.full_attention(q, K, V)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None, :], torch.from_numpy(K)[None], torch.from_numpy(V)[None],
        enable_gqa=True)[0, :, 0, :].numpy()
    np.testing.assert_allclose(o, ref, atol=1e-12, rtol=1e-10)


def test_gqa_head_mapping_is_contiguous_groups():
    # KV head g holds constant value g; query head h must read KV head h // G.
    Hq, Hkv, n, D = 12, 3, 9, 8
    K = rand(Hkv, n, D)
    V = np.stack([np.full((n, D), float(g)) for g in range(Hkv)])
    o, _ = O.full_attention(rand(Hq, D), K, V)
    for h in range(Hq):
        np.testing.assert_allclose(o[h], h // (Hq // Hkv), atol=1e-13)


def test_default_scale_is_inverse_sqrt_head_dim():
    # q.k = D for these vectors, so the logit is sqrt(D) with scale 1/sqrt(D).
    D = 64
    K = np.stack([np.ones(D), np.zeros(D)])
    V = np.stack([np.ones(D), np.zeros(D)])
    o, _ = O.full_attention(np.ones((1, D)), K[None], V[None])
    w = math.exp(math.sqrt(D)) / (math.exp(math.sqrt(D)) + 1)
    np.testing.assert_allclose(o[0], w, atol=1e-14)


# ----------------------------------------------------------------- page scores
@pytest.mark.parametrize("n", [1, 15, 16, 17, 100, 1024])
def test_sum_scores_add_up_to_query_heads(n):
    _, p = O.full_attention(rand(12, 32), rand(4, n, 32), rand(4, n, 32))
    S = O.page_scores(p, 16, O.HEAD_SUM)
    assert len(S) == -(-n // 16)
    assert abs(S.sum() - 12) < 1e-12


def test_single_page_score_equals_query_heads():
    _, p = O.full_attention(rand(7, 64), rand(1, 11, 64), rand(1, 11, 64))
    np.testing.assert_allclose(O.page_scores(p, 16), [7.0], atol=1e-13)


def test_scores_match_library_softmax_mass_per_page():
    Hq, Hkv, n, D = 8, 2, 70, 32
    q, K = rand(Hq, D), rand(Hkv, n, D)
    _, p = O.full_attention(q, K, rand(Hkv, n, D))
    Kx = torch.from_numpy(K).repeat_interleave(Hq // Hkv, 0)
    probs = torch.softmax(torch.einsum("hd,hnd->hn", torch.from_numpy(q), Kx) / math.sqrt(D), -1)
    mass = [probs[:, j * 16:(j + 1) * 16].sum().item() for j in range(5)]
    np.testing.assert_allclose(O.page_scores(p, 16), mass, atol=1e-12)
    maxmass = [probs[:, j * 16:(j + 1) * 16].max(0).values.sum().item() for j in range(5)]
    np.testing.assert_allclose(O.page_scores(p, 16, O.HEAD_MAX), maxmass, atol=1e-12)


def test_head_modes_agree_with_one_query_head_and_max_bounds():
    _, p1 = O.full_attention(rand(1, 16), rand(1, 90, 16), rand(1, 90, 16))
    np.testing.assert_allclose(O.page_scores(p1, 16, O.HEAD_MAX), O.page_scores(p1, 16, O.HEAD_SUM), atol=0)
    _, p = O.full_attention(rand(6, 16), rand(2, 90, 16), rand(2, 90, 16))
    tot = O.page_scores(p, 16, O.HEAD_MAX).sum()
    assert 1 - 1e-12 <= tot <= 6 + 1e-12


def test_planted_token_puts_one_per_head_in_its_page():
    Hq, n, D = 4, 200, 16
    K = rand(1, n, D) * 1e-3
    q = np.zeros((Hq, D)); q[:, 3] = 1.0
    K[0, 141, 3] = 1e4
    _, p = O.full_attention(q, K, rand(1, n, D), 1.0)
    S = O.page_scores(p, 16)
    assert abs(S[141 // 16] - Hq) < 1e-9


# ----------------------------------------------------------------- selection
def _brute_force_topk(S, candidates, k):
    """The unique k-subset C with (S_c > S_u) or (S_c == S_u and c < u) for all c in C, u outside."""
    if len(candidates) <= k:
        return list(candidates)
    found = []
    for C in itertools.combinations(candidates, k):
        rest = [u for u in candidates if u not in C]
        if all(S[c] > S[u] or (S[c] == S[u] and c < u) for c in C for u in rest):
            found.append(list(C))
    assert len(found) == 1
    return found[0]


@pytest.mark.parametrize("trial", range(40))
def test_selection_matches_brute_force_with_ties(trial):
    r = np.random.default_rng(trial)
    N = int(r.integers(1, 9))
    n = int(r.integers((N - 1) * 16 + 1, N * 16 + 1))
    S = r.integers(0, 3, size=N).astype(np.float64)     # small integers: many exact ties
    k = int(r.integers(0, 6))
    sink = int(r.choice([0, 1, 16, 20]))
    rec = int(r.choice([0, 1, 16, 17, 40]))
    sel = O.select_pages(S, n, 16, k, sink, rec)
    forced = set(O.sink_page_set(n, 16, sink)) | set(O.recency_page_set(n, 16, rec))
    cands = [j for j in range(N) if j not in forced]
    expect = sorted(forced | set(_brute_force_topk(S, cands, k)))
    assert sel == expect


def test_selection_matches_stable_library_sort():
    r = np.random.default_rng(7)
    for _ in range(50):
        N = int(r.integers(5, 300))
        n = N * 16 - int(r.integers(0, 16))
        S = np.round(r.random(N), 2)                    # ties likely
        k = int(r.integers(1, N))
        sel = O.select_pages(S, n, 16, k, 16, 64)
        forced = set(O.sink_page_set(n, 16, 16)) | set(O.recency_page_set(n, 16, 64))
        cands = torch.tensor([j for j in range(N) if j not in forced], dtype=torch.long)
        order = torch.sort(-torch.from_numpy(S)[cands], stable=True).indices
        top = set(cands[order[:k]].tolist())
        assert sel == sorted(forced | top)


def test_sink_and_recency_always_selected():
    r = np.random.default_rng(3)
    for _ in range(100):
        N = int(r.integers(1, 200))
        n = N * 16 - int(r.integers(0, 16))
        sink, rec = int(r.integers(0, 64)), int(r.integers(0, 300))
        S = r.random(N)
        sel = set(O.select_pages(S, n, 16, int(r.integers(0, 10)), sink, rec))
        assert set(range(-(-min(sink, n) // 16))) <= sel
        if rec:
            assert set(range(max(n - rec, 0) // 16, N)) <= sel
            # the page of token n - rec is the first recency page; the one before is not forced
        assert (N - 1) in sel or rec == 0


def test_budget_covering_all_pages_selects_all():
    S = np.random.default_rng(0).random(40)
    assert O.select_pages(S, 40 * 16 - 3, 16, 40, 0, 0) == list(range(40))


def test_one_page_context_selects_page_zero():
    for n in (1, 7, 16):
        assert O.select_pages(np.array([0.3]), n, 16, 4, 16, 64) == [0]
        assert O.select_pages(np.array([0.3]), n, 16, 0, 0, 0) == []
        assert O.select_pages(np.array([0.3]), n, 16, 1, 0, 0) == [0]


def test_recency_and_sink_page_counts_of_tiny_workload():
    # 1024 tokens, 16-token sink, 64-token window: page 0 and the last 4 pages.
    assert O.sink_page_set(1024, 16, 16) == [0]
    assert O.recency_page_set(1024, 16, 64) == [60, 61, 62, 63]
    # unaligned end: the window reaches into one more page
    assert O.recency_page_set(1030, 16, 64) == [60, 61, 62, 63, 64]


# ----------------------------------------------------------------- sparse attention
def test_sparse_with_all_pages_equals_full():
    q, K, V = rand(8, 64), rand(2, 333, 64), rand(2, 333, 64)
    full, _ = O.full_attention(q, K, V)
    sp = O.sparse_attention(q, K, V, list(range(21)), 16)
    np.testing.assert_allclose(sp, full, atol=1e-12)


def test_sparse_equals_library_attention_on_gathered_tokens():
    Hq, Hkv, n, D = 8, 2, 333, 64
    q, K, V = rand(Hq, D), rand(Hkv, n, D), rand(Hkv, n, D)
    pages = [0, 3, 4, 11, 20]                            # page 20 is the partial last page (tokens 320..332)
    t = [i for j in pages for i in range(j * 16, min(j * 16 + 16, n))]
    assert len(t) == 4 * 16 + 13
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None], torch.from_numpy(K[:, t])[None], torch.from_numpy(V[:, t])[None],
        enable_gqa=True)[0, :, 0].numpy()
    np.testing.assert_allclose(O.sparse_attention(q, K, V, pages, 16), ref, atol=1e-12)


# ----------------------------------------------------------------- stack
def _stack_inputs(L, Hq, Hkv, n, D, seed):
    r = np.random.default_rng(seed)
    qs = [r.standard_normal((Hq, D)) for _ in range(L)]
    kvs = [(r.standard_normal((Hkv, n, D)), r.standard_normal((Hkv, n, D))) for _ in range(L)]
    return qs, kvs


def test_stack_all_full_equals_per_layer_full():
    qs, kvs = _stack_inputs(4, 8, 2, 100, 32, 0)
    outs, sels = O.stack_step(["full"] * 4, lambda l: qs[l], lambda l: kvs[l], 100, 16, 2, 16, 32)
    assert sels == {}
    for l in range(4):
        np.testing.assert_allclose(outs[l], O.full_attention(qs[l], *kvs[l])[0], atol=0)


def test_stack_sparse_layers_use_latest_delta_selection():
    qs, kvs = _stack_inputs(6, 8, 2, 300, 32, 1)
    kinds = ["full", "delta", "sparse", "delta", "sparse", "sparse"]
    outs, sels = O.stack_step(kinds, lambda l: qs[l], lambda l: kvs[l], 300, 16, 3, 16, 32)
    assert set(sels) == {1, 3}
    np.testing.assert_allclose(outs[1], O.full_attention(qs[1], *kvs[1])[0], atol=0)
    for l, src in ((2, 1), (4, 3), (5, 3)):
        np.testing.assert_allclose(outs[l], O.sparse_attention(qs[l], *kvs[l], sels[src][1], 16), atol=0)


def test_delta_selection_recovers_planted_pages():
    # Each planted token carries a huge logit; with budget 3 its pages are exactly the top-3.
    Hq, Hkv, n, D = 4, 1, 400, 16
    K = rand(Hkv, n, D) * 0.01
    q = np.zeros((Hq, D)); q[:, 0] = 1.0
    for t in (50, 130, 222):
        K[0, t, 0] = 30.0
    _, p = O.full_attention(q, K, rand(Hkv, n, D), 1.0)
    sel = O.select_pages(O.page_scores(p, 16), n, 16, 3, 16, 32)
    assert sel == [0, 3, 8, 13, 23, 24]


# ----------------------------------------------------------------- layer-shift calibration
def test_layer_shift_closed_forms():
    x = np.array([3.0, 1.0, 0.0, 2.0])
    assert abs(O.layer_shift(x, x)) < 1e-15
    assert abs(O.layer_shift(x, 5 * x)) < 1e-15                     # scale invariant
    assert abs(O.layer_shift([1, 0, 0], [0, 2, 0]) - 1.0) < 1e-15   # orthogonal
    assert abs(O.layer_shift([1, 0], [1, 1]) - (1 - 1 / math.sqrt(2))) < 1e-15
    assert O.layer_shift([0, 0], [1, 2]) == 1.0


def test_layer_shift_matches_library_cosine():
    a, b = RNG.random(300), RNG.random(300)
    ref = 1 - torch.nn.functional.cosine_similarity(torch.from_numpy(a), torch.from_numpy(b), dim=0).item()
    assert abs(O.layer_shift(a, b) - ref) < 1e-12


def test_choose_delta_layers_rules():
    shift = np.array([0, 0, 0.1, 0.9, 0.85, 0.2, 0.7, 0.1, 0.8])
    assert O.choose_delta_layers(shift, 1) == [2]
    # by shift: 3 (one layer from 2: skipped), 4, 8, then 6
    assert O.choose_delta_layers(shift, 3, min_gap=2) == [2, 4, 8]
    assert O.choose_delta_layers(shift, 4, min_gap=2) == [2, 4, 6, 8]
    assert O.choose_delta_layers(shift, 3, min_gap=1) == [2, 3, 4]
