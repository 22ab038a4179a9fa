"""Planted mistakes in the oracle must trip at least one pin.

Each case swaps one oracle function for a plausibly wrong variant (on the CPU,
inside this test only) and checks that a named pin from
``test_oracle_pins`` then fails.
"""
import numpy as np
import pytest

from oracle import delta_oracle as O
from tests import test_oracle_pins as pins


def _wrong_scale(q, K, V, scale=None):
    return _orig_full(q, K, V, 1.0 / q.shape[1] if scale is None else scale)


def _wrong_gqa(q, K, V, scale=None):
    Hq, D = q.shape
    Hkv = K.shape[0]
    scale = O.default_scale(D) if scale is None else scale
    o = np.empty((Hq, D)); p = np.empty((Hq, K.shape[1]))
    for h in range(Hq):                      # interleaved instead of contiguous groups
        oh, ph = O.softmax_attention(q[h:h + 1], K[h % Hkv], V[h % Hkv], scale)
        o[h], p[h] = oh[0], ph[0]
    return o, p


def _wrong_tie(S, n, P, k, sink, rec):
    N = O.num_pages(n, P)
    forced = set(O.sink_page_set(n, P, sink)) | set(O.recency_page_set(n, P, rec))
    cands = [j for j in range(N) if j not in forced]
    chosen = cands if len(cands) <= k else sorted(cands, key=lambda j: (-S[j], -j))[:k]
    return sorted(forced | set(chosen))


def _wrong_recency(n, P, r):
    if r <= 0 or n <= 0:
        return []
    return list(range(-(-max(n - r, 0) // P), O.num_pages(n, P)))


def _dropped_tail_page(p, P, mode=O.HEAD_SUM):
    S = _orig_scores(p, P, mode)
    if p.shape[1] % P:
        S[-1] = 0.0
    return S


def _wrong_sparse(q, K, V, pages, P, scale=None):
    t = np.concatenate([np.arange(j * P, (j + 1) * P) for j in pages])   # ignores the context end
    t = t[t < K.shape[1] - 1]
    o, _ = O.full_attention(q, K[:, t], V[:, t], scale)
    return o


_orig_full = O.full_attention
_orig_scores = O.page_scores

CASES = [
    ("full_attention", _wrong_scale, lambda: pins.test_default_scale_is_inverse_sqrt_head_dim()),
    ("full_attention", _wrong_scale, lambda: pins.test_full_attention_matches_torch_sdpa(28, 4, 333, 128)),
    ("full_attention", _wrong_gqa, lambda: pins.test_gqa_head_mapping_is_contiguous_groups()),
    ("select_pages", _wrong_tie, lambda: [pins.test_selection_matches_brute_force_with_ties(t) for t in range(40)]),
    ("recency_page_set", _wrong_recency, lambda: pins.test_recency_and_sink_page_counts_of_tiny_workload()),
    ("page_scores", _dropped_tail_page, lambda: pins.test_sum_scores_add_up_to_query_heads(17)),
    ("sparse_attention", _wrong_sparse, lambda: pins.test_sparse_equals_library_attention_on_gathered_tokens()),
]


@pytest.mark.parametrize("name,bad,pin", CASES, ids=[f"{c[0]}-{c[1].__name__}" for c in CASES])
def test_planted_mistake_is_caught(monkeypatch, name, bad, pin):
    monkeypatch.setattr(O, name, bad)
    with pytest.raises(AssertionError):
        pin()
