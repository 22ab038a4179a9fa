"""Plain fp64 CPU oracle of the DELTA decode attention stack.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import or call this
module; only the tests, the smoke check and the CPU-baseline leg of the
benchmark do.  It shares no code with the CUDA path.

It restates the method of "DELTA: Dynamic Layer-Aware Token Attention for
Efficient Long-Context Reasoning" (ai.info summary, section "Methodology in
Plain English"; authors' abstract), with these readings where the page leaves
a step open:

* attention is ordinary scaled-dot-product softmax attention of the current
  token's query against every cached token (scale 1/sqrt(D), no mask beyond
  the context length, the current token included);
* grouped-query attention: query head h reads KV head h // G, G = Hq / Hkv;
* a delta-layer's own output is full attention (it attends to every token while scoring);
* the page score is the softmax probability summed over all query heads of
  the sequence and over the page's tokens (HEAD_SUM).  The page's own wording,
  the maximum weight across heads per token summed over the page, is kept as
  the HEAD_MAX mode;
* selection: sink pages (those overlapping the first ``sink_tokens`` tokens)
  and recency pages (those overlapping the last ``recency_tokens`` tokens) are
  always kept, and ``k = budget_tokens / P`` more pages are taken from the
  remaining ones by score, higher first, equal scores to the lower page index;
  the result is the ascending union;
* a sparse layer attends only to the tokens of the selected pages of the most
  recent delta-layer of the same decode step, softmax renormalised over them.

Everything is computed directly from its definition: probabilities are formed
explicitly and page scores are sums of those probabilities, so the GPU's
split/partial decomposition is checked, not copied.
"""
from __future__ import annotations

import numpy as np

HEAD_SUM = "sum"
HEAD_MAX = "max"


def softmax_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float):
    """Scaled-dot-product attention of queries against one KV head.

    q: [G, D]; K, V: [n, D].  Returns (o [G, D], p [G, n]), fp64.
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    s = (q @ K.T) * scale                           # logits s_t = (q . k_t) / sqrt(D)
    s_max = s.max(axis=1, keepdims=True)
    e = np.exp(s - s_max)
    p = e / e.sum(axis=1, keepdims=True)            # softmax over the n tokens
    return p @ V, p


def default_scale(head_dim: int) -> float:
    return 1.0 / np.sqrt(head_dim)


def full_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float | None = None):
    """Decode attention of one sequence over its whole cache (GQA).

    q: [Hq, D]; K, V: [Hkv, n, D].  Returns (o [Hq, D], p [Hq, n]).
    """
    Hq, D = q.shape
    Hkv = K.shape[0]
    if Hq % Hkv:
        raise ValueError("query heads must be a multiple of KV heads")
    G = Hq // Hkv
    scale = default_scale(D) if scale is None else scale
    o = np.empty((Hq, D), dtype=np.float64)
    p = np.empty((Hq, K.shape[1]), dtype=np.float64)
    for g in range(Hkv):
        og, pg = softmax_attention(q[g * G:(g + 1) * G], K[g], V[g], scale)
        o[g * G:(g + 1) * G] = og
        p[g * G:(g + 1) * G] = pg
    return o, p


def num_pages(n: int, page_size: int) -> int:
    return -(-n // page_size)


def page_scores(p: np.ndarray, page_size: int, mode: str = HEAD_SUM) -> np.ndarray:
    """Per-page score from token probabilities p [Hq, n].

    HEAD_SUM: S_j = sum over heads h and tokens t of page j of p[h, t].
    HEAD_MAX: S_j = sum over tokens t of page j of max_h p[h, t].
    """
    Hq, n = p.shape
    N = num_pages(n, page_size)
    if mode == HEAD_SUM:
        token = p.sum(axis=0)
    elif mode == HEAD_MAX:
        token = p.max(axis=0)
    else:
        raise ValueError(mode)
    S = np.zeros(N, dtype=np.float64)
    for j in range(N):
        S[j] = token[j * page_size:min((j + 1) * page_size, n)].sum()
    return S


def sink_page_set(n: int, page_size: int, sink_tokens: int) -> list:
    """Pages overlapping the first sink_tokens tokens of an n-token context."""
    return list(range(num_pages(min(sink_tokens, n), page_size)))


def recency_page_set(n: int, page_size: int, recency_tokens: int) -> list:
    """Pages overlapping the last recency_tokens tokens of an n-token context."""
    if recency_tokens <= 0 or n <= 0:
        return []
    first = max(n - recency_tokens, 0) // page_size
    return list(range(first, num_pages(n, page_size)))


def select_pages(S: np.ndarray, n: int, page_size: int, budget_pages: int,
                 sink_tokens: int, recency_tokens: int) -> list:
    """Ascending selected logical pages: sink U recency U top-k of the others.

    Top-k orders candidates by score descending and, among equal scores, by
    page index ascending, and takes the first k = budget_pages of them.
    """
    N = num_pages(n, page_size)
    assert len(S) >= N
    forced = set(sink_page_set(n, page_size, sink_tokens)) | set(recency_page_set(n, page_size, recency_tokens))
    candidates = [j for j in range(N) if j not in forced]
    if len(candidates) <= budget_pages:
        chosen = candidates
    else:
        chosen = sorted(candidates, key=lambda j: (-S[j], j))[:budget_pages]
    return sorted(forced | set(chosen))


def page_tokens(pages, n: int, page_size: int) -> np.ndarray:
    """Token positions (< n) of the given logical pages, in page order."""
    idx = [np.arange(j * page_size, min((j + 1) * page_size, n)) for j in pages]
    return np.concatenate(idx) if idx else np.zeros(0, dtype=np.int64)


def sparse_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, pages, page_size: int,
                     scale: float | None = None):
    """Attention restricted to the tokens of the selected pages.  Returns o [Hq, D]."""
    n = K.shape[1]
    t = page_tokens(pages, n, page_size)
    o, _ = full_attention(q, K[:, t], V[:, t], scale)
    return o


def stack_step(kinds, q_of, kv_of, n: int, page_size: int, budget_pages: int,
               sink_tokens: int, recency_tokens: int, mode: str = HEAD_SUM,
               scale: float | None = None, layers=None):
    """One decode step of one sequence through a layer stack.

    kinds: layer kinds ("full" | "delta" | "sparse") in order.
    q_of(l) -> [Hq, D]; kv_of(l) -> (K [Hkv, n, D], V [Hkv, n, D]).
    Returns ({layer: o}, {delta layer: (scores, selection)}).  ``layers``
    restricts which outputs are computed (selections are always refreshed).
    """
    outs, sels = {}, {}
    sel = None
    for l, kind in enumerate(kinds):
        want = layers is None or l in layers
        if kind == "sparse" and not want:
            continue
        K, V = kv_of(l)
        if kind in ("full", "delta"):
            o, p = full_attention(q_of(l), K, V, scale)
            if kind == "delta":
                S = page_scores(p, page_size, mode)
                sel = select_pages(S, n, page_size, budget_pages, sink_tokens, recency_tokens)
                sels[l] = (S, sel)
        else:
            if sel is None:
                raise ValueError("a sparse layer needs an earlier delta-layer")
            o = sparse_attention(q_of(l), K, V, sel, page_size, scale)
        if want:
            outs[l] = o
    return outs, sels


def layer_shift(scores_a: np.ndarray, scores_b: np.ndarray) -> float:
    """Inter-layer shift 1 - cos(S_a, S_b) of two layers' page-score vectors.

    The calibration of the delta-layers (ai.info summary, "Methodology in Plain English") averages
    1 - cosine similarity between consecutive layers' attention; the page-level attention map of a
    layer is read here as its vector of page scores.  Zero vectors give a shift of 1.
    """
    a = np.asarray(scores_a, dtype=np.float64)
    b = np.asarray(scores_b, dtype=np.float64)
    na, nb = np.sqrt((a * a).sum()), np.sqrt((b * b).sum())
    if na == 0.0 or nb == 0.0:
        return 1.0
    return 1.0 - float((a * b).sum() / (na * nb))


def choose_delta_layers(shift: np.ndarray, count: int, first: int = 2, min_gap: int = 2) -> list:
    """Delta-layer placement from per-layer shifts (shift[l] = shift between layers l-1 and l).

    Reading of the calibration step (ai.info summary, "Methodology in Plain English"): the page
    fixes layer 2 as the first delta-layer and asks for the rest at layers of large shift spread
    over the depth of the model.  Here layer `first` is taken, then candidates in decreasing
    shift order (equal shifts: lower layer first), each kept when it lies at least `min_gap`
    layers from every layer already kept, until `count` layers are kept.
    """
    L = len(shift)
    chosen = [first]
    for l in sorted(range(first + 1, L), key=lambda l: (-shift[l], l)):
        if len(chosen) >= count:
            break
        if all(abs(l - c) >= min_gap for c in chosen):
            chosen.append(l)
    return sorted(chosen)
