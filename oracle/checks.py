"""Comparison of a GPU page selection with the oracle's — TEST INFRASTRUCTURE ONLY.

Selections are compared exactly, except where the oracle's k-th and (k+1)-th candidate
scores lie within ``TIE_REL`` (relative) plus ``TIE_ABS`` (absolute) of each other: pages
inside that near-tied band may be swapped, since rounding in a different summation order may
legitimately reorder them.  Every page outside the band, the sink pages and the recency pages
must agree exactly.

``TIE_ABS`` is the GPU selection's resolution: it sums each page's score in fixed point with
unit 2^-55, every KV head's share rounded on its own (at most 32 KV heads, so at most 2^-51
of rounding per page), which cannot order two scores closer than that; 2^-50 covers it.
"""
from __future__ import annotations

import numpy as np

from . import delta_oracle as O

TIE_REL = 1e-4
TIE_ABS = 2.0 ** -50


def selection_ok(gpu_sel, S_oracle: np.ndarray, n: int, budget_pages: int, sink_tokens: int,
                 recency_tokens: int, page_size: int = 16):
    """True if the GPU selection equals the oracle's, up to swaps among near-tied boundary pages.

    Returns (ok, exact, oracle_selection).
    """
    ref = O.select_pages(S_oracle, n, page_size, budget_pages, sink_tokens, recency_tokens)
    gpu_sel = list(gpu_sel)
    if gpu_sel == ref:
        return True, True, ref
    if gpu_sel != sorted(set(gpu_sel)) or len(gpu_sel) != len(ref):
        return False, False, ref
    N = O.num_pages(n, page_size)
    forced = set(O.sink_page_set(n, page_size, sink_tokens)) | set(O.recency_page_set(n, page_size, recency_tokens))
    cands = sorted((j for j in range(N) if j not in forced), key=lambda j: (-S_oracle[j], j))
    if len(cands) <= budget_pages or budget_pages == 0:
        return False, False, ref
    kth = S_oracle[cands[budget_pages - 1]]
    nxt = S_oracle[cands[budget_pages]]
    band = TIE_REL * abs(kth) + TIE_ABS
    if abs(kth - nxt) >= band:
        return False, False, ref
    tied = {j for j in cands if abs(S_oracle[j] - kth) < band}
    if not forced <= set(gpu_sel):
        return False, False, ref
    sure = set(ref) - tied
    if not sure <= set(gpu_sel):
        return False, False, ref
    extra = set(gpu_sel) - set(ref)
    return extra <= tied, False, ref
