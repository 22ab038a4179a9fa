"""Shared test helpers: oracle inputs from the generator, tolerances, selection comparison."""
from __future__ import annotations

import numpy as np

from oracle import delta_oracle as O
from synth import rng

# Output tolerances (stated with the workloads): fp32 max-abs <= 1e-5;
# bf16 max-abs <= 2e-2 and relative L2 <= 5e-3.  Near-tie rule for selections: sets must be
# identical unless the oracle's k-th and (k+1)-th candidate scores differ by < 1e-4 relative.
F32_MAX_ABS = 1e-5
BF16_MAX_ABS = 2e-2
BF16_REL_L2 = 5e-3
TIE_REL = 1e-4


def oracle_kv(case, layer: int, b: int, n: int | None = None):
    """(K, V) [Hkv, n, D] fp64 of one sequence from the host generator."""
    c = case.cfg
    K = np.stack([case.kv_logical(rng.T_K, layer, b, g, n) for g in range(c.num_kv_heads)]).astype(np.float64)
    V = np.stack([case.kv_logical(rng.T_V, layer, b, g, n) for g in range(c.num_kv_heads)]).astype(np.float64)
    return K, V


def assert_close(gpu: np.ndarray, ref: np.ndarray, dtype: str, what: str = ""):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(gpu - ref)
    mx = float(err.max()) if err.size else 0.0
    if dtype == "f32":
        assert mx <= F32_MAX_ABS, f"{what}: max abs err {mx:.3e} > {F32_MAX_ABS}"
    else:
        rel = float(np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-30))
        assert mx <= BF16_MAX_ABS, f"{what}: max abs err {mx:.3e} > {BF16_MAX_ABS}"
        assert rel <= BF16_REL_L2, f"{what}: rel L2 {rel:.3e} > {BF16_REL_L2}"
    return mx


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
    if abs(kth - nxt) >= TIE_REL * abs(kth):
        return False, False, ref
    tied = {j for j in cands if abs(S_oracle[j] - kth) < TIE_REL * abs(kth)}
    if not forced <= set(gpu_sel):
        return False, False, ref
    sure = set(ref) - tied
    if not sure <= set(gpu_sel):
        return False, False, ref
    extra = set(gpu_sel) - set(ref)
    return extra <= tied, False, ref
