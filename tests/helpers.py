"""Shared test helpers: oracle inputs from the generator, tolerances, selection comparison."""
from __future__ import annotations

import numpy as np

from oracle import delta_oracle as O  # noqa: F401
from oracle.checks import TIE_ABS, TIE_REL, selection_ok  # noqa: F401  (one definition for tests and bench)
from synth import rng

# Output tolerances (stated with the workloads): fp32 max-abs <= 1e-5;
# bf16 max-abs <= 2e-2 and relative L2 <= 5e-3.  Near-tie rule for selections: sets must be
# identical unless the oracle's k-th and (k+1)-th candidate scores differ by < 1e-4 relative
# plus 2^-50 absolute (the GPU's fixed-point score resolution).
F32_MAX_ABS = 1e-5
BF16_MAX_ABS = 2e-2
BF16_REL_L2 = 5e-3


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
