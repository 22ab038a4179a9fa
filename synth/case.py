"""Host-side construction of one synthetic decode workload.

A ``Case`` fixes, for a workload and a decode step: the per-sequence context
lengths, the shared CSR page table (logical page -> physical page, shuffled in
the pool), the queries of every layer, the appended token's k and v, and the
planted salient keys.  Every bulk K/V element is the counter-based generator
value of ``synth.rng`` at (tensor, layer, b, kv head, position, dim), rounded
to the storage dtype, except at planted positions, where the stored key is
``0.5*k + 3*q_hat`` with ``q_hat`` the unit-norm mean of the G current queries
of that KV head, rounded to the storage dtype.

Everything here runs on the host and is shared by both sides: the oracle reads
``kv_logical``; the GPU side fills its pools with the CUDA generator (same
values) and scatters ``planted_rows`` over them.
"""
from __future__ import annotations

import numpy as np

from . import rng
from .configs import StackConfig

__all__ = ["Case"]


class Case:
    def __init__(self, cfg: StackConfig, step: int = 0):
        self.cfg = cfg
        self.step = step
        self.key = rng.stream_key(cfg.seed, cfg.cfg_id)
        P = cfg.page_size
        self.n = np.array(cfg.contexts(step), dtype=np.int64)            # tokens attended per sequence
        self.n0 = np.array(cfg.contexts(0), dtype=np.int64)              # at the first step of the trajectory
        # Pages are allocated for the longest context the trajectory reaches.
        self.n_max_traj = np.array(cfg.contexts(cfg.steps - 1), dtype=np.int64)
        pages_needed = -(-self.n_max_traj // P)
        self.pages_per_seq = pages_needed.astype(np.int64)
        total = int(pages_needed.sum())
        pool = cfg.pool_pages_per_layer or total
        if pool < total:
            raise ValueError("pool too small for the sequences")
        self.num_phys_pages = pool
        perm = rng.permutation(self.key, rng.SALT_PAGE_PERM, pool)[:total]                # distinct physical pages
        self.page_indptr = np.zeros(cfg.batch + 1, dtype=np.int32)
        self.page_indptr[1:] = np.cumsum(pages_needed)
        self.page_indices = perm.astype(np.int32)
        self.max_pages_per_seq = int(pages_needed.max())
        self._q = {}
        self._plant_cache = {}

    # ---------------------------------------------------------------- queries
    def q_step(self) -> int:
        """Step index the queries are drawn at (the drift trajectory holds its queries)."""
        return 0 if self.cfg.drift_every else self.step

    def q(self, layer: int) -> np.ndarray:
        """[B, Hq, D] float32 stored values of the queries of a layer."""
        if layer not in self._q:
            c = self.cfg
            out = np.empty((c.batch, c.num_q_heads, c.head_dim), dtype=np.float32)
            for b in range(c.batch):
                for h in range(c.num_q_heads):
                    out[b, h] = rng.normal_block(self.key, rng.T_Q, layer, b, h, [self.q_step()], c.head_dim)[0]
            self._q[layer] = rng.round_to_dtype(out, c.dtype)
        return self._q[layer]

    # ---------------------------------------------------------------- planted keys
    def planted_positions(self, layer: int, b: int, g: int, step: int | None = None) -> np.ndarray:
        """Sorted planted positions of (layer, b, kv head g) at a step (empty when unplanted)."""
        c = self.cfg
        if c.planted == 0:
            return np.zeros(0, dtype=np.int64)
        step = self.step if step is None else step
        base = self._base_positions(layer, b, g)
        if c.drift_every:
            base = base + c.drift_shift * (step // c.drift_every)
        return np.sort(base)

    def _base_positions(self, layer: int, b: int, g: int) -> np.ndarray:
        ck = (layer, b, g)
        if ck in self._plant_cache:
            return self._plant_cache[ck]
        c = self.cfg
        lo = c.sink_tokens
        n0 = int(self.n0[b])                       # planted positions are drawn once, at the first step
        if c.drift_every:
            # every shifted block must stay inside the prefilled zone
            hi = n0 - 1 - c.recency_tokens - c.drift_shift * ((c.steps - 1) // c.drift_every)
        else:
            hi = n0 - c.recency_tokens
        hi = min(hi, n0 - 1)                       # the current token is never planted
        count = min(c.planted, max(hi - lo, 0))   # short contexts plant fewer keys
        if count == 0:
            out = np.zeros(0, dtype=np.int64)
            self._plant_cache[ck] = out
            return out
        if layer == 0:
            prev = None
        else:
            prev = self._base_positions(layer - 1, b, g)
        keep = min(int(round(c.planted_overlap * count)), len(prev)) if prev is not None else 0
        uid = (layer * 64 + b) * 64 + g
        chosen = []
        if keep:
            order = rng.permutation(self.key, rng.SALT_PLANT_KEEP + uid, len(prev))
            chosen = [int(prev[i]) for i in order[:keep]]
        taken = set(chosen)
        draw = 0
        while len(chosen) < count:
            p = int(rng.randint(self.key, rng.aux_counter(rng.SALT_PLANT_DRAW + uid, [draw]), lo, hi)[0])
            draw += 1
            if p not in taken:
                taken.add(p)
                chosen.append(p)
        out = np.array(chosen, dtype=np.int64)
        self._plant_cache[ck] = out
        return out

    def q_hat(self, layer: int, b: int, g: int) -> np.ndarray:
        """Unit-norm mean of the G queries of kv head g (float32)."""
        G = self.cfg.group
        m = self.q(layer)[b, g * G:(g + 1) * G].astype(np.float64).mean(axis=0)
        return (m / np.linalg.norm(m)).astype(np.float32)

    def planted_rows(self, layer: int, b: int, g: int, step: int | None = None):
        """(positions, [n_planted, D] float32 stored key rows) for (layer, b, g)."""
        pos = self.planted_positions(layer, b, g, step)
        if pos.size == 0:
            return pos, np.zeros((0, self.cfg.head_dim), dtype=np.float32)
        base = rng.round_to_dtype(
            rng.normal_block(self.key, rng.T_K, layer, b, g, pos, self.cfg.head_dim), self.cfg.dtype)
        rows = np.float32(0.5) * base + np.float32(3.0) * self.q_hat(layer, b, g)[None, :]
        return pos, rng.round_to_dtype(rows, self.cfg.dtype)

    # ---------------------------------------------------------------- KV values
    def kv_base(self, tensor: int, layer: int, b: int, g: int, pos) -> np.ndarray:
        """Generator values (stored dtype, as float32) with no planting, [len(pos), D]."""
        return rng.normal_block_stored(self.key, tensor, layer, b, g, np.asarray(pos), self.cfg.head_dim,
                                       self.cfg.dtype)

    def kv_logical(self, tensor: int, layer: int, b: int, g: int, n: int | None = None) -> np.ndarray:
        """[n, D] float32 stored K or V of sequence b, kv head g, positions 0..n-1, planting applied."""
        n = int(self.n[b]) if n is None else n
        out = self.kv_base(tensor, layer, b, g, np.arange(n))
        if tensor == rng.T_K:
            pos, rows = self.planted_rows(layer, b, g)
            m = pos < n
            out[pos[m]] = rows[m]
        return out

    def new_token(self, tensor: int, layer: int) -> np.ndarray:
        """[B, Hkv, D] float32 stored k or v of the token appended at this step (position n_b - 1)."""
        c = self.cfg
        out = np.empty((c.batch, c.num_kv_heads, c.head_dim), dtype=np.float32)
        for b in range(c.batch):
            for g in range(c.num_kv_heads):
                out[b, g] = self.kv_base(tensor, layer, b, g, [int(self.n[b]) - 1])[0]
        return out

    # ---------------------------------------------------------------- helpers
    def phys_page(self, b: int, logical_page: int) -> int:
        return int(self.page_indices[self.page_indptr[b] + logical_page])

    def kv_len(self) -> np.ndarray:
        return self.n.astype(np.int32)
