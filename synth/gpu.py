"""Device copies of a synthetic workload (pools, page table, queries, appended tokens).

Holds no attention arithmetic.  Bulk K/V values are written on the device by
``libsynth_fill.so`` (bit-identical to ``synth.rng``); planted salient-key rows are
computed on the host by ``synth.case`` and scattered into the pools.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

from . import rng
from .case import Case

_LIB = None


def fill_lib():
    global _LIB
    if _LIB is None:
        path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsynth_fill.so")
        if not os.path.exists(path):
            raise ImportError(f"{path} is missing: run `python -m long_context_layer_b200.build`")
        lib = ctypes.CDLL(path)
        lib.synth_fill_kv.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_uint64, ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_void_p]
        lib.synth_fill_kv.restype = ctypes.c_int
        lib.synth_fill_tokens.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int, ctypes.c_float,
                                          ctypes.c_void_p]
        lib.synth_fill_tokens.restype = ctypes.c_int
        _LIB = lib
    return _LIB


def torch_dtype(cfg) -> torch.dtype:
    return torch.bfloat16 if cfg.dtype == "bf16" else torch.float32


def to_device(x: np.ndarray, dtype: torch.dtype, device) -> torch.Tensor:
    """float32 stored values -> tensor of the storage dtype (exact: values are already rounded)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device=device).to(dtype)


class DeviceCase:
    """Device-resident buffers of a ``Case``.

    prefill: number of leading tokens of each sequence written into the pools; the
    default n_b - 1 leaves the current token for ``kv_append``.  ``prefill="all"``
    writes every attended token (for tests that skip the append).
    """

    def __init__(self, case: Case, device="cuda", layers=None, prefill="append", pool_pages: int | None = None,
                 garbage: float | None = None):
        self.case = case
        cfg = case.cfg
        self.cfg = cfg
        self.device = torch.device(device)
        self.dtype = torch_dtype(cfg)
        self.layers = list(range(cfg.num_layers)) if layers is None else list(layers)
        self.indptr = torch.from_numpy(case.page_indptr).to(self.device)
        self.indices = torch.from_numpy(case.page_indices).to(self.device)
        self.kv_len = torch.from_numpy(case.kv_len()).to(self.device)
        self.num_phys_pages = case.num_phys_pages if pool_pages is None else pool_pages
        fill = case.n - (1 if prefill == "append" else 0)
        self.fill_len = torch.from_numpy(fill.astype(np.int32)).to(self.device)
        B, Hq, Hkv, D = cfg.batch, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim
        self.k_pools, self.v_pools = [], []
        for l in self.layers:
            kp = torch.empty((self.num_phys_pages, Hkv, 16, D), dtype=self.dtype, device=self.device)
            vp = torch.empty_like(kp)
            if garbage is not None:           # what unwritten cache slots hold (e.g. NaN)
                kp.fill_(garbage)
                vp.fill_(garbage)
            self._fill(kp, rng.T_K, l)
            self._fill(vp, rng.T_V, l)
            self._plant(kp, l)
            self.k_pools.append(kp)
            self.v_pools.append(vp)
        self.q = torch.stack([to_device(case.q(l), self.dtype, self.device) for l in self.layers])
        self.k_new = torch.stack([to_device(case.new_token(rng.T_K, l), self.dtype, self.device) for l in self.layers])
        self.v_new = torch.stack([to_device(case.new_token(rng.T_V, l), self.dtype, self.device) for l in self.layers])
        self.out = torch.zeros((len(self.layers), B, Hq, D), dtype=self.dtype, device=self.device)
        torch.cuda.synchronize(self.device)

    def _fill(self, pool: torch.Tensor, tensor: int, layer: int) -> None:
        c = self.cfg
        st = torch.cuda.current_stream(self.device).cuda_stream
        r = fill_lib().synth_fill_kv(pool.data_ptr(), 1 if c.dtype == "bf16" else 0, self.num_phys_pages,
                                     c.num_kv_heads, c.head_dim, self.indptr.data_ptr(), self.indices.data_ptr(),
                                     self.fill_len.data_ptr(), c.batch, self.case.max_pages_per_seq,
                                     self.case.key, tensor, layer, float(rng.NORMAL_SCALE), st)
        if r != 0:
            raise RuntimeError(f"synth_fill_kv failed ({r})")

    def planted_index(self, layer: int, step: int | None = None):
        """(phys pages, kv heads, slots, rows) of every planted key of a layer."""
        c, case = self.cfg, self.case
        P, G, S, R = [], [], [], []
        for b in range(c.batch):
            for g in range(c.num_kv_heads):
                pos, rows = case.planted_rows(layer, b, g, step)
                if pos.size == 0:
                    continue
                P.append(case.page_indices[case.page_indptr[b] + pos // 16])
                G.append(np.full(pos.size, g))
                S.append(pos % 16)
                R.append(rows)
        if not P:
            return None
        return np.concatenate(P), np.concatenate(G), np.concatenate(S), np.concatenate(R)

    def _plant(self, pool: torch.Tensor, layer: int) -> None:
        idx = self.planted_index(layer)
        if idx is None:
            return
        p, g, s, rows = idx
        dev = self.device
        pool[torch.from_numpy(p.astype(np.int64)).to(dev), torch.from_numpy(g.astype(np.int64)).to(dev),
             torch.from_numpy(s.astype(np.int64)).to(dev)] = to_device(rows, self.dtype, dev)

    def fill_new_tokens(self, pos: torch.Tensor) -> None:
        """k_new / v_new of every layer <- generator values at positions pos[b] (device int32)."""
        c = self.cfg
        assert self.layers == list(range(len(self.layers)))
        st = torch.cuda.current_stream(self.device).cuda_stream
        for tensor, buf in ((rng.T_K, self.k_new), (rng.T_V, self.v_new)):
            r = fill_lib().synth_fill_tokens(buf.data_ptr(), 1 if c.dtype == "bf16" else 0, len(self.layers), c.batch,
                                             c.num_kv_heads, c.head_dim, pos.data_ptr(), self.case.key, tensor,
                                             float(rng.NORMAL_SCALE), st)
            if r != 0:
                raise RuntimeError(f"synth_fill_tokens failed ({r})")

    def replant(self, step: int) -> None:
        """Drift: move every layer's planted keys to their positions at `step` (the previous
        positions get their generator values back)."""
        c, case = self.cfg, self.case
        if c.planted == 0 or not c.drift_every:
            return
        prev_step = max(step - c.drift_every, 0)
        dev = self.device
        for li, l in enumerate(self.layers):
            P, G, S, R = [], [], [], []
            for b in range(c.batch):
                for g in range(c.num_kv_heads):
                    old = case.planted_positions(l, b, g, prev_step)
                    P.append(case.page_indices[case.page_indptr[b] + old // 16])
                    G.append(np.full(old.size, g))
                    S.append(old % 16)
                    R.append(case.kv_base(rng.T_K, l, b, g, old))
            dev_idx = lambda a: torch.from_numpy(np.concatenate(a).astype(np.int64)).to(dev)
            # restore first, then plant (two scatters: an old and a new position may coincide)
            self.k_pools[li][dev_idx(P), dev_idx(G), dev_idx(S)] = to_device(np.concatenate(R), self.dtype, dev)
            p, g, s_, rows = self.planted_index(l, step)
            self.k_pools[li][torch.from_numpy(p.astype(np.int64)).to(dev), torch.from_numpy(g.astype(np.int64)).to(dev),
                             torch.from_numpy(s_.astype(np.int64)).to(dev)] = to_device(rows, self.dtype, dev)

    def pool_row(self, layer_idx: int, tensor: int, b: int, g: int, pos: int) -> torch.Tensor:
        c = self.case
        phys = c.page_indices[c.page_indptr[b] + pos // 16]
        pool = self.k_pools[layer_idx] if tensor == rng.T_K else self.v_pools[layer_idx]
        return pool[phys, g, pos % 16]
