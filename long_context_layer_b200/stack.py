"""One DELTA decode step over a whole layer stack, through the C ABI.

Layer schedule (DELTA: Dynamic Layer-Aware Token Attention, ai.info summary,
"Methodology in Plain English"): layers before the first delta-layer run full
attention; a delta-layer runs full attention and refreshes the page selection;
every other layer runs sparse attention over the selection of the most recent
delta-layer of the same decode step.  The step starts by appending the current
token's k and v to every layer's paged pool in one launch (the cache is kept in full).

The runner only sequences C-ABI calls on one CUDA stream; it can capture the
whole step in a CUDA graph so one replay launches every kernel of the step.
"""
from __future__ import annotations

import torch

from . import _native as N

FULL, DELTA, SPARSE = "full", "delta", "sparse"


def layer_kinds(num_layers: int, delta_layers) -> list:
    first = min(delta_layers)
    return [DELTA if l in delta_layers else (FULL if l < first else SPARSE) for l in range(num_layers)]


class DeltaStack:
    """Buffers and call sequence of one decode step.

    Tensors (all on one CUDA device):
      indptr [B+1], indices [nnz], kv_len [B]  int32 page table shared by all layers
      k_pools[l], v_pools[l]                   [num_phys_pages, Hkv, 16, D] per layer
      q [L, B, Hq, D], k_new / v_new [L, B, Hkv, D], out [L, B, Hq, D]
    """

    def __init__(self, kinds, num_q_heads: int, num_kv_heads: int, head_dim: int, dtype: torch.dtype,
                 indptr: torch.Tensor, indices: torch.Tensor, kv_len: torch.Tensor, max_pages_per_seq: int,
                 num_phys_pages: int, budget_pages: int = 0, sink_tokens: int = 0, recency_tokens: int = 0,
                 sm_scale: float = 0.0, keep_scores: bool = False, reduce: int = N.DELTA_HEAD_SUM):
        self.kinds = list(kinds)
        self.device = indptr.device
        self.batch = int(kv_len.numel())
        self.dtype = dtype
        dt = N.DELTA_BF16 if dtype == torch.bfloat16 else N.DELTA_F32
        if dtype not in (torch.bfloat16, torch.float32):
            raise ValueError("dtype must be bfloat16 or float32")
        self.desc = N.DeltaDesc(num_q_heads, num_kv_heads, head_dim, 16, dt, sm_scale, num_phys_pages)
        self.indptr, self.indices, self.kv_len = indptr, indices, kv_len
        self.pt = N.DeltaPageTable(indptr.data_ptr(), indices.data_ptr(), kv_len.data_ptr(), self.batch,
                                   max_pages_per_seq)
        self.sp = N.DeltaSelectParams(budget_pages, sink_tokens, recency_tokens, reduce)
        self.max_pages = max_pages_per_seq
        self.ws_bytes = N.workspace_size_reduce(self.desc, self.batch, max_pages_per_seq, reduce)
        self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=self.device)
        N.workspace_init(self.workspace, self.ws_bytes, torch.cuda.current_stream(self.device).cuda_stream)
        self.sel_stride = max(N.sel_capacity(self.sp), 1)
        self.delta_layers = [l for l, k in enumerate(self.kinds) if k == DELTA]
        nd = max(len(self.delta_layers), 1)
        self.sel_cnt = torch.zeros(nd, self.batch, dtype=torch.int32, device=self.device)
        self.sel_pages = torch.zeros(nd, self.batch, self.sel_stride, dtype=torch.int32, device=self.device)
        self.page_scores = (torch.zeros(nd, self.batch, max_pages_per_seq, dtype=torch.float32, device=self.device)
                            if keep_scores else None)
        if any(k == SPARSE for k in self.kinds):
            first_sparse = self.kinds.index(SPARSE)
            if not any(k == DELTA for k in self.kinds[:first_sparse]):
                raise ValueError("a sparse layer needs an earlier delta-layer")
        self.graph = None

    # ------------------------------------------------------------------ one step
    def launches_per_step(self, append: bool = True) -> int:
        # a delta-layer scoring with HEAD_SUM selects its pages inside its decode kernel; HEAD_MAX
        # adds a selection kernel
        per = {FULL: 1, DELTA: 1 if self.sp.reduce == N.DELTA_HEAD_SUM else 2, SPARSE: 1}
        return sum(per[k] for k in self.kinds) + (1 if append else 0)

    def step(self, q, k_new, v_new, k_pools, v_pools, out, append: bool = True, stream: int | None = None):
        st = torch.cuda.current_stream(self.device).cuda_stream if stream is None else stream
        d, pt = self.desc, self.pt
        cur = -1
        if append:      # every layer's new token in one launch (layers do not read each other's pools)
            N.kv_append_layers(d, pt, k_new, v_new, k_pools, v_pools, st)
        for l, kind in enumerate(self.kinds):
            # a sparse layer after a sparse layer uses the settled entry: the selection and the
            # appended tokens were final before the previous sparse layer began (it waited on the
            # delta-layer that wrote the selection), so this layer may read them early
            self._layer(l, kind, cur, q, k_pools, v_pools, out, st)
            if kind == DELTA:
                cur = self.delta_layers.index(l)

    # ------------------------------------------------------------------ host buffers
    def step_host(self, q_host, k_new_host, v_new_host, k_pools, v_pools, out_host, q_dev, k_new_dev, v_new_dev,
                  out_dev, append: bool = True, early_layers: int = 2, out_chunks: int = 8):
        """One decode step whose inputs and outputs live in (pinned) host memory.

        On a copy stream: the first `early_layers` layers' q and appended tokens, then every other
        layer's, which arrive while the first layers compute (the append runs as two launches, one
        per group of layers).  The outputs return to the host on another stream in about `out_chunks`
        groups of consecutive layers, each as soon as its last layer is done (the last layer on its
        own, so that only its output is copied after the final kernel).  The compute stream
        joins the copy streams at those few points only, so most consecutive kernels keep their
        programmatic-launch overlap.  *_dev are device staging buffers of the same shapes.
        Everything is enqueued on the current stream (graph-capturable); out_host is complete once
        that stream reaches the end of the step.
        """
        main = torch.cuda.current_stream(self.device)
        if not hasattr(self, "_up"):
            self._up = torch.cuda.Stream(self.device)
            self._down = torch.cuda.Stream(self.device)
        up, down = self._up, self._down
        L = len(self.kinds)
        early = max(1, min(early_layers, L))
        up.wait_stream(main)
        down.wait_stream(main)
        groups = [(0, early)] + ([(early, L)] if early < L else [])
        ready = []
        with torch.cuda.stream(up):
            for a, b in groups:
                q_dev[a:b].copy_(q_host[a:b], non_blocking=True)
                k_new_dev[a:b].copy_(k_new_host[a:b], non_blocking=True)
                v_new_dev[a:b].copy_(v_new_host[a:b], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(up)
                ready.append(ev)
        st = main.cuda_stream
        per = -(-max(L - 1, 1) // max(1, out_chunks))
        cur, c0 = -1, 0
        for gi, (a, b) in enumerate(groups):
            main.wait_event(ready[gi])
            if append:
                N.kv_append_layers(self.desc, self.pt, k_new_dev[a:b], v_new_dev[a:b], k_pools[a:b], v_pools[a:b], st)
            for l in range(a, b):
                kind = self.kinds[l]
                self._layer(l, kind, cur, q_dev, k_pools, v_pools, out_dev, st)
                if kind == DELTA:
                    cur = self.delta_layers.index(l)
                if l + 1 - c0 == per or l >= L - 2:
                    done = torch.cuda.Event()
                    done.record(main)
                    down.wait_event(done)
                    with torch.cuda.stream(down):
                        out_host[c0:l + 1].copy_(out_dev[c0:l + 1], non_blocking=True)
                    c0 = l + 1
        main.wait_stream(up)
        main.wait_stream(down)

    def _layer(self, l, kind, cur, q, k_pools, v_pools, out, st):
        d, pt, ws, wb = self.desc, self.pt, self.workspace, self.ws_bytes
        if kind == FULL:
            N.full_attn(d, pt, q[l], k_pools[l], v_pools[l], out[l], ws, wb, st)
        elif kind == DELTA:
            c = self.delta_layers.index(l)
            scores = self.page_scores[c] if self.page_scores is not None else None
            N.select_attn(d, pt, self.sp, q[l], k_pools[l], v_pools[l], out[l], self.sel_cnt[c], self.sel_pages[c],
                          self.sel_stride, scores, ws, wb, st)
        elif l > 0 and self.kinds[l - 1] == SPARSE:
            N.sparse_attn_settled(d, pt, self.sel_cnt[cur], self.sel_pages[cur], self.sel_stride, q[l], k_pools[l],
                                  v_pools[l], out[l], ws, wb, st)
        else:
            N.sparse_attn(d, pt, self.sel_cnt[cur], self.sel_pages[cur], self.sel_stride, q[l], k_pools[l],
                          v_pools[l], out[l], ws, wb, st)

    # ------------------------------------------------------------------ CUDA graph
    def capture(self, *args, **kw) -> torch.cuda.CUDAGraph:
        """Capture one step (same arguments as step) into a CUDA graph and return it."""
        s = torch.cuda.Stream(self.device)
        s.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(s):
            self.step(*args, **kw)          # warm: sets per-device kernel attributes outside capture
        torch.cuda.current_stream(self.device).wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.step(*args, **kw)
        self.graph = g
        return g

    def selection(self, delta_index: int = -1) -> list:
        """Host copy of a delta-layer's selection: list (per sequence) of ascending logical pages."""
        cnt = self.sel_cnt[delta_index].cpu().tolist()
        pages = self.sel_pages[delta_index].cpu()
        return [pages[b, :cnt[b]].tolist() for b in range(self.batch)]

    # ------------------------------------------------------------------ calibration
    def calibration_shifts(self, q, k_pools, v_pools, out, stream: int | None = None) -> torch.Tensor:
        """Per-layer shift [L, B]: shift[l][b] = 1 - cos(page scores of layer l-1, of layer l).

        Every layer from 1 on runs as a delta-layer (full attention plus page scores) on the
        current cache; layers 0 and 1 get shift 0.  DELTA's calibration (ai.info summary,
        "Methodology in Plain English") averages such shifts over several steps and inputs
        and places the delta-layers where they are large.
        """
        st = torch.cuda.current_stream(self.device).cuda_stream if stream is None else stream
        L = len(self.kinds)
        scores = torch.zeros(L, self.batch, self.max_pages, dtype=torch.float32, device=self.device)
        shift = torch.zeros(L, self.batch, dtype=torch.float32, device=self.device)
        sel_cnt = torch.zeros(self.batch, dtype=torch.int32, device=self.device)
        sel_pages = torch.zeros(self.batch, self.sel_stride, dtype=torch.int32, device=self.device)
        for l in range(1, L):
            N.select_attn(self.desc, self.pt, self.sp, q[l], k_pools[l], v_pools[l], out[l], sel_cnt, sel_pages,
                          self.sel_stride, scores[l], self.workspace, self.ws_bytes, st)
            if l >= 2:
                N.layer_shift(self.pt, scores[l - 1], scores[l], shift[l], st)
        return shift


def choose_delta_layers(shift, count: int, first: int = 2, min_gap: int = 2) -> list:
    """Delta-layer placement from per-layer shifts (shift[l]: between layers l-1 and l), computed by
    the library's host function delta_choose_layers (the rule is stated in include/delta_attn.h)."""
    return N.choose_layers(shift, count, first, min_gap)
