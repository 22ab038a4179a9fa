"""The five synthetic decode workloads and their layer schedules.

Each workload is a stack of layers of three kinds (DELTA: Dynamic Layer-Aware
Token Attention, ai.info summary, "Methodology in Plain English"): the layers
before the first delta-layer run full attention, the delta-layers run full
attention and refresh the page selection, and every other layer attends only to
the pages chosen by the latest delta-layer.  The delta-layer indices of the
Qwen-7B / Llama-8B / Qwen-14B-shaped stacks follow the calibrated lists under
"Main Findings" (the last bullet) of the same page where the workload names them.

Token/page arithmetic follows the same page ("Main Findings", fifth bullet):
a budget of K pages of P=16 tokens is K*16 tokens (64 pages are 1k tokens), and
the recency window of 8 pages covers 128 tokens.
"""
from __future__ import annotations

from dataclasses import dataclass

from . import rng

PAGE_SIZE = 16

FULL, DELTA, SPARSE = "full", "delta", "sparse"


@dataclass(frozen=True)
class StackConfig:
    name: str
    cfg_id: int
    dtype: str                      # "f32" | "bf16": storage type of q, k, v, o
    num_layers: int
    delta_layers: tuple
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    batch: int
    budget_tokens: int
    sink_tokens: int
    recency_tokens: int
    context: int = 0                # fixed n_b (tokens attended, current token included); 0 -> drawn
    context_range: tuple = ()       # (lo, hi) inclusive range for per-sequence draws
    context_list: tuple = ()        # explicit n_b per sequence (overrides the two above)
    planted: int = 0                # salient keys per (layer, b, kv head)
    planted_overlap: float = 0.8
    pool_pages_per_layer: int = 0   # 0 -> exactly the pages the sequences need
    steps: int = 1                  # decode steps of the trajectory (drift workload)
    drift_every: int = 0
    drift_shift: int = 0
    seed: int = 0
    page_size: int = PAGE_SIZE

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def budget_pages(self) -> int:
        return self.budget_tokens // self.page_size

    def layer_kinds(self) -> list:
        first = min(self.delta_layers)
        kinds = []
        for l in range(self.num_layers):
            if l in self.delta_layers:
                kinds.append(DELTA)
            elif l < first:
                kinds.append(FULL)
            else:
                kinds.append(SPARSE)
        return kinds

    def contexts(self, step: int = 0) -> list:
        """n_b for every sequence at a decode step (the appended token included)."""
        if self.context_list:
            base = list(self.context_list)
        elif self.context:
            base = [self.context] * self.batch
        else:
            lo, hi = self.context_range
            key = rng.stream_key(self.seed, self.cfg_id)
            base = [int(x) for x in rng.randint(key, rng.aux_counter(rng.SALT_CONTEXT, range(self.batch)), lo, hi + 1)]
        return [n + step for n in base]

    def max_context(self) -> int:
        top = max(self.context_list) if self.context_list else (self.context if self.context else self.context_range[1])
        return top + self.steps - 1

    def with_(self, **kw) -> "StackConfig":
        d = dict(self.__dict__)
        d.update(kw)
        return StackConfig(**d)


def sink_pages(sink_tokens: int, page_size: int = PAGE_SIZE) -> int:
    """Pages overlapping the first sink_tokens tokens."""
    return -(-sink_tokens // page_size)


def recency_pages_max(recency_tokens: int, page_size: int = PAGE_SIZE) -> int:
    """Upper bound on pages overlapping the last recency_tokens tokens (one more when unaligned)."""
    return 0 if recency_tokens <= 0 else -(-recency_tokens // page_size) + 1


def sel_capacity(cfg: StackConfig) -> int:
    """Room for one sequence's selection list: k + sink + recency pages (+1 for an unaligned end)."""
    return cfg.budget_pages + sink_pages(cfg.sink_tokens, cfg.page_size) + recency_pages_max(cfg.recency_tokens, cfg.page_size)


TINY = StackConfig(
    name="tiny-f32", cfg_id=1, dtype="f32", num_layers=4, delta_layers=(1,),
    num_q_heads=8, num_kv_heads=1, head_dim=64, batch=1, context=1024,
    budget_tokens=8 * 16, sink_tokens=16, recency_tokens=64)

QWEN7B_8K = StackConfig(
    name="qwen7b-b1-8k-bf16", cfg_id=2, dtype="bf16", num_layers=28, delta_layers=(2, 14),
    num_q_heads=28, num_kv_heads=4, head_dim=128, batch=1, context=8192,
    budget_tokens=1024, sink_tokens=16, recency_tokens=256, planted=32)

QWEN7B_B8_VAR = StackConfig(
    name="qwen7b-b8-16k32k-bf16", cfg_id=3, dtype="bf16", num_layers=28, delta_layers=(2, 14),
    num_q_heads=28, num_kv_heads=4, head_dim=128, batch=8, context_range=(16384, 32768),
    budget_tokens=2048, sink_tokens=16, recency_tokens=512, planted=32,
    pool_pages_per_layer=69905)

LLAMA8B_64K = StackConfig(
    name="llama3-8b-b4-64k-bf16", cfg_id=4, dtype="bf16", num_layers=32, delta_layers=(2, 12, 22),
    num_q_heads=32, num_kv_heads=8, head_dim=128, batch=4, context=65536,
    budget_tokens=4096, sink_tokens=16, recency_tokens=512, planted=32)

DRIFT_48L = StackConfig(
    name="drift-48l-b16-16k-bf16", cfg_id=5, dtype="bf16", num_layers=48, delta_layers=(2, 6, 42),
    num_q_heads=40, num_kv_heads=8, head_dim=128, batch=16, context=16385,
    budget_tokens=2048, sink_tokens=16, recency_tokens=512, planted=32,
    steps=1000, drift_every=100, drift_shift=256)

CONFIGS = {c.cfg_id: c for c in (TINY, QWEN7B_8K, QWEN7B_B8_VAR, LLAMA8B_64K, DRIFT_48L)}


def kv_bytes_per_token(num_layers: int, num_kv_heads: int, head_dim: int, elem_bytes: int) -> int:
    """KV-cache bytes one token occupies across a model (K and V, every layer)."""
    return num_layers * num_kv_heads * head_dim * 2 * elem_bytes
