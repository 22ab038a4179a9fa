"""fp64 CPU oracle of the DELTA decode stack — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product path (``long_context_layer_b200``) never does, and the two share no
code; the only common inputs come from the seeded generators in ``synth``.
"""
from .delta_oracle import (  # noqa: F401
    HEAD_MAX, HEAD_SUM, choose_delta_layers, default_scale, layer_shift, full_attention, num_pages, page_scores, page_tokens,
    recency_page_set, select_pages, sink_page_set, softmax_attention, sparse_attention, stack_step,
)
