"""Token/page/byte accounting of the workloads, pinned to the figures the DELTA page prints."""
import json
import os

from synth import configs as C


def _golden(golden_dir):
    with open(os.path.join(golden_dir, "paper_constants.json")) as f:
        return json.load(f)


def test_page_budget_token_conversions(golden_dir):
    g = _golden(golden_dir)
    P = g["page_size"]["value"]
    assert P == C.PAGE_SIZE
    for key in ("budget_1k", "recency_main", "budget_4k", "budget_8k"):
        assert g[key]["pages"] * P == g[key]["tokens"]
        cfg = C.TINY.with_(budget_tokens=g[key]["tokens"])
        assert cfg.budget_pages == g[key]["pages"]


def test_kv_cache_size_exceeds_printed_bound(golden_dir):
    k = _golden(golden_dir)["kv_cache_llama3_8b"]
    per_tok = C.kv_bytes_per_token(k["layers"], k["kv_heads"], k["head_dim"], k["elem_bytes"])
    assert per_tok == 131072
    total = per_tok * k["context"] * k["batch"]
    assert total > k["lower_bound_bytes"]
    assert total == 549755813888


def test_layer_schedules(golden_dir):
    g = _golden(golden_dir)["delta_layers"]
    for name, d in g.items():
        if name == "cite":
            continue
        assert d["delta"][0] == 2
    # the drift workload takes the 48-layer DS-Qwen-14B list
    assert list(C.DRIFT_48L.delta_layers) == g["DS-Qwen-14B"]["delta"]
    assert C.DRIFT_48L.num_layers == g["DS-Qwen-14B"]["layers"]
    for cfg in C.CONFIGS.values():
        kinds = cfg.layer_kinds()
        first = min(cfg.delta_layers)
        assert all(k == C.FULL for k in kinds[:first])
        assert all(kinds[l] == C.DELTA for l in cfg.delta_layers)
        assert kinds.count(C.SPARSE) == cfg.num_layers - first - len(cfg.delta_layers)
    assert C.QWEN7B_8K.layer_kinds()[:3] == [C.FULL, C.FULL, C.DELTA]
    assert C.TINY.layer_kinds() == [C.FULL, C.DELTA, C.SPARSE, C.SPARSE]


def test_selection_capacities():
    assert C.sel_capacity(C.TINY) == 8 + 1 + 5
    assert C.sel_capacity(C.QWEN7B_8K) == 64 + 1 + 17
    assert C.sel_capacity(C.LLAMA8B_64K) == 256 + 1 + 33
