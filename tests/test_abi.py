"""The C-ABI library loads, exports every symbol the header declares, and rejects bad
arguments on the host before launching anything (no GPU needed for these paths)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "delta_attn.h")


@pytest.fixture(scope="module")
def L():
    import __graft_entry__
    __graft_entry__._build_module().build()
    import long_context_layer_b200 as lib
    return lib


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:size_t|delta_status|int32_t|const char\*)\s+(delta_\w+)\s*\(", text, re.M)))


def test_header_declares_the_four_calls():
    fns = declared_functions()
    for name in ("delta_kv_append", "delta_full_attn", "delta_select_attn", "delta_sparse_attn"):
        assert name in fns


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", L._native.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [f for f in declared_functions() if f not in exported]
    assert not missing, missing
    assert sorted(L._native.EXPORTED) == declared_functions()


def test_status_strings(L):
    for s in range(6):
        assert L.status_string(s) and L.status_string(s) != "unknown status"
    assert L.status_string(99) == "unknown status"


def _desc(L, **kw):
    d = dict(num_q_heads=28, num_kv_heads=4, head_dim=128, page_size=16, dtype=L.DELTA_BF16, sm_scale=0.0,
             num_phys_pages=512)
    d.update(kw)
    return L.DeltaDesc(**d)


FAKE = 1 << 40  # never dereferenced: every call below fails validation first


def _pt(L, batch=1, maxp=512):
    return L.DeltaPageTable(FAKE, FAKE, FAKE, batch, maxp)


@pytest.mark.parametrize("kw,status", [
    (dict(num_q_heads=27), 1),          # not a multiple of the KV heads
    (dict(head_dim=96), 2),             # unsupported head dim
    (dict(page_size=32), 2),            # unsupported page size
    (dict(num_q_heads=36), 2),          # group of 9 > 8
    (dict(dtype=7), 1),
    (dict(sm_scale=-1.0), 1),
])
def test_bad_descriptor_rejected(L, kw, status):
    s = L.full_attn(_desc(L, **kw), _pt(L), FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, 0, check=False)
    assert s == status


def test_null_pointers_and_workspace_rejected(L):
    d = _desc(L)
    assert L.full_attn(d, _pt(L), None, FAKE, FAKE, FAKE, FAKE, 1 << 30, 0, check=False) == 1
    assert L.full_attn(d, L.DeltaPageTable(None, FAKE, FAKE, 1, 512), FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, 0,
                       check=False) == 1
    assert L.full_attn(d, _pt(L), FAKE, FAKE, FAKE, FAKE, None, 1 << 30, 0, check=False) == 3
    assert L.full_attn(d, _pt(L), FAKE, FAKE, FAKE, FAKE, FAKE + 8, 1 << 30, 0, check=False) == 3   # misaligned
    need = L.workspace_size(d, 1, 512)
    assert need > 0
    assert L.full_attn(d, _pt(L), FAKE, FAKE, FAKE, FAKE, FAKE, need - 1, 0, check=False) == 3
    assert L.full_attn(d, _pt(L), FAKE + 4, FAKE, FAKE, FAKE, FAKE, need, 0, check=False) == 1     # misaligned q


def test_select_arguments_rejected(L):
    d = _desc(L)
    sp = L.DeltaSelectParams(64, 16, 256, L.DELTA_HEAD_SUM)
    cap = L.sel_capacity(sp)
    assert cap == 64 + 1 + 17
    ws = L.workspace_size(d, 1, 512)
    args = (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE)
    assert L.select_attn(d, _pt(L), sp, *args[:4], FAKE, FAKE, cap - 1, None, FAKE, ws, 0, check=False) == 1
    sp_max = L.DeltaSelectParams(64, 16, 256, L.DELTA_HEAD_MAX)
    ws_max = L.workspace_size_reduce(d, 1, 512, L.DELTA_HEAD_MAX)
    assert ws_max == ws + 28 * 512 * 16 * 4          # per-token logits of every query head
    assert L.workspace_size_reduce(d, 1, 512, L.DELTA_HEAD_SUM) == ws
    assert L.workspace_size_reduce(d, 1, 512, 7) == 0
    assert L.select_attn(d, _pt(L), sp_max, *args[:4], FAKE, FAKE, cap, None, FAKE, ws, 0, check=False) == 3
    sp_bad_mode = L.DeltaSelectParams(64, 16, 256, 5)
    assert L.select_attn(d, _pt(L), sp_bad_mode, *args[:4], FAKE, FAKE, cap, None, FAKE, ws, 0, check=False) == 1
    sp_bad = L.DeltaSelectParams(-1, 16, 256, L.DELTA_HEAD_SUM)
    assert L.select_attn(d, _pt(L), sp_bad, *args[:4], FAKE, FAKE, cap, None, FAKE, ws, 0, check=False) == 1
    assert L.select_attn(d, _pt(L, maxp=40000), sp, *args[:4], FAKE, FAKE, cap, None, FAKE,
                         L.workspace_size(d, 1, 40000), 0, check=False) == 2
    assert L.select_attn(d, _pt(L), sp, *args[:4], None, FAKE, cap, None, FAKE, ws, 0, check=False) == 1


def test_sparse_and_append_arguments_rejected(L):
    d = _desc(L)
    ws = L.workspace_size(d, 1, 512)
    assert L.sparse_attn(d, _pt(L), None, FAKE, 10, FAKE, FAKE, FAKE, FAKE, FAKE, ws, 0, check=False) == 1
    assert L.sparse_attn(d, _pt(L), FAKE, FAKE, 0, FAKE, FAKE, FAKE, FAKE, FAKE, ws, 0, check=False) == 1
    assert L.sparse_attn_settled(d, _pt(L), None, FAKE, 10, FAKE, FAKE, FAKE, FAKE, FAKE, ws, 0, check=False) == 1
    assert L.sparse_attn_settled(d, _pt(L), FAKE, FAKE, 0, FAKE, FAKE, FAKE, FAKE, FAKE, ws, 0, check=False) == 1
    assert L.sparse_attn_settled(d, _pt(L), FAKE, FAKE, 10, FAKE, FAKE, FAKE, FAKE, None, ws, 0, check=False) == 3
    assert L.layer_shift(_pt(L), None, FAKE, FAKE, 0, check=False) == 1
    assert L.kv_append(d, _pt(L), None, FAKE, FAKE, FAKE, 0, check=False) == 1
    assert L.kv_append(_desc(L, head_dim=80), _pt(L), FAKE, FAKE, FAKE, FAKE, 0, check=False) == 2


def test_empty_batch_is_a_no_op(L):
    d = _desc(L)
    pt = L.DeltaPageTable(None, None, None, 0, 0)
    assert L.full_attn(d, pt, None, None, None, None, None, 0, 0, check=False) == 0
    assert L.kv_append(d, pt, None, None, None, None, 0, check=False) == 0


def test_stack_placement_rule_matches_the_oracle():
    # the library's delta-layer placement (delta_choose_layers, a host function) equals the oracle's on random shifts,
    # ties included
    import numpy as np
    from oracle import delta_oracle as O
    from long_context_layer_b200.stack import choose_delta_layers
    r = np.random.default_rng(7)
    for _ in range(200):
        L = int(r.integers(4, 49))
        shift = np.round(r.random(L), 1)          # coarse values: many exact ties
        shift[:2] = 0.0
        count = int(r.integers(1, 6))
        gap = int(r.integers(1, 4))
        assert choose_delta_layers(shift, count, min_gap=gap) == O.choose_delta_layers(shift, count, min_gap=gap)


def test_choose_layers_rejects_bad_arguments(L):
    import ctypes
    from long_context_layer_b200 import _native as N
    shift = (ctypes.c_float * 4)(0, 0, 0.5, float("nan"))
    out = (ctypes.c_int32 * 4)()
    n = ctypes.c_int32(0)
    assert N.lib.delta_choose_layers(shift, 4, 2, 2, 1, out, ctypes.byref(n)) == N.DELTA_ERR_INVALID_ARG   # NaN
    ok = (ctypes.c_float * 4)(0, 0, 0.5, 0.7)
    assert N.lib.delta_choose_layers(ok, 4, 2, 4, 1, out, ctypes.byref(n)) == N.DELTA_ERR_INVALID_ARG     # first
    assert N.lib.delta_choose_layers(ok, 4, 2, 2, -1, out, ctypes.byref(n)) == N.DELTA_ERR_INVALID_ARG    # gap
    assert N.lib.delta_choose_layers(ok, 4, 3, 2, 1, out, ctypes.byref(n)) == N.DELTA_OK
    assert [out[i] for i in range(n.value)] == [2, 3]        # only two layers after layer 1
