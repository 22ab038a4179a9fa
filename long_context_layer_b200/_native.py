"""ctypes binding of include/delta_attn.h (argument marshalling only).

Every function takes device pointers as integers or torch CUDA tensors and passes
them unchanged to the C ABI; all computation happens in libdelta_attn.so.  Importing
this module fails loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdelta_attn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m long_context_layer_b200.build` "
        "(there is no fallback implementation)")

lib = ctypes.CDLL(LIB_PATH)

DELTA_OK, DELTA_ERR_INVALID_ARG, DELTA_ERR_UNSUPPORTED, DELTA_ERR_WORKSPACE, DELTA_ERR_CUDA, DELTA_ERR_BOUNDS = range(6)
DELTA_F32, DELTA_BF16 = 0, 1
DELTA_HEAD_SUM, DELTA_HEAD_MAX = 0, 1

EXPORTED = [
    "delta_workspace_size", "delta_workspace_size_reduce", "delta_workspace_init", "delta_sel_capacity", "delta_kv_append",
    "delta_kv_append_layers",
    "delta_full_attn", "delta_full_attn_noalloc", "delta_select_attn", "delta_sparse_attn",
    "delta_sparse_attn_settled",
    "delta_layer_shift", "delta_choose_layers", "delta_read_device_error",
    "delta_status_string",
]


class DeltaDesc(ctypes.Structure):
    _fields_ = [("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("sm_scale", ctypes.c_float),
                ("num_phys_pages", ctypes.c_int64)]


class DeltaPageTable(ctypes.Structure):
    _fields_ = [("page_indptr", ctypes.c_void_p), ("page_indices", ctypes.c_void_p),
                ("kv_len", ctypes.c_void_p), ("batch", ctypes.c_int32),
                ("max_pages_per_seq", ctypes.c_int32)]


class DeltaSelectParams(ctypes.Structure):
    _fields_ = [("budget_pages", ctypes.c_int32), ("sink_tokens", ctypes.c_int32),
                ("recency_tokens", ctypes.c_int32), ("reduce", ctypes.c_int32)]


_vp, _sz, _i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
_D, _PT, _SP = ctypes.POINTER(DeltaDesc), ctypes.POINTER(DeltaPageTable), ctypes.POINTER(DeltaSelectParams)

lib.delta_workspace_size.argtypes = [_D, _i32, _i32]
lib.delta_workspace_size.restype = _sz
lib.delta_workspace_size_reduce.argtypes = [_D, _i32, _i32, _i32]
lib.delta_workspace_size_reduce.restype = _sz
lib.delta_workspace_init.argtypes = [_vp, _sz, _vp]
lib.delta_workspace_init.restype = _i32
lib.delta_sel_capacity.argtypes = [_SP, _i32]
lib.delta_sel_capacity.restype = _i32
lib.delta_kv_append.argtypes = [_D, _PT, _vp, _vp, _vp, _vp, _vp]
lib.delta_kv_append.restype = _i32
_vpp = ctypes.POINTER(ctypes.c_void_p)
lib.delta_kv_append_layers.argtypes = [_D, _PT, _i32, _vpp, _vpp, _vpp, _vpp, _vp]
lib.delta_kv_append_layers.restype = _i32
lib.delta_full_attn.argtypes = [_D, _PT, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
lib.delta_full_attn.restype = _i32
lib.delta_full_attn_noalloc.argtypes = [_D, _PT, _vp, _vp, _vp, _vp, _vp]
lib.delta_full_attn_noalloc.restype = _i32
lib.delta_select_attn.argtypes = [_D, _PT, _SP, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _sz, _vp]
lib.delta_select_attn.restype = _i32
lib.delta_sparse_attn.argtypes = [_D, _PT, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
lib.delta_sparse_attn.restype = _i32
lib.delta_sparse_attn_settled.argtypes = [_D, _PT, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
lib.delta_sparse_attn_settled.restype = _i32
lib.delta_layer_shift.argtypes = [_PT, _vp, _vp, _vp, _vp]
lib.delta_layer_shift.restype = _i32
lib.delta_choose_layers.argtypes = [ctypes.POINTER(ctypes.c_float), _i32, _i32, _i32, _i32,
                                    ctypes.POINTER(_i32), ctypes.POINTER(_i32)]
lib.delta_choose_layers.restype = _i32
lib.delta_read_device_error.argtypes = [_vp, ctypes.POINTER(_i32), _vp]
lib.delta_read_device_error.restype = _i32
lib.delta_status_string.argtypes = [_i32]
lib.delta_status_string.restype = ctypes.c_char_p


class DeltaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} (status {status})")
        self.status = status


def ptr(x) -> int | None:
    """Device address of a torch tensor, an int, or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def status_string(status: int) -> str:
    return lib.delta_status_string(status).decode()


def _check(status: int, where: str) -> int:
    if status != DELTA_OK:
        raise DeltaError(status, where)
    return status


def workspace_size(desc: DeltaDesc, batch: int, max_pages_per_seq: int) -> int:
    return lib.delta_workspace_size(ctypes.byref(desc), batch, max_pages_per_seq)


def workspace_size_reduce(desc: DeltaDesc, batch: int, max_pages_per_seq: int, reduce: int) -> int:
    return lib.delta_workspace_size_reduce(ctypes.byref(desc), batch, max_pages_per_seq, reduce)


def workspace_init(workspace, nbytes: int, stream: int = 0) -> None:
    _check(lib.delta_workspace_init(ptr(workspace), nbytes, stream), "delta_workspace_init")


def sel_capacity(sp: DeltaSelectParams, page_size: int = 16) -> int:
    return lib.delta_sel_capacity(ctypes.byref(sp), page_size)


def kv_append(desc, pt, k_new, v_new, k_pool, v_pool, stream: int = 0, check: bool = True) -> int:
    s = lib.delta_kv_append(ctypes.byref(desc), ctypes.byref(pt), ptr(k_new), ptr(v_new), ptr(k_pool),
                            ptr(v_pool), stream)
    return _check(s, "delta_kv_append") if check else s


def _ptr_array(xs):
    return (ctypes.c_void_p * len(xs))(*[ptr(x) for x in xs])


def kv_append_layers(desc, pt, k_new, v_new, k_pools, v_pools, stream: int = 0, check: bool = True) -> int:
    """k_new, v_new, k_pools, v_pools: sequences (one entry per layer) of device tensors or pointers."""
    n = len(k_pools)
    s = lib.delta_kv_append_layers(ctypes.byref(desc), ctypes.byref(pt), n, _ptr_array([k_new[l] for l in range(n)]),
                                   _ptr_array([v_new[l] for l in range(n)]), _ptr_array(list(k_pools)),
                                   _ptr_array(list(v_pools)), stream)
    return _check(s, "delta_kv_append_layers") if check else s


def full_attn(desc, pt, q, k_pool, v_pool, o, workspace, ws_bytes: int, stream: int = 0, check: bool = True) -> int:
    s = lib.delta_full_attn(ctypes.byref(desc), ctypes.byref(pt), ptr(q), ptr(k_pool), ptr(v_pool), ptr(o),
                            ptr(workspace), ws_bytes, stream)
    return _check(s, "delta_full_attn") if check else s


def full_attn_noalloc(desc, pt, q, k_pool, v_pool, o, stream: int = 0, check: bool = True) -> int:
    """delta_full_attn with the library's own fixed scratch instead of a caller workspace."""
    s = lib.delta_full_attn_noalloc(ctypes.byref(desc), ctypes.byref(pt), ptr(q), ptr(k_pool), ptr(v_pool), ptr(o),
                                    stream)
    return _check(s, "delta_full_attn_noalloc") if check else s


def select_attn(desc, pt, sp, q, k_pool, v_pool, o, sel_cnt, sel_pages, sel_stride: int, page_scores,
                workspace, ws_bytes: int, stream: int = 0, check: bool = True) -> int:
    s = lib.delta_select_attn(ctypes.byref(desc), ctypes.byref(pt), ctypes.byref(sp), ptr(q), ptr(k_pool),
                              ptr(v_pool), ptr(o), ptr(sel_cnt), ptr(sel_pages), sel_stride, ptr(page_scores),
                              ptr(workspace), ws_bytes, stream)
    return _check(s, "delta_select_attn") if check else s


def sparse_attn(desc, pt, sel_cnt, sel_pages, sel_stride: int, q, k_pool, v_pool, o, workspace, ws_bytes: int,
                stream: int = 0, check: bool = True) -> int:
    s = lib.delta_sparse_attn(ctypes.byref(desc), ctypes.byref(pt), ptr(sel_cnt), ptr(sel_pages), sel_stride,
                              ptr(q), ptr(k_pool), ptr(v_pool), ptr(o), ptr(workspace), ws_bytes, stream)
    return _check(s, "delta_sparse_attn") if check else s


def sparse_attn_settled(desc, pt, sel_cnt, sel_pages, sel_stride: int, q, k_pool, v_pool, o, workspace,
                        ws_bytes: int, stream: int = 0, check: bool = True) -> int:
    s = lib.delta_sparse_attn_settled(ctypes.byref(desc), ctypes.byref(pt), ptr(sel_cnt), ptr(sel_pages), sel_stride,
                                      ptr(q), ptr(k_pool), ptr(v_pool), ptr(o), ptr(workspace), ws_bytes, stream)
    return _check(s, "delta_sparse_attn_settled") if check else s


def layer_shift(pt, scores_a, scores_b, shift_out, stream: int = 0, check: bool = True) -> int:
    s = lib.delta_layer_shift(ctypes.byref(pt), ptr(scores_a), ptr(scores_b), ptr(shift_out), stream)
    return _check(s, "delta_layer_shift") if check else s


def choose_layers(shift, count: int, first: int = 2, min_gap: int = 2) -> list:
    """delta_choose_layers on a host sequence of per-layer shifts; returns the ascending layer ids."""
    vals = [float(x) for x in shift]
    arr = (ctypes.c_float * len(vals))(*vals)
    out = (_i32 * max(count, 1))()
    n = _i32(0)
    _check(lib.delta_choose_layers(arr, len(vals), count, first, min_gap, out, ctypes.byref(n)),
           "delta_choose_layers")
    return [int(out[i]) for i in range(n.value)]


def read_device_error(workspace, stream: int = 0) -> tuple:
    flags = _i32(0)
    s = lib.delta_read_device_error(ptr(workspace), ctypes.byref(flags), stream)
    return s, flags.value
