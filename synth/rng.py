"""Counter-based random numbers shared by the oracle side and the GPU side.

This module holds no attention arithmetic.  It defines one pure function of an
integer counter, so any element of any synthetic tensor can be regenerated on
the host at any time, and a CUDA fill kernel (``synth/csrc/synth_fill.cu``)
produces bit-identical values on the device.

Definition (both sides implement exactly this):

* ``mix64(z)`` is the splitmix64 output finaliser (Steele, Lea, Flood,
  "Fast splittable pseudorandom number generators", OOPSLA 2014):
  ``z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27; z *= 0x94D049BB133111EB;
  z ^= z >> 31`` on unsigned 64-bit integers with wrap-around.
* ``bits(key, c) = mix64(key + (c + 1) * 0x9E3779B97F4A7C15)`` — the c-th
  output of a splitmix64 stream whose state starts at ``key``.
* ``normal(bits)``: the four 16-bit fields u0..u3 of the 64 bits are summed,
  ``S = u0+u1+u2+u3``; the value is ``float32(S - 131070) * float32(sqrt(3)/65536)``,
  one IEEE-754 single multiply rounded to nearest.  This is the Irwin-Hall
  sum of four uniforms standardised to mean 0, variance 1 (range +-3.464); it is
  exact integer arithmetic up to one correctly rounded multiply, so host and
  device agree bit for bit.
* ``bf16`` storage rounds the float32 value to nearest-even on its upper 16 bits.
"""
from __future__ import annotations

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
NORMAL_SCALE = np.float32(np.sqrt(3.0) / 65536.0)

# Tensor ids in the element counter.
T_K, T_V, T_Q, T_AUX = 0, 1, 2, 3

# Bit layout of an element counter: d (8) | pos (20) | head (6) | b (6) | layer (6) | tensor.
D_BITS, POS_BITS, HEAD_BITS, B_BITS, LAYER_BITS = 8, 20, 6, 6, 6
MAX_D = 1 << D_BITS
MAX_POS = 1 << POS_BITS


def mix64(z: np.ndarray) -> np.ndarray:
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, cfg_id: int) -> int:
    """Start state of the stream for one (seed, workload) pair."""
    z = np.uint64((seed * 0x100000001B3 + cfg_id * 0x9E3779B1 + 0x5851F42D4C957F2D) & 0xFFFFFFFFFFFFFFFF)
    return int(mix64(z))


def bits(key: int, counter: np.ndarray) -> np.ndarray:
    c = np.asarray(counter, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + (c + np.uint64(1)) * GOLDEN
    return mix64(z)


def normal_from_bits(b: np.ndarray) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint64)
    m = np.uint64(0xFFFF)
    s = ((b & m) + ((b >> np.uint64(16)) & m) + ((b >> np.uint64(32)) & m) + (b >> np.uint64(48))).astype(np.int64)
    return (s - 131070).astype(np.float32) * NORMAL_SCALE


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest-even); returns the 16-bit patterns as uint16."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    return (u >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_to_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    """Value as stored in the given dtype, returned as float32."""
    x = np.asarray(x, dtype=np.float32)
    if dtype == "bf16":
        return bf16_bits_to_f32(f32_to_bf16_bits(x))
    if dtype == "f32":
        return x
    raise ValueError(dtype)


def element_counter(tensor: int, layer: int, b: int, head: int, pos, d) -> np.ndarray:
    """Counter of element (tensor, layer, b, head, pos, d); pos and d broadcast."""
    assert 0 <= layer < (1 << LAYER_BITS) and 0 <= b < (1 << B_BITS) and 0 <= head < (1 << HEAD_BITS)
    hi = ((tensor << LAYER_BITS | layer) << B_BITS | b) << HEAD_BITS | head
    pos = np.asarray(pos, dtype=np.uint64)
    d = np.asarray(d, dtype=np.uint64)
    return (np.uint64(hi) << np.uint64(POS_BITS + D_BITS)) | (pos << np.uint64(D_BITS)) | d


def normal_block(key: int, tensor: int, layer: int, b: int, head: int, pos: np.ndarray, dim: int) -> np.ndarray:
    """[len(pos), dim] float32 generator values for one (tensor, layer, b, head)."""
    pos = np.asarray(pos, dtype=np.uint64).reshape(-1, 1)
    d = np.arange(dim, dtype=np.uint64).reshape(1, -1)
    return normal_from_bits(bits(key, element_counter(tensor, layer, b, head, pos, d)))


_HOST_LIB = None


def _host_lib():
    """The C copy of this generator (synth/csrc/synth_host.c), or None when it is not built."""
    global _HOST_LIB
    if _HOST_LIB is None:
        import ctypes
        import os
        path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsynth_host.so")
        if not os.path.exists(path):
            _HOST_LIB = False
        else:
            lib = ctypes.CDLL(path)
            lib.synth_host_normal_block.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                    ctypes.c_int, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                                    ctypes.c_float, ctypes.c_int, ctypes.c_void_p]
            lib.synth_host_normal_block.restype = ctypes.c_int
            _HOST_LIB = lib
    return _HOST_LIB or None


def normal_block_stored(key: int, tensor: int, layer: int, b: int, head: int, pos, dim: int, dtype: str,
                        use_c: bool = True) -> np.ndarray:
    """round_to_dtype(normal_block(...), dtype): the stored values, [len(pos), dim] float32.

    Uses the C copy of the generator when it is built (same bits, much faster), else numpy.
    """
    lib = _host_lib() if use_c else None
    p = np.ascontiguousarray(np.asarray(pos, dtype=np.int64).reshape(-1))
    if lib is None or dtype not in ("bf16", "f32") or (p.size and (p.min() < 0 or p.max() >= MAX_POS)):
        # (positions outside the counter field keep numpy's wrap-around semantics)
        return round_to_dtype(normal_block(key, tensor, layer, b, head, p, dim), dtype)
    out = np.empty((p.size, dim), dtype=np.float32)
    r = lib.synth_host_normal_block(key, tensor, layer, b, head, p.ctypes.data, p.size, dim, float(NORMAL_SCALE),
                                    1 if dtype == "bf16" else 0, out.ctypes.data)
    if r != 0:
        raise ValueError(f"synth_host_normal_block failed ({r})")
    return out


# Salts of the auxiliary draws (host-side choices).  An aux counter is salt << 20 | index.
SALT_PAGE_PERM = 1
SALT_CONTEXT = 2
SALT_PLANT_KEEP = 1 << 18     # + (layer*64 + b)*64 + g
SALT_PLANT_DRAW = 2 << 18     # + (layer*64 + b)*64 + g
AUX_INDEX_BITS = 20


def aux_counter(salt: int, index) -> np.ndarray:
    assert 0 <= salt < (1 << 26)
    idx = np.asarray(index, dtype=np.uint64)
    return (np.uint64(salt) << np.uint64(AUX_INDEX_BITS)) + idx


def uniform_u64(key: int, counters: np.ndarray) -> np.ndarray:
    """Raw 64-bit draws on the auxiliary tensor id (host-side choices: lengths, shuffles, positions)."""
    c = np.asarray(counters, dtype=np.uint64) | (np.uint64(T_AUX) << np.uint64(LAYER_BITS + B_BITS + HEAD_BITS + POS_BITS + D_BITS))
    return bits(key, c)


def randint(key: int, counters: np.ndarray, low: int, high: int) -> np.ndarray:
    """Integers in [low, high) from aux draws (multiply-high reduction of the top 32 bits)."""
    span = high - low
    assert span > 0
    u = uniform_u64(key, counters) >> np.uint64(32)
    with np.errstate(over="ignore"):
        return (low + ((u * np.uint64(span)) >> np.uint64(32))).astype(np.int64)


def permutation(key: int, salt: int, n: int) -> np.ndarray:
    """A permutation of range(n): stable argsort of aux draws."""
    assert n <= (1 << AUX_INDEX_BITS)
    return np.argsort(uniform_u64(key, aux_counter(salt, np.arange(n))), kind="stable").astype(np.int64)
