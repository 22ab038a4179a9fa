"""The seeded input generator: determinism, distribution, rounding and workload structure."""
import numpy as np
import torch

from synth import configs as C
from synth import rng
from synth.case import Case


def test_splitmix64_reference_values():
    # splitmix64 seeded with 0: first outputs as published with the algorithm (Vigna's reference code).
    out = rng.bits(0, np.arange(3))
    assert [int(x) for x in out] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_generator_is_deterministic_and_pure():
    k = rng.stream_key(0, 2)
    a = rng.normal_block(k, rng.T_K, 3, 0, 1, np.arange(100), 128)
    b = rng.normal_block(k, rng.T_K, 3, 0, 1, np.arange(100), 128)
    assert np.array_equal(a, b)
    c = rng.normal_block(k, rng.T_K, 3, 0, 1, np.arange(40, 60), 128)
    assert np.array_equal(a[40:60], c)


def test_normal_moments_and_range():
    x = rng.normal_block(rng.stream_key(0, 9), rng.T_V, 0, 0, 0, np.arange(4096), 128).ravel()
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01
    assert np.abs(x).max() <= 2 * np.sqrt(3) + 1e-6


def test_bf16_rounding_matches_torch_nearest_even():
    x = rng.normal_block(rng.stream_key(1, 1), rng.T_K, 0, 0, 0, np.arange(512), 128).ravel()
    x = np.concatenate([x, np.float32([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8])])  # exact ties
    ours = rng.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_page_table_is_a_valid_shuffled_mapping():
    case = Case(C.QWEN7B_B8_VAR)
    ind, ptr = case.page_indices, case.page_indptr
    assert len(set(ind.tolist())) == len(ind)
    assert ind.min() >= 0 and ind.max() < case.num_phys_pages == 69905
    for b in range(8):
        assert ptr[b + 1] - ptr[b] == -(-case.n[b] // 16)
        assert 16384 <= case.n[b] <= 32768
    assert not np.array_equal(ind, np.sort(ind))


def test_planted_positions_follow_the_recipe():
    case = Case(C.QWEN7B_8K)
    cfg = case.cfg
    for g in range(cfg.num_kv_heads):
        prev = None
        for layer in range(6):
            pos = case.planted_positions(layer, 0, g)
            assert len(set(pos.tolist())) == 32
            assert pos.min() >= cfg.sink_tokens and pos.max() < case.n[0] - cfg.recency_tokens
            if prev is not None:
                assert len(set(pos.tolist()) & set(prev.tolist())) >= 26
            prev = pos


def test_planted_keys_raise_their_logits():
    case = Case(C.QWEN7B_8K)
    q = case.q(5)[0]
    K = case.kv_logical(rng.T_K, 5, 0, 2)
    pos = case.planted_positions(5, 0, 2)
    s = q[14:21] @ K.T / np.sqrt(128)
    other = np.setdiff1d(np.arange(K.shape[0]), pos)
    assert s[:, pos].mean() > s[:, other].mean() + 0.5


def test_drift_positions_shift_every_block():
    case = Case(C.DRIFT_48L)
    p0 = case.planted_positions(10, 3, 1, step=0)
    p1 = case.planted_positions(10, 3, 1, step=99)
    p2 = case.planted_positions(10, 3, 1, step=100)
    assert np.array_equal(p0, p1) and np.array_equal(p2, p0 + 256)
    last = case.planted_positions(10, 3, 1, step=999)
    assert last.max() < 16384 - 512


def test_host_c_generator_equals_numpy_generator_bit_for_bit():
    # synth/csrc/synth_host.c restates the generator in C for speed; it must give the same bits
    assert rng._host_lib() is not None, "libsynth_host.so is not built"
    r = np.random.default_rng(7)
    for dtype in ("bf16", "f32"):
        for _ in range(20):
            key = int(r.integers(0, 2 ** 63))
            t, l, b, h = int(r.integers(0, 4)), int(r.integers(0, 64)), int(r.integers(0, 64)), int(r.integers(0, 64))
            pos = r.integers(0, 1 << 20, size=int(r.integers(1, 50)))
            dim = int(r.choice([64, 128, 256, 7]))
            c = rng.normal_block_stored(key, t, l, b, h, pos, dim, dtype)
            ref = rng.round_to_dtype(rng.normal_block(key, t, l, b, h, pos, dim), dtype)
            assert np.array_equal(c.view(np.uint32), ref.view(np.uint32))
