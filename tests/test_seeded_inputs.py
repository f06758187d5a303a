"""The seeded input generator: reproducible, counter-based, right distribution."""
import numpy as np
import torch

import seeded_inputs as si


def test_deterministic_and_seed_dependent():
    a = si.packed_qkv(2, 17, 3, 8, 5)
    b = si.packed_qkv(2, 17, 3, 8, 5)
    c = si.packed_qkv(2, 17, 3, 8, 6)
    assert a.shape == (2, 17, 3, 3, 8) and a.dtype == np.uint16
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c)


def test_counter_based_slices():
    """Any element range regenerates on its own (odd starts included)."""
    full = si.normals(123, 0, 1001)
    for start, count in [(0, 1), (1, 5), (7, 100), (500, 501)]:
        assert np.array_equal(si.normals(123, start, count), full[start:start + count])


def test_threaded_fill_matches_serial():
    a = si.packed_qkv(3, 97, 4, 64, 77, threads=1)
    b = si.packed_qkv(3, 97, 4, 64, 77, threads=4)
    assert np.array_equal(a, b)


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 7.0
    x[:4] = [0.0, -0.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8]  # ties to even
    ours = si.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = si.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_moments_and_slot_sigmas():
    c = si.SIGLIP_SO400M14_224PX_2VIEWS  # Q, K with variance 2; V with variance 1
    x = si.bf16_bits_to_f32(c.qkv(0)).astype(np.float64)
    q, k, v = x[:, :, 0], x[:, :, 1], x[:, :, 2]
    for arr, var in [(q, 2.0), (k, 2.0), (v, 1.0)]:
        assert abs(arr.mean()) < 0.02
        assert abs(arr.var() - var) < 0.03 * var
    y = si.bf16_bits_to_f32(si.VIT_B16_224PX_3VIEWS.qkv(0)).astype(np.float64)
    assert abs(y.var() - 1.0) < 0.02


def test_config_table():
    shapes = [(c.B, c.N, c.H, c.d) for c in si.WORKLOADS]
    assert shapes == [(1, 50, 12, 64), (3, 197, 12, 64), (3, 257, 16, 64), (2, 256, 16, 72),
                      (256, 577, 16, 64)]
    assert si.VIT_B16_112PX_1VIEW.scale == 0.125 and si.VIT_B16_112PX_1VIEW.seed(0) == 0
    assert [c.calls for c in si.WORKLOADS] == [1, 12, 24, 27, 1]
    assert abs(si.SIGLIP_SO400M14_224PX_2VIEWS.scale - 72 ** -0.5) < 1e-15
    assert si.VIT_L14_336PX_B256.flops() == 4 * 256 * 16 * 577 * 577 * 64
    seeds = {c.seed(i) for c in si.WORKLOADS for i in range(c.calls)}
    assert len(seeds) == sum(c.calls for c in si.WORKLOADS)
