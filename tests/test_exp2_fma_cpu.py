"""The FMA-pipe exponential of the attention kernel (ptx.cuh, exp2_fma_pair), checked on
the CPU: its constants are read from the source and its steps emulated in float32
(round to the nearest integer by adding 1.5 * 2^23, the cubic in Horner form on the
remainder in [-1/2, 1/2], the integer added to the exponent field).  The weights it
produces are rounded to bf16 (relative error up to 2^-9) before P V, so its own error
must stay far below that; exactly representable powers of two must come out exact to
within the polynomial's error at f = 0."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _coefficients():
    src = open(os.path.join(ROOT, "vit_self_attention_b200", "csrc", "ptx.cuh")).read()
    body = src[src.index("void exp2_fma_pair("):]
    body = body[:body.index("\n}\n")]
    nums = [float(v) for v in re.findall(r"f32x2_pack\(([0-9.]+)f, \1f\)", body)
            if float(v) < 2.0]
    # Horner order in the source: c3, c2, then c1, then c0.
    assert len(nums) == 4, nums
    c3, c2, c1, c0 = nums
    assert "12582912.0f" in body  # 1.5 * 2^23
    assert "<< 23" in body
    return [np.float32(v) for v in (c0, c1, c2, c3)]


def _emulate(a):
    c0, c1, c2, c3 = _coefficients()
    magic = np.float32(12582912.0)
    ac = np.maximum(a.astype(np.float32), np.float32(-126.0))
    t = (ac + magic).astype(np.float32)
    r = (t - magic).astype(np.float32)
    f = (ac - r).astype(np.float32)
    q = (c3 * f + c2).astype(np.float32)
    q = (q * f + c1).astype(np.float32)
    q = (q * f + c0).astype(np.float32)
    bits = q.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32), f


def test_relative_error_over_the_argument_range():
    rng = np.random.default_rng(7)
    a = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001),
                        rng.uniform(-30.0, 8.0, 1_000_000)]).astype(np.float32)
    y, f = _emulate(a)
    assert float(np.abs(f).max()) <= 0.5
    ref = np.exp2(a.astype(np.float64))
    rel = np.abs(y.astype(np.float64) - ref) / ref
    assert float(rel.max()) < 1e-4, float(rel.max())
    assert float(rel.max()) < 2.0 ** -9 / 20  # far below P's bf16 rounding


def test_integers_masked_keys_and_clamp():
    y, _ = _emulate(np.arange(-120, 9, dtype=np.float32))
    ref = np.exp2(np.arange(-120, 9, dtype=np.float64))
    assert np.all(np.abs(y / ref - 1.0) < 1e-4)
    # Masked keys (-inf) and very negative arguments give the clamp's 2^-126 (about 1e-38):
    # positive, finite and negligible next to any unmasked weight (>= 2^-8 of the largest).
    y, _ = _emulate(np.array([-np.inf, -1e30, -127.5, -126.0], dtype=np.float32))
    assert np.all(np.isfinite(y)) and np.all(y > 0) and np.all(y < 2.0 ** -125)
