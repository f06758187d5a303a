"""The allocation-free linear entry point (fixed device workspace) against the
regular one.  Named to be collected last; it also passes when run alone.

Some callers cannot allocate device memory (code recorded into a stream
capture, or a runtime that owns all device memory); vla_linear_fwd_static
serves them with a fixed device array as its split-K scratch.  Both entry
points make the same choices (tile width, K split) when the regular one is
given a workspace of the same size, so the outputs must be identical bytes.
Two calls in a row check that the shared static array carries nothing over
from one call to the next (its arrival counters are cleared by every call).
"""
import math

import numpy as np
import pytest
import torch

import seeded_inputs as si
from gpu_helpers import needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _case(M, K, N, seed, residual):
    x = _dev(si.normal_bf16(seed, (M, K)))
    w = _dev(si.normal_bf16(seed + 1, (N, K), 0.0, 1.0 / math.sqrt(K)))
    b = _dev(si.normal_bf16(seed + 2, (N,), 0.0, 0.1))
    r = _dev(si.normal_bf16(seed + 3, (M, N))) if residual else None
    return x, w, b, r


def test_static_workspace_linear_matches_regular_entry_point():
    import vit_self_attention_b200 as vab
    nbytes = vab.vla_linear_static_workspace_bytes()
    assert nbytes == 8 << 20
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    cases = [(64, 16384, 256, 1000, True),    # few tiles and a long K: split K
             (64, 16384, 256, 1500, True),    # the same shape again: the array is reused
             (771, 1024, 1024, 2000, True)]   # output linear + residual, ViT-L/14 x 3 views
    for M, K, N, seed, residual in cases:      # two calls in a row
        x, w, b, r = _case(M, K, N, seed, residual)
        y_static = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        y_regular = torch.empty_like(y_static)
        assert vab.vla_linear_fwd_static(x, w, b, r, y_static, M, K, N) == vab.OK
        assert vab.vla_linear_fwd(x, w, b, r, y_regular, M, K, N, ws, nbytes) == vab.OK
        torch.cuda.synchronize()
        assert torch.isfinite(y_static.float()).all()
        assert torch.equal(y_static, y_regular), f"M={M} K={K} N={N}"


def test_static_workspace_linear_warm_calls_allocate_nothing():
    """After one warm call (which does the per-device set-up), further calls change
    neither torch's allocated bytes nor the device's free memory."""
    import vit_self_attention_b200 as vab
    from cuda.bindings import runtime as cudart
    M, K, N = 64, 16384, 256  # a split-K shape: the fixed array holds its partial sums
    x, w, b, r = _case(M, K, N, 3000, True)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    assert vab.vla_linear_fwd_static(x, w, b, r, y, M, K, N) == vab.OK
    torch.cuda.synchronize()
    alloc0 = torch.cuda.memory_allocated()
    err, free0, _ = cudart.cudaMemGetInfo()
    assert int(err) == 0
    for _ in range(5):
        assert vab.vla_linear_fwd_static(x, w, b, r, y, M, K, N) == vab.OK
    torch.cuda.synchronize()
    err, free1, _ = cudart.cudaMemGetInfo()
    assert int(err) == 0
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 == free0, f"device free memory changed by {free0 - free1} bytes"
