"""Checks that pin the fp64 oracle to facts fixed outside itself.

Each ``pin_*`` function takes an ``oracle.OracleLib`` and raises
``AssertionError`` when the library disagrees with a closed form, a worked
example, an invariant of the attention definition, a pure-Python brute force
or PyTorch's own CPU scaled-dot-product attention.  ``test_oracle_pins`` runs
them against the real oracle; ``test_oracle_mutants`` runs them against
deliberately broken copies of the oracle source and requires each copy to fail
at least one pin.

Definitions being pinned (multi-head self-attention of the ViT block, as in the
Pi0 Flash Attention tutorial, sections 1 and 3.2):
``o[b,i,h,:] = sum_j softmax_j(scale * q[b,i,h,:] . k[b,j,h,:]) v[b,j,h,:]``;
and the layers around it: LayerNorm over the last dimension and the linear layer
``x @ w.T + bias (+ res)`` (FluxVLA inference-acceleration page: norm fusion,
and section 3's cublasLt fused GEMM + bias (+ residual)).
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

import seeded_inputs as si

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "closed_forms.json")


def _rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} != {b.shape}"
    assert np.all(np.isfinite(a)), f"{what}: non-finite values"
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol, f"{what}: max |err| {err:.3e} > {tol:.1e}"


def pin_golden_closed_forms(lib):
    """Hand-derived worked examples (tests/golden/closed_forms.json)."""
    with open(GOLDEN) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        k = np.array(c["k"], dtype=np.float64)
        v = np.array(c["v"], dtype=np.float64)
        q = np.array(c["q"], dtype=np.float64)
        if q.shape[0] < k.shape[0]:
            q = np.repeat(q, k.shape[0], axis=0)[: k.shape[0]]
        want = np.array(c["o"], dtype=np.float64)
        if want.shape[0] < k.shape[0]:
            want = np.repeat(want, k.shape[0], axis=0)[: k.shape[0]]
        o = lib.attention_f64(q[None, :, None, :], k[None, :, None, :], v[None, :, None, :],
                              c["scale"])
        _close(o[0, :, 0, :], want, c["tol"], c["name"])


def pin_single_token(lib):
    """N = 1: the only weight is 1, so o equals the value row exactly."""
    r = _rng(1)
    q, k, v = (r.standard_normal((3, 1, 4, 72)) for _ in range(3))
    o = lib.attention_f64(q, k, v, 0.3)
    _close(o, v, 0.0, "N=1 -> o == v")


def pin_two_tokens_sigmoid(lib):
    """N = 2: o_i = sigmoid(s_i0 - s_i1) v_0 + sigmoid(s_i1 - s_i0) v_1."""
    r = _rng(2)
    q, k, v = (r.standard_normal((2, 2, 3, 8)) for _ in range(3))
    scale = 0.7
    o = lib.attention_f64(q, k, v, scale)
    want = np.empty_like(o)
    for b in range(2):
        for h in range(3):
            for i in range(2):
                s0 = scale * float(np.dot(q[b, i, h], k[b, 0, h]))
                s1 = scale * float(np.dot(q[b, i, h], k[b, 1, h]))
                w0 = 1.0 / (1.0 + math.exp(s1 - s0))
                w1 = 1.0 / (1.0 + math.exp(s0 - s1))
                want[b, i, h] = w0 * v[b, 0, h] + w1 * v[b, 1, h]
    _close(o, want, 1e-14, "N=2 sigmoid closed form")


def pin_identical_values(lib):
    """Every value row equal to one vector u: the weights sum to 1, so o rows equal u."""
    r = _rng(3)
    B, N, H, d = 2, 37, 3, 16
    q, k = r.standard_normal((B, N, H, d)), r.standard_normal((B, N, H, d))
    u = r.standard_normal((B, 1, H, d))
    v = np.broadcast_to(u, (B, N, H, d)).copy()
    o = lib.attention_f64(q, k, v, 1.3)
    _close(o, v, 1e-13, "identical V rows")


def pin_zero_query_mean(lib):
    """Q = 0: all logits are 0, so o is the plain mean of the value rows."""
    r = _rng(4)
    B, N, H, d = 2, 29, 2, 8
    q = np.zeros((B, N, H, d))
    k, v = r.standard_normal((B, N, H, d)), r.standard_normal((B, N, H, d))
    o = lib.attention_f64(q, k, v, 0.125)
    want = np.broadcast_to(v.mean(axis=1, keepdims=True), v.shape)
    _close(o, want, 1e-14, "Q=0 -> mean of V")


def pin_probs_rows(lib):
    """Softmax rows are non-negative, sum to 1, and are proportional to exp(logit)."""
    r = _rng(5)
    B, N, H, d = 2, 19, 2, 8
    q, k = r.standard_normal((B, N, H, d)), r.standard_normal((B, N, H, d))
    scale = 0.9
    p = lib.probs_f64(q, k, scale)
    assert np.all(p >= 0.0), "negative softmax weight"
    _close(p.sum(axis=-1), np.ones((B, H, N)), 1e-14, "softmax rows sum to 1")
    s = scale * np.einsum("bihc,bjhc->bhij", q, k)
    # log-ratio test: log p_ij - log p_i0 == s_ij - s_i0
    _close(np.log(p) - np.log(p[..., :1]), s - s[..., :1], 1e-12, "softmax log-ratios")


def pin_joint_kv_permutation(lib):
    """Permuting the key and value rows by the same permutation leaves o unchanged;
    permuting the query rows permutes the output rows."""
    r = _rng(6)
    B, N, H, d = 2, 23, 2, 8
    q, k, v = (r.standard_normal((B, N, H, d)) for _ in range(3))
    o = lib.attention_f64(q, k, v, 0.5)
    perm = r.permutation(N)
    o2 = lib.attention_f64(q, k[:, perm], v[:, perm], 0.5)
    _close(o2, o, 1e-13, "joint K/V permutation")
    o3 = lib.attention_f64(q[:, perm], k, v, 0.5)
    _close(o3, o[:, perm], 1e-13, "query permutation equivariance")
    # permuting only V must change the result (a K/V mix-up would hide here)
    o4 = lib.attention_f64(q, k, v[:, perm], 0.5)
    assert np.max(np.abs(o4 - o)) > 1e-3, "o does not depend on which value row goes with which key"


def pin_head_batch_independence(lib):
    """Each (b, h) slice is computed on its own: it equals a B = H = 1 call on that slice."""
    r = _rng(7)
    B, N, H, d = 3, 21, 4, 8
    q, k, v = (r.standard_normal((B, N, H, d)) for _ in range(3))
    o = lib.attention_f64(q, k, v, 0.6)
    for b in range(B):
        for h in range(H):
            sl = (slice(b, b + 1), slice(None), slice(h, h + 1), slice(None))
            oh = lib.attention_f64(q[sl], k[sl], v[sl], 0.6)
            _close(oh, o[sl], 0.0, f"slice b={b} h={h}")


def pin_hard_attention(lib):
    """A large scale with a unique maximising key gives that key's value row."""
    r = _rng(8)
    B, N, H, d = 1, 40, 2, 8
    q, k, v = (r.standard_normal((B, N, H, d)) for _ in range(3))
    scale = 1.0e4
    o = lib.attention_f64(q, k, v, scale)
    s = np.einsum("bihc,bjhc->bhij", q, k)
    top = np.argsort(s, axis=-1)
    for b in range(B):
        for h in range(H):
            for i in range(N):
                j1, j2 = top[b, h, i, -1], top[b, h, i, -2]
                gap = scale * (s[b, h, i, j1] - s[b, h, i, j2])
                if gap > 60.0:  # every other weight below e^-60
                    _close(o[b, i, h], v[b, j1, h], 1e-15, f"hard attention row {i}")


def pin_brute_force_python(lib):
    """Pure-Python loops over a tiny problem, written from the definition."""
    r = _rng(9)
    B, N, H, d = 2, 5, 2, 3
    q, k, v = (r.standard_normal((B, N, H, d)) for _ in range(3))
    scale = 0.8
    o = lib.attention_f64(q, k, v, scale)
    want = np.zeros_like(o)
    for b in range(B):
        for h in range(H):
            for i in range(N):
                logits = [scale * sum(q[b, i, h, c] * k[b, j, h, c] for c in range(d))
                          for j in range(N)]
                w = [math.exp(x) for x in logits]
                tot = math.fsum(w)
                for c in range(d):
                    want[b, i, h, c] = math.fsum(w[j] * v[b, j, h, c] for j in range(N)) / tot
    _close(o, want, 1e-14, "pure-Python brute force")


def _torch_sdpa(q, k, v, scale):
    import torch
    import torch.nn.functional as F
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).permute(0, 2, 1, 3)  # [B,H,N,d]
    o = F.scaled_dot_product_attention(t(q), t(k), t(v), scale=scale)
    return o.permute(0, 2, 1, 3).contiguous().numpy()


def _widen(bits):
    return si.bf16_bits_to_f32(bits).astype(np.float64)


def pin_torch_sdpa_workloads(lib, workloads=si.ENCODER_WORKLOADS):
    """PyTorch's CPU scaled_dot_product_attention in fp64 on the seeded encoder workload
    inputs, sliced from the packed buffer by numpy (independently of the oracle's own
    slicing)."""
    for c in workloads:
        bits = c.qkv(0)
        x = _widen(bits)
        q, k, v = x[:, :, 0], x[:, :, 1], x[:, :, 2]
        want = _torch_sdpa(q, k, v, c.scale)
        got = lib.attention_packed_bf16(bits, c.scale)
        _close(got, want, 1e-12, f"{c.name} vs torch SDPA fp64")
        got2 = lib.attention_f64(q, k, v, c.scale)
        _close(got2, want, 1e-12, f"{c.name} fp64 entry vs torch SDPA fp64")


def pin_torch_sdpa_large_slice(lib):
    """One image of the 336px ViT-L/14 shape (N = 577, H = 16, d = 64) against torch SDPA."""
    c = si.VIT_L14_336PX_B256
    bits = si.packed_qkv(1, c.N, c.H, c.d, c.seed(0))
    x = _widen(bits)
    want = _torch_sdpa(x[:, :, 0], x[:, :, 1], x[:, :, 2], c.scale)
    got = lib.attention_packed_bf16(bits, c.scale)
    _close(got, want, 1e-12, "N=577 slice vs torch SDPA fp64")


def pin_d72_zero_padding(lib):
    """Zero channels appended to q, k and v (72 -> 80) change neither the logits nor the
    first 72 output channels, provided the scale stays 1/sqrt(72)."""
    r = _rng(10)
    B, N, H = 2, 33, 2
    q, k, v = (r.standard_normal((B, N, H, 72)) for _ in range(3))
    scale = 1.0 / math.sqrt(72.0)
    o = lib.attention_f64(q, k, v, scale)
    pad = lambda a: np.concatenate([a, np.zeros((B, N, H, 8))], axis=-1)
    o80 = lib.attention_f64(pad(q), pad(k), pad(v), scale)
    _close(o80[..., :72], o, 1e-15, "72 -> 80 zero padding")
    _close(o80[..., 72:], np.zeros((B, N, H, 8)), 0.0, "padded channels stay zero")


def pin_rows_entry(lib):
    """The sampled-rows entry returns exactly the full computation's rows."""
    c = si.VIT_L14_224PX_3VIEWS
    bits = c.qkv(3)
    full = lib.attention_packed_bf16(bits, c.scale)
    rows = [(0, 0, 0), (2, 15, 256), (1, 7, 128), (2, 3, 1)]
    got = lib.attention_rows_packed_bf16(bits, c.scale, rows)
    for r_, (b, h, n) in enumerate(rows):
        _close(got[r_], full[b, n, h], 0.0, f"row {(b, h, n)}")


# --------------------------------------------------------------- LayerNorm
# y[m,i] = (x[m,i] - mean_m) / sqrt(var_m + eps) * gamma[i] + beta[i], biased variance
# ("FluxVLA docs, inference acceleration", Triton fused kernels: norm fusion).

def _bits(a):
    """Exact bf16 bit patterns of values that bf16 represents exactly."""
    a = np.asarray(a, dtype=np.float32)
    bits = si.f32_to_bf16_bits(a)
    assert np.array_equal(si.bf16_bits_to_f32(bits), a), "value not exact in bf16"
    return bits


def _bf16(a):
    return si.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def pin_layernorm_closed_forms(lib):
    """Constant rows give beta; a row of +a / -a gives +-a/sqrt(a^2 + eps) * gamma + beta;
    with gamma = 1, beta = 0 every row has mean 0 and variance var / (var + eps)."""
    W = 12
    gamma = _bf16(np.linspace(0.5, 2.0, W))
    beta = _bf16(np.linspace(-1.0, 1.0, W))
    x = _bits(np.full((3, W), [[2.0], [-7.5], [0.0]]))
    y = lib.layernorm_bf16(x, gamma, beta, 1e-6)
    _close(y, np.broadcast_to(si.bf16_bits_to_f32(beta), (3, W)), 0.0, "constant rows -> beta")
    a, eps = 3.0, 0.25
    row = np.array([a if i % 2 == 0 else -a for i in range(W)])
    y = lib.layernorm_bf16(_bits(row[None]), gamma, beta, eps)[0]
    want = row / math.sqrt(a * a + eps) * si.bf16_bits_to_f32(gamma) + si.bf16_bits_to_f32(beta)
    _close(y, want, 1e-12, "two-valued row")
    one, zero = _bits(np.ones(64)), _bits(np.zeros(64))
    x = _bf16(_rng(3).normal(0.4, 1.7, size=(5, 64)))
    eps = 0.5
    y = lib.layernorm_bf16(x, one, zero, eps)
    xv = si.bf16_bits_to_f32(x).astype(np.float64)
    var = xv.var(axis=1)
    _close(y.mean(axis=1), np.zeros(5), 1e-12, "output mean")
    _close(y.var(axis=1), var / (var + eps), 1e-12, "output variance")


def pin_layernorm_shift_invariance(lib):
    """With eps = 0 the result ignores a constant shift and a positive scale of the row
    (values chosen exactly representable after the shift and scale)."""
    W = 32
    gamma = _bf16(_rng(4).normal(size=W))
    beta = _bf16(_rng(5).normal(size=W))
    base = _rng(6).integers(-40, 40, size=(4, W)).astype(np.float64)
    y0 = lib.layernorm_bf16(_bits(base), gamma, beta, 0.0)
    y1 = lib.layernorm_bf16(_bits(base + 24.0), gamma, beta, 0.0)
    y2 = lib.layernorm_bf16(_bits(base * 4.0), gamma, beta, 0.0)
    _close(y1, y0, 1e-12, "shift")
    _close(y2, y0, 1e-12, "scale")


def pin_layernorm_brute_force_and_torch(lib):
    """Pure-Python loops on tiny rows, and torch's fp64 layer_norm on a ViT-width batch."""
    import torch
    W, M, eps = 7, 3, 1e-5
    x = _bf16(_rng(7).normal(size=(M, W)))
    g = _bf16(_rng(8).normal(size=W))
    b = _bf16(_rng(9).normal(size=W))
    xv, gv, bv = (si.bf16_bits_to_f32(t).astype(float).tolist() for t in (x, g, b))
    want = []
    for r in xv:
        mu = sum(r) / W
        var = sum((v - mu) ** 2 for v in r) / W
        want.append([(r[i] - mu) / math.sqrt(var + eps) * gv[i] + bv[i] for i in range(W)])
    _close(lib.layernorm_bf16(x, g, b, eps), np.array(want), 1e-12, "brute-force LayerNorm")
    W, M = 768, 40
    x = _bf16(_rng(10).normal(0.1, 1.3, size=(M, W)))
    g = _bf16(_rng(11).normal(1.0, 0.2, size=W))
    b = _bf16(_rng(12).normal(0.0, 0.2, size=W))
    tw = lambda t: torch.from_numpy(si.bf16_bits_to_f32(t).astype(np.float64))
    want = torch.nn.functional.layer_norm(tw(x), (W,), tw(g), tw(b), 1e-6).numpy()
    _close(lib.layernorm_bf16(x, g, b, 1e-6), want, 1e-10, "torch layer_norm fp64")


# ------------------------------------------------------------------ linear
# y[m,n] = sum_k x[m,k] w[n,k] + bias[n] + res[m,n]  (same page, section 3: cublasLt
# fused GEMM + bias (+ residual); the Pi0 tutorial's qkv linear feeds attention).

def pin_linear_closed_forms(lib):
    """Identity weights return x + bias, zero weights return bias, a rank-1 weight
    u v^T returns (x . v) u + bias, and a residual is added once."""
    K = 16
    x = _bf16(_rng(13).normal(size=(6, K)))
    xv = si.bf16_bits_to_f32(x).astype(np.float64)
    bias = _bf16(_rng(14).normal(size=K))
    bv = si.bf16_bits_to_f32(bias).astype(np.float64)
    _close(lib.linear_bf16(x, _bits(np.eye(K)), bias), xv + bv, 1e-12, "identity weight")
    _close(lib.linear_bf16(x, _bits(np.zeros((5, K))), bias[:5]), np.broadcast_to(bv[:5], (6, 5)),
           0.0, "zero weight")
    u = np.array([1.0, -2.0, 0.5, 4.0, 0.25])
    v = _rng(15).integers(-3, 4, size=K).astype(np.float64)
    w = _bits(np.outer(u, v))
    _close(lib.linear_bf16(x, w), np.outer(xv @ v, u), 1e-12, "rank-1 weight")
    res = _bf16(_rng(16).normal(size=(6, 5)))
    rv = si.bf16_bits_to_f32(res).astype(np.float64)
    w = _bf16(_rng(17).normal(size=(5, K)))
    _close(lib.linear_bf16(x, w, bias[:5], res) - lib.linear_bf16(x, w, bias[:5]), rv, 1e-12,
           "residual")


def pin_linear_permutation_and_linearity(lib):
    """A permutation weight permutes the input features; the map is linear in x."""
    K = 24
    perm = _rng(18).permutation(K)
    P = np.zeros((K, K))
    P[np.arange(K), perm] = 1.0
    x = _bf16(_rng(19).normal(size=(3, K)))
    xv = si.bf16_bits_to_f32(x).astype(np.float64)
    _close(lib.linear_bf16(x, _bits(P)), xv[:, perm], 0.0, "permutation weight")
    w = _bf16(_rng(20).normal(size=(9, K)))
    a = _rng(21).integers(-8, 8, size=(4, K)).astype(np.float64)
    b = _rng(22).integers(-8, 8, size=(4, K)).astype(np.float64)
    _close(lib.linear_bf16(_bits(a + b), w),
           lib.linear_bf16(_bits(a), w) + lib.linear_bf16(_bits(b), w), 1e-9, "linearity")


def pin_linear_brute_force_and_torch(lib):
    """Pure-Python loops on a tiny case (weights [N, K] as nn.Linear stores them), and
    torch's fp64 addmm on the ViT-B/16 qkv shape."""
    import torch
    M, K, N = 3, 5, 4
    x = _bf16(_rng(23).normal(size=(M, K)))
    w = _bf16(_rng(24).normal(size=(N, K)))
    b = _bf16(_rng(25).normal(size=N))
    xv, wv, bv = (si.bf16_bits_to_f32(t).astype(float).tolist() for t in (x, w, b))
    want = [[sum(xv[m][k] * wv[n][k] for k in range(K)) + bv[n] for n in range(N)]
            for m in range(M)]
    _close(lib.linear_bf16(x, w, b), np.array(want), 1e-12, "brute-force linear")
    M, K, N = 50, 768, 2304
    x = _bf16(_rng(26).normal(size=(M, K)))
    w = _bf16(_rng(27).normal(size=(N, K)) / math.sqrt(K))
    b = _bf16(_rng(28).normal(size=N))
    tw = lambda t: torch.from_numpy(si.bf16_bits_to_f32(t).astype(np.float64))
    want = torch.addmm(tw(b), tw(x), tw(w).T).numpy()
    _close(lib.linear_bf16(x, w, b), want, 1e-10, "torch addmm fp64")


# ------------------------------------------------------------ bf16 rounding
# Round to nearest, ties to even, of the residual stream's sum (the fused residual
# add + LayerNorm stores s = x + r in bf16).

def pin_round_bf16_ties_and_torch(lib):
    """Hand-worked ties and edges, then torch's float32 -> bfloat16 conversion (round to
    nearest even) on random float32 values, subnormals and ties included."""
    import torch
    cases = [(1.0, 0x3F80), (1.0 + 2.0 ** -8, 0x3F80),           # tie -> even (down)
             (1.0 + 3 * 2.0 ** -8, 0x3F82),                         # tie -> even (up)
             (1.0 + 2.0 ** -8 + 2.0 ** -30, 0x3F81),                # just above a tie
             (-3.0, 0xC040), (0.0, 0x0000), (-0.0, 0x8000),
             (2.0 ** -133, 0x0001), (1.5 * 2.0 ** -133, 0x0002),    # subnormal tie -> even
             (2.0 ** -134, 0x0000),                                 # subnormal tie -> zero
             (255.5 * 2.0 ** 120, 0x7F80), (255.25 * 2.0 ** 120, 0x7F7F)]
    got = lib.round_bf16(np.array([v for v, _ in cases]))
    for (v, want), g in zip(cases, got):
        assert int(g) == want, f"round_bf16({v!r}) = {int(g):#06x}, want {want:#06x}"
    rng = _rng(40)
    v = rng.normal(size=4000).astype(np.float32) * np.float32(3.0)
    ties = (_bf16(rng.normal(size=500)).astype(np.uint32) << 16) | np.uint32(0x8000)
    tiny = rng.normal(size=500).astype(np.float32) * np.float32(1e-39)
    v = np.concatenate([v, ties.view(np.float32), tiny])
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = lib.round_bf16(v.astype(np.float64))
    assert np.array_equal(got, want), f"{int((got != want).sum())} roundings differ from torch"


# ------------------------------------------------- residual add + LayerNorm
# s = bf16(x + r), y = LayerNorm(s)  ("FluxVLA docs, inference acceleration", Triton
# fused kernels: residual add + LayerNorm in one kernel).

def pin_add_layernorm_reductions(lib):
    """r = 0 gives s = x and y = LayerNorm(x); sums that bf16 holds exactly are exact;
    the add is symmetric; torch's bf16 add gives the same stream bits."""
    import torch
    W = 48
    x = _bf16(_rng(41).normal(size=(5, W)))
    g = _bf16(_rng(42).normal(1.0, 0.3, size=W))
    b = _bf16(_rng(43).normal(0.0, 0.3, size=W))
    s, y = lib.add_layernorm_bf16(x, _bits(np.zeros((5, W))), g, b, 1e-6)
    assert np.array_equal(s, x), "r = 0 must leave the stream unchanged"
    _close(y, lib.layernorm_bf16(x, g, b, 1e-6), 0.0, "r = 0 reduces to LayerNorm")
    xi = _rng(44).integers(-60, 60, size=(3, W)).astype(np.float64)
    ri = _rng(45).integers(-60, 60, size=(3, W)).astype(np.float64)
    s, _ = lib.add_layernorm_bf16(_bits(xi), _bits(ri), g, b, 1e-6)
    assert np.array_equal(s, _bits(xi + ri)), "exact integer sums"
    r = _bf16(_rng(46).normal(0.0, 4.0, size=(5, W)))
    s1, y1 = lib.add_layernorm_bf16(x, r, g, b, 1e-5)
    s2, y2 = lib.add_layernorm_bf16(r, x, g, b, 1e-5)
    assert np.array_equal(s1, s2)
    _close(y1, y2, 0.0, "symmetric add")
    tx = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16)
    tr = torch.from_numpy(r.view(np.int16)).view(torch.bfloat16)
    want = (tx + tr).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(s1, want), "stream bits differ from torch's bf16 add"


def pin_add_layernorm_torch(lib):
    """torch: the bf16 residual add, then fp64 layer_norm of the stored stream, at the
    ViT-L width."""
    import torch
    M, W = 30, 1024
    x = _bf16(_rng(47).normal(0.2, 1.5, size=(M, W)))
    r = _bf16(_rng(48).normal(-0.1, 0.8, size=(M, W)))
    g = _bf16(_rng(49).normal(1.0, 0.2, size=W))
    b = _bf16(_rng(50).normal(0.0, 0.2, size=W))
    tb = lambda t: torch.from_numpy(t.view(np.int16)).view(torch.bfloat16)
    stream = (tb(x) + tb(r)).double()
    want = torch.nn.functional.layer_norm(stream, (W,), tb(g).double(), tb(b).double(), 1e-6)
    s, y = lib.add_layernorm_bf16(x, r, g, b, 1e-6)
    _close(y, want.numpy(), 1e-10, "torch add + layer_norm fp64")


# --------------------------------------------------------- linear + GELU
# y = gelu(x @ w.T + bias), tanh form (same page, same section: matrix multiply with
# bias and activation fused).

def pin_linear_gelu_torch_and_erf(lib):
    """torch's fp64 tanh GELU after addmm; within the tanh form's published gap
    (< 5e-4) of the exact x Phi(x), and measurably not the exact form."""
    import torch
    from scipy.special import erf
    M, K, N = 40, 1152, 512
    x = _bf16(_rng(51).normal(size=(M, K)))
    w = _bf16(_rng(52).normal(size=(N, K)) * 2.0 / math.sqrt(K))
    b = _bf16(_rng(53).normal(size=N))
    tw = lambda t: torch.from_numpy(si.bf16_bits_to_f32(t).astype(np.float64))
    pre = torch.addmm(tw(b), tw(x), tw(w).T)
    want = torch.nn.functional.gelu(pre, approximate="tanh").numpy()
    got = lib.linear_gelu_bf16(x, w, b)
    _close(got, want, 1e-12, "torch gelu(tanh) fp64")
    a = pre.numpy()
    exact = 0.5 * a * (1.0 + erf(a / math.sqrt(2.0)))
    gap = np.abs(got - exact).max()
    assert gap < 5e-4, f"tanh GELU {gap} away from the exact form"
    assert gap > 1e-4, "this is the exact (erf) GELU, not the tanh form"


def pin_linear_gelu_closed_forms(lib):
    """gelu(0) = 0; gelu(a) = a for large a and 0 for large -a; gelu(a) - gelu(-a) = a
    (odd part of the tanh form), checked through weights w and -w."""
    K = 16
    x = _bf16(_rng(54).normal(size=(4, K)))
    zero_w = _bits(np.zeros((8, K)))
    _close(lib.linear_gelu_bf16(x, zero_w), np.zeros((4, 8)), 0.0, "gelu(0)")
    big = _bits(np.array([10.0, -10.0, 24.0, -24.0, 0.0, 0.0, 0.0, 0.0]))
    y = lib.linear_gelu_bf16(x, zero_w, big)
    _close(y[:, :4], np.broadcast_to([10.0, 0.0, 24.0, 0.0], (4, 4)), 1e-12, "saturation")
    w = _bf16(_rng(55).normal(size=(8, K)))
    minus_w = w ^ np.uint16(0x8000)
    diff = lib.linear_gelu_bf16(x, w) - lib.linear_gelu_bf16(x, minus_w)
    _close(diff, lib.linear_bf16(x, w), 1e-12, "odd part")


ALL_PINS = [
    pin_golden_closed_forms,
    pin_single_token,
    pin_two_tokens_sigmoid,
    pin_identical_values,
    pin_zero_query_mean,
    pin_probs_rows,
    pin_joint_kv_permutation,
    pin_head_batch_independence,
    pin_hard_attention,
    pin_brute_force_python,
    pin_torch_sdpa_workloads,
    pin_d72_zero_padding,
    pin_rows_entry,
    pin_layernorm_closed_forms,
    pin_layernorm_shift_invariance,
    pin_layernorm_brute_force_and_torch,
    pin_linear_closed_forms,
    pin_linear_permutation_and_linearity,
    pin_linear_brute_force_and_torch,
    pin_round_bf16_ties_and_torch,
    pin_add_layernorm_reductions,
    pin_add_layernorm_torch,
    pin_linear_gelu_torch_and_erf,
    pin_linear_gelu_closed_forms,
]
