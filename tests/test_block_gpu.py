"""LayerNorm, residual add + LayerNorm, linear and linear + GELU layers around the
attention core vs. the fp64 oracle, and whole encoder layers stage by stage.

Stage-wise: every GPU stage is compared with the oracle on identical bf16 inputs
(the GPU's own bf16 output of the previous stage feeds the oracle's next stage).
Tolerance: the attention stage keeps the attention bound (max |err| <= 2e-2,
mean |err| <= 2e-3); LayerNorm and linear outputs use the bound derived from their
arithmetic: the output is an fp32 result (the GEMM's accumulation with bias, GELU and
residual applied in the same fp32 epilogue) rounded to bf16 once, at most 2^-9 of what it
rounds, so elementwise |err| <= 2^-8 (|x w^T + b| + |res|) + 2^-10 and the mean error
<= 2^-9 of the mean magnitude (an absolute bound like the attention's would not fit:
these outputs reach |y| ~ 6, where one bf16 ulp is 0.03).  The residual stream of the
fused add + LayerNorm is compared bit for bit (one rounding of an exact sum).  The GELU
output adds the error of the epilogue's tanh, the hardware approximation's absolute
error below 2^-10.9, i.e. under 2^-11 |a| for pre-activation a, which the magnitude
|y| + |a| / 8 covers.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import seeded_inputs as si
from gpu_helpers import assert_close_bf16, assert_parity, needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]

# (name, B, N, H, d): the encoder workloads; width W = H d, tokens M = B N.
ENCODERS = [(c.name, c.B, c.N, c.H, c.d) for c in si.ENCODER_WORKLOADS]


def dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def host(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def ln_inputs(M, W, seed):
    return (si.normal_bf16(seed, (M, W), 0.2, 1.3), si.normal_bf16(seed + 1, (W,), 1.0, 0.1),
            si.normal_bf16(seed + 2, (W,), 0.0, 0.1))


def linear_inputs(M, K, N, seed):
    return (si.normal_bf16(seed, (M, K)), si.normal_bf16(seed + 1, (N, K), 0.0, 1.0 / math.sqrt(K)),
            si.normal_bf16(seed + 2, (N,), 0.0, 0.1))


@pytest.mark.parametrize("name,B,N,H,d", ENCODERS)
def test_layernorm_encoder_widths(name, B, N, H, d):
    import vit_self_attention_b200 as vab
    M, W = B * N, H * d
    x, g, b = ln_inputs(M, W, 100 + W)
    got = vab.layernorm(dev(x), dev(g), dev(b), 1e-6)
    torch.cuda.synchronize()
    assert_close_bf16(f64(got), oracle.layernorm_bf16(x, g, b, 1e-6), f"LayerNorm {name}")


@pytest.mark.parametrize("M,W", [(1, 8), (7, 16), (33, 248), (5, 256), (9, 264), (3, 2048),
                                 (1000, 768)])
def test_layernorm_edge_shapes_and_in_place(M, W):
    import vit_self_attention_b200 as vab
    x, g, b = ln_inputs(M, W, 200 + M + W)
    want = oracle.layernorm_bf16(x, g, b, 1e-5)
    xt = dev(x)
    got = vab.layernorm(xt, dev(g), dev(b), 1e-5)
    torch.cuda.synchronize()
    assert_close_bf16(f64(got), want, f"LayerNorm M={M} W={W}")
    vab.layernorm(xt, dev(g), dev(b), 1e-5, out=xt)  # in place
    torch.cuda.synchronize()
    assert_close_bf16(f64(xt), want, f"LayerNorm in place M={M} W={W}")


@pytest.mark.parametrize("name,B,N,H,d", ENCODERS)
def test_qkv_linear_encoder_shapes(name, B, N, H, d):
    import vit_self_attention_b200 as vab
    M, K = B * N, H * d
    x, w, b = linear_inputs(M, K, 3 * K, 300 + K)
    got = vab.linear(dev(x), dev(w), dev(b))
    torch.cuda.synchronize()
    assert_close_bf16(f64(got), oracle.linear_bf16(x, w, b), f"qkv linear {name}")


@pytest.mark.parametrize("M,K,N,bias,res", [(1, 8, 8, True, False), (5, 16, 24, False, False),
                                            (129, 768, 768, True, True), (77, 64, 200, False, True),
                                            (1000, 1024, 1024, True, True)])
def test_linear_bias_residual_variants(M, K, N, bias, res):
    import vit_self_attention_b200 as vab
    x, w, b = linear_inputs(M, K, N, 400 + M + K + N)
    r = si.normal_bf16(500 + M, (M, N)) if res else None
    got = vab.linear(dev(x), dev(w), dev(b) if bias else None, dev(r) if res else None)
    torch.cuda.synchronize()
    want = oracle.linear_bf16(x, w, b if bias else None, r)
    assert_close_bf16(f64(got), want, f"linear M={M} K={K} N={N} bias={bias} res={res}",
                      mag=residual_magnitude(x, w, b if bias else None, r))


@pytest.mark.parametrize("M,K,N,res,ws", [
    (64, 16384, 256, True, True),     # few tiles and a long K: split K (16 parts)
    (64, 16384, 256, True, False),    # the same without a workspace: one part per tile
    (100, 12296, 200, True, True),    # K not a multiple of 64, ragged N: split K
    (591, 3072, 768, True, True),     # ViT-B/16 fc2 (3 views): few tiles, K too short to split
    (4096, 1024, 3072, False, True),  # 256-wide tiles, several waves over the SMs
    (300, 136, 72, True, True),       # K and N ending inside one 64-wide step / tile
    (2000, 768, 2304, False, True),   # 128-wide tiles
])
def test_linear_tile_widths_and_split_k(M, K, N, res, ws):
    """The GEMM's tile-width choices (256 / 128 / 64 columns) and its split-K path (fp32
    partial sums in the caller's workspace, added up in split order by the last arrival)
    against the oracle; without a workspace the same shape runs unsplit."""
    import vit_self_attention_b200 as vab
    x, w, b = linear_inputs(M, K, N, 900 + M + K + N)
    r = si.normal_bf16(950 + M, (M, N)) if res else None
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    wsb = vab.vla_linear_workspace_bytes() if ws else 0
    wst = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda") if ws else None
    vab.vla_linear_fwd(dev(x), dev(w), dev(b), dev(r) if res else None, y, M, K, N, wst, wsb)
    torch.cuda.synchronize()
    assert_close_bf16(f64(y), oracle.linear_bf16(x, w, b, r),
                      f"linear M={M} K={K} N={N} res={res} workspace={ws}",
                      mag=residual_magnitude(x, w, b, r))


def test_linear_gelu_split_k():
    """fc1 + GELU on a shape with few tiles and a long K (split K) and on the same shape
    unsplit: both against the oracle."""
    import vit_self_attention_b200 as vab
    M, K, N = 200, 16384, 256
    x, w, b = linear_inputs(M, K, N, 1200)
    want = oracle.linear_gelu_bf16(x, w, b)
    a = np.abs(oracle.linear_bf16(x, w, b))
    for wsb in (vab.vla_linear_workspace_bytes(), 0):
        wst = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda")
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        vab.vla_linear_gelu_fwd(dev(x), dev(w), dev(b), y, M, K, N, wst if wsb else None, wsb)
        torch.cuda.synchronize()
        assert_close_bf16(f64(y), want, f"fc1 + GELU workspace={wsb}", mag=np.abs(want) + a / 8)


def test_linear_in_place_residual():
    """y = x @ w.T + bias + y (the output projection adding into the residual stream)."""
    import vit_self_attention_b200 as vab
    M, K = 591, 768
    x, w, b = linear_inputs(M, K, K, 600)
    r = si.normal_bf16(601, (M, K))
    rt = dev(r)
    vab.linear(dev(x), dev(w), dev(b), rt, out=rt)
    torch.cuda.synchronize()
    assert_close_bf16(f64(rt), oracle.linear_bf16(x, w, b, r), "in-place residual",
                      mag=residual_magnitude(x, w, b, r))


def residual_magnitude(x, w, b, r):
    """|x @ w.T + b| + |r|: the magnitudes the two roundings of a residual linear act on."""
    if r is None:
        return np.abs(oracle.linear_bf16(x, w, b))
    return np.abs(oracle.linear_bf16(x, w, b)) + np.abs(si.bf16_bits_to_f32(r).astype(np.float64))


def block_weights(W, seed):
    return {"g": si.normal_bf16(seed, (W,), 1.0, 0.1), "be": si.normal_bf16(seed + 1, (W,), 0.0, 0.1),
            "wqkv": si.normal_bf16(seed + 2, (3 * W, W), 0.0, 1.0 / math.sqrt(W)),
            "bqkv": si.normal_bf16(seed + 3, (3 * W,), 0.0, 0.1),
            "wo": si.normal_bf16(seed + 4, (W, W), 0.0, 1.0 / math.sqrt(W)),
            "bo": si.normal_bf16(seed + 5, (W,), 0.0, 0.1)}


@pytest.mark.parametrize("name", ["vit_b16_112px_1view", "vit_b16_224px_3views",
                                  "siglip_so400m14_224px_2views"])
def test_attention_half_block_stagewise(name):
    """x -> LayerNorm -> qkv linear -> attention -> output linear + residual x, each stage
    against the oracle on the GPU's own bf16 input to that stage."""
    import vit_self_attention_b200 as vab
    c = si.workload(name)
    cfg = c.index - 1  # seed offset of this workload
    W = c.H * c.d
    x = si.normal_bf16(700 + cfg, (c.B, c.N, W))
    p = block_weights(W, 710 + cfg)
    t = {k: dev(v) for k, v in p.items()}
    xt = dev(x)
    xn = vab.layernorm(xt, t["g"], t["be"], 1e-6)
    qkv = vab.linear(xn, t["wqkv"], t["bqkv"])
    o = vab.attention(qkv.view(c.B, c.N, 3, c.H, c.d), c.scale)
    y = vab.linear(o.view(c.B, c.N, W), t["wo"], t["bo"], xt)
    torch.cuda.synchronize()
    assert_close_bf16(f64(xn), oracle.layernorm_bf16(x, p["g"], p["be"], 1e-6), "LayerNorm stage")
    assert_close_bf16(f64(qkv), oracle.linear_bf16(host(xn), p["wqkv"], p["bqkv"]), "qkv stage")
    assert_parity(f64(o), oracle.attention_packed_bf16(host(qkv).reshape(c.B, c.N, 3, c.H, c.d),
                                                       c.scale), "attention stage")
    ob = host(o).reshape(c.B, c.N, W)
    assert_close_bf16(f64(y), oracle.linear_bf16(ob, p["wo"], p["bo"], x),
                      "output projection + residual stage",
                      mag=residual_magnitude(ob, p["wo"], p["bo"], x))


def test_half_block_graph_capture():
    """Two layers of the chain captured in one CUDA graph and replayed give the same bytes
    as the eager calls."""
    import vit_self_attention_b200 as vab
    c = si.VIT_B16_224PX_3VIEWS
    W = c.H * c.d
    x0 = dev(si.normal_bf16(800, (c.B, c.N, W)))
    layers = [{k: dev(v) for k, v in block_weights(W, 810 + 10 * i).items()} for i in range(2)]
    ws = torch.empty(vab.vla_linear_workspace_bytes(), dtype=torch.uint8, device="cuda")
    bufs = {"xn": torch.empty_like(x0), "qkv": torch.empty((c.B, c.N, 3 * W), dtype=torch.bfloat16,
                                                            device="cuda"),
            "o": torch.empty((c.B, c.N, c.H, c.d), dtype=torch.bfloat16, device="cuda")}

    def run(x):
        for p in layers:
            vab.layernorm(x, p["g"], p["be"], 1e-6, out=bufs["xn"])
            vab.linear(bufs["xn"], p["wqkv"], p["bqkv"], out=bufs["qkv"], workspace=ws)
            vab.attention(bufs["qkv"].view(c.B, c.N, 3, c.H, c.d), c.scale, out=bufs["o"])
            vab.linear(bufs["o"].view(c.B, c.N, W), p["wo"], p["bo"], x, out=x, workspace=ws)

    eager = x0.clone()
    run(eager)
    torch.cuda.synchronize()
    xg = x0.clone()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run(x0.clone())  # warm-up (plans, algorithms) outside the capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        run(xg)
    xg.copy_(x0)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(xg, eager)


# MLP hidden width per encoder width: ViT-B/16 3072, ViT-L/14 4096, SigLIP-So400m 4304.
MLP = {768: 3072, 1024: 4096, 1152: 4304}


def mlp_weights(W, F, seed):
    return {"g2": si.normal_bf16(seed, (W,), 1.0, 0.1), "be2": si.normal_bf16(seed + 1, (W,), 0.0, 0.1),
            "w1": si.normal_bf16(seed + 2, (F, W), 0.0, 1.0 / math.sqrt(W)),
            "b1": si.normal_bf16(seed + 3, (F,), 0.0, 0.1),
            "w2": si.normal_bf16(seed + 4, (W, F), 0.0, 1.0 / math.sqrt(F)),
            "b2": si.normal_bf16(seed + 5, (W,), 0.0, 0.1)}


def gelu_magnitude(x, w, b):
    """|gelu(a)| + |a| / 8 for the pre-activation a = x @ w.T + b."""
    a = np.abs(oracle.linear_bf16(x, w, b))
    return np.abs(oracle.linear_gelu_bf16(x, w, b)) + a / 8.0


@pytest.mark.parametrize("name,B,N,H,d", ENCODERS)
def test_add_layernorm_encoder_widths(name, B, N, H, d):
    import vit_self_attention_b200 as vab
    M, W = B * N, H * d
    x, g, b = ln_inputs(M, W, 900 + W)
    r = si.normal_bf16(950 + W, (M, W), 0.0, 0.7)
    s, y = vab.add_layernorm(dev(x), dev(r), dev(g), dev(b), 1e-6)
    torch.cuda.synchronize()
    want_s, want_y = oracle.add_layernorm_bf16(x, r, g, b, 1e-6)
    assert np.array_equal(host(s), want_s), f"residual stream bits, {name}"
    assert_close_bf16(f64(y), want_y, f"add + LayerNorm {name}")


@pytest.mark.parametrize("M,W", [(1, 8), (7, 16), (33, 248), (9, 264), (3, 2048), (1000, 1152)])
def test_add_layernorm_edge_shapes_and_in_place(M, W):
    import vit_self_attention_b200 as vab
    x, g, b = ln_inputs(M, W, 1000 + M + W)
    r = si.normal_bf16(1001 + M + W, (M, W), 0.0, 3.0)
    want_s, want_y = oracle.add_layernorm_bf16(x, r, g, b, 1e-5)
    xt, rt = dev(x), dev(r)
    s, y = vab.add_layernorm(xt, rt, dev(g), dev(b), 1e-5)
    torch.cuda.synchronize()
    assert np.array_equal(host(s), want_s)
    assert_close_bf16(f64(y), want_y, f"add + LayerNorm M={M} W={W}")
    vab.add_layernorm(xt, rt, dev(g), dev(b), 1e-5, out_s=xt, out_y=rt)  # both in place
    torch.cuda.synchronize()
    assert np.array_equal(host(xt), want_s)
    assert_close_bf16(f64(rt), want_y, f"add + LayerNorm in place M={M} W={W}")


@pytest.mark.parametrize("name,B,N,H,d", ENCODERS)
def test_linear_gelu_mlp_shapes(name, B, N, H, d):
    import vit_self_attention_b200 as vab
    M, K = B * N, H * d
    F = MLP[K]
    x, w, b = linear_inputs(M, K, F, 1100 + K)
    got = vab.linear_gelu(dev(x), dev(w), dev(b))
    torch.cuda.synchronize()
    assert_close_bf16(f64(got), oracle.linear_gelu_bf16(x, w, b), f"fc1 + GELU {name}",
                      mag=gelu_magnitude(x, w, b))


@pytest.mark.parametrize("M,K,N,bias", [(1, 8, 8, True), (5, 16, 24, False), (77, 64, 200, True),
                                        (300, 1152, 4304, False)])
def test_linear_gelu_variants(M, K, N, bias):
    import vit_self_attention_b200 as vab
    x, w, b = linear_inputs(M, K, N, 1200 + M + K + N)
    b = b if bias else None
    got = vab.linear_gelu(dev(x), dev(w), dev(b) if bias else None)
    torch.cuda.synchronize()
    assert_close_bf16(f64(got), oracle.linear_gelu_bf16(x, w, b),
                      f"linear + GELU M={M} K={K} N={N} bias={bias}", mag=gelu_magnitude(x, w, b))


def _layer_stagewise(name, fused_norm):
    """One pre-norm encoder layer on the GPU, each stage against the oracle on the GPU's
    own bf16 input to that stage.  fused_norm: the output projection leaves the residual
    to the fused add + LayerNorm; otherwise it adds it in its epilogue and LN2 is plain."""
    import vit_self_attention_b200 as vab
    c = si.workload(name)
    cfg = c.index - 1  # seed offset of this workload
    W = c.H * c.d
    F = MLP[W]
    x = si.normal_bf16(1300 + cfg, (c.B, c.N, W))
    p = {**block_weights(W, 1310 + cfg), **mlp_weights(W, F, 1320 + cfg)}
    t = {k: dev(v) for k, v in p.items()}
    xt = dev(x)
    xn = vab.layernorm(xt, t["g"], t["be"], 1e-6)
    qkv = vab.linear(xn, t["wqkv"], t["bqkv"])
    o = vab.attention(qkv.view(c.B, c.N, 3, c.H, c.d), c.scale)
    if fused_norm:
        proj = vab.linear(o.view(c.B, c.N, W), t["wo"], t["bo"])
        h, hn = vab.add_layernorm(xt, proj, t["g2"], t["be2"], 1e-6)
    else:
        h = vab.linear(o.view(c.B, c.N, W), t["wo"], t["bo"], xt)
        hn = vab.layernorm(h, t["g2"], t["be2"], 1e-6)
    a = vab.linear_gelu(hn, t["w1"], t["b1"])
    out = vab.linear(a, t["w2"], t["b2"], h)
    torch.cuda.synchronize()
    assert_close_bf16(f64(xn), oracle.layernorm_bf16(x, p["g"], p["be"], 1e-6), "LN1")
    assert_close_bf16(f64(qkv), oracle.linear_bf16(host(xn), p["wqkv"], p["bqkv"]), "qkv")
    assert_parity(f64(o), oracle.attention_packed_bf16(host(qkv).reshape(c.B, c.N, 3, c.H, c.d),
                                                       c.scale), "attention")
    ob = host(o).reshape(c.B, c.N, W)
    if fused_norm:
        assert_close_bf16(f64(proj), oracle.linear_bf16(ob, p["wo"], p["bo"]), "output projection",
                          mag=residual_magnitude(ob, p["wo"], p["bo"], None))
        want_h, want_hn = oracle.add_layernorm_bf16(x, host(proj), p["g2"], p["be2"], 1e-6)
        assert np.array_equal(host(h), want_h), "residual stream after attention"
        assert_close_bf16(f64(hn), want_hn, "add + LN2")
    else:
        assert_close_bf16(f64(h), oracle.linear_bf16(ob, p["wo"], p["bo"], x),
                          "output projection + residual",
                          mag=residual_magnitude(ob, p["wo"], p["bo"], x))
        assert_close_bf16(f64(hn), oracle.layernorm_bf16(host(h), p["g2"], p["be2"], 1e-6), "LN2")
    hb = host(hn)
    assert_close_bf16(f64(a), oracle.linear_gelu_bf16(hb, p["w1"], p["b1"]), "fc1 + GELU",
                      mag=gelu_magnitude(hb, p["w1"], p["b1"]))
    ab, hh = host(a), host(h)
    assert_close_bf16(f64(out), oracle.linear_bf16(ab, p["w2"], p["b2"], hh), "fc2 + residual",
                      mag=residual_magnitude(ab, p["w2"], p["b2"], hh))


@pytest.mark.parametrize("name", ["vit_b16_112px_1view", "vit_b16_224px_3views",
                                  "siglip_so400m14_224px_2views"])
def test_encoder_layer_stagewise(name):
    _layer_stagewise(name, fused_norm=False)


@pytest.mark.parametrize("name", ["vit_b16_224px_3views", "siglip_so400m14_224px_2views"])
def test_encoder_layer_stagewise_fused_residual_norm(name):
    _layer_stagewise(name, fused_norm=True)


def test_encoder_layers_graph_capture():
    """Two whole encoder layers captured in one CUDA graph and replayed give the eager
    bytes."""
    import vit_self_attention_b200 as vab
    c = si.SIGLIP_SO400M14_224PX_2VIEWS
    W = c.H * c.d
    F = MLP[W]
    x0 = dev(si.normal_bf16(1400, (c.B, c.N, W)))
    layers = [{k: dev(v) for k, v in {**block_weights(W, 1410 + 10 * i),
                                       **mlp_weights(W, F, 1450 + 10 * i)}.items()}
              for i in range(2)]
    ws = torch.empty(vab.vla_linear_workspace_bytes(), dtype=torch.uint8, device="cuda")
    e = lambda *shape: torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    bufs = {"xn": e(c.B, c.N, W), "qkv": e(c.B, c.N, 3 * W), "o": e(c.B, c.N, c.H, c.d),
            "a": e(c.B, c.N, F)}

    def run(x):
        for p in layers:
            vab.layernorm(x, p["g"], p["be"], 1e-6, out=bufs["xn"])
            vab.linear(bufs["xn"], p["wqkv"], p["bqkv"], out=bufs["qkv"], workspace=ws)
            vab.attention(bufs["qkv"].view(c.B, c.N, 3, c.H, c.d), c.scale, out=bufs["o"])
            vab.linear(bufs["o"].view(c.B, c.N, W), p["wo"], p["bo"], x, out=x, workspace=ws)
            vab.layernorm(x, p["g2"], p["be2"], 1e-6, out=bufs["xn"])
            vab.linear_gelu(bufs["xn"], p["w1"], p["b1"], out=bufs["a"], workspace=ws)
            vab.linear(bufs["a"], p["w2"], p["b2"], x, out=x, workspace=ws)

    eager = x0.clone()
    run(eager)
    torch.cuda.synchronize()
    xg = x0.clone()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run(x0.clone())
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        run(xg)
    xg.copy_(x0)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(xg, eager)


def _layer_weights(W, F, seed):
    n = lambda s, shape, m, sd: si.normal_bf16(seed + s, shape, m, sd)
    return {"g": n(0, (W,), 1.0, 0.1), "be": n(1, (W,), 0.0, 0.1),
            "wq": n(2, (3 * W, W), 0.0, 1.0 / math.sqrt(W)), "bq": n(3, (3 * W,), 0.0, 0.1),
            "wo": n(4, (W, W), 0.0, 1.0 / math.sqrt(W)), "bo": n(5, (W,), 0.0, 0.1),
            "g2": n(6, (W,), 1.0, 0.1), "be2": n(7, (W,), 0.0, 0.1),
            "w1": n(8, (F, W), 0.0, 1.0 / math.sqrt(W)), "b1": n(9, (F,), 0.0, 0.1),
            "w2": n(10, (W, F), 0.0, 1.0 / math.sqrt(F)), "b2": n(11, (W,), 0.0, 0.1)}


def _oracle_layer(x, p, c):
    """One pre-norm encoder layer in the oracle, every stage's fp64 result rounded to bf16
    before the next stage reads it (the precision at which the layers hand over)."""
    W = c.H * c.d
    r = oracle.round_bf16
    xn = r(oracle.layernorm_bf16(x, p["g"], p["be"], 1e-6))
    qkv = r(oracle.linear_bf16(xn, p["wq"], p["bq"]))
    o = r(oracle.attention_packed_bf16(qkv.reshape(c.B, c.N, 3, c.H, c.d), c.scale))
    h = r(oracle.linear_bf16(o.reshape(c.B * c.N, W), p["wo"], p["bo"], x))
    hn = r(oracle.layernorm_bf16(h, p["g2"], p["be2"], 1e-6))
    a = r(oracle.linear_gelu_bf16(hn, p["w1"], p["b1"]))
    return r(oracle.linear_bf16(a, p["w2"], p["b2"], h))


def test_encoder_chain_against_oracle_chain_eager_and_graph():
    """Four whole encoder layers of the ViT-B/16 224 px workload (3 views: 591 tokens,
    width 768, MLP 3072, seeded weights per layer), run eagerly and replayed from one CUDA
    graph, against the oracle chain fed the same bf16 weights (each oracle stage reading the
    previous oracle stage's bf16-rounded output).

    Bound for L layers: each layer rounds the residual stream twice, and two correct
    evaluations whose pre-rounding values differ within the stage bounds can round an
    element to neighbouring bf16 values, one spacing (at most 2^-7 of its magnitude) apart;
    the residual path carries such a difference forward, and the branches add their own
    stage errors on top.  So the difference grows about linearly with L: mean |err| <=
    2^-8 L mean|x_L| and max |err| <= 2^-4 L rms(x_L) for the final stream x_L (a float32
    chain rounded at the same points differs from the oracle chain by 0.0013 L mean|x_L| in
    mean and 0.025-0.05 rms(x_L) at most for L <= 4)."""
    import vit_self_attention_b200 as vab
    c = si.VIT_B16_224PX_3VIEWS
    L, W, F = 4, c.H * c.d, 3072
    M = c.B * c.N
    params = [_layer_weights(W, F, 2000 + 13 * i) for i in range(L)]
    x0 = si.normal_bf16(1999, (M, W))
    want = x0
    for p in params:
        want = _oracle_layer(want, p, c)
    want64 = si.bf16_bits_to_f32(want).astype(np.float64)

    dp = [{k: dev(v) for k, v in p.items()} for p in params]
    ws = torch.empty(vab.vla_linear_workspace_bytes(), dtype=torch.uint8, device="cuda")
    xs = [dev(x0)] + [torch.empty((M, W), dtype=torch.bfloat16, device="cuda")
                      for _ in range(2 * L)]
    xn = torch.empty((M, W), dtype=torch.bfloat16, device="cuda")
    qkv = torch.empty((M, 3 * W), dtype=torch.bfloat16, device="cuda")
    o = torch.empty((c.B, c.N, c.H, c.d), dtype=torch.bfloat16, device="cuda")
    a = torch.empty((M, F), dtype=torch.bfloat16, device="cuda")

    def encoder(stream=None):
        for i, q in enumerate(dp):
            h_in, h_mid, h_out = xs[2 * i], xs[2 * i + 1], xs[2 * i + 2]
            vab.layernorm(h_in, q["g"], q["be"], 1e-6, out=xn, stream=stream)
            vab.linear(xn, q["wq"], q["bq"], out=qkv, workspace=ws, stream=stream)
            vab.attention(qkv.view(c.B, c.N, 3, c.H, c.d), c.scale, out=o, stream=stream)
            vab.linear(o.view(M, W), q["wo"], q["bo"], h_in, out=h_mid, workspace=ws,
                       stream=stream)
            vab.layernorm(h_mid, q["g2"], q["be2"], 1e-6, out=xn, stream=stream)
            vab.linear_gelu(xn, q["w1"], q["b1"], out=a, workspace=ws, stream=stream)
            vab.linear(a, q["w2"], q["b2"], h_mid, out=h_out, workspace=ws, stream=stream)

    def check(got, what):
        got = f64(got)
        assert np.all(np.isfinite(got)), what
        err = np.abs(got - want64)
        rms = float(np.sqrt((want64 ** 2).mean()))
        mean_bound = 2.0 ** -8 * L * float(np.abs(want64).mean())
        assert float(err.mean()) <= mean_bound, f"{what}: mean|err| {err.mean():.3e} > {mean_bound:.3e}"
        assert float(err.max()) <= 2.0 ** -4 * L * rms, f"{what}: max|err| {err.max():.3e}"

    encoder()
    torch.cuda.synchronize()
    eager = xs[-1].clone()
    check(eager, "eager encoder chain")

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        encoder(s)  # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        encoder(s)
    for t in xs[1:]:
        t.zero_()
    g.replay()
    torch.cuda.synchronize()
    check(xs[-1], "graph-replayed encoder chain")
    assert torch.equal(xs[-1], eager), "graph replay differs from the eager run"
    del g


@pytest.mark.parametrize("M,K,N,res", [(1, 64, 64, False), (37, 128, 200, True),
                                       (129, 256, 320, False), (300, 192, 72, True)])
def test_linear_stores_stay_inside_the_output(M, K, N, res):
    """The GEMM's output (and residual) move as TMA boxes of 32 rows x 64 columns, which
    overhang the tensor when M or N is ragged: nothing outside [M, N] may be written.  The
    output is a view into a larger buffer whose guards hold a sentinel; they must be
    unchanged and the output must match the oracle."""
    import vit_self_attention_b200 as vab
    x, w, b = linear_inputs(M, K, N, 5100 + M + K + N)
    r = si.normal_bf16(5400 + M, (M, N)) if res else None
    n_y = M * N
    guard = 8 * 1024  # elements (16 KB) on each side, 16-byte aligned
    sentinel = 0x7FA5
    big = torch.full((guard + n_y + guard,), sentinel, dtype=torch.int16, device="cuda")
    y = big[guard:guard + n_y].view(torch.bfloat16).view(M, N)
    vab.linear(dev(x), dev(w), dev(b), dev(r) if res else None, out=y)
    torch.cuda.synchronize()
    assert bool((big[:guard] == sentinel).all()), "written before the output"
    assert bool((big[guard + n_y:] == sentinel).all()), "written after the output"
    assert_close_bf16(f64(y), oracle.linear_bf16(x, w, b, r),
                      f"guarded linear M={M} K={K} N={N} res={res}",
                      mag=residual_magnitude(x, w, b, r))
