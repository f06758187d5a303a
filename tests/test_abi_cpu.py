"""The C-ABI library loads, exports every declared symbol, and validates arguments
on the host before touching a GPU (these tests need no GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vla_attn.h")


def declared_functions():
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vla_[a-z_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    assert "vla_attn_fwd" in names and "vla_attn_strerror" in names
    assert len(names) >= 8


def test_library_exports_every_declared_symbol():
    import vit_self_attention_b200 as vab
    lib = ctypes.CDLL(vab.LIBRARY_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} not exported"
    assert set(declared_functions()) == set(vab.EXPORTED_SYMBOLS)
    nm = subprocess.run(["nm", "-D", "--defined-only", vab.LIBRARY_PATH], capture_output=True,
                        text=True)
    if nm.returncode == 0:
        for name in declared_functions():
            assert re.search(rf"\bT {name}$", nm.stdout, re.M), f"{name} not a defined text symbol"


def test_build_targets_sm100a_only():
    from vit_self_attention_b200 import build
    f = build.flags()
    assert "arch=compute_100a,code=sm_100a" in f
    assert sum(1 for x in f if x == "-gencode") == 1


H, D = 12, 64
Q = 0x10000000
K = Q + H * D * 2
V = Q + 2 * H * D * 2
O = 0x20000000


def call(q=Q, k=K, v=V, o=O, B=1, N=50, h=H, d=D, scale=0.125):
    import vit_self_attention_b200 as vab
    return vab.vla_attn_fwd(q, k, v, o, B, N, h, d, scale, stream=0, check=False)


def test_argument_validation_on_host():
    import vit_self_attention_b200 as vab
    assert call(q=0) == vab.ERR_NULL
    assert call(o=0) == vab.ERR_NULL
    assert call(B=0) == vab.ERR_SHAPE
    assert call(N=0) == vab.ERR_SHAPE
    assert call(h=0) == vab.ERR_SHAPE
    assert call(N=-5) == vab.ERR_SHAPE
    assert call(d=128, k=Q + H * 128 * 2, v=Q + 4 * H * 128) == vab.ERR_UNSUPPORTED
    assert call(d=32, k=Q + H * 32 * 2, v=Q + 4 * H * 32) == vab.ERR_UNSUPPORTED
    assert call(N=16385) == vab.ERR_UNSUPPORTED
    assert call(k=K + 2) == vab.ERR_SHAPE          # not the packed relation
    assert call(v=K) == vab.ERR_SHAPE
    assert call(q=Q + 2, k=K + 2, v=V + 2) == vab.ERR_ALIGN
    assert call(o=O + 8) == vab.ERR_ALIGN
    assert call(scale=0.0) == vab.ERR_SCALE
    assert call(scale=-1.0) == vab.ERR_SCALE
    assert call(scale=float("inf")) == vab.ERR_SCALE
    assert call(scale=float("nan")) == vab.ERR_SCALE


def test_valid_arguments_without_gpu_fail_cleanly():
    import torch

    import vit_self_attention_b200 as vab
    if torch.cuda.is_available():
        pytest.skip("this checks the no-GPU path")
    assert call() in (vab.ERR_CUDA, vab.ERR_DEVICE)
    assert vab.vla_attn_launch_count() == 0


def test_strerror_and_limits():
    import vit_self_attention_b200 as vab
    for st in range(-9, 1):
        assert vab.vla_attn_strerror(st)
    assert "unknown" in vab.vla_attn_strerror(-99)
    assert vab.vla_attn_max_tokens(64) == 16384 and vab.vla_attn_max_tokens(72) == 16384
    assert vab.vla_attn_max_tokens(128) == 0


def test_host_entry_validation():
    import vit_self_attention_b200 as vab
    st = vab.vla_attn_fwd_host(0, O, Q, O, 1, 50, H, D, 0.125, stream=0, check=False)
    assert st == vab.ERR_NULL
    st = vab.vla_attn_fwd_host(0x1000, 0x2000, Q, O, 1, 50, H, D, -1.0, stream=0, check=False)
    assert st == vab.ERR_SCALE


def test_product_package_has_no_oracle_or_fallback():
    """The CUDA package never imports the oracle nor carries a CPU/torch compute path."""
    pkg = os.path.join(ROOT, "vit_self_attention_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if not fn.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                continue
            with open(os.path.join(dirpath, fn)) as f:
                src = f.read()
            assert "oracle" not in src.lower(), f"{fn} mentions the oracle"
            assert "scaled_dot_product_attention" not in src, f"{fn} has a torch attention path"
            assert "softmax(" not in src.replace("softmax(Q", "").replace("softmax(q", ""), fn


def test_layernorm_and_linear_validation_on_host():
    """The LayerNorm and linear entry points reject bad arguments before touching a GPU."""
    import math as _m

    import vit_self_attention_b200 as vab
    X, G, B_, Y = 0x10000000, 0x11000000, 0x12000000, 0x13000000

    def ln(x=X, g=G, b=B_, y=Y, M=4, W=768, eps=1e-6):
        return vab.vla_layernorm_fwd(x, g, b, y, M, W, eps, stream=0, check=False)

    assert ln(x=None) == vab.ERR_NULL and ln(g=None) == vab.ERR_NULL and ln(y=None) == vab.ERR_NULL
    assert ln(M=0) == vab.ERR_SHAPE and ln(W=0) == vab.ERR_SHAPE
    assert ln(W=12) == vab.ERR_UNSUPPORTED and ln(W=2056) == vab.ERR_UNSUPPORTED
    assert ln(eps=-1.0) == vab.ERR_SCALE and ln(eps=_m.nan) == vab.ERR_SCALE
    assert ln(x=X + 2) == vab.ERR_ALIGN and ln(b=B_ + 8) == vab.ERR_ALIGN

    W_, BI, R, WS = 0x14000000, 0x15000000, 0x16000000, 0x17000000

    def lin(x=X, w=W_, bias=BI, res=R, y=Y, M=4, K=768, N=2304, ws=WS, wsb=1 << 20):
        return vab.vla_linear_fwd(x, w, bias, res, y, M, K, N, ws, wsb, stream=0, check=False)

    assert lin(x=None) == vab.ERR_NULL and lin(w=None) == vab.ERR_NULL
    assert lin(y=None) == vab.ERR_NULL and lin(ws=None) == vab.ERR_NULL
    assert lin(M=0) == vab.ERR_SHAPE and lin(K=-8) == vab.ERR_SHAPE
    assert lin(K=12) == vab.ERR_UNSUPPORTED and lin(N=10) == vab.ERR_UNSUPPORTED
    assert lin(bias=BI + 2) == vab.ERR_ALIGN and lin(res=R + 4) == vab.ERR_ALIGN
    assert lin(ws=WS + 8) == vab.ERR_ALIGN
    assert vab.vla_linear_workspace_bytes() >= 1 << 20


def test_add_layernorm_and_linear_gelu_validation_on_host():
    """The fused residual add + LayerNorm and the linear + GELU entry points reject bad
    arguments before touching a GPU."""
    import math as _m

    import vit_self_attention_b200 as vab
    X, R, G, B_, S, Y = (0x10000000 + i * 0x1000000 for i in range(6))

    def aln(x=X, r=R, g=G, b=B_, s=S, y=Y, M=4, W=1024, eps=1e-6):
        return vab.vla_add_layernorm_fwd(x, r, g, b, s, y, M, W, eps, stream=0, check=False)

    for kw in ("x", "r", "g", "b", "s", "y"):
        assert aln(**{kw: None}) == vab.ERR_NULL, kw
    assert aln(M=0) == vab.ERR_SHAPE and aln(W=-8) == vab.ERR_SHAPE
    assert aln(W=20) == vab.ERR_UNSUPPORTED and aln(W=4096) == vab.ERR_UNSUPPORTED
    assert aln(eps=-1e-6) == vab.ERR_SCALE and aln(eps=_m.inf) == vab.ERR_SCALE
    assert aln(r=R + 2) == vab.ERR_ALIGN and aln(s=S + 8) == vab.ERR_ALIGN

    W_, BI, WS = 0x17000000, 0x18000000, 0x19000000

    def lg(x=X, w=W_, bias=BI, y=Y, M=4, K=1152, N=4304, ws=WS, wsb=1 << 20):
        return vab.vla_linear_gelu_fwd(x, w, bias, y, M, K, N, ws, wsb, stream=0, check=False)

    assert lg(x=None) == vab.ERR_NULL and lg(w=None) == vab.ERR_NULL and lg(y=None) == vab.ERR_NULL
    assert lg(ws=None) == vab.ERR_NULL
    assert lg(M=0) == vab.ERR_SHAPE and lg(N=-8) == vab.ERR_SHAPE
    assert lg(K=12) == vab.ERR_UNSUPPORTED and lg(N=4302) == vab.ERR_UNSUPPORTED
    assert lg(bias=BI + 2) == vab.ERR_ALIGN and lg(y=Y + 4) == vab.ERR_ALIGN
