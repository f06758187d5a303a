"""B200 (sm_100a) self-attention core of a ViT / SigLIP vision encoder.

Thin ctypes binding over ``libvla_attn.so`` (C ABI in ``include/vla_attn.h``):
argument marshalling only -- every step of the computation runs in the CUDA
kernels of that library.  There is no CPU or PyTorch fallback: importing this
package fails loudly when the library has not been built.

Operation: ``o = softmax(q k^T * scale) v`` per image and head over the packed
``[B, N, 3, H, d]`` bf16 QKV that a ViT block's qkv linear emits (the
multi-head self-attention of the Pi0 Flash Attention tutorial, sections 1 and
3.2), output ``[B, N, H, d]`` bf16.
"""
from __future__ import annotations

import ctypes
import math
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIBRARY_PATH = os.path.join(_PKG, "libvla_attn.so")

if not os.path.exists(LIBRARY_PATH):
    raise ImportError(
        f"{LIBRARY_PATH} is missing: build it with `python vit_self_attention_b200/build.py` "
        "(nvcc, sm_100a); there is no fallback implementation")

_lib = ctypes.CDLL(LIBRARY_PATH)

_VP = ctypes.c_void_p
_I = ctypes.c_int
_lib.vla_attn_fwd.argtypes = [_VP, _VP, _VP, _VP, _I, _I, _I, _I, ctypes.c_float, _VP]
_lib.vla_attn_fwd.restype = _I
_lib.vla_attn_fwd_host.argtypes = [_VP, _VP, _VP, _VP, _I, _I, _I, _I, ctypes.c_float, _VP]
_lib.vla_attn_fwd_host.restype = _I
_lib.vla_attn_strerror.argtypes = [_I]
_lib.vla_attn_strerror.restype = ctypes.c_char_p
_lib.vla_attn_last_device_status.argtypes = [_VP, ctypes.POINTER(_I)]
_lib.vla_attn_last_device_status.restype = _I
_lib.vla_attn_reset_device_status.argtypes = [_VP]
_lib.vla_attn_reset_device_status.restype = _I
_lib.vla_attn_max_tokens.argtypes = [_I]
_lib.vla_attn_max_tokens.restype = _I
_lib.vla_attn_launch_count.argtypes = []
_lib.vla_attn_launch_count.restype = ctypes.c_uint64
_lib.vla_attn_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
_lib.vla_attn_set_wait_limit_ns.restype = None
_lib.vla_attn_set_test_stall.argtypes = [_I]
_lib.vla_attn_set_test_stall.restype = None
_lib.vla_layernorm_fwd.argtypes = [_VP, _VP, _VP, _VP, _I, _I, ctypes.c_float, _VP]
_lib.vla_layernorm_fwd.restype = _I
_lib.vla_linear_fwd.argtypes = [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _VP, ctypes.c_size_t, _VP]
_lib.vla_linear_fwd.restype = _I
_lib.vla_linear_workspace_bytes.argtypes = []
_lib.vla_linear_workspace_bytes.restype = ctypes.c_size_t
_lib.vla_add_layernorm_fwd.argtypes = [_VP, _VP, _VP, _VP, _VP, _VP, _I, _I, ctypes.c_float, _VP]
_lib.vla_add_layernorm_fwd.restype = _I
_lib.vla_linear_gelu_fwd.argtypes = [_VP, _VP, _VP, _VP, _I, _I, _I, _VP, ctypes.c_size_t, _VP]
_lib.vla_linear_gelu_fwd.restype = _I
_lib.vla_linear_fwd_static.argtypes = [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _VP]
_lib.vla_linear_fwd_static.restype = _I
_lib.vla_linear_static_workspace_bytes.argtypes = []
_lib.vla_linear_static_workspace_bytes.restype = ctypes.c_size_t

# Status codes of include/vla_attn.h
OK = 0
ERR_NULL = -1
ERR_SHAPE = -2
ERR_UNSUPPORTED = -3
ERR_ALIGN = -4
ERR_SCALE = -5
ERR_CUDA = -6
ERR_TIMEOUT = -7
ERR_DEVICE = -8
ERR_MEMORY = -9

EXPORTED_SYMBOLS = (
    "vla_attn_fwd", "vla_attn_fwd_host", "vla_attn_strerror", "vla_attn_last_device_status",
    "vla_attn_reset_device_status", "vla_attn_max_tokens", "vla_attn_launch_count",
    "vla_attn_set_wait_limit_ns",
    "vla_attn_set_test_stall", "vla_layernorm_fwd", "vla_linear_fwd", "vla_linear_workspace_bytes",
    "vla_linear_fwd_static", "vla_linear_static_workspace_bytes", "vla_add_layernorm_fwd",
    "vla_linear_gelu_fwd",
)


class VlaAttnError(RuntimeError):
    def __init__(self, status: int):
        self.status = status
        super().__init__(f"vla_attn status {status}: {vla_attn_strerror(status)}")


def _addr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return int(x.data_ptr())


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


def vla_attn_strerror(status: int) -> str:
    return _lib.vla_attn_strerror(int(status)).decode()


def vla_attn_fwd(q, k, v, o, B: int, N: int, H: int, d: int, scale: float, stream=None,
                 check: bool = True) -> int:
    """Enqueue the attention kernel.  ``q/k/v/o`` are tensors or raw device addresses
    (``k = q + H*d``, ``v = q + 2*H*d`` elements into one packed buffer).  Returns the
    status; raises ``VlaAttnError`` on a non-zero status when ``check``."""
    st = _lib.vla_attn_fwd(_addr(q), _addr(k), _addr(v), _addr(o), int(B), int(N), int(H),
                           int(d), float(scale), _stream(stream))
    if check and st != OK:
        raise VlaAttnError(st)
    return st


def vla_attn_fwd_host(qkv_host, o_host, qkv_dev, o_dev, B: int, N: int, H: int, d: int,
                      scale: float, stream=None, check: bool = True) -> int:
    """Host-buffer variant: H2D copy, kernel, D2H copy, all enqueued on ``stream``."""
    st = _lib.vla_attn_fwd_host(_addr(qkv_host), _addr(o_host), _addr(qkv_dev), _addr(o_dev),
                                int(B), int(N), int(H), int(d), float(scale), _stream(stream))
    if check and st != OK:
        raise VlaAttnError(st)
    return st


def vla_attn_last_device_status(stream=None) -> tuple[int, int]:
    """(status, site) of the device-side status word; synchronises ``stream``."""
    site = _I(0)
    st = _lib.vla_attn_last_device_status(_stream(stream), ctypes.byref(site))
    return st, site.value


def vla_attn_reset_device_status(stream=None) -> int:
    return _lib.vla_attn_reset_device_status(_stream(stream))


def vla_attn_max_tokens(d: int) -> int:
    return _lib.vla_attn_max_tokens(int(d))


def vla_attn_launch_count() -> int:
    return int(_lib.vla_attn_launch_count())


def vla_attn_set_wait_limit_ns(ns: int) -> None:
    _lib.vla_attn_set_wait_limit_ns(int(ns))


def vla_attn_set_test_stall(enable: bool) -> None:
    """Testing hook: following launches wait on a barrier nothing completes (see the header)."""
    _lib.vla_attn_set_test_stall(1 if enable else 0)


def vla_layernorm_fwd(x, gamma, beta, y, M: int, W: int, eps: float, stream=None,
                      check: bool = True) -> int:
    """Enqueue LayerNorm over the last dimension (see include/vla_attn.h)."""
    st = _lib.vla_layernorm_fwd(_addr(x), _addr(gamma), _addr(beta), _addr(y), int(M), int(W),
                                float(eps), _stream(stream))
    if check and st != OK:
        raise VlaAttnError(st)
    return st


def vla_add_layernorm_fwd(x, r, gamma, beta, s, y, M: int, W: int, eps: float, stream=None,
                          check: bool = True) -> int:
    """Enqueue ``s = bf16(x + r)``, ``y = LayerNorm(s)`` (see include/vla_attn.h)."""
    st = _lib.vla_add_layernorm_fwd(_addr(x), _addr(r), _addr(gamma), _addr(beta), _addr(s),
                                    _addr(y), int(M), int(W), float(eps), _stream(stream))
    if check and st != OK:
        raise VlaAttnError(st)
    return st


def vla_linear_gelu_fwd(x, w, bias, y, M: int, K: int, N: int, workspace=None,
                        workspace_bytes: int = 0, stream=None, check: bool = True) -> int:
    """Enqueue ``y = gelu(x @ w.T + bias)`` (tanh GELU; see include/vla_attn.h)."""
    st = _lib.vla_linear_gelu_fwd(_addr(x), _addr(w), _addr(bias), _addr(y), int(M), int(K),
                                  int(N), _addr(workspace), int(workspace_bytes), _stream(stream))
    if check and st != OK:
        raise VlaAttnError(st)
    return st


def vla_linear_workspace_bytes() -> int:
    return int(_lib.vla_linear_workspace_bytes())


def vla_linear_fwd(x, w, bias, res, y, M: int, K: int, N: int, workspace=None,
                   workspace_bytes: int = 0, stream=None, check: bool = True) -> int:
    """Enqueue ``y = x @ w.T + bias (+ res)`` (see include/vla_attn.h)."""
    st = _lib.vla_linear_fwd(_addr(x), _addr(w), _addr(bias), _addr(res), _addr(y), int(M),
                             int(K), int(N), _addr(workspace), int(workspace_bytes),
                             _stream(stream))
    if check and st != OK:
        raise VlaAttnError(st)
    return st


def vla_linear_static_workspace_bytes() -> int:
    return int(_lib.vla_linear_static_workspace_bytes())


def vla_linear_fwd_static(x, w, bias, res, y, M: int, K: int, N: int, stream=None,
                          check: bool = True) -> int:
    """``vla_linear_fwd`` with the library's fixed device workspace (no allocation;
    overlapping calls race -- see the header)."""
    st = _lib.vla_linear_fwd_static(_addr(x), _addr(w), _addr(bias), _addr(res), _addr(y),
                                    int(M), int(K), int(N), _stream(stream))
    if check and st != OK:
        raise VlaAttnError(st)
    return st


def layernorm(x, gamma, beta, eps: float = 1e-6, out=None, stream=None):
    """LayerNorm of a contiguous bf16 CUDA tensor over its last dimension."""
    import torch
    if x.dtype != torch.bfloat16 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous bf16 CUDA tensor")
    W = int(x.shape[-1])
    if out is None:
        out = torch.empty_like(x)
    vla_layernorm_fwd(x, gamma, beta, out, x.numel() // W, W, eps, stream)
    return out


def add_layernorm(x, r, gamma, beta, eps: float = 1e-6, out_s=None, out_y=None, stream=None):
    """``(s, y)``: the residual stream ``s = bf16(x + r)`` and ``y = LayerNorm(s)`` for
    contiguous bf16 CUDA tensors of one shape (``out_s`` may be ``x`` or ``r``)."""
    import torch
    for t in (x, r):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("x and r must be contiguous bf16 CUDA tensors")
    if x.shape != r.shape:
        raise ValueError("x and r must have one shape")
    W = int(x.shape[-1])
    s = torch.empty_like(x) if out_s is None else out_s
    y = torch.empty_like(x) if out_y is None else out_y
    vla_add_layernorm_fwd(x, r, gamma, beta, s, y, x.numel() // W, W, eps, stream)
    return s, y


def linear_gelu(x, w, bias=None, out=None, workspace=None, stream=None):
    """``gelu(x @ w.T + bias)`` (tanh GELU) for contiguous bf16 CUDA tensors."""
    import torch
    N, K = (int(v) for v in w.shape)
    M = x.numel() // K
    if out is None:
        out = torch.empty(tuple(x.shape[:-1]) + (N,), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.empty(vla_linear_workspace_bytes(), dtype=torch.uint8, device=x.device)
    vla_linear_gelu_fwd(x, w, bias, out, M, K, N, workspace, workspace.numel(), stream)
    return out


def linear(x, w, bias=None, res=None, out=None, workspace=None, stream=None):
    """``x @ w.T + bias (+ res)`` for contiguous bf16 CUDA tensors (``w`` is ``[N, K]``)."""
    import torch
    N, K = (int(v) for v in w.shape)
    M = x.numel() // K
    if out is None:
        out = torch.empty(tuple(x.shape[:-1]) + (N,), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.empty(vla_linear_workspace_bytes(), dtype=torch.uint8, device=x.device)
    vla_linear_fwd(x, w, bias, res, out, M, K, N, workspace, workspace.numel(), stream)
    return out


def attention(qkv, scale: float | None = None, out=None, stream=None):
    """Convenience wrapper for a contiguous bf16 CUDA tensor ``qkv`` of shape
    ``[B, N, 3, H, d]``; returns ``out`` (allocated by torch if None) ``[B, N, H, d]``."""
    import torch
    if qkv.dim() != 5 or qkv.shape[2] != 3:
        raise ValueError("qkv must have shape [B, N, 3, H, d]")
    if qkv.dtype != torch.bfloat16 or not qkv.is_cuda or not qkv.is_contiguous():
        raise ValueError("qkv must be a contiguous bf16 CUDA tensor")
    B, N, _, H, d = qkv.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, N, H, d), dtype=torch.bfloat16, device=qkv.device)
    base = qkv.data_ptr()
    step = H * d * 2
    vla_attn_fwd(base, base + step, base + 2 * step, out, B, N, H, d, scale, stream)
    return out


__all__ = [
    "LIBRARY_PATH", "EXPORTED_SYMBOLS", "VlaAttnError", "vla_attn_fwd", "vla_attn_fwd_host",
    "vla_attn_strerror", "vla_attn_last_device_status", "vla_attn_reset_device_status",
    "vla_attn_max_tokens", "vla_attn_launch_count", "vla_attn_set_wait_limit_ns",
    "vla_attn_set_test_stall", "vla_layernorm_fwd", "vla_linear_fwd", "vla_linear_workspace_bytes",
    "vla_linear_fwd_static", "vla_linear_static_workspace_bytes", "vla_add_layernorm_fwd",
    "vla_linear_gelu_fwd", "layernorm", "add_layernorm", "linear", "linear_gelu", "attention",
]
