"""fp64 CPU oracle for the ViT/SigLIP self-attention core and the LayerNorm and
linear layers around it -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg use this package.  The CUDA library neither imports nor links it, and it
imports nothing from the CUDA package.

The arithmetic lives in ``vla_attn_oracle.cpp`` (plain definitions of
``O = softmax(Q K^T * scale) V`` per image and head, of LayerNorm over the last
dimension, of ``x @ w.T + bias (+ res)``, of the fused residual add + LayerNorm and
of the linear layer with a GELU, fp64 throughout); this
module only marshals numpy arrays through ctypes.  ``OracleLib`` can wrap any
build of that source (the tests compile deliberately broken copies to show
that the pins catch them); the module-level functions use the real build.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

_DP = ctypes.POINTER(ctypes.c_double)
_U16P = ctypes.POINTER(ctypes.c_uint16)
_I64P = ctypes.POINTER(ctypes.c_int64)
_I = ctypes.c_int


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


class OracleLib:
    """ctypes view of one compiled oracle library."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        lib.oracle_layernorm_bf16.argtypes = [_U16P, _U16P, _U16P, _DP, _I, _I,
                                              ctypes.c_double, _I]
        lib.oracle_layernorm_bf16.restype = _I
        lib.oracle_linear_bf16.argtypes = [_U16P, _U16P, _U16P, _U16P, _DP, _I, _I, _I, _I]
        lib.oracle_linear_bf16.restype = _I
        lib.oracle_round_bf16.argtypes = [_DP, _U16P, ctypes.c_long]
        lib.oracle_round_bf16.restype = _I
        lib.oracle_add_layernorm_bf16.argtypes = [_U16P, _U16P, _U16P, _U16P, _U16P, _DP, _I, _I,
                                                  ctypes.c_double, _I]
        lib.oracle_add_layernorm_bf16.restype = _I
        lib.oracle_linear_gelu_bf16.argtypes = [_U16P, _U16P, _U16P, _DP, _I, _I, _I, _I]
        lib.oracle_linear_gelu_bf16.restype = _I
        lib.oracle_attn_f64.argtypes = [_DP, _DP, _DP, _DP, _I, _I, _I, _I, ctypes.c_double, _I]
        lib.oracle_attn_f64.restype = _I
        lib.oracle_attn_probs_f64.argtypes = [_DP, _DP, _DP, _I, _I, _I, _I, ctypes.c_double]
        lib.oracle_attn_probs_f64.restype = _I
        lib.oracle_attn_packed_bf16.argtypes = [_U16P, _DP, _I, _I, _I, _I, ctypes.c_double, _I]
        lib.oracle_attn_packed_bf16.restype = _I
        lib.oracle_attn_rows_packed_bf16.argtypes = [_U16P, _I, _I, _I, _I, ctypes.c_double,
                                                     _I64P, _I, _DP, _I]
        lib.oracle_attn_rows_packed_bf16.restype = _I
        lib.oracle_default_threads.argtypes = []
        lib.oracle_default_threads.restype = _I
        self.path = path
        self._lib = lib

    def default_threads(self) -> int:
        """Threads a call with ``threads=0`` uses (the host's hardware concurrency)."""
        return int(self._lib.oracle_default_threads())

    def attention_f64(self, q, k, v, scale: float, threads: int = 0) -> np.ndarray:
        """``o = softmax(q k^T * scale) v`` for fp64 ``[B, N, H, d]`` arrays."""
        q = np.ascontiguousarray(q, dtype=np.float64)
        k = np.ascontiguousarray(k, dtype=np.float64)
        v = np.ascontiguousarray(v, dtype=np.float64)
        if q.ndim != 4 or q.shape != k.shape or q.shape != v.shape:
            raise ValueError("q, k, v must share one [B, N, H, d] shape")
        B, N, H, d = q.shape
        o = np.empty_like(q)
        rc = self._lib.oracle_attn_f64(_ptr(q, ctypes.c_double), _ptr(k, ctypes.c_double),
                                       _ptr(v, ctypes.c_double), _ptr(o, ctypes.c_double),
                                       B, N, H, d, float(scale), int(threads))
        if rc != 0:
            raise ValueError(f"oracle_attn_f64 rejected the input (rc={rc})")
        return o

    def probs_f64(self, q, k, scale: float) -> np.ndarray:
        """Softmax matrix ``[B, H, N, N]`` for fp64 ``[B, N, H, d]`` q and k."""
        q = np.ascontiguousarray(q, dtype=np.float64)
        k = np.ascontiguousarray(k, dtype=np.float64)
        B, N, H, d = q.shape
        p = np.empty((B, H, N, N), dtype=np.float64)
        rc = self._lib.oracle_attn_probs_f64(_ptr(q, ctypes.c_double), _ptr(k, ctypes.c_double),
                                             _ptr(p, ctypes.c_double), B, N, H, d, float(scale))
        if rc != 0:
            raise ValueError(f"oracle_attn_probs_f64 rejected the input (rc={rc})")
        return p

    def attention_packed_bf16(self, qkv_bits, scale: float, threads: int = 0) -> np.ndarray:
        """Oracle output fp64 ``[B, N, H, d]`` for packed ``[B, N, 3, H, d]`` bf16 bits."""
        qkv_bits = np.ascontiguousarray(qkv_bits, dtype=np.uint16)
        if qkv_bits.ndim != 5 or qkv_bits.shape[2] != 3:
            raise ValueError("qkv must be [B, N, 3, H, d]")
        B, N, _, H, d = qkv_bits.shape
        o = np.empty((B, N, H, d), dtype=np.float64)
        rc = self._lib.oracle_attn_packed_bf16(_ptr(qkv_bits, ctypes.c_uint16),
                                               _ptr(o, ctypes.c_double), B, N, H, d,
                                               float(scale), int(threads))
        if rc != 0:
            raise ValueError(f"oracle_attn_packed_bf16 rejected the input (rc={rc})")
        return o

    def attention_rows_packed_bf16(self, qkv_bits, scale: float, rows, threads: int = 0
                                   ) -> np.ndarray:
        """Oracle output rows ``[len(rows), d]`` for ``rows`` = iterable of ``(b, h, n)``."""
        qkv_bits = np.ascontiguousarray(qkv_bits, dtype=np.uint16)
        B, N, _, H, d = qkv_bits.shape
        idx = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
        out = np.empty((idx.shape[0], d), dtype=np.float64)
        rc = self._lib.oracle_attn_rows_packed_bf16(_ptr(qkv_bits, ctypes.c_uint16), B, N, H, d,
                                                    float(scale), _ptr(idx, ctypes.c_int64),
                                                    int(idx.shape[0]),
                                                    _ptr(out, ctypes.c_double), int(threads))
        if rc != 0:
            raise ValueError(f"oracle_attn_rows_packed_bf16 rejected the input (rc={rc})")
        return out


    def layernorm_bf16(self, x_bits, gamma_bits, beta_bits, eps: float,
                       threads: int = 0) -> np.ndarray:
        """fp64 LayerNorm over the last dimension of bf16 ``x`` (``[..., W]``)."""
        x = np.ascontiguousarray(x_bits, dtype=np.uint16)
        W = int(x.shape[-1])
        M = int(x.size // W)
        g = np.ascontiguousarray(gamma_bits, dtype=np.uint16).reshape(W)
        b = np.ascontiguousarray(beta_bits, dtype=np.uint16).reshape(W)
        out = np.empty(x.shape, dtype=np.float64)
        rc = self._lib.oracle_layernorm_bf16(_ptr(x, ctypes.c_uint16), _ptr(g, ctypes.c_uint16),
                                             _ptr(b, ctypes.c_uint16), _ptr(out, ctypes.c_double),
                                             M, W, float(eps), int(threads))
        if rc != 0:
            raise ValueError(f"oracle_layernorm_bf16 rejected the input (rc={rc})")
        return out

    def linear_bf16(self, x_bits, w_bits, bias_bits=None, res_bits=None,
                    threads: int = 0) -> np.ndarray:
        """fp64 ``x @ w.T + bias (+ res)`` for bf16 ``x [..., K]``, ``w [N, K]``."""
        x = np.ascontiguousarray(x_bits, dtype=np.uint16)
        w = np.ascontiguousarray(w_bits, dtype=np.uint16)
        N, K = (int(v) for v in w.shape)
        if x.shape[-1] != K:
            raise ValueError("x and w disagree on K")
        M = int(x.size // K)
        b = None if bias_bits is None else np.ascontiguousarray(bias_bits, dtype=np.uint16).reshape(N)
        r = None if res_bits is None else np.ascontiguousarray(res_bits, dtype=np.uint16).reshape(M, N)
        out = np.empty(x.shape[:-1] + (N,), dtype=np.float64)
        rc = self._lib.oracle_linear_bf16(
            _ptr(x, ctypes.c_uint16), _ptr(w, ctypes.c_uint16),
            None if b is None else _ptr(b, ctypes.c_uint16),
            None if r is None else _ptr(r, ctypes.c_uint16), _ptr(out, ctypes.c_double),
            M, K, N, int(threads))
        if rc != 0:
            raise ValueError(f"oracle_linear_bf16 rejected the input (rc={rc})")
        return out

    def round_bf16(self, v) -> np.ndarray:
        """bf16 bits of finite fp64 values, rounded to nearest, ties to even."""
        v = np.ascontiguousarray(v, dtype=np.float64)
        out = np.empty(v.shape, dtype=np.uint16)
        rc = self._lib.oracle_round_bf16(_ptr(v, ctypes.c_double), _ptr(out, ctypes.c_uint16),
                                         int(v.size))
        if rc != 0:
            raise ValueError("oracle_round_bf16: non-finite input")
        return out

    def add_layernorm_bf16(self, x_bits, r_bits, gamma_bits, beta_bits, eps: float,
                           threads: int = 0) -> tuple[np.ndarray, np.ndarray]:
        """``(s, y)``: the residual stream ``s = bf16(x + r)`` (bits) and fp64
        ``y = LayerNorm(s)`` over the last dimension."""
        x = np.ascontiguousarray(x_bits, dtype=np.uint16)
        r = np.ascontiguousarray(r_bits, dtype=np.uint16)
        if r.shape != x.shape:
            raise ValueError("x and r must have one shape")
        W = int(x.shape[-1])
        M = int(x.size // W)
        g = np.ascontiguousarray(gamma_bits, dtype=np.uint16).reshape(W)
        b = np.ascontiguousarray(beta_bits, dtype=np.uint16).reshape(W)
        s = np.empty(x.shape, dtype=np.uint16)
        y = np.empty(x.shape, dtype=np.float64)
        rc = self._lib.oracle_add_layernorm_bf16(
            _ptr(x, ctypes.c_uint16), _ptr(r, ctypes.c_uint16), _ptr(g, ctypes.c_uint16),
            _ptr(b, ctypes.c_uint16), _ptr(s, ctypes.c_uint16), _ptr(y, ctypes.c_double), M, W,
            float(eps), int(threads))
        if rc != 0:
            raise ValueError(f"oracle_add_layernorm_bf16 rejected the input (rc={rc})")
        return s, y

    def linear_gelu_bf16(self, x_bits, w_bits, bias_bits=None, threads: int = 0) -> np.ndarray:
        """fp64 ``gelu(x @ w.T + bias)`` (tanh form) for bf16 ``x [..., K]``, ``w [N, K]``."""
        x = np.ascontiguousarray(x_bits, dtype=np.uint16)
        w = np.ascontiguousarray(w_bits, dtype=np.uint16)
        N, K = (int(v) for v in w.shape)
        if x.shape[-1] != K:
            raise ValueError("x and w disagree on K")
        M = int(x.size // K)
        b = None if bias_bits is None else np.ascontiguousarray(bias_bits, dtype=np.uint16).reshape(N)
        out = np.empty(x.shape[:-1] + (N,), dtype=np.float64)
        rc = self._lib.oracle_linear_gelu_bf16(
            _ptr(x, ctypes.c_uint16), _ptr(w, ctypes.c_uint16),
            None if b is None else _ptr(b, ctypes.c_uint16), _ptr(out, ctypes.c_double),
            M, K, N, int(threads))
        if rc != 0:
            raise ValueError(f"oracle_linear_gelu_bf16 rejected the input (rc={rc})")
        return out


_default: OracleLib | None = None


def lib() -> OracleLib:
    """The oracle built from this directory's source (built on first use)."""
    global _default
    if _default is None:
        _default = OracleLib(_build.build())
    return _default


def default_threads() -> int:
    return lib().default_threads()


def attention_f64(q, k, v, scale: float, threads: int = 0) -> np.ndarray:
    return lib().attention_f64(q, k, v, scale, threads)


def probs_f64(q, k, scale: float) -> np.ndarray:
    return lib().probs_f64(q, k, scale)


def attention_packed_bf16(qkv_bits, scale: float, threads: int = 0) -> np.ndarray:
    return lib().attention_packed_bf16(qkv_bits, scale, threads)


def attention_rows_packed_bf16(qkv_bits, scale: float, rows, threads: int = 0) -> np.ndarray:
    return lib().attention_rows_packed_bf16(qkv_bits, scale, rows, threads)


def layernorm_bf16(x_bits, gamma_bits, beta_bits, eps: float, threads: int = 0) -> np.ndarray:
    return lib().layernorm_bf16(x_bits, gamma_bits, beta_bits, eps, threads)


def linear_bf16(x_bits, w_bits, bias_bits=None, res_bits=None, threads: int = 0) -> np.ndarray:
    return lib().linear_bf16(x_bits, w_bits, bias_bits, res_bits, threads)


def round_bf16(v) -> np.ndarray:
    return lib().round_bf16(v)


def add_layernorm_bf16(x_bits, r_bits, gamma_bits, beta_bits, eps: float, threads: int = 0):
    return lib().add_layernorm_bf16(x_bits, r_bits, gamma_bits, beta_bits, eps, threads)


def linear_gelu_bf16(x_bits, w_bits, bias_bits=None, threads: int = 0) -> np.ndarray:
    return lib().linear_gelu_bf16(x_bits, w_bits, bias_bits, threads)


SOURCE = _build.SRC

__all__ = ["OracleLib", "lib", "attention_f64", "probs_f64", "attention_packed_bf16",
           "attention_rows_packed_bf16", "layernorm_bf16", "linear_bf16", "round_bf16",
           "add_layernorm_bf16", "linear_gelu_bf16", "default_threads",
           "SOURCE"]
