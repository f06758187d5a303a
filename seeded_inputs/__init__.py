"""Seeded synthetic inputs for the ViT/SigLIP self-attention core.

This module is shared by the fp64 oracle's tests and by the CUDA path's tests
and bench, and it holds none of the attention arithmetic: it only turns a seed
into the packed ``[B, N, 3, H, d]`` bf16 QKV buffer that a ViT block's ``qkv``
linear would emit (Flash Attention tutorial for the Pi0 VLA, section 3.2: the
encoder's ``block.attn.qkv`` feeds multi-head attention).

Generator (defined here, counter-based, so any element can be regenerated on
its own):

* ``gamma = 0x9E3779B97F4A7C15``; the k-th 64-bit draw for a seed is the
  splitmix64 finaliser applied to ``seed + (k + 1) * gamma`` (mod 2**64).
* Element ``e`` (flat index in memory order of ``[B, N, 3, H, d]``) belongs to
  pair ``p = e // 2``; draws ``2p`` and ``2p + 1`` give
  ``u1 = ((a >> 11) + 1) * 2**-53`` in (0, 1] and ``u2 = (b >> 11) * 2**-53``.
* Box-Muller in fp64: ``r = sqrt(-2 ln u1)``; even ``e`` takes
  ``r cos(2 pi u2)``, odd ``e`` takes ``r sin(2 pi u2)``.
* The value is multiplied by the slot's standard deviation (Q, K slots and the
  V slot may differ), rounded to fp32 (round to nearest even) and then to bf16
  (round to nearest even on the fp32 bit pattern).

The result is returned as ``uint16`` bf16 bit patterns so that every consumer
sees the identical bytes.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_TWO_M53 = 2.0 ** -53

__all__ = [
    "AttnConfig",
    "WORKLOADS",
    "ENCODER_WORKLOADS",
    "VIT_B16_112PX_1VIEW",
    "VIT_B16_224PX_3VIEWS",
    "VIT_L14_224PX_3VIEWS",
    "SIGLIP_SO400M14_224PX_2VIEWS",
    "VIT_L14_336PX_B256",
    "workload",
    "call_seed",
    "splitmix64_draws",
    "normals",
    "packed_qkv",
    "bf16_bits_to_f32",
    "f32_to_bf16_bits",
]


def splitmix64_draws(seed: int, start: int, count: int) -> np.ndarray:
    """Draws ``start .. start+count-1`` of the counter-based splitmix64 stream."""
    k = np.arange(start, start + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + (k + np.uint64(1)) * _GAMMA
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        z = z ^ (z >> np.uint64(31))
    return z


def normals(seed: int, start: int, count: int) -> np.ndarray:
    """Standard normal fp64 values for flat element indices ``start .. start+count-1``."""
    if count <= 0:
        return np.zeros(0, dtype=np.float64)
    p0 = start // 2
    p1 = (start + count - 1) // 2
    npairs = p1 - p0 + 1
    draws = splitmix64_draws(seed, 2 * p0, 2 * npairs)
    a = draws[0::2]
    b = draws[1::2]
    u1 = ((a >> np.uint64(11)).astype(np.float64) + 1.0) * _TWO_M53
    u2 = (b >> np.uint64(11)).astype(np.float64) * _TWO_M53
    r = np.sqrt(-2.0 * np.log(u1))
    th = 2.0 * math.pi * u2
    z = np.empty(2 * npairs, dtype=np.float64)
    z[0::2] = r * np.cos(th)
    z[1::2] = r * np.sin(th)
    off = start - 2 * p0
    return z[off:off + count]


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest even) and return the bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    return (u >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 exactly."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16(seed: int, shape, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    """bf16 bit patterns (``uint16``, given shape) of ``mean + std * N(0, 1)`` draws from the
    counter-based generator, in memory order (fp64 draw, fp32 scale, bf16 round)."""
    count = int(np.prod(shape))
    z = normals(seed, 0, count)
    v = (np.float64(mean) + np.float64(std) * z).astype(np.float32)
    return f32_to_bf16_bits(v).reshape(shape)


def _fill_chunk(out: np.ndarray, seed: int, start: int, count: int, H: int, d: int,
                sigma_qk: float, sigma_v: float) -> None:
    z = normals(seed, start, count)
    if sigma_qk != 1.0 or sigma_v != 1.0:
        e = np.arange(start, start + count, dtype=np.int64)
        slot = (e // (H * d)) % 3
        sig = np.where(slot == 2, sigma_v, sigma_qk)
        z = z * sig
    out[start:start + count] = f32_to_bf16_bits(z.astype(np.float32))


def packed_qkv(B: int, N: int, H: int, d: int, seed: int,
               sigma_qk: float = 1.0, sigma_v: float = 1.0,
               threads: int | None = None) -> np.ndarray:
    """Packed ``[B, N, 3, H, d]`` bf16 bit patterns (``uint16``) for ``seed``."""
    total = B * N * 3 * H * d
    flat = np.empty(total, dtype=np.uint16)
    chunk = 1 << 22
    starts = list(range(0, total, chunk))
    if threads is None:
        threads = min(32, os.cpu_count() or 1)
    if len(starts) <= 1 or threads <= 1:
        for s in starts:
            _fill_chunk(flat, seed, s, min(chunk, total - s), H, d, sigma_qk, sigma_v)
    else:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(lambda s: _fill_chunk(flat, seed, s, min(chunk, total - s), H, d,
                                              sigma_qk, sigma_v), starts))
    return flat.reshape(B, N, 3, H, d)


@dataclass(frozen=True)
class AttnConfig:
    """One workload shape of the attention core.

    ``layers`` is the encoder depth used to turn one call's time into images/s;
    ``calls`` is how many independently seeded calls the workload defines.
    """
    index: int
    name: str
    B: int
    N: int
    H: int
    d: int
    scale: float
    sigma_qk: float
    sigma_v: float
    calls: int
    layers: int

    def seed(self, call: int) -> int:
        return call_seed(self.index, call)

    def flops(self) -> int:
        return 4 * self.B * self.H * self.N * self.N * self.d

    def bytes(self) -> int:
        return 8 * self.B * self.N * self.H * self.d

    def qkv(self, call: int = 0, threads: int | None = None) -> np.ndarray:
        return packed_qkv(self.B, self.N, self.H, self.d, self.seed(call),
                          self.sigma_qk, self.sigma_v, threads)


def call_seed(config_index: int, call: int) -> int:
    """Seed of call ``call`` of config ``config_index`` (the 112x112 case is seed 0)."""
    if config_index == 1:
        return 0 if call == 0 else 1000 + call
    return 1000 * config_index + call


WORKLOADS = (
    # ViT-B/16 at 112x112, one camera view: 49 patches + CLS.
    AttnConfig(1, "vit_b16_112px_1view", 1, 50, 12, 64, 1.0 / 8.0, 1.0, 1.0, 1, 12),
    # ViT-B/16 at 224x224, three camera views (Main/Side/Top), 12 layers.
    AttnConfig(2, "vit_b16_224px_3views", 3, 197, 12, 64, 1.0 / math.sqrt(64), 1.0, 1.0, 12, 12),
    # ViT-L/14 at 224x224, three views, 24 layers.
    AttnConfig(3, "vit_l14_224px_3views", 3, 257, 16, 64, 1.0 / math.sqrt(64), 1.0, 1.0, 24, 24),
    # SigLIP-So400m/14 at 224x224, two views, width 1152 = 16 x 72, 27 layers;
    # Q and K drawn with variance 2 for a peaked softmax.
    AttnConfig(4, "siglip_so400m14_224px_2views", 2, 256, 16, 72, 1.0 / math.sqrt(72),
               math.sqrt(2.0), 1.0, 27, 27),
    # ViT-L/14 at 336x336 (576 patches + CLS), 256 images per call.
    AttnConfig(5, "vit_l14_336px_b256", 256, 577, 16, 64, 1.0 / math.sqrt(64), 1.0, 1.0, 1, 24),
)


(VIT_B16_112PX_1VIEW, VIT_B16_224PX_3VIEWS, VIT_L14_224PX_3VIEWS, SIGLIP_SO400M14_224PX_2VIEWS,
 VIT_L14_336PX_B256) = WORKLOADS
# The camera-view encoder workloads (µs-scale calls, many layers per image batch).
ENCODER_WORKLOADS = WORKLOADS[:4]


def workload(name: str) -> AttnConfig:
    """The workload with this name (``vit_l14_336px_b256`` and so on)."""
    for c in WORKLOADS:
        if c.name == name:
            return c
    raise KeyError(name)
