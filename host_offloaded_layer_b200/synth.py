"""Seeded synthetic inputs for the layer stack (weights, activations, cotangents).

This module is the only code shared by the CUDA path, the benchmark and the
CPU oracle's tests. It holds no arithmetic of the method itself: it draws
counter-based normal variates and rounds them to bf16, nothing else.

Generator (stated here so any implementation can reproduce it bit for bit):

* ``mix64`` is the SplitMix64 output function (Steele, Lea, Flood,
  "Fast splittable pseudorandom number generators", OOPSLA 2014):
  ``z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27; z *= 0x94D049BB133111EB;
  z ^= z >> 31`` on uint64 with wrap-around.
* A tensor stream is keyed by ``(seed, layer, tensor_id)``:
  ``key = mix64(mix64(seed + GOLDEN) ^ ((layer + 1) << 20 | tensor_id))``.
* Element ``i`` draws ``w = mix64(key + (i + 1) * GOLDEN)`` (GOLDEN =
  0x9E3779B97F4A7C15), splits it into ``hi = w >> 32`` and ``lo = w & 0xffffffff``,
  forms ``u1 = (hi + 0.5) / 2**32`` and ``u2 = (lo + 0.5) / 2**32`` and returns the
  Box-Muller normal ``sqrt(-2 ln u1) * cos(2 pi u2)`` in float64, scaled by ``std``
  and rounded to float32 (round to nearest even).
* bf16 values are the float32 values rounded to nearest even on the upper 16 bits.

Weight recipe (Qwen2.5-style block, one record per layer): every matrix and
bias is N(0, 0.02); the two RMSNorm gains are exactly 1. Activations ``x0``
and the output cotangent ``dY`` are N(0, 1). Default seed 1234.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
DEFAULT_SEED = 1234
WEIGHT_STD = 0.02

# tensor ids of one layer record, in record order
TENSOR_IDS = {
    "g1": 0, "wq": 1, "wk": 2, "wv": 3, "bq": 4, "bk": 5, "bv": 6,
    "wo": 7, "g2": 8, "wg": 9, "wu": 10, "wd": 11,
}
X0_ID = 100
DY_ID = 101


def _mix64(z: np.ndarray) -> np.ndarray:
    z = z ^ (z >> np.uint64(30))
    z = z * _M1
    z = z ^ (z >> np.uint64(27))
    z = z * _M2
    return z ^ (z >> np.uint64(31))


def _mix64_scalar(z: int) -> int:
    m = (1 << 64) - 1
    z &= m
    z ^= z >> 30
    z = (z * 0xBF58476D1CE4E5B9) & m
    z ^= z >> 27
    z = (z * 0x94D049BB133111EB) & m
    return z ^ (z >> 31)


def stream_key(seed: int, layer: int, tensor_id: int) -> int:
    m = (1 << 64) - 1
    a = _mix64_scalar((seed + 0x9E3779B97F4A7C15) & m)
    return _mix64_scalar(a ^ ((((layer + 1) & 0xFFFFFFFF) << 20) | tensor_id))


def _normal_chunk(key: int, start: int, stop: int, std: float) -> np.ndarray:
    with np.errstate(over="ignore"):
        idx = np.arange(start + 1, stop + 1, dtype=np.uint64)
        w = _mix64(np.uint64(key) + idx * GOLDEN)
    hi = (w >> np.uint64(32)).astype(np.float64)
    lo = (w & np.uint64(0xFFFFFFFF)).astype(np.float64)
    u1 = (hi + 0.5) * (1.0 / 4294967296.0)
    u2 = (lo + 0.5) * (1.0 / 4294967296.0)
    z = np.sqrt(-2.0 * np.log(u1)) * np.cos((2.0 * np.pi) * u2)
    return (z * std).astype(np.float32)


_POOL: ThreadPoolExecutor | None = None


def _pool() -> ThreadPoolExecutor:
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max_workers=max(1, min(32, os.cpu_count() or 1)))
    return _POOL


def normal_f32(seed: int, layer: int, tensor_id: int, n: int, std: float = 1.0,
               out: np.ndarray | None = None) -> np.ndarray:
    """``n`` float32 normals N(0, std^2) of stream (seed, layer, tensor_id)."""
    key = stream_key(seed, layer, tensor_id)
    if out is None:
        out = np.empty(n, dtype=np.float32)
    chunk = 1 << 22
    if n <= chunk:
        out[:n] = _normal_chunk(key, 0, n, std)
        return out

    def work(s):
        e = min(n, s + chunk)
        out[s:e] = _normal_chunk(key, s, e, std)

    list(_pool().map(work, range(0, n, chunk)))
    return out


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    with np.errstate(over="ignore"):
        r = (u + rounding) >> np.uint32(16)
    nan = (u & np.uint32(0x7FFFFFFF)) > np.uint32(0x7F800000)
    r = np.where(nan, (u >> np.uint32(16)) | np.uint32(0x40), r)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """float32 values rounded to the nearest bf16 value (returned as float32)."""
    return bf16_bits_to_f32(f32_to_bf16_bits(x))


def layer_tensor_shapes(hidden: int, n_q_heads: int, n_kv_heads: int, head_dim: int,
                        ffn: int, qkv_bias: bool = True) -> dict[str, tuple[int, ...]]:
    """Shapes of one layer's tensors, nn.Linear style W[out, in]."""
    hq, hkv = n_q_heads * head_dim, n_kv_heads * head_dim
    shapes = {
        "g1": (hidden,), "wq": (hq, hidden), "wk": (hkv, hidden), "wv": (hkv, hidden),
        "bq": (hq,), "bk": (hkv,), "bv": (hkv,),
        "wo": (hidden, hq), "g2": (hidden,),
        "wg": (ffn, hidden), "wu": (ffn, hidden), "wd": (hidden, ffn),
    }
    if not qkv_bias:
        for k in ("bq", "bk", "bv"):
            shapes.pop(k)
    return shapes


def layer_weights_f32(shapes: dict[str, tuple[int, ...]], seed: int, layer: int,
                      std: float = WEIGHT_STD) -> dict[str, np.ndarray]:
    """fp32 master values of one layer: N(0, std^2) matrices and biases, gains 1."""
    out = {}
    for name, shp in shapes.items():
        n = int(np.prod(shp))
        if name in ("g1", "g2"):
            out[name] = np.ones(shp, dtype=np.float32)
        else:
            out[name] = normal_f32(seed, layer, TENSOR_IDS[name], n, std).reshape(shp)
    return out


def activations_bf16_bits(seed: int, which: int, B: int, T: int, H: int) -> np.ndarray:
    """x0 (``which=X0_ID``) or dY (``which=DY_ID``) as bf16 bits, shape [B, T, H]."""
    return f32_to_bf16_bits(normal_f32(seed, -1, which, B * T * H, 1.0)).reshape(B, T, H)
