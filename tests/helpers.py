"""Shared helpers of the GPU parity tests (inputs, device transfer, error metric)."""
from __future__ import annotations

import numpy as np

from host_offloaded_layer_b200 import _lib as L
from host_offloaded_layer_b200 import synth

TOL = 2e-2  # relative Frobenius error per tensor (bf16 operands, fp32 accumulation)


def branch_tol(x, y_ref) -> float:
    """Error budget of a residual branch (Y - X) when the residual stream is stored in bf16.

    The GPU stores the layer's two residual sums (x2 and y) as bf16. The error of
    rounding the oracle's own Y to bf16, e_r = ||bf16(Y) - Y||, measures one such
    rounding; two of them, with a factor 2 of slack each, are allowed on top of
    the parity tolerance, relative to the branch ||Y - X||."""
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y_ref, dtype=np.float64)
    e_r = np.linalg.norm(synth.bf16_round(y.astype(np.float32)).astype(np.float64) - y)
    return TOL + 4.0 * e_r / max(np.linalg.norm(y - x), 1e-30)


def rel(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def dev_bf16(bits: np.ndarray):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy())
    return t.view(torch.bfloat16).cuda()


def dev_f32(arr: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32)).cuda()


def host_f64(t) -> np.ndarray:
    import torch
    if t.dtype == torch.bfloat16:
        return bits_to_f64(t.view(torch.int16).cpu().numpy().view(np.uint16))
    return t.detach().cpu().numpy().astype(np.float64)


def empty_bf16(*shape):
    import torch
    return torch.empty(*shape, dtype=torch.bfloat16, device="cuda")


def empty_f32(*shape):
    import torch
    return torch.empty(*shape, dtype=torch.float32, device="cuda")


def workspace(nbytes: int):
    import torch
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device="cuda")


def shape_dict(cfg) -> dict:
    return dict(hidden=cfg.hidden, n_q_heads=cfg.n_q_heads, n_kv_heads=cfg.n_kv_heads, head_dim=cfg.head_dim,
                ffn=cfg.ffn, qkv_bias=bool(cfg.qkv_bias))


def layer_record(cfg, seed: int, layer: int, std: float = synth.WEIGHT_STD, gain_std: float = 0.0):
    """(bf16 record bits, {name: float64 bf16 values}) of one layer.

    Matrices and biases are the synthetic N(0, std) draws; gains are 1, or
    1 + N(0, gain_std) when gain_std > 0 (to exercise the gain gradients)."""
    shapes = synth.layer_tensor_shapes(**shape_dict(cfg))
    f32 = synth.layer_weights_f32(shapes, seed, layer, std)
    if gain_std > 0:
        for i, g in enumerate(("g1", "g2")):
            f32[g] = (1.0 + synth.normal_f32(seed, layer, 50 + i, shapes[g][0], gain_std)).astype(np.float32)
    off = L.mt_layer_param_offsets(cfg)
    rec = np.zeros(off.record_elems, dtype=np.uint16)
    w64 = {}
    for name, arr in f32.items():
        bits = synth.f32_to_bf16_bits(arr.ravel())
        o = getattr(off, name)
        rec[o:o + bits.size] = bits
        w64[name] = bits_to_f64(bits).reshape(arr.shape)
    return rec, w64


def grads_from_record(cfg, rec_f32: np.ndarray) -> dict:
    off = L.mt_layer_param_offsets(cfg)
    shapes = synth.layer_tensor_shapes(**shape_dict(cfg))
    out = {}
    for name, shp in shapes.items():
        o = getattr(off, name)
        n = int(np.prod(shp))
        out[name] = np.asarray(rec_f32[o:o + n], dtype=np.float64).reshape(shp)
    return out


def oracle_cfg(cfg):
    from oracle import OracleCfg
    return OracleCfg(hidden=cfg.hidden, n_q_heads=cfg.n_q_heads, n_kv_heads=cfg.n_kv_heads, head_dim=cfg.head_dim,
                     ffn=cfg.ffn, qkv_bias=bool(cfg.qkv_bias), rms_eps=float(np.float32(cfg.rms_eps)),
                     rope_theta=float(np.float32(cfg.rope_theta)))
