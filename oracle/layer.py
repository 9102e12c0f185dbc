"""Plain float64 forward and backward of a Qwen2.5-style decoder layer stack.

TEST INFRASTRUCTURE ONLY (see the package docstring). Nothing here is called
by the product path.

Source of the computation. The MegaTrain pages ("MegaTrain: Full Precision
Training of 100B+ Parameter Large Language Models on a Single GPU", the
listing page's Table 2) train Qwen2.5-7B/14B/32B/72B models but never write the
decoder block out. This oracle takes the plainest reading that the rest of the
pages and the model family support:

    h1 = RMSNorm(x; g1)                      pre-norm, eps inside the root
    q, k, v = h1 Wq^T + bq, h1 Wk^T + bk, h1 Wv^T + bv   (bias on QKV only)
    q, k = RoPE(q), RoPE(k)                  rotate-half pairs (i, i + d/2)
    o_h = softmax(q_h k_c^T / sqrt(d), causal) v_c,  c = floor(h * nkv / nq)
    x2 = x + concat_h(o_h) Wo^T              no output bias
    h2 = RMSNorm(x2; g2)
    y = x2 + (silu(h2 Wg^T) * (h2 Wu^T)) Wd^T

The backward is the explicit adjoint of each of those steps, with every
weight and bias gradient summed over all B*T tokens. The stack's loss is
sum(Y * dY), so dY is the top cotangent. parity pinned: see
tests/test_oracle_pins.py (finite differences, brute-force attention, RoPE and
RMSNorm closed forms and invariants, special cases).

Everything is computed in float64 (``dtype`` may be set to float32 for
timing only). Inputs are the bf16 values of the weights, x and dY, upcast.
Matrix products use numpy's matmul; nothing is tiled, fused or reordered.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class OracleCfg:
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    qkv_bias: bool = True
    rms_eps: float = 1e-6
    rope_theta: float = 1e6


# ---------------------------------------------------------------- RMSNorm
def rmsnorm_fwd(x: np.ndarray, g: np.ndarray, eps: float):
    """y = x / sqrt(mean_j x_j^2 + eps) * g over the last axis.

    Returns (y, rstd) with rstd = 1 / sqrt(mean x^2 + eps) per row.
    """
    ms = np.mean(x * x, axis=-1, keepdims=True)
    rstd = 1.0 / np.sqrt(ms + eps)
    return x * rstd * g, rstd[..., 0]


def rmsnorm_bwd(dy: np.ndarray, x: np.ndarray, g: np.ndarray, rstd: np.ndarray):
    """Adjoint of :func:`rmsnorm_fwd`.

    With xh = x * rstd: dx = rstd * (g*dy - xh * mean_j(xh_j * g_j * dy_j)),
    dg = sum over rows of dy * xh.
    """
    r = rstd[..., None]
    xh = x * r
    gdy = g * dy
    dx = r * (gdy - xh * np.mean(xh * gdy, axis=-1, keepdims=True))
    dg = np.sum((dy * xh).reshape(-1, x.shape[-1]), axis=0)
    return dx, dg


# ---------------------------------------------------------------- RoPE
def rope_tables(T: int, d: int, theta: float, dtype=np.float64):
    """cos/sin of angle t * theta^(-2i/d) for t < T, i < d/2 (shape [T, d/2]).

    Angles are formed in float64 whatever ``dtype`` is.
    """
    i = np.arange(d // 2, dtype=np.float64)
    omega = theta ** (-2.0 * i / d)
    ang = np.arange(T, dtype=np.float64)[:, None] * omega[None, :]
    return np.cos(ang).astype(dtype), np.sin(ang).astype(dtype)


def rope_apply(u: np.ndarray, cos: np.ndarray, sin: np.ndarray, inverse: bool = False):
    """Rotate-half RoPE on u of shape [B, T, heads, d].

    Pair (u_i, u_{i+d/2}) becomes (u_i cos a - u_{i+d/2} sin a,
    u_{i+d/2} cos a + u_i sin a). ``inverse`` rotates by -a, which is also the
    adjoint (the rotation is orthogonal), so it serves as the RoPE backward.
    """
    h = u.shape[-1] // 2
    c = cos[None, :, None, :]
    s = -sin[None, :, None, :] if inverse else sin[None, :, None, :]
    a, b = u[..., :h], u[..., h:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


# ---------------------------------------------------------------- attention
def _kv_head(h: int, nq: int, nkv: int) -> int:
    return (h * nkv) // nq


def attention_fwd(q: np.ndarray, k: np.ndarray, v: np.ndarray):
    """Causal grouped-query softmax attention.

    q [B,T,nq,d], k and v [B,T,nkv,d]. For query head h the key/value head is
    c = floor(h*nkv/nq) (contiguous groups). s_tu = q_t . k_u / sqrt(d) for
    u <= t, p = softmax_u(s) with the row maximum subtracted, o_t = sum_u p_tu v_u.
    Returns (o [B,T,nq,d], lse [B,nq,T]) with lse_t = log sum_u exp(s_tu).
    """
    B, T, nq, d = q.shape
    nkv = k.shape[2]
    scale = 1.0 / np.sqrt(d)
    mask = np.triu(np.ones((T, T), dtype=bool), k=1)  # u > t is masked
    o = np.empty_like(q)
    lse = np.empty((B, nq, T), dtype=q.dtype)
    for b in range(B):
        for h in range(nq):
            c = _kv_head(h, nq, nkv)
            s = (q[b, :, h, :] @ k[b, :, c, :].T) * scale
            s = np.where(mask, -np.inf, s)
            m = np.max(s, axis=1, keepdims=True)
            e = np.exp(s - m)
            l = np.sum(e, axis=1, keepdims=True)
            o[b, :, h, :] = (e / l) @ v[b, :, c, :]
            lse[b, h, :] = (m + np.log(l))[:, 0]
    return o, lse


def attention_bwd(do: np.ndarray, q: np.ndarray, k: np.ndarray, v: np.ndarray,
                  o: np.ndarray, lse: np.ndarray):
    """Adjoint of :func:`attention_fwd`.

    P = exp(S - lse); dV = P^T dO; dP = dO V^T; D = rowsum(dO * O);
    dS = P * (dP - D); dQ = dS K / sqrt(d); dK = dS^T Q / sqrt(d). The
    query heads of a group add into their shared key/value head.
    """
    B, T, nq, d = q.shape
    nkv = k.shape[2]
    scale = 1.0 / np.sqrt(d)
    mask = np.triu(np.ones((T, T), dtype=bool), k=1)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(nq):
            c = _kv_head(h, nq, nkv)
            s = (q[b, :, h, :] @ k[b, :, c, :].T) * scale
            p = np.where(mask, 0.0, np.exp(s - lse[b, h, :, None]))
            dv[b, :, c, :] += p.T @ do[b, :, h, :]
            dp = do[b, :, h, :] @ v[b, :, c, :].T
            D = np.sum(do[b, :, h, :] * o[b, :, h, :], axis=1, keepdims=True)
            ds = p * (dp - D)
            dq[b, :, h, :] = (ds @ k[b, :, c, :]) * scale
            dk[b, :, c, :] += (ds.T @ q[b, :, h, :]) * scale
    return dq, dk, dv


# ---------------------------------------------------------------- SwiGLU
def _sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def swiglu_fwd(g: np.ndarray, u: np.ndarray):
    """m = silu(g) * u with silu(z) = z * sigmoid(z)."""
    return g * _sigmoid(g) * u


def swiglu_bwd(dm: np.ndarray, g: np.ndarray, u: np.ndarray):
    """dg = dm * u * sigmoid(g) * (1 + g * (1 - sigmoid(g))), du = dm * silu(g)."""
    sg = _sigmoid(g)
    dg = dm * u * sg * (1.0 + g * (1.0 - sg))
    du = dm * g * sg
    return dg, du


# ---------------------------------------------------------------- layer
def _lin(x, w, b=None):
    y = x @ w.T
    return y if b is None else y + b


def layer_fwd(cfg: OracleCfg, w: dict, x: np.ndarray):
    """Forward of one layer on x [B,T,H]; returns (y, cache for layer_bwd)."""
    B, T, H = x.shape
    nq, nkv, d = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim
    h1, rstd1 = rmsnorm_fwd(x, w["g1"], cfg.rms_eps)
    q = _lin(h1, w["wq"], w.get("bq")).reshape(B, T, nq, d)
    k = _lin(h1, w["wk"], w.get("bk")).reshape(B, T, nkv, d)
    v = _lin(h1, w["wv"], w.get("bv")).reshape(B, T, nkv, d)
    cos, sin = rope_tables(T, d, cfg.rope_theta, x.dtype)
    qr, kr = rope_apply(q, cos, sin), rope_apply(k, cos, sin)
    o, lse = attention_fwd(qr, kr, v)
    o2 = o.reshape(B, T, nq * d)
    x2 = x + _lin(o2, w["wo"])
    h2, rstd2 = rmsnorm_fwd(x2, w["g2"], cfg.rms_eps)
    gt = _lin(h2, w["wg"])
    ut = _lin(h2, w["wu"])
    m = swiglu_fwd(gt, ut)
    y = x2 + _lin(m, w["wd"])
    cache = dict(x=x, h1=h1, rstd1=rstd1, qr=qr, kr=kr, v=v, o=o, o2=o2, lse=lse,
                 x2=x2, h2=h2, rstd2=rstd2, g=gt, u=ut, m=m, cos=cos, sin=sin)
    return y, cache


def _wgrad(dy2d, x2d):
    """dW = dY^T X summed over every token row."""
    return dy2d.T @ x2d


def layer_bwd(cfg: OracleCfg, w: dict, cache: dict, dy: np.ndarray):
    """Adjoint of :func:`layer_fwd`; returns (dx, grads dict keyed like w)."""
    B, T, H = dy.shape
    nq, nkv, d = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim
    M = B * T
    c = cache
    gr = {}
    # y = x2 + m Wd^T
    dy2 = dy.reshape(M, H)
    gr["wd"] = _wgrad(dy2, c["m"].reshape(M, -1))
    dm = dy @ w["wd"]
    dg, du = swiglu_bwd(dm, c["g"], c["u"])
    gr["wg"] = _wgrad(dg.reshape(M, -1), c["h2"].reshape(M, H))
    gr["wu"] = _wgrad(du.reshape(M, -1), c["h2"].reshape(M, H))
    dh2 = dg @ w["wg"] + du @ w["wu"]
    dx2n, gr["g2"] = rmsnorm_bwd(dh2, c["x2"], w["g2"], c["rstd2"])
    dx2 = dy + dx2n
    # x2 = x + o2 Wo^T
    gr["wo"] = _wgrad(dx2.reshape(M, H), c["o2"].reshape(M, -1))
    do = (dx2 @ w["wo"]).reshape(B, T, nq, d)
    dqr, dkr, dv = attention_bwd(do, c["qr"], c["kr"], c["v"], c["o"], c["lse"])
    dq = rope_apply(dqr, c["cos"], c["sin"], inverse=True).reshape(B, T, nq * d)
    dk = rope_apply(dkr, c["cos"], c["sin"], inverse=True).reshape(B, T, nkv * d)
    dv = dv.reshape(B, T, nkv * d)
    h1 = c["h1"].reshape(M, H)
    gr["wq"] = _wgrad(dq.reshape(M, -1), h1)
    gr["wk"] = _wgrad(dk.reshape(M, -1), h1)
    gr["wv"] = _wgrad(dv.reshape(M, -1), h1)
    if cfg.qkv_bias:
        gr["bq"] = dq.reshape(M, -1).sum(axis=0)
        gr["bk"] = dk.reshape(M, -1).sum(axis=0)
        gr["bv"] = dv.reshape(M, -1).sum(axis=0)
    dh1 = dq @ w["wq"] + dk @ w["wk"] + dv @ w["wv"]
    dxn, gr["g1"] = rmsnorm_bwd(dh1, c["x"], w["g1"], c["rstd1"])
    dx = dx2 + dxn
    return dx, gr


def stack_fwd_bwd(cfg: OracleCfg, ws: list, x0: np.ndarray, dy: np.ndarray):
    """Full-activation forward then backward of len(ws) layers.

    x_{l+1} = layer_l(x_l); loss = sum(Y * dY). Returns (Y, dX0, [grads_l]).
    """
    caches = []
    x = x0
    for w in ws:
        x, cache = layer_fwd(cfg, w, x)
        caches.append(cache)
    y = x
    g = dy
    grads = [None] * len(ws)
    for l in range(len(ws) - 1, -1, -1):
        g, grads[l] = layer_bwd(cfg, ws[l], caches[l], g)
    return y, g, grads
