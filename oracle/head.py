"""Plain float64 embedding, final RMSNorm, LM head and cross-entropy.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The MegaTrain pages count the embedding and the LM head in the model's
parameters (Table 5's totals reproduce only with them) but do not write them
out; the plainest reading for the Qwen2.5 family (Table 2) is an untied
embedding E [V, H], a final RMSNorm with gain gf, an LM head W [V, H] and the
mean token cross-entropy against the next-token targets:

    x0 = E[tokens];  h = RMSNorm(y; gf);  z = h W^T
    loss = mean_t (logsumexp_v z_tv - z_t,target_t)

with the adjoints dz = (softmax(z) - onehot(target)) / n_tokens,
dW = dz^T h, dh = dz W, and dE[v] = sum of dx0 over the tokens equal to v.
parity pinned: tests/test_oracle_pins.py (finite differences, closed forms).
"""
from __future__ import annotations

import numpy as np

from .layer import rmsnorm_bwd, rmsnorm_fwd


def embed_fwd(tokens: np.ndarray, E: np.ndarray) -> np.ndarray:
    """x0[b, t] = E[tokens[b, t]]."""
    return E[tokens]


def embed_bwd(tokens: np.ndarray, dx0: np.ndarray, vocab: int) -> np.ndarray:
    """dE[v] = sum of dx0[b, t] over the (b, t) with tokens[b, t] == v."""
    H = dx0.shape[-1]
    dE = np.zeros((vocab, H), dtype=dx0.dtype)
    np.add.at(dE, tokens.reshape(-1), dx0.reshape(-1, H))
    return dE


def head_loss_fwd_bwd(y: np.ndarray, gf: np.ndarray, W: np.ndarray, targets: np.ndarray, eps: float):
    """Mean cross-entropy of the LM head on the stack output y [B, T, H].

    Returns (loss, dy, dgf, dW)."""
    B, T, H = y.shape
    n = B * T
    h, rstd = rmsnorm_fwd(y, gf, eps)
    z = h.reshape(n, H) @ W.T
    zmax = z.max(axis=1, keepdims=True)
    lse = (zmax + np.log(np.exp(z - zmax).sum(axis=1, keepdims=True)))[:, 0]
    tgt = targets.reshape(-1)
    loss = float(np.mean(lse - z[np.arange(n), tgt]))
    dz = np.exp(z - lse[:, None])
    dz[np.arange(n), tgt] -= 1.0
    dz /= n
    dW = dz.T @ h.reshape(n, H)
    dh = (dz @ W).reshape(B, T, H)
    dy, dgf = rmsnorm_bwd(dh, y, gf, rstd)
    return loss, dy, dgf, dW
