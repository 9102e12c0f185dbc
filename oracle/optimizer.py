"""Plain float64 AdamW, the CPU optimizer step of the memory-centric design.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The blog summary of MegaTrain (design point 1) keeps Adam momentum and
variance in host memory and runs the optimizer step entirely on the CPU. The
update is AdamW with decoupled weight decay (Loshchilov and Hutter,
"Decoupled Weight Decay Regularization", ICLR 2019, Algorithm 2, with the
schedule multiplier fixed at 1):

    m = b1 m + (1 - b1) g
    v = b2 v + (1 - b2) g^2
    w = w - lr * (m / (1 - b1^t) / (sqrt(v / (1 - b2^t)) + eps) + wd * w)

parity pinned: tests/test_oracle_pins.py (first step from zero state,
zero gradient, constant gradient).
"""
from __future__ import annotations

import numpy as np


def adamw_step(w, m, v, g, t, lr, beta1, beta2, eps, weight_decay):
    """Returns (w, m, v) after step t (t >= 1)."""
    w = np.asarray(w, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    m = beta1 * np.asarray(m, dtype=np.float64) + (1.0 - beta1) * g
    v = beta2 * np.asarray(v, dtype=np.float64) + (1.0 - beta2) * g * g
    m_hat = m / (1.0 - beta1 ** t)
    v_hat = v / (1.0 - beta2 ** t)
    w = w - lr * (m_hat / (np.sqrt(v_hat) + eps) + weight_decay * w)
    return w, m, v
