"""Pins of the CPU oracle to facts other than itself (no GPU needed).

Each test checks the oracle against a closed form, an invariant, a
brute-force loop written separately here, or central finite differences, so
that a dropped term, a wrong sign or index, or a transposed operand anywhere
in oracle/layer.py fails at least one of them.
"""
import math

import numpy as np
import pytest

from oracle import layer as O

TINY = O.OracleCfg(hidden=16, n_q_heads=4, n_kv_heads=2, head_dim=4, ffn=24,
                   qkv_bias=True, rms_eps=1e-6, rope_theta=1e4)


def _weights(cfg, rng, gains_random=True):
    H, hq, hkv, F = cfg.hidden, cfg.n_q_heads * cfg.head_dim, cfg.n_kv_heads * cfg.head_dim, cfg.ffn
    w = {
        "g1": 1.0 + 0.3 * rng.standard_normal(H) if gains_random else np.ones(H),
        "wq": 0.3 * rng.standard_normal((hq, H)),
        "wk": 0.3 * rng.standard_normal((hkv, H)),
        "wv": 0.3 * rng.standard_normal((hkv, H)),
        "bq": 0.2 * rng.standard_normal(hq),
        "bk": 0.2 * rng.standard_normal(hkv),
        "bv": 0.2 * rng.standard_normal(hkv),
        "wo": 0.3 * rng.standard_normal((H, hq)),
        "g2": 1.0 + 0.3 * rng.standard_normal(H) if gains_random else np.ones(H),
        "wg": 0.3 * rng.standard_normal((F, H)),
        "wu": 0.3 * rng.standard_normal((F, H)),
        "wd": 0.3 * rng.standard_normal((H, F)),
    }
    return w


def _loss_stack(cfg, ws, x, dy):
    for w in ws:
        x, _ = O.layer_fwd(cfg, w, x)
    return float(np.sum(x * dy))


# ------------------------------------------------------------ finite differences
@pytest.mark.parametrize("n_layers", [1, 2])
def test_backward_matches_central_differences(n_layers):
    """Every gradient of the stack equals its fp64 central difference."""
    rng = np.random.default_rng(7 + n_layers)
    B, T = 2, 5
    ws = [_weights(TINY, rng) for _ in range(n_layers)]
    x = rng.standard_normal((B, T, TINY.hidden))
    dy = rng.standard_normal((B, T, TINY.hidden))
    _, dx, grads = O.stack_fwd_bwd(TINY, ws, x, dy)
    h = 1e-6

    def check(analytic, perturb):
        v = rng.standard_normal(analytic.shape)
        lp = perturb(h * v)
        lm = perturb(-h * v)
        fd = (lp - lm) / (2 * h)
        an = float(np.sum(analytic * v))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (fd, an)

    check(dx, lambda e: _loss_stack(TINY, ws, x + e, dy))
    for li in range(n_layers):
        for name in ws[li]:
            def perturb(e, li=li, name=name):
                ws2 = [dict(w) for w in ws]
                ws2[li][name] = ws[li][name] + e
                return _loss_stack(TINY, ws2, x, dy)
            check(grads[li][name], perturb)


def test_attention_backward_matches_central_differences():
    rng = np.random.default_rng(3)
    B, T, nq, nkv, d = 2, 6, 4, 2, 4
    q = rng.standard_normal((B, T, nq, d))
    k = rng.standard_normal((B, T, nkv, d))
    v = rng.standard_normal((B, T, nkv, d))
    do = rng.standard_normal((B, T, nq, d))
    o, lse = O.attention_fwd(q, k, v)
    dq, dk, dv = O.attention_bwd(do, q, k, v, o, lse)
    h = 1e-6
    for arr, g, idx in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        e = rng.standard_normal(arr.shape)
        args_p = [q, k, v]
        args_m = [q, k, v]
        args_p[idx] = arr + h * e
        args_m[idx] = arr - h * e
        fd = (np.sum(O.attention_fwd(*args_p)[0] * do) - np.sum(O.attention_fwd(*args_m)[0] * do)) / (2 * h)
        assert abs(fd - np.sum(g * e)) < 1e-7 * max(1.0, abs(fd))


# ------------------------------------------------------------ attention
def _naive_attention(q, k, v):
    """Separately written loops: exp without max subtraction, explicit sums."""
    B, T, nq, d = q.shape
    nkv = k.shape[2]
    grp = nq // nkv
    o = np.zeros_like(q)
    lse = np.zeros((B, nq, T))
    for b in range(B):
        for h in range(nq):
            c = h // grp
            for t in range(T):
                w = [math.exp(sum(q[b, t, h, j] * k[b, u, c, j] for j in range(d)) / math.sqrt(d))
                     for u in range(t + 1)]
                z = sum(w)
                for j in range(d):
                    o[b, t, h, j] = sum(w[u] * v[b, u, c, j] for u in range(t + 1)) / z
                lse[b, h, t] = math.log(z)
    return o, lse


def test_attention_matches_bruteforce_gqa():
    rng = np.random.default_rng(11)
    q = rng.standard_normal((2, 7, 6, 4))
    k = rng.standard_normal((2, 7, 2, 4))
    v = rng.standard_normal((2, 7, 2, 4))
    o, lse = O.attention_fwd(q, k, v)
    o2, lse2 = _naive_attention(q, k, v)
    np.testing.assert_allclose(o, o2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lse2, rtol=1e-12, atol=1e-12)


def test_attention_single_token_returns_its_value_head():
    rng = np.random.default_rng(12)
    q = rng.standard_normal((3, 1, 4, 8))
    k = rng.standard_normal((3, 1, 2, 8))
    v = rng.standard_normal((3, 1, 2, 8))
    o, lse = O.attention_fwd(q, k, v)
    for h in range(4):
        np.testing.assert_allclose(o[:, 0, h], v[:, 0, h // 2], rtol=0, atol=1e-15)
        np.testing.assert_allclose(lse[:, h, 0], np.sum(q[:, 0, h] * k[:, 0, h // 2], -1) / np.sqrt(8), atol=1e-14)


def test_attention_zero_queries_give_causal_running_mean():
    """q = 0 makes every score equal: o_t is the mean of v_0..v_t of its group."""
    rng = np.random.default_rng(13)
    T = 9
    q = np.zeros((1, T, 4, 4))
    k = rng.standard_normal((1, T, 2, 4))
    v = rng.standard_normal((1, T, 2, 4))
    o, lse = O.attention_fwd(q, k, v)
    csum = np.cumsum(v, axis=1) / np.arange(1, T + 1)[None, :, None, None]
    for h in range(4):
        np.testing.assert_allclose(o[:, :, h], csum[:, :, h // 2], atol=1e-14)
        np.testing.assert_allclose(lse[0, h], np.log(np.arange(1, T + 1)), atol=1e-14)


def test_gqa_equals_mha_with_repeated_heads():
    rng = np.random.default_rng(14)
    q = rng.standard_normal((2, 6, 8, 4))
    k = rng.standard_normal((2, 6, 2, 4))
    v = rng.standard_normal((2, 6, 2, 4))
    o, _ = O.attention_fwd(q, k, v)
    o_mha, _ = O.attention_fwd(q, np.repeat(k, 4, axis=2), np.repeat(v, 4, axis=2))
    np.testing.assert_allclose(o, o_mha, atol=1e-14)


# ------------------------------------------------------------ RoPE
def test_rope_closed_form_rotates_pairs_i_and_i_plus_half():
    d, T, theta = 4, 6, 100.0
    cos, sin = O.rope_tables(T, d, theta)
    for idx, omega in ((0, 1.0), (1, 0.1)):  # omega_i = theta^(-2i/d)
        u = np.zeros((1, T, 1, d))
        u[..., idx] = 1.0
        r = O.rope_apply(u, cos, sin)
        t = np.arange(T)
        np.testing.assert_allclose(r[0, :, 0, idx], np.cos(omega * t), atol=1e-15)
        np.testing.assert_allclose(r[0, :, 0, idx + d // 2], np.sin(omega * t), atol=1e-15)
        others = [j for j in range(d) if j not in (idx, idx + d // 2)]
        assert np.all(r[0, :, 0, others] == 0.0)


def test_rope_relative_position_invariance():
    rng = np.random.default_rng(21)
    d, T, s = 8, 20, 7
    cos, sin = O.rope_tables(T + s, d, 1e4)
    qv = rng.standard_normal(d)
    kv = rng.standard_normal(d)
    u = np.tile(qv, (1, T + s, 1, 1))
    w = np.tile(kv, (1, T + s, 1, 1))
    rq, rk = O.rope_apply(u, cos, sin), O.rope_apply(w, cos, sin)
    for m, n in ((3, 1), (12, 5), (4, 4)):
        a = np.dot(rq[0, m, 0], rk[0, n, 0])
        b = np.dot(rq[0, m + s, 0], rk[0, n + s, 0])
        assert abs(a - b) < 1e-12


def test_rope_inverse_undoes_rotation():
    rng = np.random.default_rng(22)
    u = rng.standard_normal((2, 9, 3, 8))
    cos, sin = O.rope_tables(9, 8, 1e6)
    np.testing.assert_allclose(O.rope_apply(O.rope_apply(u, cos, sin), cos, sin, inverse=True), u, atol=1e-14)


def test_attention_output_invariant_to_position_shift():
    rng = np.random.default_rng(23)
    T, s, d = 8, 5, 8
    q = rng.standard_normal((1, T, 2, d))
    k = rng.standard_normal((1, T, 1, d))
    v = rng.standard_normal((1, T, 1, d))
    cos, sin = O.rope_tables(T + s, d, 1e4)
    o0, _ = O.attention_fwd(O.rope_apply(q, cos[:T], sin[:T]), O.rope_apply(k, cos[:T], sin[:T]), v)
    o1, _ = O.attention_fwd(O.rope_apply(q, cos[s:], sin[s:]), O.rope_apply(k, cos[s:], sin[s:]), v)
    np.testing.assert_allclose(o0, o1, atol=1e-12)


# ------------------------------------------------------------ RMSNorm
def test_rmsnorm_scale_invariance_and_closed_form():
    rng = np.random.default_rng(31)
    x = rng.standard_normal((4, 10))
    g = rng.standard_normal(10)
    y1, _ = O.rmsnorm_fwd(x, g, 0.0)
    y2, _ = O.rmsnorm_fwd(3.7 * x, g, 0.0)
    np.testing.assert_allclose(y1, y2, atol=1e-14)
    c = -0.25
    y, rstd = O.rmsnorm_fwd(np.full((1, 6), c), np.arange(6.0), 1e-2)
    np.testing.assert_allclose(y[0], np.arange(6.0) * c / math.sqrt(c * c + 1e-2), atol=1e-15)
    np.testing.assert_allclose(rstd, [1 / math.sqrt(c * c + 1e-2)], atol=1e-15)
    # rows with a known mean square: x = (3, 4) has mean square 12.5
    y, _ = O.rmsnorm_fwd(np.array([[3.0, 4.0]]), np.ones(2), 0.0)
    np.testing.assert_allclose(y, [[3 / math.sqrt(12.5), 4 / math.sqrt(12.5)]], atol=1e-15)


def test_rmsnorm_backward_orthogonal_to_input_at_zero_eps():
    rng = np.random.default_rng(32)
    x = rng.standard_normal((5, 12))
    g = rng.standard_normal(12)
    dy = rng.standard_normal((5, 12))
    _, rstd = O.rmsnorm_fwd(x, g, 0.0)
    dx, _ = O.rmsnorm_bwd(dy, x, g, rstd)
    np.testing.assert_allclose(np.sum(dx * x, axis=1), 0.0, atol=1e-12)


# ------------------------------------------------------------ SwiGLU
def test_silu_derivative_pointwise():
    z = np.linspace(-6, 6, 49)
    u = np.ones_like(z)
    h = 1e-6
    fd = (O.swiglu_fwd(z + h, u) - O.swiglu_fwd(z - h, u)) / (2 * h)
    dg, du = O.swiglu_bwd(np.ones_like(z), z, u)
    np.testing.assert_allclose(dg, fd, atol=1e-9)
    np.testing.assert_allclose(du, z / (1 + np.exp(-z)), atol=1e-15)
    assert O.swiglu_fwd(np.array([0.0]), np.array([5.0]))[0] == 0.0
    np.testing.assert_allclose(O.swiglu_fwd(np.array([40.0]), np.array([2.0])), [80.0], rtol=1e-15)


# ------------------------------------------------------------ whole layer
def test_zero_output_projections_make_the_layer_identity():
    rng = np.random.default_rng(41)
    w = _weights(TINY, rng)
    w["wo"] = np.zeros_like(w["wo"])
    w["wd"] = np.zeros_like(w["wd"])
    x = rng.standard_normal((2, 5, TINY.hidden))
    dy = rng.standard_normal((2, 5, TINY.hidden))
    y, dx, (gr,) = O.stack_fwd_bwd(TINY, [w], x, dy)
    np.testing.assert_array_equal(y, x)
    np.testing.assert_allclose(dx, dy, atol=0)
    for name in ("wq", "wk", "wv", "bq", "bk", "bv", "g1", "wg", "wu", "g2"):
        assert np.all(gr[name] == 0), name
    assert np.any(gr["wo"] != 0) and np.any(gr["wd"] != 0)


def test_gradients_vanish_and_are_linear_in_dy():
    rng = np.random.default_rng(42)
    w = _weights(TINY, rng)
    x = rng.standard_normal((2, 5, TINY.hidden))
    _, dx0, (g0,) = O.stack_fwd_bwd(TINY, [w], x, np.zeros_like(x))
    assert np.all(dx0 == 0) and all(np.all(v == 0) for v in g0.values())
    d1 = rng.standard_normal(x.shape)
    d2 = rng.standard_normal(x.shape)
    _, a, (ga,) = O.stack_fwd_bwd(TINY, [w], x, d1)
    _, b, (gb,) = O.stack_fwd_bwd(TINY, [w], x, d2)
    _, c, (gc,) = O.stack_fwd_bwd(TINY, [w], x, 2.0 * d1 - 0.5 * d2)
    np.testing.assert_allclose(c, 2.0 * a - 0.5 * b, atol=1e-12)
    for n in ga:
        np.testing.assert_allclose(gc[n], 2.0 * ga[n] - 0.5 * gb[n], atol=1e-11)


def test_single_token_layer_closed_form():
    """At T = 1 attention returns the value head and RoPE is the identity (angle 0)."""
    rng = np.random.default_rng(43)
    cfg = TINY
    w = _weights(cfg, rng)
    x = rng.standard_normal((3, 1, cfg.hidden))
    y, _ = O.layer_fwd(cfg, w, x)
    for b in range(3):
        xv = x[b, 0]
        h1 = xv / math.sqrt(np.mean(xv ** 2) + cfg.rms_eps) * w["g1"]
        vv = np.array([sum(w["wv"][i, j] * h1[j] for j in range(cfg.hidden)) + w["bv"][i]
                       for i in range(cfg.n_kv_heads * cfg.head_dim)])
        d = cfg.head_dim
        o = np.concatenate([vv[(h // 2) * d:(h // 2 + 1) * d] for h in range(cfg.n_q_heads)])
        x2 = xv + np.array([sum(w["wo"][i, j] * o[j] for j in range(len(o))) for i in range(cfg.hidden)])
        h2 = x2 / math.sqrt(np.mean(x2 ** 2) + cfg.rms_eps) * w["g2"]
        gg = np.array([sum(w["wg"][f, j] * h2[j] for j in range(cfg.hidden)) for f in range(cfg.ffn)])
        uu = np.array([sum(w["wu"][f, j] * h2[j] for j in range(cfg.hidden)) for f in range(cfg.ffn)])
        m = gg / (1 + np.exp(-gg)) * uu
        yy = x2 + np.array([sum(w["wd"][i, f] * m[f] for f in range(cfg.ffn)) for i in range(cfg.hidden)])
        np.testing.assert_allclose(y[b, 0], yy, atol=1e-12)


def test_weight_gradient_against_textbook_loops():
    rng = np.random.default_rng(44)
    w = _weights(TINY, rng)
    x = rng.standard_normal((2, 3, TINY.hidden))
    dy = rng.standard_normal((2, 3, TINY.hidden))
    y, cache = O.layer_fwd(TINY, w, x)
    _, gr = O.layer_bwd(TINY, w, cache, dy)
    m = cache["m"]
    H, F = TINY.hidden, TINY.ffn
    for i in range(H):
        for f in range(F):
            s = sum(dy[b, t, i] * m[b, t, f] for b in range(2) for t in range(3))
            assert abs(gr["wd"][i, f] - s) < 1e-12


# ------------------------------------------------------------ AdamW
from oracle.optimizer import adamw_step  # noqa: E402


def test_adamw_first_step_closed_form():
    rng = np.random.default_rng(51)
    w = rng.standard_normal(50)
    g = rng.standard_normal(50)
    lr, eps, wd = 1e-3, 1e-8, 0.1
    w1, m1, v1 = adamw_step(w, np.zeros(50), np.zeros(50), g, 1, lr, 0.9, 0.999, eps, wd)
    np.testing.assert_allclose(m1, 0.1 * g, rtol=1e-12)
    np.testing.assert_allclose(v1, 0.001 * g * g, rtol=1e-12)
    # bias correction makes the first step lr * g / (|g| + eps) plus the decoupled decay
    np.testing.assert_allclose(w1, w - lr * (g / (np.abs(g) + eps) + wd * w), rtol=1e-12, atol=1e-15)


def test_adamw_zero_gradient_only_decays():
    w = np.linspace(-2, 2, 9)
    w1, m1, v1 = adamw_step(w, np.zeros(9), np.zeros(9), np.zeros(9), 1, 0.01, 0.9, 0.999, 1e-8, 0.5)
    np.testing.assert_array_equal(m1, 0.0)
    np.testing.assert_allclose(w1, w * (1 - 0.01 * 0.5), rtol=1e-15)


def test_adamw_constant_gradient_moves_by_lr_per_step():
    g = np.array([3.0, -0.5, 1e-3])
    w, m, v = np.zeros(3), np.zeros(3), np.zeros(3)
    for t in range(1, 6):
        w, m, v = adamw_step(w, m, v, g, t, 0.01, 0.9, 0.99, 1e-12, 0.0)
    np.testing.assert_allclose(w, -5 * 0.01 * g / (np.abs(g) + 1e-12), rtol=1e-9)


# ------------------------------------------------------------ embedding, LM head, cross-entropy
from oracle import head as HD  # noqa: E402


def test_head_loss_gradients_match_central_differences():
    rng = np.random.default_rng(71)
    B, T, H, V = 2, 3, 8, 11
    y = rng.standard_normal((B, T, H))
    gf = 1.0 + 0.2 * rng.standard_normal(H)
    W = 0.5 * rng.standard_normal((V, H))
    tgt = rng.integers(0, V, size=(B, T))
    loss, dy, dgf, dW = HD.head_loss_fwd_bwd(y, gf, W, tgt, 1e-6)
    h = 1e-6
    for arr, g, name in ((y, dy, "y"), (gf, dgf, "gf"), (W, dW, "W")):
        e = rng.standard_normal(arr.shape)
        args_p = {"y": y, "gf": gf, "W": W}
        args_m = dict(args_p)
        args_p[name] = arr + h * e
        args_m[name] = arr - h * e
        lp = HD.head_loss_fwd_bwd(args_p["y"], args_p["gf"], args_p["W"], tgt, 1e-6)[0]
        lm = HD.head_loss_fwd_bwd(args_m["y"], args_m["gf"], args_m["W"], tgt, 1e-6)[0]
        assert abs((lp - lm) / (2 * h) - np.sum(g * e)) < 1e-7, name


def test_head_loss_closed_forms():
    # all-zero logits: every token's loss is log V, and each dW row is the softmax-minus-onehot weighting
    B, T, H, V = 1, 4, 6, 5
    y = np.random.default_rng(72).standard_normal((B, T, H))
    W = np.zeros((V, H))
    tgt = np.array([[0, 1, 1, 4]])
    loss, dy, dgf, dW = HD.head_loss_fwd_bwd(y, np.ones(H), W, tgt, 1e-6)
    assert abs(loss - np.log(V)) < 1e-12
    assert np.all(dy == 0) and np.all(dgf == 0)
    h, _ = O.rmsnorm_fwd(y, np.ones(H), 1e-6)
    counts = np.bincount(tgt.reshape(-1), minlength=V)
    expect = (h.reshape(-1, H).sum(axis=0)[None, :] / V - np.stack(
        [h.reshape(-1, H)[tgt.reshape(-1) == v].sum(axis=0) for v in range(V)])) / (B * T)
    np.testing.assert_allclose(dW, expect, atol=1e-14)
    assert counts.sum() == B * T


def test_embedding_backward_is_a_scatter_add():
    rng = np.random.default_rng(73)
    tok = np.array([[3, 1, 3], [0, 3, 2]])
    dx = rng.standard_normal((2, 3, 4))
    dE = HD.embed_bwd(tok, dx, 5)
    np.testing.assert_allclose(dE[3], dx[0, 0] + dx[0, 2] + dx[1, 1], atol=1e-15)
    np.testing.assert_array_equal(dE[4], 0.0)
    E = rng.standard_normal((5, 4))
    np.testing.assert_array_equal(HD.embed_fwd(tok, E)[1, 2], E[2])
