"""Embedding, final RMSNorm, LM head and cross-entropy on the B200 through the
C ABI, against the CPU oracle (oracle/head.py)."""
import numpy as np
import pytest

import helpers as H
from host_offloaded_layer_b200 import _lib as L
from host_offloaded_layer_b200 import synth
from oracle import head as HD

pytestmark = pytest.mark.gpu


def _bits(seed, tid, n, std=1.0):
    return synth.f32_to_bf16_bits(synth.normal_f32(seed, 9, tid, n, std))


@pytest.mark.parametrize("M,Hd,V,chunk", [(256, 256, 1000, 384), (128, 3584, 152064, 16384)])
def test_head_loss_matches_oracle(M, Hd, V, chunk):
    import torch
    y = _bits(1, 1, M * Hd).reshape(M, Hd)
    gf = synth.f32_to_bf16_bits((1.0 + synth.normal_f32(1, 9, 2, Hd, 0.1)).astype(np.float32))
    W = _bits(1, 3, V * Hd, 0.05).reshape(V, Hd)
    tgt = np.random.default_rng(5).integers(0, V, size=M).astype(np.int32)
    loss = torch.zeros(1, dtype=torch.float32, device="cuda")
    dy = H.empty_bf16(M, Hd)
    dgf = H.empty_f32(Hd)
    dW = torch.full((V, Hd), float("nan"), dtype=torch.float32, device="cuda")
    ws = H.workspace(L.mt_head_workspace_bytes(M, Hd, V, chunk))
    t_d = torch.from_numpy(tgt).cuda()
    args = (H.dev_bf16(y), H.dev_bf16(gf), H.dev_bf16(W), t_d, M, Hd, V, 1e-6, chunk, loss, dy, dgf, dW, ws,
            ws.numel())
    L.mt_head_loss_fwd_bwd(*args)
    torch.cuda.synchronize()
    assert L.mt_device_error(clear=True) == 0
    l_ref, dy_ref, dgf_ref, dW_ref = HD.head_loss_fwd_bwd(H.bits_to_f64(y)[None], H.bits_to_f64(gf),
                                                          H.bits_to_f64(W), tgt[None], 1e-6)
    assert abs(loss.item() - l_ref) / abs(l_ref) < 1e-3
    assert H.rel(H.host_f64(dy), dy_ref[0]) < H.TOL
    assert H.rel(H.host_f64(dgf), dgf_ref) < H.TOL
    assert H.rel(H.host_f64(dW), dW_ref) < H.TOL
    # bitwise repeatable
    dW2 = torch.zeros_like(dW)
    L.mt_head_loss_fwd_bwd(*args[:12], dW2, ws, ws.numel())
    torch.cuda.synchronize()
    assert torch.equal(dW, dW2)


def test_embedding_gather_and_scatter_add():
    import torch
    M, Hd, V = 1000, 512, 300
    rng = np.random.default_rng(8)
    tok = rng.integers(0, V // 3, size=M).astype(np.int32)  # many repeats, some rows unused
    E = _bits(2, 1, V * Hd).reshape(V, Hd)
    dx = _bits(2, 2, M * Hd).reshape(M, Hd)
    x = H.empty_bf16(M, Hd)
    bad = torch.zeros(1, dtype=torch.int32, device="cuda")
    t_d = torch.from_numpy(tok).cuda()
    L.mt_embed_fwd(t_d, H.dev_bf16(E), x, M, Hd, V, bad)
    order = np.empty(M, np.int32)
    start = np.empty(V + 1, np.int32)
    L.mt_embed_sort(tok, M, V, order, start)
    dE = torch.full((V, Hd), float("nan"), dtype=torch.float32, device="cuda")
    L.mt_embed_bwd(torch.from_numpy(order).cuda(), torch.from_numpy(start).cuda(), H.dev_bf16(dx), dE, Hd, V)
    torch.cuda.synchronize()
    assert bad.item() == 0
    assert np.array_equal(H.host_f64(x), H.bits_to_f64(E)[tok])
    np.testing.assert_allclose(H.host_f64(dE), HD.embed_bwd(tok, H.bits_to_f64(dx), V), rtol=1e-5, atol=1e-5)
    bad_tok = torch.from_numpy(np.array([0, V, -1, 5], np.int32)).cuda()
    x2 = H.empty_bf16(4, Hd)
    L.mt_embed_fwd(bad_tok, H.dev_bf16(E), x2, 4, Hd, V, bad)
    torch.cuda.synchronize()
    assert bad.item() == 2
