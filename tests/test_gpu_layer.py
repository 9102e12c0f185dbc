"""The stateless layer templates (forward; recompute + backward) on the B200
through the C ABI, against the CPU oracle: output, input gradient and every
weight/bias/gain gradient, relative Frobenius error <= 2e-2 per tensor."""
import numpy as np
import pytest

import helpers as H
from host_offloaded_layer_b200 import _lib as L
from host_offloaded_layer_b200 import synth
from oracle import layer as O

pytestmark = pytest.mark.gpu

CASES = {
    # the one-layer config: hidden 256, 4/2 heads of 64, FFN 688, batch 2 x 128
    "tiny": (dict(hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64, ffn=688), 2, 128, 0),
    # the same shape with weights of std 1/sqrt(hidden): the residual branches are as
    # large as the input, so Y - X and dX - dY are held to the plain 2e-2 tolerance
    "tiny_strong_branch": (dict(hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64, ffn=688), 2, 128, 0),
    # ragged sequence, MLP in 64-token chunks
    "tiny_ragged_chunked": (dict(hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64, ffn=688), 3, 100, 64),
    # head_dim 128, a group of 7 query heads per kv head (the 7B ratio), no QKV bias
    "gqa7_nobias": (dict(hidden=896, n_q_heads=7, n_kv_heads=1, head_dim=128, ffn=2048, qkv_bias=False), 2, 96, 0),
    # MHA
    "mha": (dict(hidden=512, n_q_heads=4, n_kv_heads=4, head_dim=128, ffn=1376), 1, 200, 0),
    # the Qwen2.5-7B layer shape at reduced batch
    "qwen7b_b1_t128": (dict(hidden=3584, n_q_heads=28, n_kv_heads=4, head_dim=128, ffn=18944), 1, 128, 0),
    "qwen7b_b2_t128": (dict(hidden=3584, n_q_heads=28, n_kv_heads=4, head_dim=128, ffn=18944), 2, 128, 0),
    # one whole 1024-token sequence: eight 128-row query blocks per head, the persistent attention
    # schedules, and every weight gradient summed over 1024 tokens
    "qwen7b_b1_t1024": (dict(hidden=3584, n_q_heads=28, n_kv_heads=4, head_dim=128, ffn=18944), 1, 1024, 0),
    # the Qwen2.5-14B layer shape
    "qwen14b_b1_t64": (dict(hidden=5120, n_q_heads=40, n_kv_heads=8, head_dim=128, ffn=13824), 1, 64, 0),
    "qwen14b_b1_t1024": (dict(hidden=5120, n_q_heads=40, n_kv_heads=8, head_dim=128, ffn=13824), 1, 1024, 0),
    # the long-context regime: 64 key blocks per query row on the tcgen05 attention, the MLP over four
    # 2048-token chunks (the chunked path the 32K-token workload runs), a 7:1 head group
    "gqa7_t8192_chunked": (dict(hidden=896, n_q_heads=7, n_kv_heads=1, head_dim=128, ffn=2048), 1, 8192, 2048),
}


def _run(cfg, B, T, chunk, seed=1234, std=synth.WEIGHT_STD):
    import torch
    rec, w64 = H.layer_record(cfg, seed, 0, std=std, gain_std=0.1)
    x = synth.activations_bf16_bits(seed, synth.X0_ID, B, T, cfg.hidden)
    dy = synth.activations_bf16_bits(seed, synth.DY_ID, B, T, cfg.hidden)
    w_d = H.dev_bf16(rec)
    x_d, dy_d = H.dev_bf16(x), H.dev_bf16(dy)
    y_d = H.empty_bf16(B, T, cfg.hidden)
    dx_d = H.empty_bf16(B, T, cfg.hidden)
    dw_d = torch.full((rec.size,), float("nan"), dtype=torch.float32, device="cuda")
    ws = H.workspace(L.mt_layer_workspace_bytes(cfg, B, T, chunk))
    L.mt_layer_fwd(cfg, w_d, x_d, y_d, B, T, chunk, ws, ws.numel())
    L.mt_layer_recompute_bwd(cfg, w_d, x_d, dy_d, dx_d, dw_d, B, T, chunk, ws, ws.numel())
    torch.cuda.synchronize()
    assert L.mt_device_error(clear=True) == 0
    return rec, w64, x, dy, H.host_f64(y_d), H.host_f64(dx_d), dw_d.cpu().numpy()


@pytest.mark.parametrize("name", list(CASES))
def test_layer_matches_oracle(name):
    shape, B, T, chunk = CASES[name]
    cfg = L.make_cfg(**shape)
    std = 1.0 / np.sqrt(shape["hidden"]) if name == "tiny_strong_branch" else synth.WEIGHT_STD
    rec, w64, x, dy, y, dx, dw = _run(cfg, B, T, chunk, std=std)
    ocfg = H.oracle_cfg(cfg)
    x64, dy64 = H.bits_to_f64(x), H.bits_to_f64(dy)
    y_ref, cache = O.layer_fwd(ocfg, w64, x64)
    dx_ref, g_ref = O.layer_bwd(ocfg, w64, cache, dy64)
    errs = {"Y": H.rel(y, y_ref), "dX": H.rel(dx, dx_ref)}
    got = H.grads_from_record(cfg, dw)
    for k, v in g_ref.items():
        errs["d" + k] = H.rel(got[k], v)
    bad = {k: v for k, v in errs.items() if not v <= H.TOL}
    # the residual branches alone, within the bf16 residual-stream budget
    br = {"Y-X": (H.rel(y - x64, y_ref - x64), H.branch_tol(x64, y_ref)),
          "dX-dY": (H.rel(dx - dy64, dx_ref - dy64), H.branch_tol(dy64, dx_ref))}
    bad.update({k: v for k, v in br.items() if not v[0] <= v[1]})
    if name == "tiny_strong_branch":  # branches as large as the input: the plain tolerance
        bad.update({k: v for k, v in br.items() if not v[0] <= H.TOL})
    assert not bad, f"{name}: {bad} (all: {errs}, branches: {br})"


def test_layer_backward_is_bitwise_reproducible():
    cfg = L.make_cfg(**CASES["tiny"][0])
    a = _run(cfg, 2, 128, 0)
    b = _run(cfg, 2, 128, 0)
    assert np.array_equal(a[5], b[5]) and np.array_equal(a[6].view(np.uint32), b[6].view(np.uint32))


def test_chunked_mlp_matches_unchunked():
    cfg = L.make_cfg(**CASES["tiny"][0])
    full = _run(cfg, 2, 128, 0)
    ch = _run(cfg, 2, 128, 96)  # ragged last chunk (256 = 96 + 96 + 64)
    assert np.array_equal(full[4], ch[4]), "forward rows are independent of the chunking"
    assert H.rel(ch[6], full[6]) < 1e-5


def test_gradient_record_padding_is_untouched():
    cfg = L.make_cfg(hidden=264, n_q_heads=3, n_kv_heads=1, head_dim=64, ffn=520)
    off = L.mt_layer_param_offsets(cfg)
    assert off.record_elems > off.param_count  # this shape has padding between blocks
    *_, dw = _run(cfg, 1, 64, 0)
    used = np.zeros(off.record_elems, dtype=bool)
    for name, shp in synth.layer_tensor_shapes(**H.shape_dict(cfg)).items():
        o = getattr(off, name)
        used[o:o + int(np.prod(shp))] = True
    assert np.all(np.isfinite(dw[used]))
    assert np.all(np.isnan(dw[~used])), "padding of the gradient record was written"
