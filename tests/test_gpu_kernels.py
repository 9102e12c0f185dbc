"""Block kernels on the B200 through the C ABI, against the CPU oracle.

Every input is seeded and synthetic; outputs are compared element by element
(relative Frobenius error) with the oracle's float64 result on the same bf16
inputs. Sizes span several tiles and include ragged tails.
"""
import numpy as np
import pytest

import helpers as H
from host_offloaded_layer_b200 import _lib as L
from host_offloaded_layer_b200 import synth
from oracle import layer as O

pytestmark = pytest.mark.gpu


def _bits(seed, tid, n, std=1.0):
    return synth.f32_to_bf16_bits(synth.normal_f32(seed, 7, tid, n, std))


def _check_dev_error():
    assert L.mt_device_error(clear=True) == 0


# ------------------------------------------------------------------ GEMM
@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1), (1, 0), (1, 1)])
@pytest.mark.parametrize("M,N,K", [(256, 512, 256), (200, 300, 136), (2048, 4096, 512), (96, 40, 1000),
                                   (600, 1100, 8200)])  # K >= 8192, a few tiles: the 256 x 256 tile
def test_gemm_layouts_match_fp64_matmul(a_mn, b_mn, M, N, K):
    import torch
    lda = ((M if a_mn else K) + 7) // 8 * 8 + 8
    ldb = ((N if b_mn else K) + 7) // 8 * 8 + 16
    a_rows, a_cols = (K, M) if a_mn else (M, K)
    b_rows, b_cols = (K, N) if b_mn else (N, K)
    A = _bits(1, 1, a_rows * lda).reshape(a_rows, lda)
    B = _bits(1, 2, b_rows * ldb).reshape(b_rows, ldb)
    A64 = H.bits_to_f64(A)[:, :a_cols]
    B64 = H.bits_to_f64(B)[:, :b_cols]
    Am = A64.T if a_mn else A64   # logical [M, K]
    Bm = B64.T if b_mn else B64   # logical [N, K]
    ref = Am @ Bm.T
    dA, dB = H.dev_bf16(A), H.dev_bf16(B)
    ldc = (N + 7) // 8 * 8 + 8
    C = torch.zeros(M, ldc, dtype=torch.float32, device="cuda")
    L.mt_gemm_bf16(dA, lda, a_mn, dB, ldb, b_mn, C, ldc, 1, 0, M, N, K)
    torch.cuda.synchronize()
    _check_dev_error()
    got = H.host_f64(C)[:, :N]
    assert H.rel(got, ref) < 1e-5
    assert np.all(H.host_f64(C)[:, N:] == 0), "wrote past N"
    # bf16 output with bias and residual
    bias = _bits(1, 3, N)
    res = _bits(1, 4, M * ldc).reshape(M, ldc)
    Cb = torch.zeros(M, ldc, dtype=torch.bfloat16, device="cuda")
    L.mt_gemm_bf16(dA, lda, a_mn, dB, ldb, b_mn, Cb, ldc, 0, 0, M, N, K, H.dev_bf16(bias), H.dev_bf16(res), ldc)
    torch.cuda.synchronize()
    ref_b = ref + H.bits_to_f64(bias)[None, :] + H.bits_to_f64(res)[:, :N]
    assert H.rel(H.host_f64(Cb)[:, :N], ref_b) < 1e-2
    # fp32 accumulate: C += A B^T
    L.mt_gemm_bf16(dA, lda, a_mn, dB, ldb, b_mn, C, ldc, 1, 1, M, N, K)
    torch.cuda.synchronize()
    assert H.rel(H.host_f64(C)[:, :N], 2 * ref) < 1e-5
    _check_dev_error()


def test_gemm_is_deterministic_and_covers_many_waves():
    import torch
    M, N, K = 4096, 4608, 3584  # 32 x 18 tiles: several persistent waves per CTA
    A = H.dev_bf16(_bits(2, 1, M * K).reshape(M, K))
    B = H.dev_bf16(_bits(2, 2, N * K).reshape(N, K))
    C1 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    C2 = torch.empty_like(C1)
    L.mt_gemm_bf16(A, K, 0, B, K, 0, C1, N, 0, 0, M, N, K)
    L.mt_gemm_bf16(A, K, 0, B, K, 0, C2, N, 0, 0, M, N, K)
    torch.cuda.synchronize()
    assert torch.equal(C1.view(torch.int16), C2.view(torch.int16))
    rows = torch.randint(0, M, (64,), generator=torch.Generator().manual_seed(0)).cuda()
    r64 = H.host_f64(A[rows]) @ H.host_f64(B).T
    assert H.rel(H.host_f64(C1[rows]), r64) < 1e-2
    _check_dev_error()


def test_gemm_weight_gradient_layout_wide_tile():
    """The weight-gradient layout (both operands MN-major) with K >= 8192 runs the 256 x 512 pair
    tile when its waves of clusters pay: 2000 x 4000 is 64 wide tiles (one wave) against 128
    narrow ones (two). fp32 output, then fp32 accumulate, on sampled rows against float64, with
    ragged row and column blocks."""
    import torch
    M, N, K = 2000, 4000, 8200
    A = _bits(14, 1, K * M).reshape(K, M)  # [K, M]: M contiguous
    B = _bits(14, 2, K * N, 0.05).reshape(K, N)
    dA, dB = H.dev_bf16(A), H.dev_bf16(B)
    C = torch.zeros(M, N, dtype=torch.float32, device="cuda")
    L.mt_gemm_bf16(dA, M, 1, dB, N, 1, C, N, 1, 0, M, N, K)
    torch.cuda.synchronize()
    _check_dev_error()
    rows = np.concatenate([np.random.default_rng(4).choice(M - 16, 48, replace=False), np.arange(M - 16, M)])
    ref = H.bits_to_f64(A[:, rows]).T @ H.bits_to_f64(B)
    assert H.rel(H.host_f64(C)[rows], ref) < 1e-5
    L.mt_gemm_bf16(dA, M, 1, dB, N, 1, C, N, 1, 1, M, N, K)
    torch.cuda.synchronize()
    assert H.rel(H.host_f64(C)[rows], 2 * ref) < 1e-5
    _check_dev_error()


@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1)])
def test_gemm_long_k_many_rows_wide_tile(a_mn, b_mn):
    """At 65536 rows and more with K >= 8192 the forward and input-gradient layouts run the
    256 x 512 pair tile (the down projection and dh2 of the 96 x 1024 workload): sampled rows
    of a bf16 result with a residual against the float64 product, a ragged last row block and a
    ragged last column block (N = 1000: 514 wide tiles, whole waves of 64 to 74 clusters)."""
    import torch
    M, N, K = 65600, 1000, 8200
    A = _bits(13, 1, M * K).reshape(M, K)
    b_rows, b_cols = (K, N) if b_mn else (N, K)
    B = _bits(13, 2, b_rows * b_cols, 0.05).reshape(b_rows, b_cols)
    res = _bits(13, 3, M * N).reshape(M, N)
    C = torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")
    L.mt_gemm_bf16(H.dev_bf16(A), K, a_mn, H.dev_bf16(B), b_cols, b_mn, C, N, 0, 0, M, N, K, None, H.dev_bf16(res), N)
    torch.cuda.synchronize()
    _check_dev_error()
    rows = np.concatenate([np.random.default_rng(3).choice(M - 64, 60, replace=False), np.arange(M - 4, M)])
    b64 = H.bits_to_f64(B)
    ref = H.bits_to_f64(A[rows]) @ (b64 if b_mn else b64.T) + H.bits_to_f64(res[rows])
    assert H.rel(H.host_f64(C)[rows], ref) < 1e-2


@pytest.mark.parametrize("M,F,K", [(256, 688, 256), (200, 1000, 136), (8192, 18944, 3584)])
def test_gemm_with_swiglu_epilogue(M, F, K):
    import torch
    A = _bits(9, 1, M * K, 1.0).reshape(M, K)
    W = _bits(9, 2, 2 * F * K, 0.05).reshape(2 * F, K)
    m = torch.zeros(M, F, dtype=torch.bfloat16, device="cuda")
    gu = torch.zeros(M, 2 * F, dtype=torch.bfloat16, device="cuda")
    L.mt_gemm_swiglu_bf16(H.dev_bf16(A), K, H.dev_bf16(W), K, m, F, gu, 2 * F, M, F, K)
    torch.cuda.synchronize()
    _check_dev_error()
    rows = np.arange(M) if M <= 256 else np.random.default_rng(0).choice(M, 96, replace=False)
    a64 = H.bits_to_f64(A)[rows]
    w64 = H.bits_to_f64(W)
    g, u = a64 @ w64[:F].T, a64 @ w64[F:].T
    assert H.rel(H.host_f64(m)[rows], O.swiglu_fwd(g, u)) < 1e-2
    got = H.host_f64(gu)[rows]
    assert H.rel(got[:, :F], g) < 1e-2 and H.rel(got[:, F:], u) < 1e-2
    m2 = torch.zeros_like(m)  # without g, u
    L.mt_gemm_swiglu_bf16(H.dev_bf16(A), K, H.dev_bf16(W), K, m2, F, None, 0, M, F, K)
    torch.cuda.synchronize()
    assert torch.equal(m.view(torch.int16), m2.view(torch.int16))


@pytest.mark.parametrize("M,F,K", [(256, 688, 256), (200, 1000, 136), (8192, 18944, 3584)])
def test_gemm_with_swiglu_backward_epilogue(M, F, K):
    """dm = dY Wd with [g|u] replaced by [dg|du] in the epilogue, against the
    oracle's SwiGLU backward on the float64 product."""
    import torch
    dY = _bits(11, 1, M * K, 1.0).reshape(M, K)
    Wd = _bits(11, 2, K * F, 0.05).reshape(K, F)  # [hidden, F] as stored in the layer record
    gu = _bits(11, 3, M * 2 * F, 2.0).reshape(M, 2 * F)
    gud = H.dev_bf16(gu)
    L.mt_gemm_swiglu_bwd_bf16(H.dev_bf16(dY), K, H.dev_bf16(Wd), F, gud, 2 * F, M, F, K)
    torch.cuda.synchronize()
    _check_dev_error()
    rows = np.arange(M) if M <= 256 else np.random.default_rng(1).choice(M, 96, replace=False)
    dm = H.bits_to_f64(dY)[rows] @ H.bits_to_f64(Wd)
    g64, u64 = H.bits_to_f64(gu[rows, :F]), H.bits_to_f64(gu[rows, F:])
    dg, du = O.swiglu_bwd(dm, g64, u64)
    got = H.host_f64(gud)[rows]
    assert H.rel(got[:, :F], dg) < 1e-2
    assert H.rel(got[:, F:], du) < 1e-2
    # the same GEMM plus the stand-alone SwiGLU backward kernel agrees (dm rounded to bf16 there)
    dmd = torch.empty(M, F, dtype=torch.bfloat16, device="cuda")
    L.mt_gemm_bf16(H.dev_bf16(dY), K, 0, H.dev_bf16(Wd), F, 1, dmd, F, 0, 0, M, F, K, None, None, 0)
    dgu = H.empty_bf16(M, 2 * F)
    L.mt_swiglu_bwd(dmd, H.dev_bf16(gu), dgu, M, F)
    torch.cuda.synchronize()
    assert H.rel(got, H.host_f64(dgu)[rows]) < 1e-2


# ------------------------------------------------------------------ RMSNorm
@pytest.mark.parametrize("rows,Hd", [(256, 256), (1000, 3584), (37, 5120)])
def test_rmsnorm_forward_and_backward(rows, Hd):
    import torch
    x = _bits(3, 1, rows * Hd).reshape(rows, Hd)
    g = synth.f32_to_bf16_bits((1.0 + synth.normal_f32(3, 7, 2, Hd, 0.2)).astype(np.float32))
    dy = _bits(3, 3, rows * Hd).reshape(rows, Hd)
    dres = _bits(3, 4, rows * Hd).reshape(rows, Hd)
    eps = 1e-6
    y = H.empty_bf16(rows, Hd)
    rstd = H.empty_f32(rows)
    dx, x_d = H.empty_bf16(rows, Hd), H.dev_bf16(x)
    dg = H.empty_f32(Hd)
    L.mt_rmsnorm_fwd(x_d, H.dev_bf16(g), y, rstd, rows, Hd, eps)
    ws = H.workspace(L.mt_rmsnorm_bwd_workspace_bytes(rows, Hd))
    L.mt_rmsnorm_bwd(H.dev_bf16(dy), x_d, H.dev_bf16(g), rstd, H.dev_bf16(dres), dx, dg, rows, Hd, ws, ws.numel())
    torch.cuda.synchronize()
    x64, g64, dy64 = H.bits_to_f64(x), H.bits_to_f64(g), H.bits_to_f64(dy)
    y_ref, r_ref = O.rmsnorm_fwd(x64, g64, eps)
    assert H.rel(H.host_f64(y), y_ref) < 1e-2
    assert H.rel(H.host_f64(rstd), r_ref) < 1e-5
    dx_ref, dg_ref = O.rmsnorm_bwd(dy64, x64, g64, r_ref)
    assert H.rel(H.host_f64(dx), dx_ref + H.bits_to_f64(dres)) < 1e-2
    assert H.rel(H.host_f64(dx) - H.bits_to_f64(dres), dx_ref) < 2e-2
    assert H.rel(H.host_f64(dg), dg_ref) < 1e-4


# ------------------------------------------------------------------ RoPE, SwiGLU, colsum
@pytest.mark.parametrize("B,T,nh,d", [(2, 128, 6, 64), (1, 1000, 3, 128)])
def test_rope_matches_oracle_and_inverts(B, T, nh, d):
    import torch
    ld = nh * d + 64
    x = _bits(4, 1, B * T * ld).reshape(B, T, ld)
    xd = H.dev_bf16(x)
    L.mt_rope(xd, ld, B, T, nh, d, 1e6, False)
    torch.cuda.synchronize()
    cos, sin = O.rope_tables(T, d, 1e6)
    u = H.bits_to_f64(x)[..., :nh * d].reshape(B, T, nh, d)
    ref = O.rope_apply(u, cos, sin).reshape(B, T, nh * d)
    got = H.host_f64(xd)
    assert H.rel(got[..., :nh * d], ref) < 1e-2
    assert np.array_equal(got[..., nh * d:], H.bits_to_f64(x)[..., nh * d:]), "touched columns past the heads"
    L.mt_rope(xd, ld, B, T, nh, d, 1e6, True)
    torch.cuda.synchronize()
    assert H.rel(H.host_f64(xd)[..., :nh * d], H.bits_to_f64(x)[..., :nh * d]) < 1e-2


@pytest.mark.parametrize("rows,F", [(256, 688), (333, 18944)])
def test_swiglu_forward_and_backward(rows, F):
    import torch
    gu = _bits(5, 1, rows * 2 * F, 2.0).reshape(rows, 2 * F)
    dm = _bits(5, 2, rows * F).reshape(rows, F)
    m = H.empty_bf16(rows, F)
    dgu = H.empty_bf16(rows, 2 * F)
    gud = H.dev_bf16(gu)
    L.mt_swiglu_fwd(gud, m, rows, F)
    L.mt_swiglu_bwd(H.dev_bf16(dm), gud, dgu, rows, F)
    torch.cuda.synchronize()
    g64, u64 = H.bits_to_f64(gu[:, :F]), H.bits_to_f64(gu[:, F:])
    assert H.rel(H.host_f64(m), O.swiglu_fwd(g64, u64)) < 1e-2
    dg, du = O.swiglu_bwd(H.bits_to_f64(dm), g64, u64)
    got = H.host_f64(dgu)
    assert H.rel(got[:, :F], dg) < 1e-2
    assert H.rel(got[:, F:], du) < 1e-2


def test_colsum_fixed_order():
    import torch
    rows, cols, ld = 3001, 4608, 4616
    X = _bits(6, 1, rows * ld).reshape(rows, ld)
    out = H.empty_f32(cols)
    ws = H.workspace(L.mt_colsum_workspace_bytes(rows, cols))
    Xd = H.dev_bf16(X)
    L.mt_colsum(Xd, rows, cols, ld, out, ws, ws.numel())
    torch.cuda.synchronize()
    ref = H.bits_to_f64(X)[:, :cols].sum(axis=0)
    assert H.rel(H.host_f64(out), ref) < 1e-5
    out2 = H.empty_f32(cols)
    L.mt_colsum(Xd, rows, cols, ld, out2, ws, ws.numel())
    torch.cuda.synchronize()
    assert torch.equal(out, out2)


# ------------------------------------------------------------------ attention
ATTN_CASES = [
    (2, 128, 4, 2, 64),     # the tiny layer's heads
    (2, 100, 4, 4, 64),     # ragged T, MHA
    (1, 200, 7, 1, 128),    # ragged, group of 7 (the 7B ratio)
    (1, 320, 28, 4, 128),   # 7B heads
    (2, 64, 2, 1, 128),
    (2, 1024, 28, 4, 128),  # the 7B heads over 8 key blocks (online-softmax rescaling)
    (2, 700, 8, 2, 128),    # ragged last query block that reaches into the next sequence and past the end
    (3, 1, 7, 1, 128),      # one token: the upper key half of the only block is masked for every row
    (3, 37, 5, 5, 128),     # shorter than one key half
]


@pytest.mark.parametrize("B,T,nq,nkv,d", ATTN_CASES)
def test_attention_forward_and_backward(B, T, nq, nkv, d):
    import torch
    ld = (nq + 2 * nkv) * d
    qkv = _bits(8, 1, B * T * ld, 1.5).reshape(B, T, ld)
    do = _bits(8, 2, B * T * nq * d).reshape(B, T, nq * d)
    qkv_d = H.dev_bf16(qkv)
    o = H.empty_bf16(B, T, nq * d)
    lse = H.empty_f32(B, nq, T)
    L.mt_attention_fwd(qkv_d, ld, o, nq * d, lse, B, T, nq, nkv, d)
    torch.cuda.synchronize()
    q64 = H.bits_to_f64(qkv)
    q = q64[..., :nq * d].reshape(B, T, nq, d)
    k = q64[..., nq * d:(nq + nkv) * d].reshape(B, T, nkv, d)
    v = q64[..., (nq + nkv) * d:].reshape(B, T, nkv, d)
    o_ref, lse_ref = O.attention_fwd(q, k, v)
    assert H.rel(H.host_f64(o), o_ref.reshape(B, T, nq * d)) < 1e-2
    assert H.rel(H.host_f64(lse), lse_ref) < 1e-4
    # backward from the GPU's own o (as the layer does)
    o64 = H.host_f64(o).reshape(B, T, nq, d)
    dqkv = torch.zeros(B, T, ld, dtype=torch.bfloat16, device="cuda")
    ws = H.workspace(L.mt_attention_bwd_workspace_bytes(B, T, nq))
    L.mt_attention_bwd(qkv_d, ld, o, H.dev_bf16(do), nq * d, lse, dqkv, B, T, nq, nkv, d, ws, ws.numel())
    torch.cuda.synchronize()
    dq, dk, dv = O.attention_bwd(H.bits_to_f64(do).reshape(B, T, nq, d), q, k, v, o64, H.host_f64(lse))
    got = H.host_f64(dqkv)
    assert H.rel(got[..., :nq * d], dq.reshape(B, T, -1)) < 2e-2
    assert H.rel(got[..., nq * d:(nq + nkv) * d], dk.reshape(B, T, -1)) < 2e-2
    assert H.rel(got[..., (nq + nkv) * d:], dv.reshape(B, T, -1)) < 2e-2
    # deterministic
    dqkv2 = torch.zeros_like(dqkv)
    L.mt_attention_bwd(qkv_d, ld, o, H.dev_bf16(do), nq * d, lse, dqkv2, B, T, nq, nkv, d, ws, ws.numel())
    torch.cuda.synchronize()
    assert torch.equal(dqkv.view(torch.int16), dqkv2.view(torch.int16))
    # backward from the oracle's own o (rounded to bf16) and lse: independent of the forward kernel
    _attention_bwd_from_oracle_forward(qkv_d, q, k, v, o_ref, lse_ref, do, B, T, nq, nkv, d)


def _attention_bwd_from_oracle_forward(qkv_d, q, k, v, o_ref, lse_ref, do_bits, B, T, nq, nkv, d):
    """The backward kernel fed the oracle forward's o (bf16) and lse (fp32), against the
    oracle's backward on the same o and lse."""
    import torch
    ld = (nq + 2 * nkv) * d
    o_bits = synth.f32_to_bf16_bits(o_ref.reshape(B, T, nq * d).astype(np.float32))
    lse_f32 = np.ascontiguousarray(lse_ref, dtype=np.float32)
    dqkv = torch.zeros(B, T, ld, dtype=torch.bfloat16, device="cuda")
    ws = H.workspace(L.mt_attention_bwd_workspace_bytes(B, T, nq))
    L.mt_attention_bwd(qkv_d, ld, H.dev_bf16(o_bits), H.dev_bf16(do_bits), nq * d, H.dev_f32(lse_f32), dqkv, B, T, nq,
                       nkv, d, ws, ws.numel())
    torch.cuda.synchronize()
    _check_dev_error()
    dq, dk, dv = O.attention_bwd(H.bits_to_f64(do_bits).reshape(B, T, nq, d), q, k, v,
                                 H.bits_to_f64(o_bits).reshape(B, T, nq, d), lse_f32.astype(np.float64))
    got = H.host_f64(dqkv)
    errs = {"dq": H.rel(got[..., :nq * d], dq.reshape(B, T, -1)),
            "dk": H.rel(got[..., nq * d:(nq + nkv) * d], dk.reshape(B, T, -1)),
            "dv": H.rel(got[..., (nq + nkv) * d:], dv.reshape(B, T, -1))}
    assert all(e < 2e-2 for e in errs.values()), errs


@pytest.mark.parametrize("T", [8192, 16320])
def test_long_context_attention_matches_oracle(T):
    """Long sequences (the long-context workloads' regime): 64 and 128 key blocks per query
    row, a group of 7 query heads per key/value head (the 7B ratio) and, at 16320 tokens, a
    ragged last query block. Forward against the oracle; backward from the oracle's own
    forward outputs against the oracle's backward."""
    import torch
    B, nq, nkv, d = 1, 7, 1, 128
    ld = (nq + 2 * nkv) * d
    qkv = _bits(12, T, B * T * ld, 1.5).reshape(B, T, ld)
    do = _bits(13, T, B * T * nq * d).reshape(B, T, nq * d)
    qkv_d = H.dev_bf16(qkv)
    o = H.empty_bf16(B, T, nq * d)
    lse = H.empty_f32(B, nq, T)
    L.mt_attention_fwd(qkv_d, ld, o, nq * d, lse, B, T, nq, nkv, d)
    torch.cuda.synchronize()
    _check_dev_error()
    q64 = H.bits_to_f64(qkv)
    q = q64[..., :nq * d].reshape(B, T, nq, d)
    k = q64[..., nq * d:(nq + nkv) * d].reshape(B, T, nkv, d)
    v = q64[..., (nq + nkv) * d:].reshape(B, T, nkv, d)
    o_ref, lse_ref = O.attention_fwd(q, k, v)
    assert H.rel(H.host_f64(o), o_ref.reshape(B, T, nq * d)) < 1e-2
    assert H.rel(H.host_f64(lse), lse_ref) < 1e-4
    _attention_bwd_from_oracle_forward(qkv_d, q, k, v, o_ref, lse_ref, do, B, T, nq, nkv, d)
