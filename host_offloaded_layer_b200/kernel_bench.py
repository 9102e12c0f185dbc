"""Times one block kernel through the C ABI (CUDA events, warm-up first).

    python -m host_offloaded_layer_b200.kernel_bench gemm --M 16384 --N 4608 --K 3584 --layout kk
    python -m host_offloaded_layer_b200.kernel_bench gemm --M 98304 --N 3584 --K 3584 --layout kk --res
    python -m host_offloaded_layer_b200.kernel_bench gemm_swiglu --M 8192 --F 18944 --K 3584
    python -m host_offloaded_layer_b200.kernel_bench gemm_swiglu_bwd --M 8192 --F 18944 --K 3584
    python -m host_offloaded_layer_b200.kernel_bench attn_fwd --B 8 --T 1024 --nq 28 --nkv 4 --d 128
    python -m host_offloaded_layer_b200.kernel_bench attn_bwd --B 8 --T 1024 --nq 28 --nkv 4 --d 128
    python -m host_offloaded_layer_b200.kernel_bench rmsnorm --rows 8192 --H 3584
    python -m host_offloaded_layer_b200.kernel_bench swiglu --rows 8192 --F 18944
    python -m host_offloaded_layer_b200.kernel_bench layer --hidden 3584 --nq 28 --nkv 4 --d 128 --F 18944 --B 8 --T 1024

GEMM layouts name the majorness of A and B: ``kk`` (forward, Y = X W^T),
``km`` (input gradient, B MN-major), ``mm`` (weight gradient). Prints one
JSON line with the mean time per launch and the achieved TFLOP/s or GB/s
(algorithmic FLOPs or bytes per launch over the measured time). Inputs are
seeded synthetic normals; this is a measurement tool, not a test.
"""
from __future__ import annotations

import argparse
import json

import numpy as np


def _dev(torch, n, seed, std=1.0):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return (torch.randn(n, generator=g, device="cuda") * std).to(torch.bfloat16)


def main():
    import torch

    from host_offloaded_layer_b200 import _lib as L

    ap = argparse.ArgumentParser()
    ap.add_argument("op", choices=["gemm", "gemm_swiglu", "gemm_swiglu_bwd", "attn_fwd", "attn_bwd", "rmsnorm", "swiglu",
                                   "layer"])
    ap.add_argument("--M", type=int, default=8192)
    ap.add_argument("--N", type=int, default=4608)
    ap.add_argument("--K", type=int, default=3584)
    ap.add_argument("--layout", default="kk", choices=["kk", "km", "mk", "mm"])
    ap.add_argument("--f32", action="store_true", help="fp32 output (weight-gradient epilogue)")
    ap.add_argument("--res", action="store_true", help="add a bf16 residual (the O / down projection epilogue)")
    ap.add_argument("--B", type=int, default=8)
    ap.add_argument("--T", type=int, default=1024)
    ap.add_argument("--nq", type=int, default=28)
    ap.add_argument("--nkv", type=int, default=4)
    ap.add_argument("--d", type=int, default=128)
    ap.add_argument("--hidden", type=int, default=3584)
    ap.add_argument("--F", type=int, default=18944)
    ap.add_argument("--rows", type=int, default=8192)
    ap.add_argument("--H", type=int, default=3584)
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    a = ap.parse_args()
    L.load()
    st = torch.cuda.current_stream()

    if a.op == "gemm":
        a_mn, b_mn = a.layout[0] == "m", a.layout[1] == "m"
        A = _dev(torch, a.M * a.K, 1)
        B = _dev(torch, a.N * a.K, 2)
        C = torch.empty(a.M * a.N, dtype=torch.float32 if a.f32 else torch.bfloat16, device="cuda")
        lda = a.M if a_mn else a.K
        ldb = a.N if b_mn else a.K
        R = _dev(torch, a.M * a.N, 3) if a.res else None
        fn = lambda: L.mt_gemm_bf16(A, lda, int(a_mn), B, ldb, int(b_mn), C, a.N, int(a.f32), 0, a.M, a.N, a.K,  # noqa
                                    None, R, a.N if a.res else 0, stream=st)
        work, unit = 2.0 * a.M * a.N * a.K, "TFLOP/s"
        shape = dict(M=a.M, N=a.N, K=a.K, layout=a.layout, f32=a.f32, res=a.res)
    elif a.op == "gemm_swiglu":
        # the gate/up projection with the SwiGLU epilogue (m, and g and u for the backward)
        A = _dev(torch, a.M * a.K, 1)
        W = _dev(torch, 2 * a.F * a.K, 2, 0.02)
        m = torch.empty(a.M * a.F, dtype=torch.bfloat16, device="cuda")
        gu = torch.empty(a.M * 2 * a.F, dtype=torch.bfloat16, device="cuda")
        fn = lambda: L.mt_gemm_swiglu_bf16(A, a.K, W, a.K, m, a.F, gu, 2 * a.F, a.M, a.F, a.K, st)  # noqa: E731
        work, unit = 2.0 * a.M * 2 * a.F * a.K, "TFLOP/s"
        shape = dict(M=a.M, F=a.F, K=a.K)
    elif a.op == "gemm_swiglu_bwd":
        # dm = dY Wd with the SwiGLU backward over [g|u] in place
        dY = _dev(torch, a.M * a.K, 1)
        Wd = _dev(torch, a.K * a.F, 2, 0.02)
        gu = _dev(torch, a.M * 2 * a.F, 3)
        fn = lambda: L.mt_gemm_swiglu_bwd_bf16(dY, a.K, Wd, a.F, gu, 2 * a.F, a.M, a.F, a.K, st)  # noqa: E731
        work, unit = 2.0 * a.M * a.F * a.K, "TFLOP/s"
        shape = dict(M=a.M, F=a.F, K=a.K)
    elif a.op in ("attn_fwd", "attn_bwd"):
        ld = (a.nq + 2 * a.nkv) * a.d
        qkv = _dev(torch, a.B * a.T * ld, 1)
        o = torch.empty(a.B * a.T * a.nq * a.d, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(a.B * a.nq * a.T, dtype=torch.float32, device="cuda")
        L.mt_attention_fwd(qkv, ld, o, a.nq * a.d, lse, a.B, a.T, a.nq, a.nkv, a.d, st)
        causal = 0.5 * a.T * a.T
        if a.op == "attn_fwd":
            fn = lambda: L.mt_attention_fwd(qkv, ld, o, a.nq * a.d, lse, a.B, a.T, a.nq, a.nkv, a.d, st)  # noqa
            work = 4.0 * a.B * a.nq * a.d * causal
        else:
            do = _dev(torch, a.B * a.T * a.nq * a.d, 3)
            dqkv = torch.empty_like(qkv)
            nws = L.mt_attention_bwd_workspace_bytes(a.B, a.T, a.nq)
            ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
            fn = lambda: L.mt_attention_bwd(qkv, ld, o, do, a.nq * a.d, lse, dqkv, a.B, a.T, a.nq, a.nkv, a.d,  # noqa
                                            ws, nws, st)
            work = 10.0 * a.B * a.nq * a.d * causal  # dV, dP, dQ, dK (the recomputed S not counted)
        unit = "TFLOP/s"
        shape = dict(B=a.B, T=a.T, nq=a.nq, nkv=a.nkv, d=a.d)
    elif a.op == "rmsnorm":
        x = _dev(torch, a.rows * a.H, 1)
        g = _dev(torch, a.H, 2)
        y = torch.empty_like(x)
        rstd = torch.empty(a.rows, dtype=torch.float32, device="cuda")
        fn = lambda: L.mt_rmsnorm_fwd(x, g, y, rstd, a.rows, a.H, 1e-6, st)  # noqa
        work, unit = 4.0 * a.rows * a.H, "GB/s"
        shape = dict(rows=a.rows, H=a.H)
    elif a.op == "swiglu":
        gu = _dev(torch, a.rows * 2 * a.F, 1)
        m = torch.empty(a.rows * a.F, dtype=torch.bfloat16, device="cuda")
        fn = lambda: L.mt_swiglu_fwd(gu, m, a.rows, a.F, st)  # noqa
        work, unit = 6.0 * a.rows * a.F, "GB/s"
        shape = dict(rows=a.rows, F=a.F)
    else:
        cfg = L.make_cfg(a.hidden, a.nq, a.nkv, a.d, a.F)
        off = L.mt_layer_param_offsets(cfg)
        w = _dev(torch, off.record_elems, 1, 0.02)
        x = _dev(torch, a.B * a.T * a.hidden, 2)
        dy = _dev(torch, a.B * a.T * a.hidden, 3)
        y = torch.empty_like(x)
        dx = torch.empty_like(x)
        dw = torch.empty(off.record_elems, dtype=torch.float32, device="cuda")
        nws = L.mt_layer_workspace_bytes(cfg, a.B, a.T, 0)
        ws = torch.empty(nws, dtype=torch.uint8, device="cuda")

        def fn():
            L.mt_layer_fwd(cfg, w, x, y, a.B, a.T, 0, ws, nws, st)
            L.mt_layer_recompute_bwd(cfg, w, x, dy, dx, dw, a.B, a.T, 0, ws, nws, st)
        M = a.B * a.T
        p_lin = off.param_count - 2 * a.hidden
        f_fwd = 2.0 * M * p_lin + 2.0 * a.B * a.T * a.T * a.nq * a.d
        work, unit = f_fwd * 4, "TFLOP/s"  # forward + recompute + backward (2x)
        shape = dict(hidden=a.hidden, nq=a.nq, nkv=a.nkv, d=a.d, F=a.F, B=a.B, T=a.T)

    for _ in range(a.warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(a.reps):
        fn()
    e1.record(st)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / a.reps
    rate = work / (ms / 1e3) / (1e12 if unit == "TFLOP/s" else 1e9)
    err = L.mt_device_error(clear=True)
    print(json.dumps({"op": a.op, **shape, "ms": ms, "rate": rate, "unit": unit, "device_error": err}))
    if err:
        raise SystemExit(1)


if __name__ == "__main__":
    np.seterr(all="ignore")
    main()
