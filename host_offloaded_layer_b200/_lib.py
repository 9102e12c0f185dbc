"""ctypes binding of the C ABI declared in include/mt.h (argument marshalling only).

Every function here has the name of its C entry point, converts its
arguments (torch tensors become their device or host addresses, streams
their ``cuda_stream`` handles), calls the library and raises ``MTError`` with
``mt_last_error()`` when the status is not ``MT_OK``. No computation happens
in Python, and there is no fallback: if ``libmt.so`` is missing, ``load()``
raises.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmt.so")

c_i32, c_i64, c_u64, c_f32, c_vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_float, ctypes.c_void_p

STATUS = {
    0: "MT_OK", 1: "MT_ERR_INVALID_ARG", 2: "MT_ERR_ALIGNMENT", 3: "MT_ERR_WORKSPACE", 4: "MT_ERR_OOM",
    5: "MT_ERR_CUDA", 6: "MT_ERR_TIMEOUT", 7: "MT_ERR_SINK", 8: "MT_ERR_INJECTED", 9: "MT_ERR_UNSUPPORTED",
    10: "MT_ERR_DEVICE",
}


class MTError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS.get(code, code)}: {msg}")
        self.code = code
        self.name = STATUS.get(code, str(code))


class mt_layer_cfg(ctypes.Structure):
    _fields_ = [("hidden", c_i32), ("n_q_heads", c_i32), ("n_kv_heads", c_i32), ("head_dim", c_i32),
                ("ffn", c_i32), ("qkv_bias", c_i32), ("rms_eps", c_f32), ("rope_theta", c_f32)]


class mt_param_offsets(ctypes.Structure):
    _fields_ = [(n, c_u64) for n in ("g1", "wq", "wk", "wv", "bq", "bk", "bv", "wo", "g2", "wg", "wu", "wd",
                                     "record_elems", "param_count")]


class mt_engine_opts(ctypes.Structure):
    _fields_ = [(n, c_i32) for n in ("ckpt_interval", "n_weight_slots", "n_host_slabs", "n_dev_grad_slabs",
                                     "mlp_chunk", "resident", "timeout_ms", "fail_h2d_at", "time_gemms",
                                     "no_slab_pool", "trace", "recompute_internals")]


class mt_trace_rec(ctypes.Structure):
    _fields_ = [("kind", c_i32), ("layer", c_i32), ("begin_ms", c_f32), ("end_ms", c_f32)]


TRACE_KINDS = ("h2d", "forward", "reforward", "backward", "d2h")


class mt_trace_summary(ctypes.Structure):
    _fields_ = [("span_ms", ctypes.c_double), ("h2d_ms", ctypes.c_double), ("d2h_ms", ctypes.c_double),
                ("fwd_ms", ctypes.c_double), ("refwd_ms", ctypes.c_double), ("bwd_ms", ctypes.c_double),
                ("exposed_h2d_ms", ctypes.c_double), ("exposed_d2h_ms", ctypes.c_double),
                ("idle_other_ms", ctypes.c_double)]

    def as_dict(self) -> dict:
        return {k: getattr(self, k) for k, _ in self._fields_}


class mt_stats(ctypes.Structure):
    _fields_ = [("step_ms", ctypes.c_double),
                ("h2d_bytes", c_u64), ("d2h_bytes", c_u64), ("layer_fwd_calls", c_u64), ("layer_bwd_calls", c_u64),
                ("weight_loads", c_u64), ("exec_flops", ctypes.c_double), ("gemm_ms", ctypes.c_double),
                ("gemm_flops", ctypes.c_double), ("gemm_launches", c_u64), ("device_bytes", c_u64),
                ("sink_ms", ctypes.c_double), ("kernel_launches", c_u64), ("traced", c_i32),
                ("trace", mt_trace_summary)]


class mt_adamw_cfg(ctypes.Structure):
    _fields_ = [("lr", c_f32), ("beta1", c_f32), ("beta2", c_f32), ("eps", c_f32), ("weight_decay", c_f32),
                ("n_threads", c_i32)]


mt_grad_sink = ctypes.CFUNCTYPE(c_i32, c_i32, ctypes.POINTER(c_f32), c_u64, c_vp)
mt_head_hook = ctypes.CFUNCTYPE(c_i32, c_vp, c_vp, c_vp, c_vp)

_P = c_vp
_CFG = ctypes.POINTER(mt_layer_cfg)
# name -> (restype, argtypes); restype c_i32 means an mt_status
_SIGS = {
    "mt_last_error": (ctypes.c_char_p, []),
    "mt_device_error": (c_i32, [ctypes.POINTER(c_i32), c_i32]),
    "mt_layer_param_count": (c_u64, [_CFG]),
    "mt_layer_param_offsets": (c_i32, [_CFG, ctypes.POINTER(mt_param_offsets)]),
    "mt_layer_workspace_bytes": (c_u64, [_CFG, c_i32, c_i32, c_i32]),
    "mt_layer_fwd": (c_i32, [_CFG, _P, _P, _P, c_i32, c_i32, c_i32, _P, c_u64, _P]),
    "mt_layer_recompute_bwd": (c_i32, [_CFG, _P, _P, _P, _P, _P, c_i32, c_i32, c_i32, _P, c_u64, _P]),
    "mt_gemm_bf16": (c_i32, [_P, c_i64, c_i32, _P, c_i64, c_i32, _P, c_i64, c_i32, c_i32, c_i64, c_i64, c_i64,
                             _P, _P, c_i64, _P]),
    "mt_gemm_swiglu_bf16": (c_i32, [_P, c_i64, _P, c_i64, _P, c_i64, _P, c_i64, c_i64, c_i64, c_i64, _P]),
    "mt_gemm_swiglu_bwd_bf16": (c_i32, [_P, c_i64, _P, c_i64, _P, c_i64, c_i64, c_i64, c_i64, _P]),
    "mt_rmsnorm_fwd": (c_i32, [_P, _P, _P, _P, c_i64, c_i32, c_f32, _P]),
    "mt_rmsnorm_bwd_workspace_bytes": (c_u64, [c_i64, c_i32]),
    "mt_rmsnorm_bwd": (c_i32, [_P, _P, _P, _P, _P, _P, _P, c_i64, c_i32, _P, c_u64, _P]),
    "mt_rmsnorm_bwd_noalloc": (c_i32, [_P, _P, _P, _P, _P, _P, _P, c_i64, c_i32, _P]),
    "mt_rope": (c_i32, [_P, c_i64, c_i32, c_i32, c_i32, c_i32, c_f32, c_i32, _P]),
    "mt_swiglu_fwd": (c_i32, [_P, _P, c_i64, c_i32, _P]),
    "mt_swiglu_bwd": (c_i32, [_P, _P, _P, c_i64, c_i32, _P]),
    "mt_colsum_workspace_bytes": (c_u64, [c_i64, c_i64]),
    "mt_colsum": (c_i32, [_P, c_i64, c_i64, c_i64, _P, _P, c_u64, _P]),
    "mt_attention_fwd": (c_i32, [_P, c_i64, _P, c_i64, _P, c_i32, c_i32, c_i32, c_i32, c_i32, _P]),
    "mt_attention_bwd_workspace_bytes": (c_u64, [c_i32, c_i32, c_i32]),
    "mt_attention_bwd": (c_i32, [_P, c_i64, _P, _P, c_i64, _P, _P, c_i32, c_i32, c_i32, c_i32, c_i32, _P, c_u64,
                                 _P]),
    "mt_host_store_create": (c_i32, [_CFG, c_i32, c_i32, ctypes.POINTER(c_vp)]),
    "mt_host_store_master": (c_vp, [c_vp, c_i32]),
    "mt_host_store_bf16": (c_vp, [c_vp, c_i32]),
    "mt_host_store_refresh_bf16": (c_i32, [c_vp, c_i32]),
    "mt_host_store_destroy": (None, [c_vp]),
    "mt_engine_workspace_bytes": (c_u64, [_CFG, c_i32, c_i32, c_i32, ctypes.POINTER(mt_engine_opts)]),
    "mt_engine_create": (c_i32, [_CFG, c_i32, c_i32, c_i32, ctypes.POINTER(mt_engine_opts), _P, c_u64, _P, _P, _P,
                                 ctypes.POINTER(c_vp)]),
    "mt_stream_step": (c_i32, [c_vp, c_vp, _P, _P, _P, _P, mt_grad_sink, c_vp]),
    "mt_stream_step_hooked": (c_i32, [c_vp, c_vp, _P, _P, _P, _P, mt_grad_sink, c_vp, mt_head_hook, c_vp]),
    "mt_stream_step_host": (c_i32, [c_vp, c_vp, _P, _P, _P, _P, mt_grad_sink, c_vp]),
    "mt_engine_trace": (c_i32, [c_vp, ctypes.POINTER(mt_trace_rec), c_i32, ctypes.POINTER(c_i32)]),
    "mt_trace_summarize": (c_i32, [ctypes.POINTER(mt_trace_rec), c_i32, ctypes.POINTER(mt_trace_summary)]),
    "mt_engine_stats": (c_i32, [c_vp, ctypes.POINTER(mt_stats)]),
    "mt_engine_reset": (c_i32, [c_vp]),
    "mt_engine_destroy": (None, [c_vp]),
    "mt_embed_fwd": (c_i32, [_P, _P, _P, c_i64, c_i32, c_i32, _P, _P]),
    "mt_embed_sort": (c_i32, [_P, c_i64, c_i32, _P, _P]),
    "mt_embed_bwd": (c_i32, [_P, _P, _P, _P, c_i32, c_i32, _P]),
    "mt_head_workspace_bytes": (c_u64, [c_i64, c_i32, c_i32, c_i32]),
    "mt_head_loss_fwd_bwd": (c_i32, [_P, _P, _P, _P, c_i64, c_i32, c_i32, c_f32, c_i32, _P, _P, _P, _P, _P, c_u64,
                                     _P]),
    "mt_adamw_update": (c_i32, [_P, _P, _P, _P, c_u64, ctypes.POINTER(mt_adamw_cfg), c_i64]),
    "mt_host_optimizer_create": (c_i32, [c_vp, ctypes.POINTER(mt_adamw_cfg), ctypes.POINTER(c_vp)]),
    "mt_host_optimizer_sink": (c_i32, [c_i32, ctypes.POINTER(c_f32), c_u64, c_vp]),
    "mt_host_optimizer_destroy": (None, [c_vp]),
    "mt_schedule_len": (c_i32, [c_i32, c_i32]),
    "mt_schedule": (c_i32, [c_i32, c_i32, c_i32, ctypes.POINTER(c_i32), ctypes.POINTER(c_i32),
                            ctypes.POINTER(c_i32), ctypes.POINTER(c_i32)]),
}
_lib: ctypes.CDLL | None = None


def load() -> ctypes.CDLL:
    """Loads libmt.so (built in-tree by host_offloaded_layer_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m host_offloaded_layer_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if hasattr(x, "ctypes"):  # numpy array
        return x.ctypes.data
    raise TypeError(f"cannot take the address of {type(x)}")


def _stream(s) -> int | None:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def last_error() -> str:
    return load().mt_last_error().decode(errors="replace")


def mt_last_error() -> str:
    """The calling thread's last error message (same as last_error())."""
    return last_error()


def _check(code: int) -> None:
    if code != 0:
        raise MTError(code, last_error())


def make_cfg(hidden, n_q_heads, n_kv_heads, head_dim, ffn, qkv_bias=True, rms_eps=1e-6, rope_theta=1e6):
    return mt_layer_cfg(hidden, n_q_heads, n_kv_heads, head_dim, ffn, 1 if qkv_bias else 0, rms_eps, rope_theta)


# ---------------------------------------------------------------- thin wrappers
def mt_device_error(clear: bool = True) -> int:
    v = c_i32(0)
    _check(load().mt_device_error(ctypes.byref(v), 1 if clear else 0))
    return v.value


def mt_layer_param_count(cfg) -> int:
    return load().mt_layer_param_count(ctypes.byref(cfg))


def mt_layer_param_offsets(cfg) -> mt_param_offsets:
    o = mt_param_offsets()
    _check(load().mt_layer_param_offsets(ctypes.byref(cfg), ctypes.byref(o)))
    return o


def mt_layer_workspace_bytes(cfg, B, T, mlp_chunk=0) -> int:
    return load().mt_layer_workspace_bytes(ctypes.byref(cfg), B, T, mlp_chunk)


def mt_layer_fwd(cfg, w, x, y, B, T, mlp_chunk, ws, ws_bytes, stream=None):
    _check(load().mt_layer_fwd(ctypes.byref(cfg), _ptr(w), _ptr(x), _ptr(y), B, T, mlp_chunk, _ptr(ws), ws_bytes,
                               _stream(stream)))


def mt_layer_recompute_bwd(cfg, w, x, dy, dx, dw, B, T, mlp_chunk, ws, ws_bytes, stream=None):
    _check(load().mt_layer_recompute_bwd(ctypes.byref(cfg), _ptr(w), _ptr(x), _ptr(dy), _ptr(dx), _ptr(dw), B, T,
                                         mlp_chunk, _ptr(ws), ws_bytes, _stream(stream)))


def mt_gemm_bf16(A, lda, a_mn_major, Bm, ldb, b_mn_major, C, ldc, c_f32, accumulate, M, N, K, bias=None,
                 residual=None, ldr=0, stream=None):
    _check(load().mt_gemm_bf16(_ptr(A), lda, a_mn_major, _ptr(Bm), ldb, b_mn_major, _ptr(C), ldc, c_f32, accumulate,
                               M, N, K, _ptr(bias), _ptr(residual), ldr, _stream(stream)))


def mt_gemm_swiglu_bf16(A, lda, Wgu, ldw, m, ldm, gu, ld_gu, M, F, K, stream=None):
    _check(load().mt_gemm_swiglu_bf16(_ptr(A), lda, _ptr(Wgu), ldw, _ptr(m), ldm, _ptr(gu), ld_gu, M, F, K,
                                      _stream(stream)))


def mt_gemm_swiglu_bwd_bf16(dY, ld_dy, Wd, ldw, gu, ld_gu, M, F, K, stream=None):
    _check(load().mt_gemm_swiglu_bwd_bf16(_ptr(dY), ld_dy, _ptr(Wd), ldw, _ptr(gu), ld_gu, M, F, K, _stream(stream)))


def mt_rmsnorm_fwd(x, g, y, rstd, rows, H, eps, stream=None):
    _check(load().mt_rmsnorm_fwd(_ptr(x), _ptr(g), _ptr(y), _ptr(rstd), rows, H, eps, _stream(stream)))


def mt_rmsnorm_bwd_workspace_bytes(rows, H) -> int:
    return load().mt_rmsnorm_bwd_workspace_bytes(rows, H)


def mt_rmsnorm_bwd(dy, x, g, rstd, dres, dx, dg, rows, H, ws, ws_bytes, stream=None):
    _check(load().mt_rmsnorm_bwd(_ptr(dy), _ptr(x), _ptr(g), _ptr(rstd), _ptr(dres), _ptr(dx), _ptr(dg), rows, H,
                                 _ptr(ws), ws_bytes, _stream(stream)))


def mt_rmsnorm_bwd_noalloc(dy, x, g, rstd, dres, dx, dg, rows, H, stream=None):
    _check(load().mt_rmsnorm_bwd_noalloc(_ptr(dy), _ptr(x), _ptr(g), _ptr(rstd), _ptr(dres), _ptr(dx), _ptr(dg), rows,
                                         H, _stream(stream)))


def mt_rope(x, ld, B, T, n_heads, head_dim, theta, inverse, stream=None):
    _check(load().mt_rope(_ptr(x), ld, B, T, n_heads, head_dim, theta, 1 if inverse else 0, _stream(stream)))


def mt_swiglu_fwd(gu, m, rows, F, stream=None):
    _check(load().mt_swiglu_fwd(_ptr(gu), _ptr(m), rows, F, _stream(stream)))


def mt_swiglu_bwd(dm, gu, dgu, rows, F, stream=None):
    _check(load().mt_swiglu_bwd(_ptr(dm), _ptr(gu), _ptr(dgu), rows, F, _stream(stream)))


def mt_colsum_workspace_bytes(rows, cols) -> int:
    return load().mt_colsum_workspace_bytes(rows, cols)


def mt_colsum(X, rows, cols, ld, out, ws, ws_bytes, stream=None):
    _check(load().mt_colsum(_ptr(X), rows, cols, ld, _ptr(out), _ptr(ws), ws_bytes, _stream(stream)))


def mt_attention_fwd(qkv, ld_qkv, o, ld_o, lse, B, T, nq, nkv, d, stream=None):
    _check(load().mt_attention_fwd(_ptr(qkv), ld_qkv, _ptr(o), ld_o, _ptr(lse), B, T, nq, nkv, d, _stream(stream)))


def mt_attention_bwd_workspace_bytes(B, T, nq) -> int:
    return load().mt_attention_bwd_workspace_bytes(B, T, nq)


def mt_attention_bwd(qkv, ld_qkv, o, d_o, ld_o, lse, dqkv, B, T, nq, nkv, d, ws, ws_bytes, stream=None):
    _check(load().mt_attention_bwd(_ptr(qkv), ld_qkv, _ptr(o), _ptr(d_o), ld_o, _ptr(lse), _ptr(dqkv), B, T, nq, nkv,
                                   d, _ptr(ws), ws_bytes, _stream(stream)))


def mt_host_store_create(cfg, n_layers, keep_fp32_master=True) -> int:
    h = c_vp()
    _check(load().mt_host_store_create(ctypes.byref(cfg), n_layers, 1 if keep_fp32_master else 0, ctypes.byref(h)))
    return h.value


def mt_host_store_master(store, layer) -> int:
    return load().mt_host_store_master(store, layer) or 0


def mt_host_store_bf16(store, layer) -> int:
    return load().mt_host_store_bf16(store, layer) or 0


def mt_host_store_refresh_bf16(store, n_threads=0):
    _check(load().mt_host_store_refresh_bf16(store, n_threads))


def mt_host_store_destroy(store):
    load().mt_host_store_destroy(store)


def make_opts(ckpt_interval=4, n_weight_slots=0, n_host_slabs=0, n_dev_grad_slabs=0, mlp_chunk=0, resident=0,
              timeout_ms=0, fail_h2d_at=0, time_gemms=0, no_slab_pool=0, trace=0,
              recompute_internals=0) -> mt_engine_opts:
    return mt_engine_opts(ckpt_interval, n_weight_slots, n_host_slabs, n_dev_grad_slabs, mlp_chunk, resident,
                          timeout_ms, fail_h2d_at, time_gemms, no_slab_pool, trace, recompute_internals)


def mt_engine_workspace_bytes(cfg, n_layers, B, T, opts) -> int:
    return load().mt_engine_workspace_bytes(ctypes.byref(cfg), n_layers, B, T, ctypes.byref(opts))


def mt_engine_create(cfg, n_layers, B, T, opts, dev_ws, dev_ws_bytes, compute, prefetch, offload) -> int:
    h = c_vp()
    _check(load().mt_engine_create(ctypes.byref(cfg), n_layers, B, T, ctypes.byref(opts), _ptr(dev_ws), dev_ws_bytes,
                                   _stream(compute), _stream(prefetch), _stream(offload), ctypes.byref(h)))
    return h.value


_NULL_SINK = ctypes.cast(None, mt_grad_sink)


def mt_stream_step(engine, store, x0, dy_top, y_top, dx0, sink=None, user=None):
    _check(load().mt_stream_step(engine, store, _ptr(x0), _ptr(dy_top), _ptr(y_top), _ptr(dx0),
                                 sink if sink is not None else _NULL_SINK, user))


_NULL_HOOK = ctypes.cast(None, mt_head_hook)


def mt_stream_step_hooked(engine, store, x0, dy_top, y_top, dx0, sink=None, user=None, hook=None, hook_user=None):
    _check(load().mt_stream_step_hooked(engine, store, _ptr(x0), _ptr(dy_top), _ptr(y_top), _ptr(dx0),
                                        sink if sink is not None else _NULL_SINK, user,
                                        hook if hook is not None else _NULL_HOOK, hook_user))


def mt_stream_step_host(engine, store, x0, dy_top, y_top, dx0, sink=None, user=None):
    _check(load().mt_stream_step_host(engine, store, _ptr(x0), _ptr(dy_top), _ptr(y_top), _ptr(dx0),
                                      sink if sink is not None else _NULL_SINK, user))


def mt_engine_stats(engine) -> mt_stats:
    s = mt_stats()
    _check(load().mt_engine_stats(engine, ctypes.byref(s)))
    return s


def mt_engine_trace(engine, cap=4096) -> list:
    """The last step's timeline: [{kind, layer, begin_ms, end_ms}] in issue order."""
    recs = (mt_trace_rec * cap)()
    n = c_i32(0)
    _check(load().mt_engine_trace(engine, recs, cap, ctypes.byref(n)))
    return [{"kind": TRACE_KINDS[r.kind], "layer": r.layer, "begin_ms": r.begin_ms, "end_ms": r.end_ms}
            for r in recs[:min(n.value, cap)]]


def mt_trace_summarize(records) -> dict:
    """Overlap summary of timeline records ({kind, layer, begin_ms, end_ms}, kinds named as
    mt_engine_trace gives them): per-phase times and the exposed transfer time."""
    arr = (mt_trace_rec * max(1, len(records)))()
    for i, r in enumerate(records):
        arr[i] = mt_trace_rec(TRACE_KINDS.index(r["kind"]), r["layer"], r["begin_ms"], r["end_ms"])
    out = mt_trace_summary()
    _check(load().mt_trace_summarize(arr, len(records), ctypes.byref(out)))
    return out.as_dict()


def mt_engine_reset(engine):
    _check(load().mt_engine_reset(engine))


def mt_engine_destroy(engine):
    load().mt_engine_destroy(engine)


def mt_schedule_len(n_layers, K) -> int:
    return load().mt_schedule_len(n_layers, K)


def mt_schedule(n_layers, K, n_slots):
    n = load().mt_schedule_len(n_layers, K)
    arrs = [(c_i32 * n)() for _ in range(4)]
    _check(load().mt_schedule(n_layers, K, n_slots, *arrs))
    return [list(a) for a in arrs]


def mt_adamw_update(w, m, v, g, n, cfg, t):
    _check(load().mt_adamw_update(_ptr(w), _ptr(m), _ptr(v), _ptr(g), n, ctypes.byref(cfg), t))


def mt_host_optimizer_create(store, cfg) -> int:
    h = c_vp()
    _check(load().mt_host_optimizer_create(store, ctypes.byref(cfg), ctypes.byref(h)))
    return h.value


def mt_host_optimizer_destroy(opt):
    load().mt_host_optimizer_destroy(opt)


def mt_host_optimizer_sink(layer, grad, n, opt):
    """Applies one layer's gradient record (host fp32, n elements) to the optimizer `opt` directly."""
    _check(load().mt_host_optimizer_sink(layer, ctypes.cast(_ptr(grad), ctypes.POINTER(c_f32)), n, opt))


def optimizer_sink():
    """The library's AdamW sink as a callable for mt_stream_step (pass the optimizer as `user`)."""
    return ctypes.cast(load().mt_host_optimizer_sink, mt_grad_sink)


def mt_embed_fwd(tokens, E, x, M, H, V, bad_tokens, stream=None):
    _check(load().mt_embed_fwd(_ptr(tokens), _ptr(E), _ptr(x), M, H, V, _ptr(bad_tokens), _stream(stream)))


def mt_embed_sort(tokens, M, V, order, start):
    _check(load().mt_embed_sort(_ptr(tokens), M, V, _ptr(order), _ptr(start)))


def mt_embed_bwd(order, start, dx, dE, H, V, stream=None):
    _check(load().mt_embed_bwd(_ptr(order), _ptr(start), _ptr(dx), _ptr(dE), H, V, _stream(stream)))


def mt_head_workspace_bytes(M, H, V, vocab_chunk) -> int:
    return load().mt_head_workspace_bytes(M, H, V, vocab_chunk)


def mt_head_loss_fwd_bwd(y, gf, W, targets, M, H, V, eps, vocab_chunk, loss, dy, dgf, dW, ws, ws_bytes, stream=None):
    _check(load().mt_head_loss_fwd_bwd(_ptr(y), _ptr(gf), _ptr(W), _ptr(targets), M, H, V, eps, vocab_chunk,
                                       _ptr(loss), _ptr(dy), _ptr(dgf), _ptr(dW), _ptr(ws), ws_bytes,
                                       _stream(stream)))
