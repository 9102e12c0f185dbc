"""The streaming engine on the B200: a whole training step over a layer stack
(forward with checkpoints every K layers, segment re-forward, recompute and
backward, weights streamed from the pinned host store, gradients offloaded
through the slab pool) against the oracle, bit-exactness of the streamed
schedule to the device-resident run, and host-side failure handling."""
import ctypes
import time

import numpy as np
import pytest

import helpers as H
from host_offloaded_layer_b200 import _lib as L
from host_offloaded_layer_b200 import synth
from oracle import layer as O

pytestmark = pytest.mark.gpu

TINY = dict(hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64, ffn=688)


QWEN7B = dict(hidden=3584, n_q_heads=28, n_kv_heads=4, head_dim=128, ffn=18944)

_RECORDS = {}


@pytest.fixture(scope="module", autouse=True)
def _free_records():
    yield
    _RECORDS.clear()  # the 7B layers' float64 copies are 1.9 GB each


def _records(shape, n_layers, seed):
    """(bf16 record bits, float64 weights) of each layer, generated once per shape and seed."""
    key = (tuple(sorted(shape.items())), seed)
    have = _RECORDS.setdefault(key, [])
    cfg = L.make_cfg(**shape)
    while len(have) < n_layers:
        have.append(H.layer_record(cfg, seed, len(have), gain_std=0.1))
    return have[:n_layers]


class Stack:
    """Host store + engine for one configuration (seeded synthetic weights)."""

    def __init__(self, shape, n_layers, B, T, seed=1234, **opts):
        import torch
        self.cfg = L.make_cfg(**shape)
        self.L, self.B, self.T = n_layers, B, T
        self.store = L.mt_host_store_create(self.cfg, n_layers, True)
        off = L.mt_layer_param_offsets(self.cfg)
        self.rec_elems = off.record_elems
        recs = _records(shape, n_layers, seed)
        self.w64 = [w64 for _, w64 in recs]
        for l, (rec, _) in enumerate(recs):
            master = np.ctypeslib.as_array((ctypes.c_float * rec.size).from_address(L.mt_host_store_master(self.store, l)))
            master[:] = synth.bf16_bits_to_f32(rec)  # bf16-representable values: RNE keeps them
        L.mt_host_store_refresh_bf16(self.store, 0)
        for l, (rec, _) in enumerate(recs):
            bf = np.ctypeslib.as_array((ctypes.c_uint16 * self.rec_elems).from_address(L.mt_host_store_bf16(self.store, l)))
            assert np.array_equal(bf, rec)
        self.opts = L.make_opts(**opts)
        nbytes = L.mt_engine_workspace_bytes(self.cfg, n_layers, B, T, self.opts)
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        self.streams = [torch.cuda.Stream() for _ in range(3)]
        self.eng = L.mt_engine_create(self.cfg, n_layers, B, T, self.opts, self.ws, nbytes, *self.streams)
        self.x = synth.activations_bf16_bits(seed, synth.X0_ID, B, T, shape["hidden"])
        self.dy = synth.activations_bf16_bits(seed, synth.DY_ID, B, T, shape["hidden"])
        self.grads = {}

        def sink(layer, ptr, n, user):
            self.grads[layer] = np.ctypeslib.as_array(ptr, shape=(n,)).copy()
            return 0

        self.sink = L.mt_grad_sink(sink)

    def step(self, sink=None):
        import torch
        x_d, dy_d = H.dev_bf16(self.x), H.dev_bf16(self.dy)
        y = H.empty_bf16(self.B, self.T, self.cfg.hidden)
        dx = H.empty_bf16(self.B, self.T, self.cfg.hidden)
        torch.cuda.synchronize()
        self.grads = {}
        L.mt_stream_step(self.eng, self.store, x_d, dy_d, y, dx, sink or self.sink)
        torch.cuda.synchronize()
        assert L.mt_device_error(clear=True) == 0
        return y, dx, dict(self.grads)

    def close(self):
        L.mt_engine_destroy(self.eng)
        L.mt_host_store_destroy(self.store)
        del self.ws


def _check_against_oracle(s, y, dx, grads):
    """Y, dX, the residual branch and every layer's gradient record against the oracle's stack."""
    ocfg = H.oracle_cfg(s.cfg)
    x64 = H.bits_to_f64(s.x)
    y_ref, dx_ref, g_ref = O.stack_fwd_bwd(ocfg, s.w64, x64, H.bits_to_f64(s.dy))
    errs = {"Y": H.rel(H.host_f64(y), y_ref), "dX": H.rel(H.host_f64(dx), dx_ref)}
    bad = {k: v for k, v in errs.items() if not v < H.TOL}
    br = H.rel(H.host_f64(y) - x64, y_ref - x64)
    if not br < H.branch_tol(x64, y_ref):
        bad["Y-X"] = br
    assert sorted(grads) == list(range(s.L))
    for l in range(s.L):
        got = H.grads_from_record(s.cfg, grads[l])
        for k, v in g_ref[l].items():
            e = H.rel(got[k], v)
            if not e < H.TOL:
                bad[f"layer{l}.d{k}"] = e
    assert not bad, bad


def _as_bits(t):
    import torch
    return t.view(torch.int16).cpu().numpy()


@pytest.mark.parametrize("n_layers,K", [(3, 2), (4, 4), (5, 1)])
def test_streamed_step_matches_oracle(n_layers, K):
    s = Stack(TINY, n_layers, 2, 128, ckpt_interval=K)
    try:
        y, dx, grads = s.step()
        _check_against_oracle(s, y, dx, grads)
        st = L.mt_engine_stats(s.eng)
        assert st.layer_bwd_calls == n_layers
        assert st.d2h_bytes == n_layers * s.rec_elems * 4
    finally:
        s.close()


def test_streamed_7b_shape_step_matches_oracle():
    """Three Qwen2.5-7B-shaped layers on 1 x 1024 tokens with K = 2 (a re-forwarded
    segment, a recomputed one and the top layer's reuse): the tcgen05 attention,
    the 2-SM GEMMs at the layer's real widths and the engine's piecewise weight
    upload and gradient offload at 7B record sizes, against the oracle per tensor."""
    s = Stack(QWEN7B, 3, 1, 1024, ckpt_interval=2)
    try:
        y, dx, grads = s.step()
        _check_against_oracle(s, y, dx, grads)
    finally:
        s.close()


def test_streamed_long_context_chunked_step_matches_oracle():
    """Two layers at 8192 tokens with the MLP in 2048-token chunks (K = 2, one segment: the forward keeps
    both layers' internals, the attention half only, and the backward recomputes the MLP chunks): the
    chunked path of the long-context workloads through the engine, against the oracle per tensor."""
    shape = dict(hidden=896, n_q_heads=7, n_kv_heads=1, head_dim=128, ffn=2048)
    s = Stack(shape, 2, 1, 8192, ckpt_interval=2, mlp_chunk=2048)
    try:
        y, dx, grads = s.step()
        _check_against_oracle(s, y, dx, grads)
    finally:
        s.close()


def _bit_exact_runs(shape, n_layers, B, T, K, variants):
    runs = {}
    for name, opts in variants.items():
        s = Stack(shape, n_layers, B, T, **{"ckpt_interval": K, **opts})
        try:
            y, dx, g = s.step()
            y2, dx2, g2 = s.step()  # a second step reuses every buffer
            runs[name] = (_as_bits(y), _as_bits(dx), g)
            assert np.array_equal(_as_bits(y), _as_bits(y2)) and np.array_equal(_as_bits(dx), _as_bits(dx2))
            for l in g:
                assert np.array_equal(g[l].view(np.uint32), g2[l].view(np.uint32))
        finally:
            s.close()
    ref = runs.pop("resident")
    for name, (y, dx, g) in runs.items():
        assert np.array_equal(y, ref[0]), name
        assert np.array_equal(dx, ref[1]), name
        for l in ref[2]:
            assert np.array_equal(g[l].view(np.uint32), ref[2][l].view(np.uint32)), (name, l)


def test_7b_shape_streamed_schedules_are_bit_exact_to_resident():
    """At the 7B layer shape: double-buffered streaming, a single weight slot and the
    pool-less offload give the resident run's Y, dX and gradient records bit for bit."""
    _bit_exact_runs(QWEN7B, 3, 1, 1024, 2, {"resident": dict(resident=1), "double": dict(),
                                             "single": dict(n_weight_slots=1), "nopool": dict(no_slab_pool=1),
                                             "recompute": dict(recompute_internals=1)})


def test_7b_shape_b8_streamed_is_bit_exact_to_resident():
    """8 x 1024 tokens: the weight-gradient GEMMs run the 256 x 512 tile (K = 8192)."""
    _bit_exact_runs(QWEN7B, 3, 8, 1024, 2, {"resident": dict(resident=1), "double": dict()})


def test_streamed_schedules_are_bit_exact_to_resident():
    # recompute_internals: every backward recomputes its layer's internals instead of reusing the
    # segment re-forward's; the kernels are deterministic, so the results are the same bits
    _bit_exact_runs(TINY, 5, 2, 128, 2, {"resident": dict(resident=1), "double": dict(),
                                          "single": dict(n_weight_slots=1),
                                          "pool1": dict(n_host_slabs=1, n_dev_grad_slabs=1),
                                          "nopool": dict(no_slab_pool=1),
                                          "recompute": dict(recompute_internals=1),
                                          "recompute_k3": dict(recompute_internals=1, ckpt_interval=3),
                                          "k3": dict(ckpt_interval=3)})


def test_host_buffer_step_equals_device_step():
    import torch
    s = Stack(TINY, 2, 2, 128, ckpt_interval=2)
    try:
        y, dx, g = s.step()
        xh = torch.from_numpy(s.x.view(np.int16).copy()).pin_memory()
        dyh = torch.from_numpy(s.dy.view(np.int16).copy()).pin_memory()
        yh = torch.empty_like(xh).pin_memory()
        dxh = torch.empty_like(xh).pin_memory()
        s.grads = {}
        L.mt_stream_step_host(s.eng, s.store, xh, dyh, yh, dxh, s.sink)
        assert np.array_equal(yh.numpy(), _as_bits(y))
        assert np.array_equal(dxh.numpy(), _as_bits(dx))
        for l in g:
            assert np.array_equal(s.grads[l].view(np.uint32), g[l].view(np.uint32))
    finally:
        s.close()


def test_injected_copy_failure_then_reset_and_recover():
    s = Stack(TINY, 3, 2, 128, ckpt_interval=2, fail_h2d_at=2)
    try:
        with pytest.raises(L.MTError) as e:
            s.step()
        assert e.value.name == "MT_ERR_INJECTED"
        L.mt_engine_reset(s.eng)
        y, dx, g = s.step()  # the injected copy has passed; the step now completes
        ref = Stack(TINY, 3, 2, 128, ckpt_interval=2)
        try:
            y2, dx2, g2 = ref.step()
        finally:
            ref.close()
        assert np.array_equal(_as_bits(y), _as_bits(y2)) and np.array_equal(_as_bits(dx), _as_bits(dx2))
    finally:
        s.close()


def test_sink_error_is_reported_and_engine_recovers():
    s = Stack(TINY, 3, 2, 128, ckpt_interval=2)
    try:
        calls = []

        def bad(layer, ptr, n, user):
            calls.append(layer)
            return 7 if layer == 1 else 0

        bad_sink = L.mt_grad_sink(bad)
        with pytest.raises(L.MTError) as e:
            s.step(sink=bad_sink)
        assert e.value.name == "MT_ERR_SINK"
        assert calls[:2] == [2, 1]
        L.mt_engine_reset(s.eng)
        y, dx, g = s.step()
        assert sorted(g) == [0, 1, 2]
    finally:
        s.close()


def test_slow_sink_times_out_with_a_clean_status():
    s = Stack(TINY, 3, 2, 128, ckpt_interval=2, n_host_slabs=1, timeout_ms=300)
    try:
        def slow(layer, ptr, n, user):
            time.sleep(1.0)
            return 0

        slow_sink = L.mt_grad_sink(slow)
        with pytest.raises(L.MTError) as e:
            s.step(sink=slow_sink)
        assert e.value.name == "MT_ERR_TIMEOUT"
        time.sleep(1.5)
        L.mt_engine_reset(s.eng)
        y, dx, g = s.step()
        assert sorted(g) == [0, 1, 2]
    finally:
        s.close()


def test_cpu_optimizer_sink_closes_the_training_loop():
    """The library's AdamW sink updates each layer's fp32 master from its streamed
    gradient record and refreshes the bf16 copy the next step streams."""
    from oracle.optimizer import adamw_step
    ref = Stack(TINY, 3, 2, 128, ckpt_interval=2)
    try:
        _, _, grads = ref.step()
    finally:
        ref.close()
    s = Stack(TINY, 3, 2, 128, ckpt_interval=2)
    cfg = L.mt_adamw_cfg(1e-2, 0.9, 0.95, 1e-8, 0.1, 0)
    opt = L.mt_host_optimizer_create(s.store, cfg)
    try:
        off = L.mt_layer_param_offsets(s.cfg)
        n = off.record_elems
        masters0 = [np.ctypeslib.as_array((ctypes.c_float * n).from_address(L.mt_host_store_master(s.store, l))).copy()
                    for l in range(3)]
        import torch
        x_d, dy_d = H.dev_bf16(s.x), H.dev_bf16(s.dy)
        y = H.empty_bf16(2, 128, TINY["hidden"])
        dx = H.empty_bf16(2, 128, TINY["hidden"])
        L.mt_stream_step(s.eng, s.store, x_d, dy_d, y, dx, L.optimizer_sink(), opt)
        torch.cuda.synchronize()
        for l in range(3):
            master = np.ctypeslib.as_array((ctypes.c_float * n).from_address(L.mt_host_store_master(s.store, l)))
            bf = np.ctypeslib.as_array((ctypes.c_uint16 * n).from_address(L.mt_host_store_bf16(s.store, l)))
            g = grads[l].astype(np.float64)
            used = np.zeros(n, dtype=bool)
            for name, shp in synth.layer_tensor_shapes(**H.shape_dict(s.cfg)).items():
                o = getattr(off, name)
                used[o:o + int(np.prod(shp))] = True
            w_ref, _, _ = adamw_step(masters0[l][used], 0.0, 0.0, g[used], 1, 1e-2, 0.9, 0.95, 1e-8, 0.1)
            assert np.max(np.abs(master[used] - w_ref)) < 1e-5
            assert np.array_equal(bf[used], synth.f32_to_bf16_bits(master[used]))
        # the next step streams the updated weights
        y2 = H.empty_bf16(2, 128, TINY["hidden"])
        L.mt_stream_step(s.eng, s.store, x_d, dy_d, y2, dx, L.optimizer_sink(), opt)
        torch.cuda.synchronize()
        assert not torch.equal(y.view(torch.int16), y2.view(torch.int16))
    finally:
        L.mt_host_optimizer_destroy(opt)
        s.close()


def test_full_model_step_with_embedding_and_head_hook():
    """Embedding -> streamed layer stack -> (hook) final norm + LM head + loss ->
    streamed backward -> embedding gradient, against the oracle end to end."""
    import torch

    from oracle import head as HD
    V, Lyr, B, T = 1000, 2, 2, 128
    s = Stack(TINY, Lyr, B, T, ckpt_interval=2)
    try:
        Hd = TINY["hidden"]
        M = B * T
        rng = np.random.default_rng(17)
        tok = rng.integers(0, V, size=M).astype(np.int32)
        tgt = np.roll(tok, -1).astype(np.int32)
        E = synth.f32_to_bf16_bits(synth.normal_f32(3, 0, 1, V * Hd, 1.0)).reshape(V, Hd)
        W = synth.f32_to_bf16_bits(synth.normal_f32(3, 0, 2, V * Hd, 0.05)).reshape(V, Hd)
        gf = synth.f32_to_bf16_bits(np.ones(Hd, np.float32))
        E_d, W_d, gf_d = H.dev_bf16(E), H.dev_bf16(W), H.dev_bf16(gf)
        tok_d, tgt_d = torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda()
        x0 = H.empty_bf16(B, T, Hd)
        bad = torch.zeros(1, dtype=torch.int32, device="cuda")
        L.mt_embed_fwd(tok_d, E_d, x0, M, Hd, V, bad)
        loss = torch.zeros(1, dtype=torch.float32, device="cuda")
        dgf = H.empty_f32(Hd)
        dWh = H.empty_f32(V, Hd)
        chunk = 384
        ws = H.workspace(L.mt_head_workspace_bytes(M, Hd, V, chunk))

        def hook(y_ptr, dy_ptr, stream, user):
            try:
                L.mt_head_loss_fwd_bwd(y_ptr, gf_d, W_d, tgt_d, M, Hd, V, 1e-6, chunk, loss, dy_ptr, dgf, dWh, ws,
                                       ws.numel(), stream)
                return 0
            except L.MTError as e:
                return e.code

        c_hook = L.mt_head_hook(hook)
        y = H.empty_bf16(B, T, Hd)
        dy = H.empty_bf16(B, T, Hd)
        dx0 = H.empty_bf16(B, T, Hd)
        torch.cuda.synchronize()
        s.grads = {}
        L.mt_stream_step_hooked(s.eng, s.store, x0, dy, y, dx0, s.sink, None, c_hook, None)
        order = np.empty(M, np.int32)
        start = np.empty(V + 1, np.int32)
        L.mt_embed_sort(tok, M, V, order, start)
        dE = H.empty_f32(V, Hd)
        L.mt_embed_bwd(torch.from_numpy(order).cuda(), torch.from_numpy(start).cuda(), dx0, dE, Hd, V)
        torch.cuda.synchronize()
        assert L.mt_device_error(clear=True) == 0 and bad.item() == 0
        # the oracle, end to end
        ocfg = H.oracle_cfg(s.cfg)
        x64 = HD.embed_fwd(tok.reshape(B, T), H.bits_to_f64(E))
        yy = x64
        for w in s.w64:
            yy, _ = O.layer_fwd(ocfg, w, yy)
        l_ref, dy_ref, dgf_ref, dW_ref = HD.head_loss_fwd_bwd(yy, H.bits_to_f64(gf), H.bits_to_f64(W),
                                                              tgt.reshape(B, T), 1e-6)
        _, dx_ref, g_ref = O.stack_fwd_bwd(ocfg, s.w64, x64, dy_ref)
        dE_ref = HD.embed_bwd(tok.reshape(B, T), dx_ref, V)
        assert abs(loss.item() - l_ref) / l_ref < 1e-3
        assert H.rel(H.host_f64(dy), dy_ref) < H.TOL
        assert H.rel(H.host_f64(dWh), dW_ref) < H.TOL and H.rel(H.host_f64(dgf), dgf_ref) < H.TOL
        assert H.rel(H.host_f64(dx0), dx_ref) < H.TOL
        assert H.rel(H.host_f64(dE), dE_ref) < H.TOL
        for l in range(Lyr):
            got = H.grads_from_record(s.cfg, s.grads[l])
            for k, v in g_ref[l].items():
                assert H.rel(got[k], v) < H.TOL, (l, k)
    finally:
        s.close()


def test_traced_step_gives_an_ordered_timeline():
    """trace = 1: every weight upload, layer call and gradient offload of the last step, in issue
    order, with the dependencies the engine enforces visible in the times."""
    s = Stack(TINY, 5, 2, 64, ckpt_interval=2, trace=1)
    try:
        with pytest.raises(L.MTError):  # nothing traced before the first step
            L.mt_engine_trace(s.eng)
        y0, dx0, g0 = s.step()
        tl = L.mt_engine_trace(s.eng)
        kinds = [r["kind"] for r in tl]
        assert kinds.count("forward") == 5 and kinds.count("backward") == 5 and kinds.count("d2h") == 5
        assert kinds.count("reforward") == 2  # segments [0,2) and [2,4) are re-run; the last is not
        assert kinds.count("h2d") >= 5
        for r in tl:
            assert -1e-3 <= r["begin_ms"] <= r["end_ms"], r
        bwd_end = {r["layer"]: r["end_ms"] for r in tl if r["kind"] == "backward"}
        for r in tl:
            if r["kind"] == "d2h":  # a layer's last gradient piece leaves after its backward
                assert r["end_ms"] >= bwd_end[r["layer"]] - 1e-3, r
        fwd = [r for r in tl if r["kind"] == "forward"]
        assert [r["layer"] for r in fwd] == list(range(5))
        assert all(a["end_ms"] <= b["begin_ms"] + 1e-3 for a, b in zip(fwd, fwd[1:]))  # one compute stream
        # the stats carry the timeline's summary: per-phase device times and exposed transfer time
        st = L.mt_engine_stats(s.eng)
        assert st.traced == 1
        tr = st.trace.as_dict()
        assert tr == pytest.approx(L.mt_trace_summarize(tl))
        busy = tr["fwd_ms"] + tr["refwd_ms"] + tr["bwd_ms"]
        assert busy > 0 and tr["h2d_ms"] > 0 and tr["d2h_ms"] > 0
        assert busy + tr["exposed_h2d_ms"] + tr["exposed_d2h_ms"] + tr["idle_other_ms"] == pytest.approx(tr["span_ms"])
        # tracing changes no result
        y1, dx1, g1 = s.step()
        assert np.array_equal(_as_bits(y0), _as_bits(y1)) and np.array_equal(_as_bits(dx0), _as_bits(dx1))
        assert all(np.array_equal(g0[k], g1[k]) for k in g0)
    finally:
        s.close()


def test_bench_store_fill_without_the_master_gives_the_same_bf16_record():
    """bench.py fills a host store without an fp32 master (when the host's memory cannot hold every rank's)
    one record at a time through an fp32 scratch; the bf16 copy streamed to the GPU is bitwise the one the
    master-plus-refresh path gives."""
    import importlib.util
    import os
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(os.path.dirname(os.path.dirname(
        os.path.abspath(__file__))), "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    cfg = L.make_cfg(**TINY)
    rec = L.mt_layer_param_offsets(cfg).record_elems
    a = L.mt_host_store_create(cfg, 2, True)
    b = L.mt_host_store_create(cfg, 2, False)
    try:
        bench.fill_store(L, a, cfg, 2, master=True)
        bench.fill_store(L, b, cfg, 2, master=False)
        assert L.mt_host_store_master(b, 0) is None or L.mt_host_store_master(b, 0) == 0
        for l in range(2):
            ba = np.ctypeslib.as_array((ctypes.c_uint16 * rec).from_address(L.mt_host_store_bf16(a, l)))
            bb = np.ctypeslib.as_array((ctypes.c_uint16 * rec).from_address(L.mt_host_store_bf16(b, l)))
            assert np.array_equal(ba, bb), l
    finally:
        L.mt_host_store_destroy(a)
        L.mt_host_store_destroy(b)
