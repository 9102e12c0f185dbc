"""Host-side logic that needs no GPU: the C-ABI library loads and exports every
entry point of include/mt.h, the layer record geometry, the streaming
schedule, argument validation, and the throughput formula."""
import json
import os
import re

import pytest

from host_offloaded_layer_b200 import _lib as L
from host_offloaded_layer_b200 import metrics

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden")

QWEN7B = dict(hidden=3584, n_q_heads=28, n_kv_heads=4, head_dim=128, ffn=18944)
QWEN14B = dict(hidden=5120, n_q_heads=40, n_kv_heads=8, head_dim=128, ffn=13824)
TINY = dict(hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64, ffn=688)


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "mt.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    # function declarations: a return type, the name, "(" (function-pointer typedefs are "(*name)")
    names = re.findall(r"\b(?:mt_status|uint64_t|int32_t|void|float|mt_bf16|char)\s*\*?\s*(mt_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def test_library_exports_every_declared_entry_point(lib):
    names = _declared_functions()
    assert len(names) >= 30
    for n in names:
        assert hasattr(lib, n), n
        assert n in L._SIGS, f"binding lacks {n}"


def test_param_count_reproduces_table5_depth_study():
    g = json.load(open(os.path.join(GOLDEN, "table5_depth.json")))
    cfg = L.make_cfg(g["hidden"], g["n_q_heads"], g["n_kv_heads"], g["head_dim"], g["ffn"])
    p_layer = L.mt_layer_param_count(cfg)
    assert p_layer == 233057792
    rows = g["rows"]
    # per-layer count from the depth deltas alone (no vocabulary assumption)
    for (l0, p0), (l1, p1) in zip(rows, rows[1:]):
        assert abs((p1 - p0) * 1e9 / (l1 - l0) - p_layer) / p_layer < 5e-3
    # totals with the untied embedding + head of the Qwen2.5 vocabulary
    for layers, billions in rows:
        total = layers * p_layer + 2 * 152064 * g["hidden"]
        assert abs(total / 1e9 - billions) <= 0.01


def test_record_layout_contiguity_and_alignment():
    for shape in (QWEN7B, QWEN14B, TINY):
        cfg = L.make_cfg(**shape)
        o = L.mt_layer_param_offsets(cfg)
        H, F = shape["hidden"], shape["ffn"]
        hq = shape["n_q_heads"] * shape["head_dim"]
        hkv = shape["n_kv_heads"] * shape["head_dim"]
        assert o.wk == o.wq + hq * H and o.wv == o.wk + hkv * H
        assert o.bk == o.bq + hq and o.bv == o.bk + hkv
        assert o.wu == o.wg + F * H
        for blk in (o.g1, o.wq, o.bq, o.wo, o.g2, o.wg, o.wd, o.record_elems):
            assert blk % 128 == 0
        ends = [o.g1 + H, o.wv + hkv * H, o.bv + hkv, o.wo + H * hq, o.g2 + H, o.wu + F * H, o.wd + H * F]
        starts = [o.g1, o.wq, o.bq, o.wo, o.g2, o.wg, o.wd]
        for a, b in zip(ends[:-1], starts[1:]):
            assert a <= b
        assert ends[-1] <= o.record_elems
        assert o.param_count == L.mt_layer_param_count(cfg)
    assert L.mt_layer_param_count(L.make_cfg(**QWEN14B)) == 275268608
    assert L.mt_layer_param_count(L.make_cfg(**TINY)) == 726016


def test_device_workspace_does_not_grow_with_depth():
    """MegaTrain Table 5: device allocation is the same at every depth."""
    cfg = L.make_cfg(**QWEN7B)
    opts = L.make_opts(ckpt_interval=4)
    base = L.mt_engine_workspace_bytes(cfg, 4, 1, 1024, opts)
    assert base > 0
    # only the checkpoint stash (one activation per K layers) depends on depth
    act = 1 * 1024 * 3584 * 2
    for layers in (28, 42, 180):
        extra = L.mt_engine_workspace_bytes(cfg, layers, 1, 1024, opts) - base
        assert extra == ((layers + 3) // 4 - 1) * act


@pytest.mark.parametrize("n_layers,K,R", [(4, 4, 4), (28, 4, 4), (6, 2, 2), (5, 1, 2), (7, 3, 3), (3, 4, 1)])
def test_schedule_holds_each_layer_when_used(n_layers, K, R):
    layer, kind, slot, load = L.mt_schedule(n_layers, K, R)
    # forward 0..L-1, then per segment: re-forward of all but the last, backward descending
    assert layer[:n_layers] == list(range(n_layers)) and set(kind[:n_layers]) == {0}
    bwd = [l for l, k in zip(layer, kind) if k == 2]
    assert bwd == list(range(n_layers - 1, -1, -1))
    holds = [None] * R
    loads = 0
    for i in range(len(layer)):
        assert 0 <= slot[i] < R
        if load[i]:
            holds[slot[i]] = layer[i]
            loads += 1
        assert holds[slot[i]] == layer[i]
        if i > 0 and R > 1:
            assert not (load[i] and slot[i] == slot[i - 1]), "a load must not evict the layer in use"
    # with a K-slot ring each layer streams in at most twice per step (forward and
    # its backward segment); a single buffer may also reload for the re-forward
    assert loads <= (2 if R >= K else 3) * n_layers
    if R >= n_layers:
        assert loads == n_layers


def test_python_binding_has_every_declared_entry_point():
    """The binding offers a function of the same name for every call the header declares."""
    decl = set(re.findall(r"\b(?:mt_status|uint64_t|int32_t|void|float|mt_bf16|char)\s*\*?\s*(mt_[a-z0-9_]+)\s*\(",
                          open(os.path.join(ROOT, "include", "mt.h")).read()))
    missing = sorted(n for n in decl if not callable(getattr(L, n, None)))
    assert not missing, missing
    assert L.mt_schedule_len(4, 4) == len(L.mt_schedule(4, 4, 4)[0])


def test_invalid_arguments_are_rejected_without_a_gpu():
    with pytest.raises(L.MTError) as e:
        L.mt_layer_param_offsets(L.make_cfg(256, 4, 3, 64, 688))
    assert e.value.name == "MT_ERR_INVALID_ARG"
    assert L.mt_layer_param_count(L.make_cfg(0, 4, 2, 64, 688)) == 0
    with pytest.raises(L.MTError) as e:
        L.mt_gemm_bf16(None, 8, 0, None, 8, 0, None, 8, 0, 0, 8, 8, 8)
    assert e.value.name == "MT_ERR_INVALID_ARG"
    with pytest.raises(L.MTError) as e:
        L.mt_gemm_bf16(16, 8, 0, 16, 8, 0, 16, 8, 0, 1, 8, 8, 8)  # accumulate into bf16
    assert e.value.name == "MT_ERR_INVALID_ARG"
    with pytest.raises(L.MTError) as e:
        L.mt_gemm_bf16(16, 12, 0, 16, 8, 0, 16, 8, 0, 0, 8, 8, 8)  # lda not a multiple of 8
    assert e.value.name == "MT_ERR_ALIGNMENT"
    assert L.mt_layer_workspace_bytes(L.make_cfg(256, 4, 2, 64, 688), 0, 128, 0) == 0
    with pytest.raises(L.MTError) as e:
        L.mt_attention_fwd(16, 512, 16, 256, 16, 1, 8, 4, 2, 96)
    assert e.value.name == "MT_ERR_UNSUPPORTED"
    opts = L.make_opts(ckpt_interval=0)
    assert L.mt_engine_workspace_bytes(L.make_cfg(**TINY), 2, 1, 8, opts) == 0
    with pytest.raises(L.MTError) as e:
        L.mt_engine_trace(None)
    assert e.value.name == "MT_ERR_INVALID_ARG"
    with pytest.raises(L.MTError) as e:  # the hooked step checks its arguments before any work
        L.mt_stream_step_hooked(None, None, None, None, None, None)
    assert e.value.name == "MT_ERR_INVALID_ARG"
    with pytest.raises(L.MTError) as e:
        L.mt_gemm_swiglu_bwd_bf16(16, 8, 16, 8, 16, 8, 8, 8, 8)  # ld_gu < 2 F
    assert e.value.name == "MT_ERR_INVALID_ARG"
    with pytest.raises(L.MTError) as e:
        L.mt_gemm_swiglu_bwd_bf16(16, 8, 16, 8, 16, 12, 8, 6, 8)  # F not a multiple of 8
    assert e.value.name == "MT_ERR_ALIGNMENT"
    with pytest.raises(L.MTError) as e:
        L.mt_head_loss_fwd_bwd(16, 16, 16, 16, 8, 12, 16, 1e-6, 8, 16, 16, 16, 16, 16, 1 << 20)  # H % 8
    assert e.value.name == "MT_ERR_INVALID_ARG"


def test_tflops_formula_reproduces_table7_long_context_rows():
    g = json.load(open(os.path.join(GOLDEN, "table7_longctx.json")))
    m = g["model"]
    for r in g["rows"]:
        tf = metrics.sustained_tflops(m["N"], m["L"], m["H"], r["B"], r["T"], r["step_s"])
        assert abs(tf - r["tflops"]) / r["tflops"] < 1e-3, (r, tf)
    assert metrics.tokens_per_s(96, 1024, 2.0) == 49152.0


def test_cpu_adamw_matches_oracle_over_three_steps():
    import numpy as np

    from oracle.optimizer import adamw_step
    rng = np.random.default_rng(61)
    n = 3_000_001  # several threads' worth, odd length
    w = rng.standard_normal(n).astype(np.float32)
    m = np.zeros(n, np.float32)
    v = np.zeros(n, np.float32)
    cfg = L.mt_adamw_cfg(1e-3, 0.9, 0.95, 1e-8, 0.01, 0)
    w64, m64, v64 = w.astype(np.float64), m.astype(np.float64), v.astype(np.float64)
    for t in range(1, 4):
        g = rng.standard_normal(n).astype(np.float32)
        L.mt_adamw_update(w, m, v, g, n, cfg, t)
        w64, m64, v64 = adamw_step(w64, m64, v64, g.astype(np.float64), t, 1e-3, 0.9, 0.95, 1e-8, 0.01)
    assert np.max(np.abs(w - w64)) < 1e-6
    assert np.max(np.abs(m - m64)) < 1e-6 and np.max(np.abs(v - v64)) < 1e-6
    with pytest.raises(L.MTError):
        L.mt_adamw_update(w, m, v, g, n, cfg, 0)


def test_bench_reference_arm_prints_one_json_line():
    """`bench.py --impl reference` times the CPU oracle and prints the contract's line."""
    import subprocess
    import sys
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "1",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOPS" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_embedding_sort_is_stable_and_complete():
    import numpy as np
    tok = np.array([3, 1, 3, 0, 3, 1], np.int32)
    order = np.empty(6, np.int32)
    start = np.empty(5, np.int32)
    L.mt_embed_sort(tok, 6, 4, order, start)
    assert list(start) == [0, 1, 3, 3, 6]
    assert list(order) == [3, 1, 5, 0, 2, 4]
    with pytest.raises(L.MTError):
        L.mt_embed_sort(np.array([4], np.int32), 1, 4, order, start)


def test_gemm_traffic_is_tied_to_the_gemm_code_not_its_comments(tmp_path, monkeypatch):
    """bench.py reports the committed GEMM DRAM traffic only for the code it was measured on:
    the hash ignores // comments and blank lines, and any code change (or another workload)
    turns the figure into null."""
    import importlib
    import shutil
    import sys
    sys.path.insert(0, ROOT)
    bench = importlib.import_module("bench")
    csrc = tmp_path / "host_offloaded_layer_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    for f in ("gemm.cu", "tcgen05.cuh"):
        shutil.copy(os.path.join(ROOT, "host_offloaded_layer_b200", "csrc", f), csrc / f)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.gemm_source_hash()
    (tmp_path / "profiles" / "gemm2_kernel_traffic.txt").write_text(
        "# header: with a colon\nkernel_code_sha256: %s\nworkload: w\ndram_bytes_per_launch: 123\n" % h)
    assert bench.gemm_traffic("w") == 123.0
    assert bench.gemm_traffic("other") is None
    g = csrc / "gemm.cu"
    g.write_text(g.read_text() + "\n// a comment only\n\n")
    assert bench.gemm_source_hash() == h and bench.gemm_traffic("w") == 123.0
    g.write_text(g.read_text() + "static int changed_code = 1;\n")
    assert bench.gemm_source_hash() != h and bench.gemm_traffic("w") is None


def test_trace_summary_attributes_idle_compute_to_the_copies_in_flight():
    """A hand-made two-layer timeline: the compute stream waits 2 ms for the first upload,
    runs, waits 1 ms for the second upload, runs the backward, then waits 1.5 ms for the
    last gradient offload to drain; a 0.5 ms gap with nothing in flight counts as neither."""
    recs = [
        {"kind": "h2d", "layer": 0, "begin_ms": 0.0, "end_ms": 2.0},
        {"kind": "h2d", "layer": 1, "begin_ms": 2.0, "end_ms": 5.0},
        {"kind": "forward", "layer": 0, "begin_ms": 2.0, "end_ms": 4.0},
        {"kind": "forward", "layer": 1, "begin_ms": 5.0, "end_ms": 6.0},
        {"kind": "backward", "layer": 1, "begin_ms": 6.5, "end_ms": 9.0},
        {"kind": "d2h", "layer": 1, "begin_ms": 8.0, "end_ms": 10.5},
        {"kind": "reforward", "layer": 0, "begin_ms": 9.0, "end_ms": 9.25},
        {"kind": "backward", "layer": 0, "begin_ms": 9.25, "end_ms": 10.0},
        {"kind": "d2h", "layer": 0, "begin_ms": 10.0, "end_ms": 11.5},
    ]
    s = L.mt_trace_summarize(recs)
    assert s["span_ms"] == pytest.approx(11.5)
    assert s["h2d_ms"] == pytest.approx(5.0) and s["d2h_ms"] == pytest.approx(4.0)
    assert s["fwd_ms"] == pytest.approx(3.0) and s["refwd_ms"] == pytest.approx(0.25)
    assert s["bwd_ms"] == pytest.approx(3.25)
    assert s["exposed_h2d_ms"] == pytest.approx(2.0 + 1.0)
    assert s["exposed_d2h_ms"] == pytest.approx(1.5)
    assert s["idle_other_ms"] == pytest.approx(0.5)
    # every instant of the span is either compute or one of the three idle kinds
    busy = s["fwd_ms"] + s["refwd_ms"] + s["bwd_ms"]
    assert busy + s["exposed_h2d_ms"] + s["exposed_d2h_ms"] + s["idle_other_ms"] == pytest.approx(s["span_ms"])
    assert L.mt_trace_summarize([])["span_ms"] == 0.0
    with pytest.raises(L.MTError):
        L.mt_trace_summarize([{"kind": "forward", "layer": 0, "begin_ms": 2.0, "end_ms": 1.0}])


def test_bench_peak_choice_and_cpu_step_extrapolation():
    """The bench takes the sustained bf16 peak unless the run's SM clock was above the clock
    that peak was measured at, and extrapolates the oracle's step time from its sample
    (exact when the sample is one layer of the workload itself)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    peaks = {"bf16_tflops": 1700.0, "bf16_tflops_sustained": 1400.0, "bf16_sustained_sm_mhz": 1350}
    assert bench.pick_peak(peaks, "measured", 1300.0)["chosen"] == 1400.0
    assert bench.pick_peak(peaks, "measured", 1950.0)["chosen"] == 1700.0
    assert bench.pick_peak({"bf16_tflops": 1700.0}, "measured", None)["chosen"] == 1700.0
    cfg = dict(shape=dict(hidden=3584), L=1, B=1, T=1024)
    assert bench.oracle_step_extrapolated(cfg, 233_057_792, 2.0, 1024) == pytest.approx(2.0)
    cfg28 = dict(shape=dict(hidden=3584), L=28, B=96, T=1024)
    assert bench.oracle_step_extrapolated(cfg28, 233_057_792, 2.0, 1024) == pytest.approx(28 * 96 * 2.0)
    # attention's share grows with T^2: doubling T more than doubles the step
    long = dict(shape=dict(hidden=3584), L=1, B=1, T=2048)
    assert bench.oracle_step_extrapolated(long, 233_057_792, 2.0, 1024) > 4.0


def test_sweep_points_fit_the_device_and_the_host():
    """Every point of bench.py's depth / width / context sweeps (MegaTrain Tables 5-7) sizes an engine
    workspace that fits a B200's 180 GB and a pinned bf16 store plus gradient slabs within 190 GB of host
    memory; the depth sweep's device workspace grows only by the checkpoint stash (one [B, T, H] bf16
    activation per K layers)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    ws = {}
    for sweep, points in bench.SWEEPS.items():
        for pt in points:
            cfg = L.make_cfg(**pt["shape"])
            opts = L.make_opts(ckpt_interval=pt["K"], mlp_chunk=pt["chunk"],
                               recompute_internals=pt.get("recompute_internals", 0))
            n = L.mt_engine_workspace_bytes(cfg, pt["L"], pt["B"], pt["T"], opts)
            rec = L.mt_layer_param_offsets(cfg).record_elems
            assert 0 < n < 180e9, (sweep, pt["label"], n)
            assert pt["L"] * rec * 2 + 3 * rec * 4 < 190e9, (sweep, pt["label"])
            ws[(sweep, pt["L"])] = n
    depth = sorted((L_, n) for (s, L_), n in ws.items() if s == "depth")
    act = 32 * 1024 * 3584 * 2
    for (l0, n0), (l1, n1) in zip(depth, depth[1:]):
        assert n1 - n0 == ((l1 + 3) // 4 - (l0 + 3) // 4) * act
    w = bench.width_shape(3.5)
    assert (w["hidden"], w["ffn"], w["n_q_heads"], w["n_kv_heads"]) == (12544, 66304, 98, 14)  # Table 6, 3.5x


def test_bench_keeps_the_fp32_master_unless_the_host_cannot_hold_it(monkeypatch):
    import importlib.util
    import types
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    cfg = L.make_cfg(**QWEN7B)
    args = types.SimpleNamespace(sink="none")
    monkeypatch.setenv("LOCAL_WORLD_SIZE", "1")
    assert bench.keep_master(L, cfg, 1, args)  # one 7B layer: 1.4 GB
    monkeypatch.setenv("LOCAL_WORLD_SIZE", "100000")
    assert not bench.keep_master(L, cfg, 28, args)  # far beyond any host
    assert bench.keep_master(L, cfg, 28, types.SimpleNamespace(sink="adamw"))  # the optimizer needs it
