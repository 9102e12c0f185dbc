"""Benchmark of the streamed decoder-stack training step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 2] [--impl ours|reference]

A step is one call of ``mt_stream_step``: forward over the whole stack with
checkpoints every K layers, then per segment re-forward, recompute and
backward, with every layer's bf16 weights streamed in from the pinned host
store and its fp32 gradients streamed out through the slab pool. Workloads
(synthetic data, seeded, N(0, 0.02) weights, N(0, 1) inputs and dY):

  1 tiny      hidden 256, 4/2 heads x 64, FFN 688, 1 layer, batch 2 x 128
  2 7b_x4     Qwen2.5-7B layer shape x 4 layers, batch 8 x 1024, K = 4
  3 7b_x28    7B shape x 28 layers, batch 96 x 1024, K = 4  (default: MegaTrain Table 4's
              "MegaTrain (full)" setting, batch size 96)
  4 14b_x48   Qwen2.5-14B shape x 48 layers, batch 64 x 1024, K = 4
  5 7b_32k    7B shape x 28 layers, batch 1 x 32768, MLP in 4096-token chunks, K = 4

The metric is sustained TFLOPS by the model-FLOPs formula 6ND + 12LHT^2
(MegaTrain Table 7 caption) with N = layers x parameters per layer, plus
tokens/s. One process per GPU; with N > 1 (torchrun) every rank runs its own
replica on its own batch (the path has no collective), the timed region is
bracketed by barriers and the slowest rank's time is used.

``--impl reference`` times the CPU oracle (float64 numpy) on a bounded
sample of the same workload and reports the same metric.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from host_offloaded_layer_b200 import metrics, synth  # noqa: E402

QWEN7B = dict(hidden=3584, n_q_heads=28, n_kv_heads=4, head_dim=128, ffn=18944)
QWEN14B = dict(hidden=5120, n_q_heads=40, n_kv_heads=8, head_dim=128, ffn=13824)
CONFIGS = {
    1: dict(name="tiny_1layer_b2x128", shape=dict(hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64, ffn=688),
            L=1, B=2, T=128, K=4, chunk=0),
    2: dict(name="qwen2.5-7b-shape_x4_b8x1024", shape=QWEN7B, L=4, B=8, T=1024, K=4, chunk=0),
    3: dict(name="qwen2.5-7b-shape_x28_b96x1024", shape=QWEN7B, L=28, B=96, T=1024, K=4, chunk=0),
    4: dict(name="qwen2.5-14b-shape_x48_b64x1024", shape=QWEN14B, L=48, B=64, T=1024, K=4, chunk=0),
    5: dict(name="qwen2.5-7b-shape_x28_b1x32768_mlpchunk4096", shape=QWEN7B, L=28, B=1, T=32768, K=4, chunk=4096),
    # MegaTrain Table 7's 128K-context row (B = 1, chunked MLP): the long-context regime, beyond the hot-path
    # workloads above; one step takes tens of seconds
    6: dict(name="qwen2.5-7b-shape_x28_b1x131072_mlpchunk4096", shape=QWEN7B, L=28, B=1, T=131072, K=4,
            chunk=4096),
}
# The ablations of MegaTrain Table 4, as engine options.
ABLATIONS = {
    "none": {},
    "single_buffer": {"n_weight_slots": 1},  # "w/o Double Buffering"
    "no_slab_pool": {"no_slab_pool": 1},     # "w/o Gradient Slab Pool"
    "ckpt1": {"ckpt_interval": 1},           # "w/ Checkpoint Interval=1"
}
VOCAB = 152064  # Qwen2.5 tokenizer (an assumption: the pages do not state it)
METRIC = "sustained TFLOPS (6ND+12LHT²) & tokens/s, streamed 7B/14B layer stack, 1 B200"
UNIT = "TFLOPS"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def _flat_items(d, prefix=""):
    for k, v in (d.items() if isinstance(d, dict) else []):
        key = f"{prefix}.{k}" if prefix else str(k)
        if isinstance(v, dict):
            yield from _flat_items(v, key)
        else:
            yield key, v


def sustained_peak_clock_mhz(peaks) -> tuple[float, str]:
    """SM clock at which the sustained bf16 peak was taken: from the peaks file when it
    records one, else the clock the profiling notes of this pool give for it (about 1.3 GHz
    under the 1000 W power cap)."""
    for k, v in _flat_items(peaks):
        kl = k.lower()
        if "sustain" in kl and ("mhz" in kl or "clock" in kl) and isinstance(v, (int, float)) and v > 100:
            return float(v), k
    return 1300.0, "assumed (sustained loop under the power cap)"


def pick_peak(peaks, src, sm_mhz):
    """The bf16 denominator for kernels timed inside a step: the sustained peak, unless the
    run's median SM clock is above the clock the sustained peak was taken at (the GPU was
    not held at that clock), in which case the burst peak."""
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sust = float(peaks.get("bf16_tflops_sustained", burst))
    clk, clk_src = sustained_peak_clock_mhz(peaks)
    use_burst = sm_mhz is not None and sm_mhz > 1.05 * clk
    return {"burst": burst, "sustained": sust, "chosen": burst if use_burst else sust,
            "which": "bf16_tflops (burst)" if use_burst else "bf16_tflops_sustained",
            "source": src, "sustained_clock_mhz": clk, "sustained_clock_source": clk_src}


def gemm_source_hash() -> str:
    """SHA-256 of the GEMM's code (gemm.cu + tcgen05.cuh) with // comments, trailing
    blanks and empty lines removed, so that an edit of comments alone keeps it."""
    import hashlib
    import re
    csrc = os.path.join(ROOT, "host_offloaded_layer_b200", "csrc")
    h = hashlib.sha256()
    for f in ("gemm.cu", "tcgen05.cuh"):
        lines = (re.sub(r"//.*$", "", ln).rstrip() for ln in open(os.path.join(csrc, f)).read().splitlines())
        h.update(("\n".join(ln for ln in lines if ln) + "\n").encode())
    return h.hexdigest()


def gemm_traffic(workload: str):
    """DRAM bytes per GEMM launch from the committed ncu summary, when that summary
    was taken on this workload with the current GEMM code (else None)."""
    path = os.path.join(ROOT, "profiles", "gemm2_kernel_traffic.txt")
    if not os.path.exists(path):
        return None
    kv = {}
    for line in open(path):
        if ":" in line and not line.startswith("#"):
            k, v = line.split(":", 1)
            kv[k.strip()] = v.strip()
    h = gemm_source_hash()
    if kv.get("kernel_code_sha256") != h or kv.get("workload") != workload:
        return None
    return float(kv["dram_bytes_per_launch"])


def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("LOCAL_RANK", "0"))


def max_over_ranks(ms: float, dist=None, device=None) -> float:
    """The slowest rank's time (all ranks call this in the same order)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job rate: the units all ranks processed over the slowest rank's time (per second)."""
    return units_per_rank * world / (ms_max / 1e3)


def model_flops(cfg, p_layer, vocab=0):
    """6ND + 12LHT^2 with N the stack's parameters (plus the untied embedding and
    LM head, 2 V H, for the whole model)."""
    sh = cfg["shape"]
    N = cfg["L"] * p_layer + 2 * vocab * sh["hidden"]
    return metrics.model_flops(N, cfg["L"], sh["hidden"], cfg["B"], cfg["T"])


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons during a region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu = gpu_index

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx.append(float(f[1]))
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- host link
def measure_link(torch, nbytes=1 << 30):
    """Pinned-memory copy bandwidth (GB/s): H2D, D2H, and both at once."""
    h = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    h2 = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    d = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    d2 = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()

    def timed(fn, reps=3):
        best = 1e9
        for _ in range(reps):
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            fn()
            torch.cuda.synchronize()
            best = min(best, time.perf_counter() - t0)
        return best

    with torch.cuda.stream(s1):
        t_h2d = timed(lambda: d.copy_(h, non_blocking=True))
        t_d2h = timed(lambda: h.copy_(d, non_blocking=True))

    def both():
        with torch.cuda.stream(s1):
            d.copy_(h, non_blocking=True)
        with torch.cuda.stream(s2):
            h2.copy_(d2, non_blocking=True)

    t_both = timed(both)
    del h, h2, d, d2
    return {"h2d_gbs": nbytes / t_h2d / 1e9, "d2h_gbs": nbytes / t_d2h / 1e9, "bidir_gbs": 2 * nbytes / t_both / 1e9}


# ---------------------------------------------------------------- CPU oracle sample
def oracle_sample(cfg, budget_s=12.0, max_tokens=1024):
    """Times the float64 oracle (forward + backward of one layer of this workload's
    shape) on one sequence of up to ``max_tokens`` tokens; returns (TFLOPS, description,
    threads, seconds per rep, tokens)."""
    from oracle import OracleCfg, layer_bwd, layer_fwd
    sh = cfg["shape"]
    T = min(cfg["T"], max_tokens)
    B = 1
    ocfg = OracleCfg(**sh)
    shapes = synth.layer_tensor_shapes(**sh)
    w = {k: synth.bf16_round(v).astype(np.float64) for k, v in synth.layer_weights_f32(shapes, 1234, 0).items()}
    x = synth.bf16_bits_to_f32(synth.activations_bf16_bits(1234, synth.X0_ID, B, T, sh["hidden"])).astype(np.float64)
    dy = synth.bf16_bits_to_f32(synth.activations_bf16_bits(1234, synth.DY_ID, B, T, sh["hidden"])).astype(np.float64)
    p_layer = sum(int(np.prod(s)) for s in shapes.values())
    flops = metrics.model_flops(p_layer, 1, sh["hidden"], B, T)
    reps, t0 = 0, time.perf_counter()
    while True:
        y, cache = layer_fwd(ocfg, w, x)
        layer_bwd(ocfg, w, cache, dy)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s or reps >= 50:
            break
    threads = os.environ.get("OPENBLAS_NUM_THREADS") or os.environ.get("OMP_NUM_THREADS") or str(os.cpu_count())
    desc = f"1 layer of the workload's shape, forward+backward, batch {B} x {T} tokens, {reps} reps in {el:.1f} s"
    return flops * reps / el / 1e12, desc, int(threads), el / reps, T


def oracle_step_extrapolated(cfg, p_layer, sec, T_s):
    """The oracle's time for one whole step of the workload (forward + backward of every
    layer on all B x T tokens, no recompute), extrapolated from one layer on T_s tokens:
    the sample's time is split in proportion to its projection FLOPs (6 P T_s) and
    attention FLOPs (12 H T_s^2); the first part scales with the tokens B T, the second
    with B T^2, and both with the layer count."""
    H = cfg["shape"]["hidden"]
    lin, att = 6.0 * p_layer * T_s, 12.0 * H * T_s ** 2
    t_lin, t_att = sec * lin / (lin + att), sec * att / (lin + att)
    B, T = cfg["B"], cfg["T"]
    return cfg["L"] * (t_lin * B * T / T_s + t_att * B * (T / T_s) ** 2)


def run_reference(args, cfg, rank, world):
    """The reference arm: the CPU oracle, timed on the host cores."""
    if rank != 0:
        return
    vals = []
    for i in range(args.warmup + args.steps):
        tf, desc, threads, sec, _ = oracle_sample(cfg, budget_s=max(1.0, 20.0 / max(1, args.steps + args.warmup)))
        if i >= args.warmup:
            vals.append(tf)
    v = statistics.median(vals)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg["name"], "sample": desc},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- ours
def fill_store(L_, store, cfg, n_layers, seed=1234, master=True):
    """The synthetic weights of every layer: into the fp32 master and then the bf16 copy (RNE), or,
    for a store without a master, one layer at a time through an fp32 scratch record."""
    off = L_.mt_layer_param_offsets(cfg)
    shapes = synth.layer_tensor_shapes(cfg.hidden, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.ffn,
                                       bool(cfg.qkv_bias))
    scratch = None if master else np.zeros(off.record_elems, dtype=np.float32)
    for l in range(n_layers):
        if master:
            ptr = L_.mt_host_store_master(store, l)
            rec = np.ctypeslib.as_array((ctypes.c_float * off.record_elems).from_address(ptr))
        else:
            rec = scratch
        for name, shp in shapes.items():
            o = getattr(off, name)
            n = int(np.prod(shp))
            if name in ("g1", "g2"):
                rec[o:o + n] = 1.0
            else:
                synth.normal_f32(seed, l, synth.TENSOR_IDS[name], n, synth.WEIGHT_STD, out=rec[o:o + n])
        if not master:
            bf = np.ctypeslib.as_array((ctypes.c_uint16 * off.record_elems).from_address(L_.mt_host_store_bf16(store, l)))
            bf[:] = synth.f32_to_bf16_bits(rec)
    if master:
        L_.mt_host_store_refresh_bf16(store, 0)


def keep_master(L_, cfg, n_layers, args) -> bool:
    """Whether this rank's host store can hold the fp32 master next to the bf16 copy: the optimizer sink
    needs it; with the no-op sink it is kept whenever the host's available memory, shared by the ranks
    of this node, holds every rank's store and slabs with 25% to spare."""
    if args.sink == "adamw":
        return True
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:
        return True
    rec = L_.mt_layer_param_offsets(cfg).record_elems
    local = int(os.environ.get("LOCAL_WORLD_SIZE", "1"))
    need = local * (n_layers * rec * 6 + 3 * rec * 4)
    return 1.25 * need <= avail


def run_ours(args, cfg, rank, world, local_rank):
    import torch
    from host_offloaded_layer_b200 import _lib as L_
    torch.cuda.set_device(local_rank)
    L_.load()
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        pg = dist
    sh = cfg["shape"]
    lcfg = L_.make_cfg(**sh)
    p_layer = L_.mt_layer_param_count(lcfg)
    nL, B, T = cfg["L"], cfg["B"], cfg["T"]
    abl = ABLATIONS[args.ablation]
    opts = L_.make_opts(ckpt_interval=abl.get("ckpt_interval", cfg["K"]), mlp_chunk=cfg["chunk"], time_gemms=1,
                        timeout_ms=120000, n_weight_slots=abl.get("n_weight_slots", 0),
                        no_slab_pool=abl.get("no_slab_pool", 0), recompute_internals=int(args.recompute_internals))
    master = keep_master(L_, lcfg, nL, args)
    store = L_.mt_host_store_create(lcfg, nL, master)
    fill_store(L_, store, lcfg, nL, master=master)
    nbytes = L_.mt_engine_workspace_bytes(lcfg, nL, B, T, opts)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    streams = [torch.cuda.Stream() for _ in range(3)]
    eng = L_.mt_engine_create(lcfg, nL, B, T, opts, ws, nbytes, *streams)
    H = sh["hidden"]
    x0 = synth.activations_bf16_bits(1234 + rank, synth.X0_ID, B, T, H)
    dy = synth.activations_bf16_bits(1234 + rank, synth.DY_ID, B, T, H)
    x_d = torch.from_numpy(x0.view(np.int16)).cuda()
    dy_d = torch.from_numpy(dy.view(np.int16)).cuda()
    y_d, dx_d = torch.empty_like(x_d), torch.empty_like(x_d)
    xh, dyh = torch.from_numpy(x0.view(np.int16)).pin_memory(), torch.from_numpy(dy.view(np.int16)).pin_memory()
    yh, dxh = torch.empty_like(xh).pin_memory(), torch.empty_like(xh).pin_memory()
    slab_count = [0]

    def sink(layer, ptr, n, user):  # the gradient record of one layer arrives in host memory
        slab_count[0] += 1
        return 0

    c_sink = L_.mt_grad_sink(sink)
    sink_user = None
    opt = None
    if args.sink == "adamw":  # the library's CPU AdamW: a full training step including the optimizer
        opt = L_.mt_host_optimizer_create(store, L_.mt_adamw_cfg(1e-5, 0.9, 0.95, 1e-8, 0.01, 0))
        c_sink, sink_user = L_.optimizer_sink(), opt
    cs = streams[0]

    def barrier():
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize()

    def timed(fn, steps):
        barrier()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(cs)
        for _ in range(steps):
            fn()
        ev1.record(cs)
        barrier()
        ms = max_over_ranks(ev0.elapsed_time(ev1), pg, "cuda")
        return ms / steps

    dev_step = lambda: L_.mt_stream_step(eng, store, x_d, dy_d, y_d, dx_d, c_sink, sink_user)  # noqa: E731
    head = None
    if args.full_model:
        # the whole model: embedding -> streamed stack -> final norm + LM head + loss (hook) -> streamed
        # backward -> embedding gradient; E, W stay on the device, tokens are synthetic
        V, chunk = VOCAB, 16384
        M = B * T
        g = torch.Generator(device="cuda").manual_seed(4321 + rank)
        E_d = (torch.randn(V, H, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
        W_d = (torch.randn(V, H, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
        gf_d = torch.ones(H, dtype=torch.bfloat16, device="cuda")
        tok = np.random.default_rng(99 + rank).integers(0, V, size=M).astype(np.int32)
        tok_d = torch.from_numpy(tok).cuda()
        tgt_d = torch.from_numpy(np.roll(tok, -1).astype(np.int32)).cuda()
        loss_d = torch.zeros(1, dtype=torch.float32, device="cuda")
        dgf_d = torch.empty(H, dtype=torch.float32, device="cuda")
        dWh_d = torch.empty(V, H, dtype=torch.float32, device="cuda")
        dE_d = torch.empty(V, H, dtype=torch.float32, device="cuda")
        bad_d = torch.zeros(1, dtype=torch.int32, device="cuda")
        nhw = L_.mt_head_workspace_bytes(M, H, V, chunk)
        hws = torch.empty(nhw, dtype=torch.uint8, device="cuda")
        order_h = torch.empty(M, dtype=torch.int32).pin_memory()
        start_h = torch.empty(V + 1, dtype=torch.int32).pin_memory()
        order_d = torch.empty(M, dtype=torch.int32, device="cuda")
        start_d = torch.empty(V + 1, dtype=torch.int32, device="cuda")
        tok_h = torch.from_numpy(tok).pin_memory()
        loss_h = torch.zeros(1, dtype=torch.float32).pin_memory()

        def hook(y_ptr, dy_ptr, stream, user):
            try:
                L_.mt_head_loss_fwd_bwd(y_ptr, gf_d, W_d, tgt_d, M, H, V, 1e-6, chunk, loss_d, dy_ptr, dgf_d, dWh_d,
                                        hws, nhw, stream)
                return 0
            except L_.MTError as e:
                return e.code

        c_hook = L_.mt_head_hook(hook)
        head = (c_hook, hws)  # keep the callback alive

        def dev_step():
            # host side of the embedding backward: the tokens' counting sort (the data loader's work)
            L_.mt_embed_sort(tok_h, M, V, order_h, start_h)
            with torch.cuda.stream(cs):
                order_d.copy_(order_h, non_blocking=True)
                start_d.copy_(start_h, non_blocking=True)
                L_.mt_embed_fwd(tok_d, E_d, x_d, M, H, V, bad_d, cs)
                L_.mt_stream_step_hooked(eng, store, x_d, dy_d, y_d, dx_d, c_sink, sink_user, c_hook, None)
                L_.mt_embed_bwd(order_d, start_d, dx_d, dE_d, H, V, cs)

        def full_host_step():  # tokens in from pinned host memory, the loss back out
            with torch.cuda.stream(cs):
                tok_d.copy_(tok_h, non_blocking=True)
            dev_step()
            with torch.cuda.stream(cs):
                loss_h.copy_(loss_d, non_blocking=True)
            cs.synchronize()
    host_step = lambda: L_.mt_stream_step_host(eng, store, xh, dyh, yh, dxh, c_sink, sink_user)  # noqa: E731
    if args.full_model:
        host_step = full_host_step
    for _ in range(args.warmup):
        dev_step()
    clocks = ClockSampler(local_rank)
    clocks.start()
    ms = timed(dev_step, args.steps)
    clk = clocks.stop()
    st = L_.mt_engine_stats(eng)  # the last timed step
    for _ in range(1):
        host_step()
    ms_e2e = timed(host_step, max(2, args.steps // 5))
    st_e2e = L_.mt_engine_stats(eng)
    assert L_.mt_device_error(clear=True) == 0, "a kernel's bounded wait ran out"
    # one more step, outside every timed region, on an engine over the same memory with the event
    # timeline on: per-phase device times and the transfer time the compute stream waited for
    L_.mt_engine_destroy(eng)
    topts = L_.mt_engine_opts.from_buffer_copy(opts)
    topts.trace = 1
    eng = L_.mt_engine_create(lcfg, nL, B, T, topts, ws, nbytes, *streams)
    dev_step()
    torch.cuda.synchronize()
    st_tr = L_.mt_engine_stats(eng)
    if args.trace and rank == 0:
        with open(args.trace, "w") as f:
            json.dump({"workload": cfg["name"], "intervals": L_.mt_engine_trace(eng)}, f, indent=0)
    link = measure_link(torch) if rank == 0 else None

    mflops = model_flops(cfg, p_layer, VOCAB if args.full_model else 0)
    value = job_throughput(mflops, world, ms) / 1e12
    e2e = job_throughput(mflops, world, ms_e2e) / 1e12
    peaks, src = load_peaks()
    pk = pick_peak(peaks, src, clk.get("sm_mhz"))
    peak_tf = pk["chosen"]
    gemm_tf = st.gemm_flops / (st.gemm_ms / 1e3) / 1e12 if st.gemm_ms > 0 else None
    line = None
    if rank == 0:
        bw = link
        t_h2d = st.h2d_bytes / (bw["h2d_gbs"] * 1e9)
        t_d2h = st.d2h_bytes / (bw["d2h_gbs"] * 1e9)
        t_bi = (st.h2d_bytes + st.d2h_bytes) / (bw["bidir_gbs"] * 1e9)

        def t_roof_at(peak):
            return max(st.exec_flops / (peak * 1e12), t_h2d, t_d2h, t_bi)

        t_comp = st.exec_flops / (peak_tf * 1e12)
        t_roof = t_roof_at(peak_tf)
        if world == 1:  # the CPU baseline is timed at one GPU only
            cpu_tf, cpu_desc, cpu_threads, cpu_sec, cpu_T = oracle_sample(cfg, budget_s=12.0)
        tr = st_tr.trace
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": cfg["name"], "layers": nL, "batch": B, "seq_len": T,
                       "ckpt_interval": abl.get("ckpt_interval", cfg["K"]), "ablation": args.ablation,
                       "full_model": bool(args.full_model),
                       "mlp_chunk": cfg["chunk"], "parallelism": f"replicas{world}" if world > 1 else "single",
                       "l2": "inputs larger than L2 (each layer's weights alone are %.0f MB)" % (p_layer * 2 / 1e6),
                       "sink": ("CPU AdamW on the fp32 master + bf16 refresh (library sink)" if args.sink == "adamw"
                                else "pinned slab handed to a no-op host callback"),
                       "host_store": ("pinned fp32 master + bf16 streaming copy" if master else
                                      "pinned bf16 streaming copy only (the host's memory could not hold every "
                                      "rank's fp32 master; the no-op sink does not read it)")},
            "tokens_per_s": B * T * world / (ms / 1e3),
            "clocks": clk,
            "e2e": {"value": e2e, "unit": UNIT,
                    "h2d_bytes_per_step": int(st_e2e.h2d_bytes) + ((2 * B * T + VOCAB + 1) * 4 if args.full_model else 0),
                    "d2h_bytes_per_step": int(st_e2e.d2h_bytes) + (4 if args.full_model else 0)},
            "gpu_launches": int(st.kernel_launches) * args.steps,
            "roofline": {"bound": "tensor", "kernel": "gemm2_kernel (tcgen05, 2-SM)", "achieved": gemm_tf,
                         "peak": peak_tf, "unit": "TFLOP/s", "frac": (gemm_tf / peak_tf) if gemm_tf else None,
                         "traffic": gemm_traffic(cfg["name"]), "traffic_unit": "bytes per launch",
                         "peak_source": f"{src} {pk['which']}",
                         "frac_of_burst": (gemm_tf / pk["burst"]) if gemm_tf else None,
                         "frac_of_sustained": (gemm_tf / pk["sustained"]) if gemm_tf else None,
                         "peak_rule": ("sustained peak unless the run's median SM clock exceeds the clock it was "
                                       f"taken at ({pk['sustained_clock_mhz']:.0f} MHz, "
                                       f"{pk['sustained_clock_source']})"),
                         "gemm_launches_per_step": int(st.gemm_launches)},
            "step_roofline": {"t_roof_ms": t_roof * 1e3, "t_step_ms": ms, "frac": t_roof / (ms / 1e3),
                              "frac_at_burst_peak": t_roof_at(pk["burst"]) / (ms / 1e3),
                              "frac_at_sustained_peak": t_roof_at(pk["sustained"]) / (ms / 1e3),
                              "t_compute_ms": t_comp * 1e3, "t_h2d_ms": t_h2d * 1e3, "t_d2h_ms": t_d2h * 1e3,
                              "t_bidir_ms": t_bi * 1e3, "exec_tflop": st.exec_flops / 1e12,
                              "model_tflop": mflops / 1e12, "h2d_bytes": int(st.h2d_bytes),
                              "d2h_bytes": int(st.d2h_bytes), "link_gbs": bw,
                              "model_flops_frac": mflops / (ms / 1e3) / (peak_tf * 1e12)},
            "timeline": {"source": "one traced step after the timed ones (CUDA events around every upload, layer "
                                   "call and offload)",
                         "step_ms": tr.span_ms, "fwd_ms": tr.fwd_ms, "refwd_ms": tr.refwd_ms, "bwd_ms": tr.bwd_ms,
                         "h2d_ms": tr.h2d_ms, "d2h_ms": tr.d2h_ms, "exposed_h2d_ms": tr.exposed_h2d_ms,
                         "exposed_d2h_ms": tr.exposed_d2h_ms, "idle_other_ms": tr.idle_other_ms},
            "cpu_baseline": None if world > 1 else {
                "value": cpu_tf, "unit": UNIT, "cores": cpu_threads, "kind": "oracle", "sample": cpu_desc,
                "step_s_extrapolated": oracle_step_extrapolated(cfg, p_layer, cpu_sec, cpu_T),
                "extrapolation": ("the oracle's forward+backward of every layer on all B x T tokens "
                                  "(no recompute), scaled from the sample: projections linearly in "
                                  "tokens, attention in B x T^2 (extrapolated, not measured)")},
            "device_workspace_gb": nbytes / 1e9,
        }
    L_.mt_engine_destroy(eng)
    if opt is not None:
        L_.mt_host_optimizer_destroy(opt)
    L_.mt_host_store_destroy(store)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- sweeps (MegaTrain Tables 5, 6, 7)
def width_shape(scale: float) -> dict:
    """The 7B layer widened by `scale` (MegaTrain Table 6 gives hidden and FFN sizes): head_dim 128
    and the 7:1 query-to-key/value head ratio of the 7B shape are kept (the pages give no heads)."""
    hidden = int(round(3584 * scale))
    nq = hidden // 128
    return dict(hidden=hidden, n_q_heads=nq, n_kv_heads=max(1, nq // 7), head_dim=128, ffn=int(round(18944 * scale)))


SWEEPS = {
    # Table 5: 7B width, depth 28 .. 180 layers
    "depth": [dict(shape=QWEN7B, L=L, B=32, T=1024, K=4, chunk=0, label=f"7b_x{L}") for L in (28, 42, 56, 84, 132, 180)],
    # Table 6: width 1.0x .. 3.5x at a fixed depth (12 layers: a 3.5x stack of 28 layers would need 160 GB of
    # pinned bf16 weights, beyond the host memory of the GPU machine next to the gradient slabs)
    "width": [dict(shape=width_shape(w), L=12, B=32, T=1024, K=4, chunk=0, label=f"width{w}x_x12")
              for w in (1.0, 1.5, 2.0, 2.5, 3.0, 3.5)],
    # Table 7's longest rows: one sequence, MLP in 4096-token chunks (at 512K the four layer-internals sets take
    # 83 GB and the whole workspace 167 GB of the B200's 192 GB)
    "context": [dict(shape=QWEN7B, L=28, B=1, T=T, K=4, chunk=4096, label=f"7b_x28_b1x{T}")
                for T in (131072, 262144, 524288)],
}


def run_sweep(args, local_rank):
    """Throughput of the streamed step across MegaTrain's depth, width and context studies. The host
    store keeps only the bf16 streaming copy (no fp32 master: the sink does not update weights), filled
    with one seeded block of 2^20 N(0, 0.02) values repeated over every record (the values do not change
    the work); one JSON line per point, with the device memory the engine uses."""
    import torch
    from host_offloaded_layer_b200 import _lib as L_
    torch.cuda.set_device(local_rank)
    L_.load()
    points = SWEEPS[args.sweep]
    if args.points:
        points = [points[i] for i in map(int, args.points.split(","))]
    block = synth.f32_to_bf16_bits(synth.normal_f32(1234, 0, 99, 1 << 20, synth.WEIGHT_STD))
    for pt in points:
        sh, nL, B, T = pt["shape"], pt["L"], pt["B"], pt["T"]
        lcfg = L_.make_cfg(**sh)
        off = L_.mt_layer_param_offsets(lcfg)
        p_layer = L_.mt_layer_param_count(lcfg)
        opts = L_.make_opts(ckpt_interval=pt["K"], mlp_chunk=pt["chunk"], timeout_ms=600000,
                            recompute_internals=pt.get("recompute_internals", 0))
        store = L_.mt_host_store_create(lcfg, nL, False)
        rec = np.resize(block, off.record_elems)
        g1, g2 = int(off.g1), int(off.g2)
        rec[g1:g1 + sh["hidden"]] = 0x3F80  # gains 1.0
        rec[g2:g2 + sh["hidden"]] = 0x3F80
        for l in range(nL):
            dst = np.ctypeslib.as_array((ctypes.c_uint16 * off.record_elems).from_address(L_.mt_host_store_bf16(store, l)))
            dst[:] = rec
        nbytes = L_.mt_engine_workspace_bytes(lcfg, nL, B, T, opts)
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        streams = [torch.cuda.Stream() for _ in range(3)]
        eng = L_.mt_engine_create(lcfg, nL, B, T, opts, ws, nbytes, *streams)
        H = sh["hidden"]
        x_d = torch.from_numpy(synth.activations_bf16_bits(1234, synth.X0_ID, B, T, H).view(np.int16)).cuda()
        dy_d = torch.from_numpy(synth.activations_bf16_bits(1234, synth.DY_ID, B, T, H).view(np.int16)).cuda()
        y_d, dx_d = torch.empty_like(x_d), torch.empty_like(x_d)
        step = lambda: L_.mt_stream_step(eng, store, x_d, dy_d, y_d, dx_d)  # noqa: E731
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        clocks = ClockSampler(local_rank)
        clocks.start()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(streams[0])
        for _ in range(args.steps):
            step()
        ev1.record(streams[0])
        torch.cuda.synchronize()
        clk = clocks.stop()
        ms = ev0.elapsed_time(ev1) / args.steps
        st = L_.mt_engine_stats(eng)
        assert L_.mt_device_error(clear=True) == 0, "a kernel's bounded wait ran out"
        mflops = metrics.model_flops(nL * p_layer, nL, H, B, T)
        rec_b = int(off.record_elems)
        persistent = (max(2, pt["K"]) * rec_b * 2 + 2 * rec_b * 4) / 1e9  # weight slots + gradient staging
        print(json.dumps({
            "sweep": args.sweep, "point": pt["label"], "layers": nL, "shape": sh, "batch": B, "seq_len": T,
            "ckpt_interval": pt["K"], "mlp_chunk": pt["chunk"],
            "recompute_internals": pt.get("recompute_internals", 0),
            "params_b": nL * p_layer / 1e9, "tflops": mflops / (ms / 1e3) / 1e12, "tokens_per_s": B * T / (ms / 1e3),
            "step_s": ms / 1e3, "steps": args.steps, "warmup": args.warmup,
            "exec_tflop_per_step": st.exec_flops / 1e12,
            "device_workspace_gb": nbytes / 1e9, "device_weights_and_grad_staging_gb": persistent,
            "host_pinned_gb": (nL * rec_b * 2 + 3 * rec_b * 4) / 1e9, "clocks": clk}), flush=True)
        L_.mt_engine_destroy(eng)
        L_.mt_host_store_destroy(store)
        del ws, x_d, dy_d, y_d, dx_d
        torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", type=int, default=3, choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--full-model", action="store_true",
                    help="add the embedding and the final norm + LM head + loss (vocabulary 152064) to the step")
    ap.add_argument("--trace", default="", metavar="PATH",
                    help="after the measurement, write the event timeline of one more step to PATH (JSON)")
    ap.add_argument("--sink", default="none", choices=["none", "adamw"],
                    help="what receives each layer's gradient record (adamw: the CPU optimizer step)")
    ap.add_argument("--ablation", default="none", choices=sorted(ABLATIONS),
                    help="engine variant of MegaTrain Table 4 (default: the full system)")
    ap.add_argument("--recompute-internals", action="store_true",
                    help="every backward recomputes its layer's internals (one layer workspace, less memory)")
    ap.add_argument("--sweep", default="", choices=["", *SWEEPS],
                    help="instead of the benchmark line: one JSON line per point of the depth (Table 5), width "
                         "(Table 6) or long-context (Table 7) study")
    ap.add_argument("--points", default="", help="with --sweep: comma-separated indices of the points to run")
    args = ap.parse_args()
    rank, world, local_rank = dist_env()
    cfg = CONFIGS[args.config]
    if args.sweep:
        run_sweep(args, local_rank)
        return
    if args.impl == "reference":
        run_reference(args, cfg, rank, world)
    else:
        run_ours(args, cfg, rank, world, local_rank)


if __name__ == "__main__":
    main()
