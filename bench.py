"""Throughput of the SVDQuant W4A4 NVFP4 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload: the FLUX-like DiT fused QKV projection (M=4608 tokens, K=3072,
N=9216, rank 32), seeded synthetic inputs from workloads.py. One step = one
forward of the layer over the batch: activation quantisation + down
projection, then the block-scaled FP4 GEMM with the fused low-rank up
projection and bias. Inputs are resident in HBM and larger than L2: every
step reads its own copy of X and of the packed weight, cycling through enough
copies that their total is at least twice the L2 size, so each step starts
with its inputs out of cache (no flush kernel runs between steps: a 256 MiB
write flush leaves DRAM busy with its write-back and is charged to the next
kernel). The timed steps are captured once into a CUDA graph and replayed
between two CUDA events on the launching stream (device time, not the host's
issue rate; ms_per_step_loop reports the same steps issued call by call).
Multi-GPU: independent replicas (the layer shards by tokens with no
exchange), max time over ranks. Rank 0 prints one JSON line.

--impl reference times the CPU oracle (float64 restatement of the layer) on
the host cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "W4A4 linear TFLOP/s and tokens/s on 1 B200; % of NVFP4 tensor peak / HBM roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
WORKLOAD = workloads.WORKLOADS[2]   # DiT fused QKV, M=4608, K=3072, N=9216, r=32
FP4_PER_BF16 = 4.0   # nominal dense fp4 / bf16 tensor throughput ratio (9 / 2.25 PFLOP/s)
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of the
# dominant kernel on this workload, from the ncu capture summarised in
# profiles/w4a4_gemm_2sm_kernel_qkv_4608x3072x9216_r32.md. Valid only for the
# kernel as captured: set to None whenever the kernel changes.
NCU_TRAFFIC_BYTES = {("dit_qkv_4608x3072x9216_r32", "w4a4_gemm_2sm_kernel"): 63436032}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def _flops(M, N, K, r):
    return 2.0 * M * N * K + 2.0 * M * r * (K + N)


def _quant_bytes(M, K, r):
    return 2 * M * K + M * K / 2 + M * K / 16 + 2 * M * r + 2 * K * r


def gpu_uuid(device: int) -> str | None:
    """nvidia-smi's identifier ("GPU-xxxxxxxx-...") of the CUDA device `device`,
    or None if it cannot be read."""
    try:
        u = str(torch.cuda.get_device_properties(device).uuid)
    except (RuntimeError, AssertionError, AttributeError):
        return None
    return u if u.startswith("GPU-") else "GPU-" + u


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 50 ms while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        # nvidia-smi numbers GPUs physically and ignores CUDA_VISIBLE_DEVICES, so
        # a CUDA ordinal may name another (possibly another user's) GPU: the
        # device is selected by its UUID (gpu_uuid), and without one nothing is
        # sampled.
        self.uuid = uuid
        self.proc = None

    def __enter__(self):
        if self.uuid is None:
            time.sleep(0.3)
            return self
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50",
                 "-i", self.uuid], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = [l.split(",") for l in (self.out or "").strip().splitlines() if l.count(",") >= 6]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "gpu_uuid": self.uuid}
        sm = [float(r[0]) for r in rows if r[0].strip().replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if "Active" == r[3 + i].strip()})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "gpu_uuid": self.uuid}


def _dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def _max_over_ranks(x: float, world: int) -> float:
    """The largest value over all ranks (every rank calls it, in the same order)."""
    if world == 1:
        return x
    import torch.distributed as dist
    device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ CPU oracle timing
def _oracle_setup(spec, X, W, b, budget_s: float):
    """Load-time work of the CPU oracle (untimed) and the size of a bounded
    sample: the first S rows of X against the first Ns output features (rows
    and output features are independent in the layer, so the sample is an
    exact slice of the workload) sized to take about `budget_s` per forward."""
    from oracle import svdq as osv
    L1, L2, _ = osv.lowrank_factors(W, spec.r)
    g_x = osv.act_global_scale(X)
    full = osv.pack_weight(W, L1, L2)
    S = 64

    def sliced(ns):
        return osv.PackedWeight(full.codes[:ns], full.scales[:ns], full.g_w, full.L1, full.L2[:, :ns])

    t0 = time.perf_counter()
    osv.forward(X[:S], sliced(128), b[:128], g_x)
    t_unit = max(time.perf_counter() - t0, 1e-3)
    ns = int(max(1, min(spec.N // 128, budget_s / t_unit))) * 128
    return sliced(ns), g_x, S, ns


def _oracle_time(X, pw, b, g_x, S, ns) -> float:
    from oracle import svdq as osv
    t0 = time.perf_counter()
    osv.forward(X[:S], pw, b[:ns], g_x)
    return time.perf_counter() - t0


def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def run_reference(args, spec):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    X, W, b = workloads.make_layer(spec)
    budget = max(0.05, min(5.0, 120.0 / max(1, args.steps + args.warmup)))
    pw, g_x, S, ns = _oracle_setup(spec, X, W, b, budget)
    times = []
    for i in range(args.warmup + args.steps):
        dt = _oracle_time(X, pw, b, g_x, S, ns)
        if i >= args.warmup:
            times.append(dt)
    t = statistics.mean(times)
    value = _flops(S, ns, spec.K, spec.r) / t / 1e12
    sample = f"first {S} rows x first {ns} of {spec.N} output features per step (float64 numpy oracle)"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD.name, "M": spec.M, "K": spec.K, "N": spec.N, "r": spec.r},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))
    return 0


# ------------------------------------------------------------------ GPU arm
def _clone_packed(svdq, pw, dev):
    """Another device copy of a packed layer (same bytes, separate memory)."""
    c = svdq.PackedWeight(pw.N, pw.K, pw.r, dev)
    for name in ("codes", "scales", "gscale", "l1t", "l2s"):
        getattr(c, name).copy_(getattr(pw, name))
    c.inv_smooth = None if pw.inv_smooth is None else pw.inv_smooth.clone()
    return c


def _gemm_kernel_name(M, N):
    """The GEMM the library dispatches to: CTA-pair 256x256 tiles when N is a
    multiple of 256 and M >= 512, else 128x128 single-CTA tiles."""
    return "w4a4_gemm_2sm_kernel" if N % 256 == 0 and M >= 512 else "w4a4_gemm_kernel"


def _gemm_pass_bytes(M, N, K, r):
    return (M * K + N * K) * (0.5 + 1.0 / 16) + 2 * M * r + 2 * r * N + 2 * N + 2 * M * N


def _pct(v, q):
    v = sorted(v)
    return v[min(len(v) - 1, max(0, int(round(q * (len(v) - 1)))))]


def _oracle_layer_rate(spec, X, W, b, budget_s):
    """The CPU oracle's forward (activation quantisation, down projection,
    4-bit product, up projection, bias; float64) on a bounded slice of one
    layer: the first S rows against the first Ns output features (rows and
    features are independent, so the slice is exact work of the layer). The
    low-rank factors are stand-ins of the right shapes (bf16 slices of W): the
    forward's cost does not depend on their values, and the LAPACK SVD of the
    large weights would dominate the bench's time. Returns (TFLOP/s, sample)."""
    from oracle import svdq as osv
    r = spec.r
    L1 = W[:r].T.contiguous()
    L2 = W[:, :r].T.contiguous()
    S = min(spec.M, 64)
    g_x = osv.act_global_scale(X[:S])

    def run(ns):
        pw = osv.pack_weight(W[:ns], L1, L2[:, :ns])
        t0 = time.perf_counter()
        osv.forward(X[:S], pw, b[:ns], g_x)
        return time.perf_counter() - t0

    unit = min(spec.N, 128)
    t_unit = max(run(unit), 1e-4)
    ns = int(max(1, min(spec.N // unit, budget_s / t_unit))) * unit
    dt = run(ns) if ns != unit else t_unit
    return _flops(S, ns, spec.K, r) / dt / 1e12, f"first {S} of {spec.M} rows x first {ns} of {spec.N} features"


def _bench_layer(svdq, spec, dev, stream, reps, peaks, oracle_budget_s):
    """One layer of a workload: cold-input steps (quantiser + GEMM, rotating
    input copies totalling at least twice the L2 size), a hot-L2 pass (the same
    inputs every step), per-kernel times, and the oracle's rate beside it."""
    M, K, N, r = spec.M, spec.K, spec.N, spec.r
    X, W, b = workloads.make_layer(spec)
    Xd, bd, Wd = X.to(dev), b.to(dev), W.to(dev)
    g_x = svdq.svdq_act_global_scale(Xd)
    L1, L2, _ = svdq.svdq_lowrank_init(Wd, r)
    pw = svdq.svdq_pack_weight(Wd, L1, L2, g_x)
    del Wd, L1, L2
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    set_bytes = Xd.numel() * 2 + sum(getattr(pw, n).numel() * getattr(pw, n).element_size()
                                     for n in ("codes", "scales", "gscale", "l1t", "l2s"))
    n_sets = max(2, -(-2 * l2_bytes // set_bytes))
    Xs = [Xd] + [Xd.clone() for _ in range(n_sets - 1)]
    pws = [pw] + [_clone_packed(svdq, pw, dev) for _ in range(n_sets - 1)]
    qa = svdq.QuantAct(M, K, r, dev)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)

    def step(j):
        svdq.svdq_quantize_act(Xs[j], pws[j], out=qa)
        svdq.svdq_w4a4_gemm(qa, pws[j], bd, out=Y)

    for i in range(max(10, n_sets)):
        step(i % n_sets)
    torch.cuda.synchronize()
    # A step of a small layer is shorter than the host needs to issue its two
    # calls, so the steps are replayed from CUDA graphs (device time; the
    # library's launches are stream-ordered and capture as they are): one graph
    # of G steps over the rotating sets (cold inputs), one of G steps on the
    # same set (hot L2), one per kernel; `reps` replays each, per-step times =
    # replay time / G.
    G = max(n_sets, 8)

    def graph_of(fn):
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side, capture_error_mode="relaxed"):
                for i in range(G):
                    fn(i)
        stream.wait_stream(side)
        return g

    def replay_times(g):
        g.replay()
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
        for e in ev:
            e[0].record(stream)
            g.replay()
            e[1].record(stream)
        torch.cuda.synchronize()
        return [e[0].elapsed_time(e[1]) / G for e in ev]

    g_cold = graph_of(lambda i: step(i % n_sets))
    g_hot = graph_of(lambda i: step(0))
    g_q = graph_of(lambda i: svdq.svdq_quantize_act(Xs[i % n_sets], pws[i % n_sets], out=qa))
    g_g = graph_of(lambda i: svdq.svdq_w4a4_gemm(qa, pws[i % n_sets], bd, out=Y))
    t_step, t_hot, t_q, t_g = (replay_times(g) for g in (g_cold, g_hot, g_q, g_g))
    # the same steps issued from the host one call at a time (includes any host gap)
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(reps):
        step(i % n_sets)
    z.record(stream)
    torch.cuda.synchronize()
    t_api = a.elapsed_time(z) / reps
    del g_cold, g_hot, g_q, g_g
    if svdq.svdq_read_device_error() != 0:
        raise RuntimeError(f"device error while timing {spec.name}")
    med, q_ms, g_ms = statistics.median(t_step), statistics.median(t_q), statistics.median(t_g)
    fp4_peak = peaks["bf16_tflops"] * FP4_PER_BF16
    o_rate, o_sample = _oracle_layer_rate(spec, X, W, b, oracle_budget_s)
    del Xs, pws, qa, Y
    return {
        "layer": spec.name, "M": M, "K": K, "N": N, "r": r, "gemm_kernel": _gemm_kernel_name(M, N),
        "input_sets": n_sets,
        "step_ms": {"median": med, "p10": _pct(t_step, 0.1), "p90": _pct(t_step, 0.9)},
        "hot_l2_step_ms": statistics.median(t_hot),
        "api_loop_step_ms": t_api,
        "tflops": _flops(M, N, K, r) / (med * 1e-3) / 1e12,
        "tokens_per_s": M / (med * 1e-3),
        "gemm_ms": g_ms,
        "gemm_frac_of_fp4_peak": 2.0 * M * N * K / (g_ms * 1e-3) / 1e12 / fp4_peak,
        "gemm_frac_of_hbm": _gemm_pass_bytes(M, N, K, r) / (g_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
        "quant_ms": q_ms,
        "quant_frac_of_hbm": _quant_bytes(M, K, r) / (q_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
        "oracle": {"tflops": o_rate, "cores": _cores(), "sample": o_sample},
    }


def bench_configs(svdq, dev, stream, reps=100, oracle_budget_s=1.0):
    """Every benchmark workload (1-5), each layer timed separately; a workload's
    time is the sum of its layers' median step times."""
    peaks, kind = _peaks()
    out = {"note": ("per layer: step = quantiser + GEMM with cold inputs (rotating copies >= 2x L2), device "
                    "time from CUDA-graph replays of the steps (median / p10 / p90 over replays); "
                    "hot_l2_step_ms with the same inputs every step; gemm_* and quant_* from graphs of one "
                    "kernel; api_loop_step_ms = the same steps issued call by call from the host; fractions of "
                    f"{kind} peaks (fp4 = bf16 burst x {FP4_PER_BF16:g}); oracle = float64 CPU oracle on a "
                    "bounded slice"), "reps": reps}
    for wid, wl in workloads.WORKLOADS.items():
        layers = [_bench_layer(svdq, spec, dev, stream, reps, peaks, oracle_budget_s) for spec in wl.layers]
        t = sum(L["step_ms"]["median"] for L in layers)
        fl = sum(_flops(L["M"], L["N"], L["K"], L["r"]) for L in layers)
        entry = {"workload": wl.name, "layers": layers}
        if wid in (3, 4):   # one block's layers in sequence: their times summed
            entry.update({"ms_sum": t, "tflops": fl / (t * 1e-3) / 1e12,
                          "tokens_per_s": wl.layers[0].M / (t * 1e-3)})
        out[str(wid)] = entry
    return out


def run_ours(args, spec):
    world, rank, local = _dist_init()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import w4a4_rank_corrected_svdq_b200 as svdq

    M, K, N, r = spec.M, spec.K, spec.N, spec.r
    X, W, b = workloads.make_layer(spec)
    Xd, bd, Wd = X.to(dev), b.to(dev), W.to(dev)
    # load time (untimed in the step): calibration, truncated SVD, residual packing
    ev_load = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    g_x = svdq.svdq_act_global_scale(Xd)          # calibration (static activation scale)
    ev_load[0].record()
    L1, L2, _ = svdq.svdq_lowrank_init(Wd, r)
    ev_load[1].record()
    pw = svdq.svdq_pack_weight(Wd, L1, L2, g_x)
    ev_load[2].record()
    torch.cuda.synchronize()
    load_ms = {"lowrank_init": ev_load[0].elapsed_time(ev_load[1]), "pack_weight": ev_load[1].elapsed_time(ev_load[2])}
    del Wd
    # Rotating input sets whose total is >= 2x L2: every step's inputs are cold.
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    set_bytes = Xd.numel() * 2 + sum(getattr(pw, n).numel() * getattr(pw, n).element_size()
                                     for n in ("codes", "scales", "gscale", "l1t", "l2s"))
    n_sets = max(2, -(-2 * l2_bytes // set_bytes))
    Xs = [Xd] + [Xd.clone() for _ in range(n_sets - 1)]
    pws = [pw] + [_clone_packed(svdq, pw, dev) for _ in range(n_sets - 1)]
    qa = svdq.QuantAct(M, K, r, dev)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    for i in range(args.warmup):
        j = i % n_sets
        svdq.svdq_quantize_act(Xs[j], pws[j], out=qa)
        svdq.svdq_w4a4_gemm(qa, pws[j], bd, out=Y)
    torch.cuda.synchronize()
    if svdq.svdq_read_device_error() != 0:
        raise RuntimeError("device error during warm-up")

    # Timed steps: the K steps (quantiser then GEMM, the GEMM a programmatic
    # dependent of the quantiser) captured once into a CUDA graph and replayed
    # inside the timed region, so the device time is not stretched by the
    # host's issue rate; one event pair on the launching stream around the
    # replay.
    def steps_graph():
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side, capture_error_mode="relaxed"):
                for i in range(args.steps):
                    j = (args.warmup + i) % n_sets
                    svdq.svdq_quantize_act(Xs[j], pws[j], out=qa)
                    svdq.svdq_w4a4_gemm(qa, pws[j], bd, out=Y)
        stream.wait_stream(side)
        return g

    graph = steps_graph()
    graph.replay()                   # upload, then one untimed replay
    torch.cuda.synchronize()
    e_a, e_b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(gpu_uuid(local)) as clk:
        e_a.record(stream)
        graph.replay()
        e_b.record(stream)
        torch.cuda.synchronize()
    _barrier(world)
    total_ms = _max_over_ranks(e_a.elapsed_time(e_b), world)
    ms_per_step = total_ms / args.steps
    del graph
    # the same steps issued call by call from the host (adds any host gap)
    e_a.record(stream)
    for i in range(args.steps):
        j = (args.warmup + i) % n_sets
        svdq.svdq_quantize_act(Xs[j], pws[j], out=qa)
        svdq.svdq_w4a4_gemm(qa, pws[j], bd, out=Y)
    e_b.record(stream)
    torch.cuda.synchronize()
    loop_ms = _max_over_ranks(e_a.elapsed_time(e_b), world) / args.steps

    # Per-kernel breakdown (separate pass, an event between the kernels).
    nb = min(args.steps, 200)
    evk = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(nb)]
    for i in range(nb):
        j = i % n_sets
        evk[i][0].record(stream)
        svdq.svdq_quantize_act(Xs[j], pws[j], out=qa)
        evk[i][1].record(stream)
        svdq.svdq_w4a4_gemm(qa, pws[j], bd, out=Y)
        evk[i][2].record(stream)
    torch.cuda.synchronize()
    quant_ms = _max_over_ranks(statistics.mean(e[0].elapsed_time(e[1]) for e in evk), world)
    gemm_ms = _max_over_ranks(statistics.mean(e[1].elapsed_time(e[2]) for e in evk), world)

    # ---- end to end through the public forward, host buffers, copies timed
    e2e_steps = min(args.steps, 50)
    Xh = X.pin_memory()
    Yh = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    ws = torch.empty(svdq.svdq_forward_workspace_size(M, K, r), dtype=torch.uint8, device=dev)
    Xe = torch.empty_like(Xd)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(2):
        Xe.copy_(Xh, non_blocking=True)
        svdq.svdq_linear_forward(Xe, pw, bd, out=Y, workspace=ws)
        Yh.copy_(Y, non_blocking=True)
    torch.cuda.synchronize()
    _barrier(world)
    e0.record(stream)
    for _ in range(e2e_steps):
        Xe.copy_(Xh, non_blocking=True)
        svdq.svdq_linear_forward(Xe, pw, bd, out=Y, workspace=ws)
        Yh.copy_(Y, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = _max_over_ranks(e0.elapsed_time(e1), world) / e2e_steps
    if svdq.svdq_read_device_error() != 0:
        raise RuntimeError("device error during timing")

    # Variants of the layer through the public API, same rotating inputs, each
    # against the plain forward: the fused QKV post-processing (per-head RMSNorm
    # of Q/K + rotary embedding in the GEMM epilogue), smoothing (lambda from
    # calibration on X; the quantiser multiplies by inv_smooth), and the dynamic
    # activation scale (an amax pass over X every call).
    n_q = min(args.steps, 200)

    def timed(fn):
        for i in range(3):
            fn(i)
        torch.cuda.synchronize()
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(n_q):
            fn(i)
        z.record(stream)
        torch.cuda.synchronize()
        return _max_over_ranks(a.elapsed_time(z), world) / n_q

    plain_ms = timed(lambda i: svdq.svdq_linear_forward(Xs[i % n_sets], pws[i % n_sets], bd, out=Y, workspace=ws))
    heads = N // 384
    qkv = None
    if N == heads * 384:
        wq = torch.ones(128, dtype=torch.bfloat16, device=dev)
        wk = torch.ones(128, dtype=torch.bfloat16, device=dev)
        cos_np, sin_np = workloads.rope_tables(M, 128)
        cos_t, sin_t = torch.from_numpy(cos_np).to(dev), torch.from_numpy(sin_np).to(dev)
        fused_ms = timed(lambda i: svdq.svdq_linear_forward_qkv(Xs[i % n_sets], pws[i % n_sets], bd, heads, wq, wk,
                                                               1e-6, cos_t, sin_t, out=Y, workspace=ws))
        qkv = {"heads": heads, "head_dim": 128, "ms_per_step": fused_ms, "plain_ms_per_step": plain_ms,
               "overhead": fused_ms / plain_ms - 1.0, "steps": n_q}
    Wv = W.to(dev)
    lam = svdq.svdq_smooth_factors(Xd, Wv, 0.5)
    L1s, L2s, _ = svdq.svdq_lowrank_init(Wv, r, smooth=lam)
    pw_s = svdq.svdq_pack_weight(Wv, L1s, L2s, 1.0, smooth=lam)
    g_s = svdq.svdq_act_global_scale(Xd, inv_smooth=pw_s.inv_smooth)
    pw_s = svdq.svdq_pack_weight(Wv, L1s, L2s, g_s, smooth=lam)
    del Wv
    pws_s = [pw_s] + [_clone_packed(svdq, pw_s, dev) for _ in range(n_sets - 1)]
    smooth_ms = timed(lambda i: svdq.svdq_linear_forward(Xs[i % n_sets], pws_s[i % n_sets], bd, out=Y, workspace=ws))
    ws_d = torch.empty(svdq.svdq_dynamic_workspace_size(M, N, K, r), dtype=torch.uint8, device=dev)
    dyn_ms = timed(lambda i: svdq.svdq_linear_forward_dynamic(Xs[i % n_sets], pws[i % n_sets], bd, out=Y,
                                                              workspace=ws_d))
    if svdq.svdq_read_device_error() != 0:
        raise RuntimeError("device error during the variant timings")
    variants = {"note": "public-API forward, same rotating inputs, one event pair around all steps",
                "steps": n_q, "plain_ms_per_step": plain_ms,
                "smoothed_ms_per_step": smooth_ms, "dynamic_scale_ms_per_step": dyn_ms}
    del pws_s, pw_s

    # AWQ W4A16 (the weight-only family for modulation layers): FLUX adaLN
    # modulation, K = 3072 -> N = 18432, M = 1 and 2 rows, six rotating copies
    # of the packed weight (larger than L2), against the HBM roofline.
    awq_out = {}
    Xm1, Wm, bm = workloads.modulation_layer(1)
    Wmd = Wm.to(dev)
    aws = [svdq.svdq_awq_pack(Wmd) for _ in range(n_sets)]
    del Wmd
    bmd = bm.to(dev)
    for Mm in (1, 2):
        Xm = workloads.modulation_layer(Mm)[0].to(dev)
        Ym = torch.empty((Mm, Wm.shape[0]), dtype=torch.bfloat16, device=dev)
        api_ms = timed(lambda i: svdq.svdq_awq_gemv(Xm, aws[i % n_sets], bmd, out=Ym))
        # The call is a few microseconds of device work, less than the host
        # needs to issue it: replay the same calls from a CUDA graph for the
        # device time per call.
        n_g = 6 * n_sets
        timing = "CUDA graph of the calls, device time per call"
        try:
            graph = torch.cuda.CUDAGraph()
            side = torch.cuda.Stream(dev)
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                with torch.cuda.graph(graph, stream=side, capture_error_mode="relaxed"):
                    for i in range(n_g):
                        svdq.svdq_awq_gemv(Xm, aws[i % n_sets], bmd, out=Ym)
            stream.wait_stream(side)
            graph.replay()
            torch.cuda.synchronize()
            g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 20
            g0.record(stream)
            for _ in range(reps):
                graph.replay()
            g1.record(stream)
            torch.cuda.synchronize()
            t_ms = g0.elapsed_time(g1) / (reps * n_g)
            del graph
        except RuntimeError as exc:  # no graph: the API loop's time (host-bound for so short a call)
            torch.cuda.synchronize()
            t_ms, timing = api_ms, f"API loop (graph capture failed: {str(exc)[:80]})"
        t_ms = _max_over_ranks(t_ms, world)
        Nm, Km = Wm.shape
        nbytes = Nm * Km // 2 + Nm * (Km // 64) * 3 + Mm * Km * 2 + Mm * Nm * 2 + Nm * 2
        gbs = nbytes / (t_ms * 1e-3) / 1e9
        awq_out[f"M{Mm}"] = {"ms": t_ms, "timing": timing,
                             "api_ms": api_ms, "algorithmic_bytes": nbytes, "gbs": gbs,
                             "frac_of_hbm": gbs / _peaks()[0]["hbm_gbs"]}
    del aws
    if svdq.svdq_read_device_error() != 0:
        raise RuntimeError("device error during the AWQ timing")
    variants["awq_w4a16_modulation_3072x18432"] = awq_out

    # MLP pair (the DiT feed-forward shapes, 3072 -> 12288 -> 3072, M = 4608):
    # the fused up projection (GELU, erf form and tanh form, and the down
    # projection's activation quantisation in its GEMM epilogue) plus the down
    # GEMM, against the unfused pair without a GELU pass (the up projection
    # writing y in bf16, the down projection reading it back), a lower bound
    # of the unfused cost.
    try:
        up_s, dn_s = workloads.WORKLOADS[3].layers[:2]
        Xu, Wu, bu = workloads.make_layer(up_s)
        Wdn, bdn = workloads.make_layer(dn_s, rows=1)[1:]
        Xud, bud, bdd = Xu.to(dev), bu.to(dev), bdn.to(dev)
        Wud = Wu.to(dev)
        Lu1, Lu2, _ = svdq.svdq_lowrank_init(Wud, up_s.r)
        pw_u = svdq.svdq_pack_weight(Wud, Lu1, Lu2, svdq.svdq_act_global_scale(Xud))
        del Wud
        Wdd = Wdn.to(dev)
        Ld1, Ld2, _ = svdq.svdq_lowrank_init(Wdd, dn_s.r)
        Mu, Fu = up_s.M, up_s.N
        Hd = torch.empty((Mu, Fu), dtype=torch.bfloat16, device=dev)
        one = torch.ones(1, dtype=torch.float32, device=dev)
        l1t_d = Ld1.t().contiguous()     # the down projection's L1^T (the layout its packed l1t holds)
        svdq.svdq_mlp_up_forward(Xud, pw_u, bud, one, l1t_d, h_out=Hd)   # calibration pass for h's scale
        g_h = svdq.svdq_act_global_scale(Hd)
        pw_d = svdq.svdq_pack_weight(Wdd, Ld1, Ld2, g_h)
        del Wdd
        qa_h = svdq.QuantAct(Mu, Fu, dn_s.r, dev)
        ws_m = torch.empty(svdq.svdq_mlp_workspace_size(Mu, Fu, up_s.K, up_s.r, dn_s.r), dtype=torch.uint8,
                           device=dev)
        ws_u = torch.empty(svdq.svdq_forward_workspace_size(Mu, up_s.K, up_s.r), dtype=torch.uint8, device=dev)
        ws_d = torch.empty(svdq.svdq_forward_workspace_size(Mu, Fu, dn_s.r), dtype=torch.uint8, device=dev)
        Yd = torch.empty((Mu, dn_s.N), dtype=torch.bfloat16, device=dev)

        def fused(i, approximate=False):
            svdq.svdq_mlp_up_forward(Xud, pw_u, bud, g_h, pw_d.l1t, approximate, out=qa_h, workspace=ws_m)
            svdq.svdq_w4a4_gemm(qa_h, pw_d, bdd, out=Yd)

        def unfused(i):
            svdq.svdq_linear_forward(Xud, pw_u, bud, out=Hd, workspace=ws_u)
            svdq.svdq_linear_forward(Hd, pw_d, bdd, out=Yd, workspace=ws_d)

        fused_ms, unfused_ms = timed(fused), timed(unfused)
        fused_tanh_ms = timed(lambda i: fused(i, True))
        if svdq.svdq_read_device_error() != 0:
            raise RuntimeError("device error during the MLP pair timing")
        pair_flops = _flops(Mu, Fu, up_s.K, up_s.r) + _flops(Mu, dn_s.N, Fu, dn_s.r)
        variants["mlp_pair_4608x3072x12288_r32"] = {
            "fused_ms_per_step": fused_ms, "fused_tanh_gelu_ms_per_step": fused_tanh_ms,
            "unfused_without_gelu_ms_per_step": unfused_ms,
            "fused_tflops": pair_flops / (fused_ms * 1e-3) / 1e12,
            "note": "one input set; the per-step working set (about 150 MB) exceeds L2"}
        del pw_u, pw_d, qa_h, ws_m, ws_u, ws_d, Hd, Yd
    except Exception as exc:  # reported, not fatal: the headline line above is complete without it
        variants["mlp_pair_4608x3072x12288_r32"] = {"error": f"{type(exc).__name__}: {str(exc)[:160]}"}

    configs = None
    if not args.no_configs:
        configs = bench_configs(svdq, dev, stream, reps=100 if args.steps >= 100 else max(args.steps, 10))

    peaks, kind = _peaks()
    gemm_name = _gemm_kernel_name(M, N)
    fp4_peak = peaks["bf16_tflops"] * FP4_PER_BF16
    gemm_tflops = 2.0 * M * N * K / (gemm_ms * 1e-3) / 1e12
    quant_gbs = _quant_bytes(M, K, r) / (quant_ms * 1e-3) / 1e9
    flops = _flops(M, N, K, r)
    value = world * flops / (ms_per_step * 1e-3) / 1e12
    tokens = world * M / (ms_per_step * 1e-3)
    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic",
        "config": {"workload": WORKLOAD.name, "M": M, "K": K, "N": N, "r": r, "global_batch_tokens": world * M,
                   "parallelism": f"replicas x{world}" if world > 1 else "single",
                   "l2": (f"inputs larger than L2: {n_sets} rotating copies of X and the packed weight "
                          f"({n_sets * set_bytes / 2**20:.0f} MiB, L2 {l2_bytes / 2**20:.0f} MiB); no flush kernel"),
                   "factors": "GPU truncated SVD of W (svdq_lowrank_init, 32 power iterations), load time"},
        "load_ms": load_ms,
        "tokens_per_s": tokens,
        "roofline": {"bound": "tensor", "achieved": gemm_tflops, "peak": fp4_peak, "unit": "TFLOP/s",
                     "frac": gemm_tflops / fp4_peak, "traffic": NCU_TRAFFIC_BYTES.get((WORKLOAD.name, gemm_name)),
                     "kernel": gemm_name, "peak_source": f"{kind} bf16 burst x {FP4_PER_BF16:g} (fp4/bf16)"},
        "ms_per_step_loop": loop_ms,
        "kernels_note": "per-kernel times from a separate pass with an event between the kernels (no overlap)",
        "kernels": {
            gemm_name: {"ms": gemm_ms, "tflops": gemm_tflops, "frac_of_fp4_peak": gemm_tflops / fp4_peak},
            "quantize_act_kernel": {"ms": quant_ms, "gbs": quant_gbs, "frac_of_hbm": quant_gbs / peaks["hbm_gbs"]},
        },
        "e2e": {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2, "ms_per_step": e2e_ms},
        "qkv_norm_rope": qkv,
        "variants": variants,
        "configs": configs,
        "gpu_launches": 2 * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        opw, og, S, ns = _oracle_setup(spec, X, W, b, budget_s=10.0)
        dt = _oracle_time(X, opw, b, og, S, ns)
        out["cpu_baseline"] = {"value": _flops(S, ns, K, r) / dt / 1e12, "unit": "TFLOP/s", "cores": _cores(),
                               "kind": "oracle",
                               "sample": f"first {S} rows x first {ns} of {N} output features, one forward"}
    if rank == 0:
        print(json.dumps(out))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-workload table (configs 1-5)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    spec = WORKLOAD.layers[0]
    if args.impl == "reference":
        return run_reference(args, spec)
    return run_ours(args, spec)


if __name__ == "__main__":
    sys.exit(main())
