#!/usr/bin/env python
"""Benchmark of the 2:4-sparse vs dense NVFP4 pipeline on the decode-shaped workload.

One step = one pass of the whole hot path over one batch of synthetic input:

    prepare_24(W)                      check + prune/compress + both NVFP4 tensor scales,
                                       one read of W
    -> quantize_nvfp4_pair(W, s_w, values, s_v)   encode both with those scales, one launch
    -> gemm_dense(X, W_nvfp4) -> gemm_sparse24(X, values_nvfp4 + meta)

(the outputs are bit-identical to check_24 -> prune_compress_24 -> quantize_nvfp4(W) ->
quantize_nvfp4(values), which read W four times).

Workload: X bf16 [8, 5120] N(0, 1), W bf16 [5120, 5120] N(0, 0.02) (the decode shape of the
pages' NVFP4 decode kernels, hidden width 5120).  Inputs live in HBM before timing starts and
rotate over 4 seeded input sets (about 440 MB in total, well beyond the 126 MB L2), so each
step reads its weight from DRAM.

The timed steps are captured in windows of up to 16 consecutive steps, one CUDA graph per
window; the timed region replays each window once, so the host pays one graph launch per
window.  An event record node inside a graph costs a few microseconds, so the timed windows
carry only one pair of events, around the dominant stage of their first step: that kernel's
launch duration (for `roofline`) is measured inside the timed region.  The per-stage breakdown
(`stages`) comes from graphs of back-to-back launches of each stage alone, run before timing.
`value` is the whole step's algorithmic HBM traffic divided by the step time (GB/s); the GEMV
comparison (dense vs 2:4 sparse: TFLOP/s, GB/s, speedup) is in `gemv`.

After the timed step (N = 1 only) the line gains `per_config`: every config of the workload
list at full size, each GEMM timed on prepared operands from CUDA-graph replays over operand
sets whose inputs exceed twice the L2 -- config 1 (FP16 toy), 2 (decode W4A16 GEMV), 3 (W4A4
4096^3: dense, element 2:4, pairwise 4:8 on the sparse FP4 MMA), 4 (routed experts), 5a / 5b
(M sweep, FP16 and NVFP4) and 5c (conv check + compress) -- each with dense and sparse time,
dense-equivalent TFLOP/s, algorithmic GB/s, arithmetic intensity, the binding roofline's
fraction and the sparse/dense speedup; `roofline_compute` is config 3's dense FP4 GEMM against
the dense FP4 tensor peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--sweep] [--no-per-config]

With --impl reference the CPU oracle (oracle/, plain scalar C) is timed on the host cores on
a bounded row sample of the same workload: that arm is a reported baseline, not the target.
Under torchrun every rank runs an independent replica (no collective on the data path);
rank 0 prints the JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

M, N, K = 8, 5120, 5120
METRIC = "2:4-sparse vs dense GEMM eff. TFLOP/s & HBM GB/s per shape; sparse/dense speedup"
WORKLOAD = ("decode_nvfp4: X bf16 [8,5120] N(0,1), W bf16 [5120,5120] N(0,0.02); step = "
            "prepare_24(W: check + prune/compress + tensor scales) + quantize_nvfp4_pair(W, values) + "
            "gemm_dense(X,W_nvfp4) + gemm_sparse24(X,values_nvfp4,meta)")
STAGES = ("prepare_24", "quantize_pair", "gemm_dense", "gemm_sparse24")
FALLBACK_HBM_GBS = 6650.0


def stage_bytes(rows: int = N) -> dict:
    """Algorithmic bytes each stage must move for `rows` weight rows, each operand once: the
    fused preparation reads W and writes the pass map, the kept values, the nibbles and 24
    bytes of counts/scales; each encode reads its input (the tensor scale is already known) and
    writes codes + block scales."""
    w = rows * K * 2                      # bf16 weight
    v = rows * K // 2 * 2                 # kept values, bf16
    meta = rows * K // 8
    x = M * K * 2
    y = M * rows * 4
    codes_w, scales_w = rows * K // 2, rows * K // 16
    codes_v, scales_v = rows * K // 4, rows * K // 32
    return {
        "prepare_24": w + rows * K // 4 + v + meta + 24,
        "quantize_pair": w + codes_w + scales_w + v + codes_v + scales_v + 16,
        "gemm_dense": codes_w + scales_w + 4 + x + y,
        "gemm_sparse24": codes_v + scales_v + 4 + meta + x + y,
    }


def gemv_flops(rows: int = N) -> float:
    return 2.0 * M * rows * K  # dense-equivalent for both GEMVs


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def traffic_record(kernel_stage: str):
    """DRAM bytes per launch from a committed ncu summary, if its kernel source is unchanged."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel_stage)
        if not rec:
            return None
        src = os.path.join(ROOT, rec["source"])
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if sha != rec["source_sha"]:
            return None
        return rec
    except Exception:
        return None


class ClockSampler:
    """Samples SM clock and throttle reasons with NVML while the timed region runs."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.nv is not None:
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ------------------------------------------------------------------------------ our arm

def max_over_ranks(ms: float, dist, device) -> float:
    """The slowest rank's time: every rank takes part and every rank gets the maximum."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_value(world: int, step_bytes: int, ms_step: float) -> float:
    """Whole-job algorithmic GB/s: each of the `world` replicas moves `step_bytes` per step."""
    return world * step_bytes / (ms_step * 1e-3) / 1e9


def run_ours(args, rank: int, world: int, dist) -> dict | None:
    import torch

    import fp16_gemm_b200 as sp
    import synth

    dev = torch.device("cuda", torch.cuda.current_device())
    bf16 = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)

    sets = []
    for i in range(args.sets):
        d = synth.decode_nvfp4(seed=i)
        s = {"x": bf16(d["X"]), "w": bf16(d["W"])}
        s["pass"] = torch.empty((N, K // 4), dtype=torch.uint8, device=dev)
        s["nfail"] = torch.empty(1, dtype=torch.int32, device=dev)
        s["v"] = torch.empty((N, K // 2), dtype=torch.bfloat16, device=dev)
        s["m"] = torch.empty(N * K // 8, dtype=torch.uint8, device=dev)
        s["ts"] = torch.empty(2, dtype=torch.float32, device=dev)
        s["wq"] = sp.NVFP4Tensor(torch.empty((N, K // 2), dtype=torch.uint8, device=dev),
                                 torch.empty((N, K // 16), dtype=torch.uint8, device=dev),
                                 torch.empty(1, dtype=torch.float32, device=dev))
        s["vq"] = sp.NVFP4Tensor(torch.empty((N, K // 4), dtype=torch.uint8, device=dev),
                                 torch.empty((N, K // 32), dtype=torch.uint8, device=dev),
                                 torch.empty(1, dtype=torch.float32, device=dev))
        s["yd"] = torch.empty((M, N), dtype=torch.float32, device=dev)
        s["ys"] = torch.empty((M, N), dtype=torch.float32, device=dev)
        sets.append(s)
    ws = torch.empty(sp.prepare_workspace_bytes(N, K), dtype=torch.uint8, device=dev)

    def stage_fns(s):
        sparse_w = sp.Sparse24(s["vq"], s["m"])
        prep = sp.Prepared24(s["pass"], s["nfail"], s["v"], s["m"], s["ts"][0:1], s["ts"][1:2])
        return [
            lambda: sp.prepare_24(s["w"], out=prep, workspace=ws),
            lambda: sp.quantize_nvfp4_pair(s["w"], prep.w_tensor_scale, s["v"], prep.v_tensor_scale,
                                           out0=s["wq"], out1=s["vq"]),
            lambda: sp.gemm_dense(s["x"], s["wq"], out=s["yd"]),
            lambda: sp.gemm_sparse24(s["x"], sparse_w, K, out=s["ys"]),
        ]

    # eager warm-up (also caches the SM count before capture)
    for s in sets:
        for f in stage_fns(s):
            f()
    torch.cuda.synchronize()
    assert sp.last_device_error() == sp.OK

    cap = torch.cuda.Stream()
    U = max(u for u in range(1, 17) if args.steps % u == 0)

    # Stage breakdown (before the timed region): each stage alone, U launches back to back over
    # the rotating input sets in one CUDA graph with events only around the whole graph (an
    # event record node costs a few microseconds, which would swamp the short kernels).  The
    # stages run in step order first, so every stage sees the operands the step gives it.
    stage_ms = []
    for si in range(len(STAGES)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            for j in range(U):
                stage_fns(sets[j % len(sets)])[si]()
        g.replay()
        torch.cuda.synchronize()
        reps = []
        for _ in range(3):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()  # the current stream, where replay() launches the graph
            g.replay()
            b.record()
            torch.cuda.synchronize()
            reps.append(a.elapsed_time(b) / U)
        stage_ms.append(statistics.median(reps))
        del g
    dom_i = max(range(len(STAGES)), key=lambda i: stage_ms[i])

    # Timed steps: windows of U consecutive steps, one CUDA graph per window, with no event
    # between stages except one pair around the dominant stage of the window's first step (that
    # kernel's launch duration, measured inside the timed region).  Replaying a window costs
    # one graph launch on the host.
    n_win = args.steps // U
    n0 = sp.kernel_launches()
    windows = []
    for wi in range(n_win):
        ev = (torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            for j in range(U):
                for si, f in enumerate(stage_fns(sets[(wi * U + j) % len(sets)])):
                    if j == 0 and si == dom_i:
                        ev[0].record()
                    f()
                    if j == 0 and si == dom_i:
                        ev[1].record()
        windows.append((g, ev))
    launches_per_step = (sp.kernel_launches() - n0) // args.steps
    torch.cuda.synchronize()

    stream = torch.cuda.current_stream()
    # warm-up: the first W steps' windows (rounded up to whole windows)
    for wi in range(min(n_win, (args.warmup + U - 1) // U)):
        windows[wi][0].replay()
    torch.cuda.synchronize()

    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    host0 = time.perf_counter()
    with ClockSampler(torch.cuda.current_device()) as clk:
        t_start.record(stream)
        for g, _ in windows:
            g.replay()
        t_end.record(stream)
        host_enqueue = time.perf_counter() - host0
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    total_ms = t_start.elapsed_time(t_end)
    dom_ms = sum(ev[0].elapsed_time(ev[1]) for _, ev in windows) / len(windows)

    total_ms = max_over_ranks(total_ms, dist, dev)
    ms_step = total_ms / args.steps
    bytes_ = stage_bytes()
    step_bytes = sum(bytes_.values())
    value = replica_value(world, step_bytes, ms_step)

    # ---------------------------------------------------------------- end to end (host buffers)
    s0 = sets[0]
    d0 = synth.decode_nvfp4(seed=0)
    hx = torch.from_numpy(d0["X"].view(np.int16)).view(torch.bfloat16).pin_memory()
    hw = torch.from_numpy(d0["W"].view(np.int16)).view(torch.bfloat16).pin_memory()
    hyd = torch.empty((M, N), dtype=torch.float32).pin_memory()
    hys = torch.empty((M, N), dtype=torch.float32).pin_memory()
    hnf = torch.empty(1, dtype=torch.int32).pin_memory()
    fns = stage_fns(s0)

    def e2e_step():
        s0["x"].copy_(hx, non_blocking=True)
        s0["w"].copy_(hw, non_blocking=True)
        for f in fns:
            f()
        hyd.copy_(s0["yd"], non_blocking=True)
        hys.copy_(s0["ys"], non_blocking=True)
        hnf.copy_(s0["nfail"], non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / args.e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, dist, dev)
    # results are still correct after all the replays (cheap sanity, outside timing)
    assert sp.last_device_error() == sp.OK
    assert int(hnf.item()) == N * K // 4  # raw normal weights: every group fails the check

    if rank != 0:
        return None

    peak, peak_kind = peaks()
    stages = {}
    for name, ms in zip(STAGES, stage_ms):
        gbs = bytes_[name] / (ms * 1e-3) / 1e9
        stages[name] = {"us": round(ms * 1e3, 3), "bytes": bytes_[name], "GB/s": round(gbs, 1),
                        "frac_hbm": round(gbs / peak, 3)}
    dom = STAGES[dom_i]
    rec = traffic_record(dom)
    achieved = round(bytes_[dom] / (dom_ms * 1e-3) / 1e9, 1)
    gd, gs = stages["gemm_dense"], stages["gemm_sparse24"]
    fl = gemv_flops()
    return {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M, "N": N, "K": K, "sets": args.sets,
                   "l2": f"{args.sets} rotating input sets (~{args.sets * 111} MB) > 126 MB L2",
                   "parallelism": f"replicas{world}" if world > 1 else "single-gpu"},
        "gemv": {
            "dense": {"us": gd["us"], "TFLOP/s": round(fl / (gd["us"] * 1e-6) / 1e12, 2),
                      "GB/s": gd["GB/s"], "bytes": gd["bytes"]},
            "sparse24": {"us": gs["us"], "TFLOP/s (dense-equiv)": round(fl / (gs["us"] * 1e-6) / 1e12, 2),
                         "GB/s": gs["GB/s"], "bytes": gs["bytes"]},
            "sparse_dense_speedup": round(gd["us"] / gs["us"], 3),
            "arith_intensity_flop_per_byte": {"dense": round(fl / gd["bytes"], 1),
                                              "sparse24": round(fl / gs["bytes"], 1)},
        },
        "stages": stages,
        "stages_note": ("per-stage kernel times from graphs of back-to-back launches of each "
                        "stage alone, run before the timed region; the step time has no stage events"),
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / peak, 3),
                     "launch_us": round(dom_ms * 1e3, 3), "launches_timed": len(windows),
                     "traffic": None if rec is None else rec["traffic_bytes_per_launch"]},
        "e2e": {"value": round(replica_value(world, step_bytes, e2e_ms), 2), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 4), "steps": args.e2e_steps,
                "h2d_bytes_per_step": hx.numel() * 2 + hw.numel() * 2,
                "d2h_bytes_per_step": hyd.numel() * 4 + hys.numel() * 4 + 4},
        "gpu_launches": int(launches_per_step * args.steps),
        "launches_per_step": int(launches_per_step),
        "host_enqueue_ms": round(host_enqueue * 1e3, 2),
        "clocks": clk.summary(),
    }


# ------------------------------------------------------------------------------ CPU oracle

def oracle_pipeline(X, Wrows):
    """One pass of the pipeline in the CPU oracle over a row sample of W."""
    import oracle
    od = oracle.BF16
    oracle.check_24(Wrows, od)
    V, meta = oracle.compress_24(Wrows, od)
    cw, sw, tw = oracle.nvfp4_encode(Wrows, od)
    cv, sv, tv = oracle.nvfp4_encode(V, od)
    Xd = oracle.to_double(X, od)
    oracle.gemm(Xd, oracle.nvfp4_decode(cw, sw, tw))
    oracle.gemm_sparse(Xd, oracle.nvfp4_decode(cv, sv, tv), meta)


def cpu_baseline(budget_s: float, steps: int = 1):
    """Times the oracle on bounded row samples; returns (GB/s, seconds, rows per step, cores)."""
    import oracle
    import synth
    d = synth.decode_nvfp4(seed=0)
    X, W = d["X"], d["W"]
    cores = oracle.max_threads()
    t0 = time.perf_counter()
    oracle_pipeline(X, np.ascontiguousarray(W[:32]))
    per_row = (time.perf_counter() - t0) / 32
    rows = int(max(8, min(N, budget_s / max(per_row, 1e-9) / steps)) // 8 * 8)
    t0 = time.perf_counter()
    for i in range(steps):
        r0 = (i * rows) % (N - rows + 1)
        oracle_pipeline(X, np.ascontiguousarray(W[r0:r0 + rows]))
    dt = time.perf_counter() - t0
    gbs = steps * sum(stage_bytes(rows).values()) / dt / 1e9
    return gbs, dt, rows, cores


# ------------------------------------------------------------------------------ per-shape sweep

L2_BYTES = 126e6


def tensor_peaks():
    """Roofline denominators: (HBM GB/s, {pipe: TFLOP/s}, {pipe: where it came from}).

    HBM copy and dense bf16 GEMM are the measured figures of MEASURED_PEAKS.json (the
    profiling recipe's fallback when absent); the other pipes take the measured bf16 figure
    times the nominal ratio (FP4 dense x 4, i.e. 9 / 2.25 PF; 2:4 pipes count dense-equivalent
    FLOPs at twice their dense rate)."""
    hbm, kind = peaks()
    bf16, bkind = 1590.0, "fallback"
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            bf16, bkind = float(json.load(f)["bf16_tflops"]), "measured bf16 GEMM"
    except Exception:
        pass
    tp = {"f16": bf16, "f16.sp": 2 * bf16, "nvfp4": 4 * bf16, "nvfp4.sp": 8 * bf16}
    src = {"hbm": kind, "f16": bkind, "f16.sp": bkind + " x 2", "nvfp4": bkind + " x 4",
           "nvfp4.sp": bkind + " x 8"}
    return hbm, tp, src


def mma_microbench():
    """{pipe: TFLOP/s} of back-to-back MMAs measured by `bench.py --peaks` (profiles/peaks.json),
    or {} when that file is absent."""
    try:
        with open(os.path.join(ROOT, "profiles", "peaks.json")) as f:
            return json.load(f)["mma_tflops"]
    except Exception:
        return {}


def _copies(set_bytes: float, lo: int = 2, hi: int = 64) -> int:
    """Operand sets to rotate over so the inputs of consecutive launches exceed twice the L2."""
    return int(max(lo, min(hi, -(-2 * L2_BYTES // max(set_bytes, 1)))))


def sweep(emit, full: bool) -> None:
    """One record per (config, shape) with dense and sparse forms side by side: GEMM time on
    prepared operands from CUDA-graph replays over rotating operand copies whose inputs total
    more than twice the L2, TFLOP/s (dense-equivalent), algorithmic GB/s, arithmetic intensity,
    the binding roofline and its fraction, and the sparse/dense speedup.  `full` adds the rows
    beyond the five configs (expert block, output-head quantisation, pairwise 4:8 on it)."""
    import torch

    import fp16_gemm_b200 as sp
    import synth

    peak_hbm, tensor_peak, peak_src = tensor_peaks()
    dev = torch.device("cuda", torch.cuda.current_device())
    t16 = lambda a, d: (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if d == "bf16"
                        else torch.from_numpy(np.ascontiguousarray(a))).to(dev)

    def timeit(fn, n_sets, reps=20):
        """Median over 5 replays of a CUDA graph of back-to-back launches cycling through the
        operand sets (at least `reps` launches and every set once), per launch in us."""
        reps = max(reps, n_sets)
        for r in range(3):
            fn(r)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=torch.cuda.Stream()):
            for r in range(reps):
                fn(r)
        g.replay()
        torch.cuda.synchronize()
        times = []
        for _ in range(5):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b) * 1e3 / reps)
        del g
        return statistics.median(times)

    def clone_op(o):
        if isinstance(o, torch.Tensor):
            return o.clone()
        return type(o)(*[clone_op(t) for t in o])

    def op_bytes(t):
        if isinstance(t, sp.NVFP4Tensor):
            return t.codes.numel() + t.scales.numel() + 4
        if isinstance(t, (sp.Sparse24, sp.Sparse48)):
            return op_bytes(t.values) + t.meta.numel()
        return t.numel() * t.element_size()

    def record(us, flops, byts, pipe):
        ai = flops / byts
        ridge = tensor_peak[pipe] * 1e12 / (peak_hbm * 1e9)
        tflops = flops / (us * 1e-6) / 1e12
        gbs = byts / (us * 1e-6) / 1e9
        bound = "hbm" if ai < ridge else "tensor"
        frac = gbs / peak_hbm if bound == "hbm" else tflops / tensor_peak[pipe]
        return {"us": round(us, 3), "TFLOP/s": round(tflops, 2), "GB/s": round(gbs, 1), "bytes": int(byts),
                "AI": round(ai, 1), "bound": bound, "pipe": pipe, "frac": round(frac, 3),
                "frac_tensor": round(tflops / tensor_peak[pipe], 3), "frac_hbm": round(gbs / peak_hbm, 3)}

    selections = []

    def case(config, workload, M, N, K, xdt, wdt, X, W):
        """X, W numpy storage; xdt in {f16, bf16, nvfp4}; wdt in {f16, bf16, nvfp4}: the dense
        GEMM on the pruned weight against the 2:4 GEMM on its compressed form."""
        x = t16(X, "f16" if xdt == "f16" else "bf16")
        if xdt == "nvfp4":
            x = sp.quantize_nvfp4(x)
        w16 = t16(W, "f16" if wdt == "f16" or (wdt == "nvfp4" and xdt == "f16") else "bf16")
        v, m = sp.prune_compress_24(w16)
        wd = sp.decompress_24(v, m, w16.shape) if wdt != "nvfp4" else w16  # dense on pruned W
        dense = sp.quantize_nvfp4(w16) if wdt == "nvfp4" else wd
        sparse = sp.Sparse24(sp.quantize_nvfp4(v) if wdt == "nvfp4" else v, m)
        del w16, wd, v
        res = {}
        flops = 2.0 * M * N * K
        for name, wop in (("dense", dense), ("sparse24", sparse)):
            wb, xb = op_bytes(wop), op_bytes(x)
            n = _copies(wb + xb)
            sets = [(x, wop)] + [(clone_op(x), clone_op(wop)) for _ in range(n - 1)]
            y = torch.empty((M, N), dtype=torch.float32, device=dev)
            sparse_ = name == "sparse24"
            ws_b = sp.gemm_workspace_bytes(x, wop, sparse_, M, N, K)
            ws = torch.empty(max(ws_b, 1), dtype=torch.uint8, device=dev) if ws_b else None
            if sparse_:
                fn = lambda r: sp.gemm_sparse24(sets[r % n][0], sets[r % n][1], K, out=y, workspace=ws)
            else:
                fn = lambda r: sp.gemm_dense(sets[r % n][0], sets[r % n][1], out=y, workspace=ws)
            us = timeit(fn, n)
            pipe = ("nvfp4" if xdt == "nvfp4" and wdt == "nvfp4" and not sparse_ else
                    "f16.sp" if sparse_ else "f16")
            res[name] = record(us, flops, xb + wb + M * N * 4, pipe)
            res[name]["input_sets"] = n
            if pipe == "nvfp4" and K % 256 == 0:
                # the same GEMM on operands already in the kernel's tile images (a weight is
                # rewritten once; the call above rewrites both operands first)
                isets = [(sp.to_mma(a), sp.to_mma(b)) for a, b in sets]
                us_i = timeit(lambda r: sp.gemm_dense(isets[r % n][0], isets[r % n][1], out=y), n)
                res["dense_tile_images"] = record(us_i, flops, xb + wb + M * N * 4, pipe)
                res["dense_tile_images"]["input_sets"] = n
                del isets
            del sets, y, ws
        # the dense / 2:4 choice the library makes for this shape without measuring (its rule
        # of measured crossovers) against the faster of the two just timed
        fmt = {"f16": sp.F16, "bf16": sp.BF16, "nvfp4": sp.NVFP4}
        sp.gemm_choice_reset()
        rule_sparse = sp.gemm_choice(fmt[xdt], fmt[wdt], M, N, K)[0]
        faster_sparse = res["sparse24"]["us"] < res["dense"]["us"]
        chosen = res["sparse24" if rule_sparse else "dense"]["us"]
        selections.append({"workload": workload, "M": M, "rule": "sparse24" if rule_sparse else "dense",
                           "faster": "sparse24" if faster_sparse else "dense",
                           "loss": round(chosen / min(res["dense"]["us"], res["sparse24"]["us"]) - 1.0, 3)})
        emit({"config": config, "sweep": workload, "M": M, "N": N, "K": K, "x": xdt, "w": wdt, **res,
              "sparse_dense_speedup": round(res["dense"]["us"] / res["sparse24"]["us"], 3),
              "selected": "sparse24" if rule_sparse else "dense"})

    def case48(config, workload, M, N, K, X, W):
        """W4A4 on the sparse FP4 MMA (pairwise 4:8 weight, activations in 32-value blocks)
        against the dense W4A4 GEMM of the same weight (NVFP4, 16-value blocks)."""
        xb, wb16 = t16(X, "bf16"), t16(W, "bf16")
        x16, x32 = sp.quantize_nvfp4(xb), sp.quantize_nvfp4_block32(xb)
        v, m = sp.prune_compress_48(wb16)
        dense, sparse = sp.quantize_nvfp4(wb16), sp.Sparse48(sp.quantize_nvfp4(v), m)
        del xb, wb16, v
        y = torch.empty((M, N), dtype=torch.float32, device=dev)
        flops = 2.0 * M * N * K
        line = {"config": config, "sweep": workload, "M": M, "N": N, "K": K, "x": "nvfp4", "w": "nvfp4"}
        for name, wop, xop, pipe in (("dense", dense, x16, "nvfp4"), ("sparse48", sparse, x32, "nvfp4.sp")):
            wbytes, xbytes = op_bytes(wop), op_bytes(xop)
            n = _copies(wbytes + xbytes)
            sets = [(xop, wop)] + [(clone_op(xop), clone_op(wop)) for _ in range(n - 1)]
            if name == "dense":
                fn = lambda r: sp.gemm_dense(sets[r % n][0], sets[r % n][1], out=y)
            else:
                fn = lambda r: sp.gemm_sparse48(sets[r % n][0], sets[r % n][1], K, out=y)
            us = timeit(fn, n)
            line[name] = record(us, flops, xbytes + wbytes + M * N * 4, pipe)
            line[name]["input_sets"] = n
            # both forms again on the kernels' tile images (the CTA-pair kernels): the weight is
            # rewritten once, the activations as a quantiser emitting images would leave them
            if name == "dense":
                isets = [(sp.to_mma(a), sp.to_mma(b)) for a, b in sets]
                fn_i = lambda r: sp.gemm_dense(isets[r % n][0], isets[r % n][1], out=y)
            else:
                isets = [(sp.b32_to_mma(a), sp.sparse48_to_mma(b, K)) for a, b in sets]
                fn_i = lambda r: sp.gemm_sparse48(isets[r % n][0], isets[r % n][1], K, out=y)
            line[name + "_tile_images"] = record(timeit(fn_i, n), flops, xbytes + wbytes + M * N * 4, pipe)
            del sets, isets
        line["sparse_dense_speedup"] = round(line["dense"]["us"] / line["sparse48"]["us"], 3)
        line["sparse_dense_speedup_tile_images"] = round(
            line["dense_tile_images"]["us"] / line["sparse48_tile_images"]["us"], 3)
        emit(line)

    # config 1: FP16 2:4 toy (L2-resident by size: a correctness configuration)
    d = synth.fp16_toy()
    case("1", "fp16_toy", 16, 256, 512, "f16", "f16", d["X"], d["W"])
    # config 2: decode-shaped W4A16 GEMV
    d = synth.decode_nvfp4()
    case("2", "decode_w4a16", 8, 5120, 5120, "bf16", "nvfp4", d["X"], d["W"])
    # config 3: prefill W4A4 4096^3, dense vs element 2:4 vs pairwise 4:8 (sparse FP4 MMA)
    d = synth.prefill_w4a4()
    case("3", "prefill_w4a4", 4096, 4096, 4096, "nvfp4", "nvfp4", d["X"], d["W"])
    case48("3", "prefill_w4a4_pairwise48", 4096, 4096, 4096, d["X"], d["W"])
    del d
    # config 4: routed experts, 4096 tokens x top-10 of 512 experts [512, 2048], bf16 x, NVFP4
    # experts dense and 2:4 (every expert is touched: each call reads all of them once, 302 MB
    # dense / 218 MB 2:4, beyond the L2)
    d = synth.moe()
    E, Ne, Ke = d["W"].shape
    xm = t16(d["X"], "bf16")
    rt = torch.from_numpy(d["routing"]).to(dev)
    wm = t16(d["W"].reshape(E * Ne, Ke), "bf16")
    del d
    _, wq, sw = sp.prepare_nvfp4_24(wm)
    del wm
    ym = torch.empty((rt.shape[0], rt.shape[1], Ne), dtype=torch.float32, device=dev)
    T, topk = rt.shape
    fl = 2.0 * T * topk * Ne * Ke
    xy = T * Ke * 2 + T * topk * Ne * 4 + T * topk * 4
    line = {"config": "4", "sweep": "moe_grouped", "experts": E, "expert_shape": [Ne, Ke], "tokens": T,
            "topk": topk, "x": "bf16", "w": "nvfp4"}
    for name, wop in (("dense", wq), ("sparse24", sw)):
        us = timeit(lambda r: sp.gemm_grouped(xm, rt, wop, E, Ne, Ke, out=ym), 1, reps=5)
        line[name] = record(us, fl, op_bytes(wop) + xy, "f16.sp" if name == "sparse24" else "f16")
    line["sparse_dense_speedup"] = round(line["dense"]["us"] / line["sparse24"]["us"], 3)
    emit(line)
    del xm, rt, wq, sw, ym
    # config 5a / 5b: M sweep at N = K = 5120, FP16 and NVFP4 (W4A16; W4A4 as an extra row)
    W16 = synth.draw(synth.rng(0), (5120, 5120), "f16")
    Wb = synth.draw(synth.rng(0), (5120, 5120), "bf16")
    for Mv in (1, 16, 128, 1024, 4096, 16384):
        X16 = synth.draw(synth.rng(Mv), (Mv, 5120), "f16")
        case("5a", "msweep_fp16", Mv, 5120, 5120, "f16", "f16", X16, W16)
        del X16
        Xb = synth.draw(synth.rng(Mv), (Mv, 5120), "bf16")
        case("5b", "msweep_nvfp4_w4a16", Mv, 5120, 5120, "bf16", "nvfp4", Xb, Wb)
        case("5b", "msweep_nvfp4_w4a4", Mv, 5120, 5120, "nvfp4", "nvfp4", Xb, Wb)
        if Mv >= 128:
            case48("5b", "msweep_w4a4_pairwise48", Mv, 5120, 5120, Xb, Wb)
        del Xb
        torch.cuda.empty_cache()
    agree = sum(c["rule"] == c["faster"] for c in selections)
    emit({"config": "selection", "sweep": "dense_sparse_selection", "shapes": len(selections),
          "rule_picks_faster": agree, "worst_loss": max(c["loss"] for c in selections), "cases": selections})
    # config 5c: conv eligibility check + compression (fp16 [256, 256, 3, 3], 5% failing groups),
    # one tensor and a batch of 512 such tensors as one [512*256, 256, 3, 3] launch
    c = synth.conv_fail5()
    for batch in (1, 512):
        wc = t16(np.ascontiguousarray(np.broadcast_to(c["W"], (batch,) + c["W"].shape)).reshape(
            (batch * 256, 256, 3, 3)), "f16")
        nb = wc.numel() * 2
        n = _copies(nb)
        wcs = [wc] + [wc.clone() for _ in range(n - 1)]
        pass_ = torch.empty((batch * 256, 64, 3, 3), dtype=torch.uint8, device=dev)
        nf = torch.empty(1, dtype=torch.int32, device=dev)
        vals = torch.empty((batch * 256, 128, 3, 3), dtype=torch.float16, device=dev)
        meta = torch.empty(batch * 256 * 64 * 9 // 2, dtype=torch.uint8, device=dev)
        us_c = timeit(lambda r: sp.check_24(wcs[r % n], sp.OP_CONV, pass_out=pass_, n_fail_out=nf), n)
        us_p = timeit(lambda r: sp.prune_compress_24(wcs[r % n], sp.OP_CONV, values_out=vals, meta_out=meta), n)
        bc, bp = nb + pass_.numel(), nb + vals.numel() * 2 + meta.numel()
        emit({"config": "5c", "sweep": "conv_check_compress", "tensors": batch, "shape": [batch * 256, 256, 3, 3],
              "input_sets": n,
              "check": {"us": round(us_c, 3), "GB/s": round(bc / us_c / 1e3, 1),
                        "frac_hbm": round(bc / us_c / 1e3 / peak_hbm, 3)},
              "compress": {"us": round(us_p, 3), "GB/s": round(bp / us_p / 1e3, 1),
                           "frac_hbm": round(bp / us_p / 1e3 / peak_hbm, 3)},
              "n_fail": int(nf.item())})
        del wc, wcs, pass_, vals, meta
    torch.cuda.empty_cache()
    if full:
        sweep_next_rows(emit, sp, synth, dev, t16, timeit, op_bytes, peak_hbm, tensor_peak)
    emit({"config": "peaks", "hbm_gbs": peak_hbm, "tensor_tflops": tensor_peak, "source": peak_src})


def sweep_next_rows(emit, sp, synth, dev, t16, timeit, op_bytes, peak_hbm, tensor_peak) -> None:
    """Rows beyond the five configs: the fused expert block, a large single-tensor quantisation
    and pairwise 4:8 check / prune on the same tensor."""
    import torch

    # routed expert block: 512 experts (gate/up [1024, 2048] packed, down [2048, 512]), 4096 bf16
    # tokens top-10, NVFP4 experts dense or 2:4; FLOPs 6 T topk H F; bytes: weights once, x, y,
    # h written and read once, the per-slot outputs written and read once (routing tables excluded)
    d = synth.moe_block()
    E, F, H = d["Wg"].shape
    xb = t16(d["X"], "bf16")
    rtb = torch.from_numpy(d["routing"]).to(dev)
    rwb = torch.from_numpy(d["router_w"]).to(dev)
    Tb, kb = rtb.shape
    wg = t16(d["Wg"].reshape(E * F, H), "bf16")
    wu = t16(d["Wu"].reshape(E * F, H), "bf16")
    wdn = t16(d["Wd"].reshape(E * H, F), "bf16")
    del d
    tsd = sp.nvfp4_group_tensor_scale([wg, wu])
    gu_d = sp.pack_gate_up(sp.quantize_nvfp4(wg, tsd), sp.quantize_nvfp4(wu, tsd))
    dn_d = sp.quantize_nvfp4(wdn)
    (vg, mg), (vu, mu) = sp.prune_compress_24(wg), sp.prune_compress_24(wu)
    del wg, wu
    tss = sp.nvfp4_group_tensor_scale([vg, vu])
    gu_s = sp.pack_gate_up(sp.Sparse24(sp.quantize_nvfp4(vg, tss), mg), sp.Sparse24(sp.quantize_nvfp4(vu, tss), mu))
    del vg, vu
    vd, md = sp.prune_compress_24(wdn)
    dn_s = sp.Sparse24(sp.quantize_nvfp4(vd), md)
    del wdn, vd
    yb = torch.empty((Tb, H), dtype=torch.float32, device=dev)
    wsb = torch.empty(sp.moe_block_workspace_bytes(Tb, kb, E, H, F), dtype=torch.uint8, device=dev)
    flb = 6.0 * Tb * kb * H * F
    xyh = Tb * H * 2 + Tb * H * 4 + 2 * Tb * kb * F * 2 + 2 * Tb * kb * H * 4
    line = {"config": "next", "sweep": "moe_block", "experts": E, "hidden": H, "inter": F, "tokens": Tb,
            "topk": kb, "x": "bf16", "w": "nvfp4", "flop": flb}
    for name, (gop, dop) in (("dense", (gu_d, dn_d)), ("sparse24", (gu_s, dn_s))):
        us = timeit(lambda r: sp.moe_block(xb, rtb, rwb, gop, dop, E, H, F, out=yb, workspace=wsb), 1, reps=3)
        byt = op_bytes(gop) + op_bytes(dop) + xyh
        line[name] = {"us": round(us, 1), "TFLOP/s": round(flb / us / 1e6, 1), "GB/s": round(byt / us / 1e3, 1),
                      "bytes": byt, "frac_hbm": round(byt / us / 1e3 / peak_hbm, 3),
                      "frac_tensor": round(flb / us / 1e6 / tensor_peak["f16"], 3)}
    line["sparse_dense_speedup"] = round(line["dense"]["us"] / line["sparse24"]["us"], 3)
    emit(line)
    del gu_d, dn_d, gu_s, dn_s, xb, yb, wsb

    # large single-tensor quantisation: a [151936, 4096] bf16 output head (~1.16 GiB -> 0.33 GiB
    # of codes + scales).  Full call: amax pass + encode pass (the tensor is 10x the L2, so it is
    # read twice); with a supplied (group-shared) scale: one pass; the group scale alone: one read.
    Wh = t16(synth.output_head()["W"], "bf16")
    R, L = Wh.shape
    qh = sp.quantize_nvfp4(Wh)
    nb_in, nb_out = Wh.numel() * 2, R * L // 2 + R * L // 16 + 4
    us_full = timeit(lambda r: sp.quantize_nvfp4(Wh, out=qh), 1, reps=5)
    ts_h = qh.tensor_scale.clone()
    us_one = timeit(lambda r: sp.quantize_nvfp4(Wh, tensor_scale=ts_h, out=qh), 1, reps=5)
    gs_out = torch.empty(1, dtype=torch.float32, device=dev)
    us_gs = timeit(lambda r: sp.nvfp4_group_tensor_scale([Wh], out=gs_out), 1, reps=5)
    alg = nb_in + nb_out
    emit({"config": "next", "sweep": "quantize_large", "shape": [R, L], "dtype": "bf16",
          "in_bytes": nb_in, "out_bytes": nb_out,
          "derived_scale": {"us": round(us_full, 1), "GB/s": round(alg / us_full / 1e3, 1),
                            "frac_hbm": round(alg / us_full / 1e3 / peak_hbm, 3),
                            "traffic_GB/s": round((2 * nb_in + nb_out) / us_full / 1e3, 1),
                            "note": "two reads of the tensor (amax, then encode)"},
          "supplied_scale": {"us": round(us_one, 1), "GB/s": round(alg / us_one / 1e3, 1),
                             "frac_hbm": round(alg / us_one / 1e3 / peak_hbm, 3)},
          "group_scale_only": {"us": round(us_gs, 1), "GB/s": round(nb_in / us_gs / 1e3, 1),
                               "frac_hbm": round(nb_in / us_gs / 1e3 / peak_hbm, 3)}})
    # pairwise 4:8 on the same tensor (check; prune + compress), 2:4 prune + compress beside it
    pass48 = torch.empty((R, L // 8), dtype=torch.uint8, device=dev)
    nf48 = torch.empty(1, dtype=torch.int32, device=dev)
    vals = torch.empty((R, L // 2), dtype=torch.bfloat16, device=dev)
    meta48 = torch.empty(R * L // 16, dtype=torch.uint8, device=dev)
    meta24 = torch.empty(R * L // 8, dtype=torch.uint8, device=dev)
    us_c48 = timeit(lambda r: sp.check_48(Wh, pass_out=pass48, n_fail_out=nf48), 1, reps=5)
    us_p48 = timeit(lambda r: sp.prune_compress_48(Wh, values_out=vals, meta_out=meta48), 1, reps=5)
    us_p24 = timeit(lambda r: sp.prune_compress_24(Wh, values_out=vals, meta_out=meta24), 1, reps=5)
    b_c48 = nb_in + pass48.numel()
    b_p48, b_p24 = nb_in + nb_in // 2 + meta48.numel(), nb_in + nb_in // 2 + meta24.numel()
    emit({"config": "next", "sweep": "pairwise48", "shape": [R, L], "dtype": "bf16",
          "check_48": {"us": round(us_c48, 1), "GB/s": round(b_c48 / us_c48 / 1e3, 1),
                       "frac_hbm": round(b_c48 / us_c48 / 1e3 / peak_hbm, 3)},
          "prune_compress_48": {"us": round(us_p48, 1), "GB/s": round(b_p48 / us_p48 / 1e3, 1),
                                "frac_hbm": round(b_p48 / us_p48 / 1e3 / peak_hbm, 3)},
          "prune_compress_24": {"us": round(us_p24, 1), "GB/s": round(b_p24 / us_p24 / 1e3, 1),
                                "frac_hbm": round(b_p24 / us_p24 / 1e3 / peak_hbm, 3)}})
    del Wh, qh, pass48, vals, meta48, meta24
    torch.cuda.empty_cache()


def per_config(lines: list) -> dict:
    """The sweep records grouped by config, for the default JSON line."""
    out: dict = {}
    for ln in lines:
        c = ln.get("config")
        if c in ("peaks", "selection"):
            out[c] = {k: v for k, v in ln.items() if k not in ("config", "cases")}
            continue
        out.setdefault(c, []).append({k: v for k, v in ln.items() if k != "config"})
    return out


def compute_roofline(lines: list):
    """The config-3 dense W4A4 GEMM (4096^3) against the dense FP4 tensor peak, with the
    pairwise-4:8 sparse FP4 GEMM of the same shape against the sparse (dense-equivalent) peak."""
    sparse = None
    for ln in lines:
        if ln.get("sweep") == "prefill_w4a4_pairwise48" and "sparse48_tile_images" in ln:
            _, tp, src = tensor_peaks()
            d = ln["sparse48_tile_images"]
            sparse = {"kernel": "gemm_nvfp4_pair_kernel (sparse): tcgen05.mma.sp cta_group::2 kind::mxf4nvf4",
                      "achieved": d["TFLOP/s"], "peak": round(tp["nvfp4.sp"], 1), "peak_kind": src["nvfp4.sp"],
                      "frac": round(d["TFLOP/s"] / tp["nvfp4.sp"], 3), "launch_us": d["us"],
                      "sparse_dense_speedup": ln.get("sparse_dense_speedup_tile_images")}
    for ln in lines:
        if ln.get("sweep") == "prefill_w4a4":
            d = ln.get("dense_tile_images", ln["dense"])
            _, tp, src = tensor_peaks()
            return {"bound": "tensor",
                    "kernel": "gemm_nvfp4_pair_kernel: W4A4 4096^3, operands as tile images (tcgen05 "
                              "cta_group::2 kind::mxf4nvf4)",
                    "achieved": d["TFLOP/s"], "peak": round(tp["nvfp4"], 1), "peak_kind": src["nvfp4"],
                    "unit": "TFLOP/s", "frac": round(d["TFLOP/s"] / tp["nvfp4"], 3), "launch_us": d["us"],
                    "row_order_operands_us": ln["dense"]["us"],
                    "mma_loop_tflops": {k: v for k, v in mma_microbench().items() if k.startswith("nvfp4")},
                    "sparse_pairwise48": sparse, "traffic": None}
    return None


def run_sweep(args) -> None:
    import torch
    torch.cuda.set_device(0)
    sweep(lambda ln: print(json.dumps(ln), flush=True), full=True)


PEAK_KINDS = (  # kind, name, FLOPs per MMA (2 M N K, K logical), rounds of four MMAs
    (0, "f16", 2 * 128 * 256 * 16, 8000),
    (1, "f16.sp", 2 * 128 * 256 * 32, 8000),
    (2, "nvfp4", 2 * 128 * 256 * 64, 8000),
    (3, "nvfp4.sp", 2 * 128 * 256 * 128, 8000),
    (4, "nvfp4.pair", 2 * 256 * 256 * 64, 8000),
)


def run_peaks(args) -> None:
    """The tensor-pipe and HBM rates this device reaches with this library's own instructions
    (back-to-back tcgen05 MMA loops on non-zero operands; a 16-byte load stream), written to
    profiles/peaks.json.  Reported beside the recipe's denominators (the driver's measured bf16
    GEMM x the nominal dtype ratio, and its measured copy bandwidth), not in their place."""
    import ctypes

    import torch

    import fp16_gemm_b200 as sp

    torch.cuda.set_device(0)
    L = sp.lib()
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    res, per = {}, {}
    with ClockSampler(0) as clk:
        for kind, name, flops, rounds in PEAK_KINDS:
            n = L.sp24_peak_ctas(kind)
            out = torch.zeros(n, dtype=torch.int64, device="cuda")
            best = None
            for _ in range(4):  # the first launch warms up; keep the fastest of the rest
                rc = L.sp24_peak_mma(kind, rounds, ctypes.c_void_p(out.data_ptr()), st)
                assert rc == sp.OK, sp.lib().sp24_status_string(rc)
                torch.cuda.synchronize()
                ns = out.cpu().numpy()
                issuers = int((ns > 0).sum())
                t = float(ns.max()) * 1e-9
                tf = issuers * 4 * rounds * flops / t / 1e12
                best = tf if best is None or tf > best else best
            assert sp.last_device_error() == sp.OK
            res[name] = round(best, 1)
            per[name] = {"issuing_ctas": issuers, "mma_per_cta": 4 * rounds, "flop_per_mma": flops}
        nbytes = 4 << 30
        buf = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        acc = torch.zeros(1, dtype=torch.int32, device="cuda")
        times = []
        for i in range(6):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            assert L.sp24_peak_read(ctypes.c_void_p(buf.data_ptr()), nbytes, ctypes.c_void_p(acc.data_ptr()), st) == sp.OK
            b.record()
            torch.cuda.synchronize()
            if i:
                times.append(a.elapsed_time(b) * 1e-3)
        hbm_read = nbytes / min(times) / 1e9
        del buf
    hbm, tp, src = tensor_peaks()
    line = {"mma_tflops": res, "mma_detail": per, "hbm_read_gbs": round(hbm_read, 1),
            "recipe_denominators": {"hbm_gbs": hbm, "tensor_tflops": tp, "source": src},
            "clocks": clk.summary(), "device": torch.cuda.get_device_name(0),
            "command": "python bench.py --peaks"}
    os.makedirs(os.path.join(ROOT, "profiles"), exist_ok=True)
    with open(os.path.join(ROOT, "profiles", "peaks.json"), "w") as f:
        json.dump(line, f, indent=1)
    print(json.dumps(line), flush=True)


def run_ncu_target(which: str) -> None:
    """Untimed: kernels run once each after a warm-up call, for an ncu capture of one family.
      decode  the decode step on its workload (prepare_vec, encode_pair_kernel, decode_tile_kernel
              dense and 2:4), twice;
      w4a4    the W4A4 GEMM at 4096^3 on tile images (gemm_nvfp4_pair_kernel), three times;
      f16     the FP16 M-sweep GEMMs at M = 4096, N = K = 5120 (gemm_f16_pair_kernel dense, then
              2:4 after its metadata image), twice;
      all     both, then the 2:4 and pairwise-4:8 W4A4 GEMMs, the FP16 M = 4096 GEMMs and the
              routed-expert workload once (several GB on the device)."""
    import torch

    import fp16_gemm_b200 as sp
    import synth

    torch.cuda.set_device(0)
    bf = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    if which in ("decode", "all"):
        d = synth.decode_nvfp4()
        x, w = bf(d["X"]), bf(d["W"])
        for _ in range(2):
            _, wq, sw = sp.prepare_nvfp4_24(w)
            sp.gemm_dense(x, wq)
            sp.gemm_sparse24(x, sw, K)
    if which in ("w4a4", "all"):
        d = synth.prefill_w4a4()
        xq, w = sp.quantize_nvfp4(bf(d["X"])), bf(d["W"])
        wq = sp.quantize_nvfp4(w)
        xi, wi = sp.to_mma(xq), sp.to_mma(wq)
        for _ in range(3):
            sp.gemm_dense(xi, wi)
    if which == "f16":
        g = synth.rng(0)
        w16 = torch.from_numpy(synth.draw(g, (5120, 5120), "f16")).cuda()
        x16 = torch.from_numpy(synth.draw(g, (4096, 5120), "f16")).cuda()
        v16, m16 = sp.prune_compress_24(w16)
        for _ in range(2):
            sp.gemm_dense(x16, w16)
            sp.gemm_sparse24(x16, sp.Sparse24(v16, m16), 5120)
    if which == "all":
        v, m = sp.prune_compress_24(w)
        vq = sp.quantize_nvfp4(v)
        v48, m48 = sp.prune_compress_48(w)
        s48, x32 = sp.Sparse48(sp.quantize_nvfp4(v48), m48), sp.quantize_nvfp4_block32(bf(d["X"]))
        for _ in range(2):
            sp.gemm_sparse24(xq, sp.Sparse24(vq, m), 4096)
            sp.gemm_sparse48(x32, s48, 4096)
        g = synth.rng(0)
        w16 = torch.from_numpy(synth.draw(g, (5120, 5120), "f16")).cuda()
        x16 = torch.from_numpy(synth.draw(g, (4096, 5120), "f16")).cuda()
        v, m = sp.prune_compress_24(w16)
        for _ in range(2):
            sp.gemm_dense(x16, w16)
            sp.gemm_sparse24(x16, sp.Sparse24(v, m), 5120)
        del w16, x16, v, m
        d = synth.moe()
        E, Ne, Ke = d["W"].shape
        xm, rt = bf(d["X"]), torch.from_numpy(d["routing"]).cuda()
        wm = bf(d["W"].reshape(E * Ne, Ke))
        del d
        _, wq, sw = sp.prepare_nvfp4_24(wm)
        del wm
        sp.gemm_grouped(xm, rt, wq, E, Ne, Ke)
        sp.gemm_grouped(xm, rt, sw, E, Ne, Ke)
    torch.cuda.synchronize()
    assert sp.last_device_error() == sp.OK
    print("ncu target done")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--sets", type=int, default=4)
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle work")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true", help="per-shape GEMM table instead of the step")
    ap.add_argument("--ncu-target", nargs="?", const="all", choices=["decode", "w4a4", "f16", "all"], default=None,
                    help="run one kernel family once, untimed (for an ncu capture); no value: all")
    ap.add_argument("--peaks", action="store_true", help="measure MMA and HBM peaks into profiles/peaks.json")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per-config GEMM table that follows the timed step")
    args = ap.parse_args()
    if args.sweep:
        run_sweep(args)
        return
    if args.ncu_target:
        run_ncu_target(args.ncu_target)
        return
    if args.peaks:
        run_peaks(args)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))

    if args.impl == "reference":
        # the CPU oracle on the host cores; under torchrun only rank 0 works
        if rank != 0:
            return
        budget = 90.0
        per_step_budget = budget / max(1, args.steps + args.warmup)
        gbs, dt, rows, cores = cpu_baseline(per_step_budget * args.steps, steps=args.steps)
        sample = f"{rows} of {N} weight rows per step (rotating), all stages, {args.steps} steps"
        line = {"metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "impl": "reference",
                "config": {"workload": WORKLOAD, "M": M, "N": N, "K": K},
                "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": cores,
                                 "kind": "oracle", "sample": sample},
                "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    import torch
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    else:
        torch.cuda.set_device(0)

    # CPU baseline first (rank 0, N=1 only), before any GPU work forks anything
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs, dt, rows, cores = cpu_baseline(args.cpu_budget)
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": f"{rows} of {N} weight rows, all six stages once ({dt:.1f} s)"}

    line = run_ours(args, rank, world, dist)
    if line is not None:
        line["cpu_baseline"] = cpu
        if world == 1 and not args.no_per_config:
            # every config at full size, each GEMM on prepared operands (CUDA-graph timing over
            # operand sets larger than the L2), after the timed step so it cannot disturb it
            lines = []
            t0 = time.perf_counter()
            with ClockSampler(torch.cuda.current_device()) as clk:
                sweep(lines.append, full=False)
            line["per_config"] = per_config(lines)
            line["per_config_clocks"] = clk.summary()
            line["per_config_seconds"] = round(time.perf_counter() - t0, 1)
            line["roofline_compute"] = compute_roofline(lines)
        print(json.dumps(line))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
