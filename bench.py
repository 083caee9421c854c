"""Benchmark of the fused SDPA forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one fused forward (one kernel launch) over the whole workload with
Q, K, V resident in HBM.  Default workload: causal LM attention, B=8, Hq=Hkv=16,
Sq=Sk=4096, d=128, bf16 -- the Sk >= 4096, d = 128 case the tensor-core target
is stated on.  Q+K+V are 402 MB, above the 126 MB L2, so no step starts with
its inputs in L2.  Under torchrun every rank runs its own copy of the workload
(independent batches, weak scaling, no data-path collective); the process
group only carries the barrier and the max-over-ranks of the timings.

`--impl reference` times the fp64 CPU oracle on the host cores instead (rank
0 only), each step a bounded random sample of the workload's rows.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention fwd TFLOP/s on 1 B200 and % of dense BF16/FP8 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="lm_causal")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--pass", dest="pass_", default="fwd", choices=["fwd", "bwd"],
                    help="bwd: time sdpa_bwd (dQ, dK, dV) on the workload, one GPU")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-config measurements added to the JSON line (1 GPU only)")
    ap.add_argument("--ref-budget-s", type=float, default=90.0,
                    help="host seconds the reference (oracle) arm spends over all its steps")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def load_traffic(workload_name):
    """DRAM bytes per launch from the committed ncu summary of this kernel
    and workload, if one exists for the current kernel build."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload_name)
    return None if e is None else e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# ranks: one process per GPU, each with its own copy of the workload
# ---------------------------------------------------------------------------
def rank_barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks_value(x, world, device):
    """Max of a per-rank scalar over all ranks (the job's time is its slowest
    rank's); a no-op for one rank."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, flops_per_rank_step, steps, ms_max):
    """Whole-job TFLOP/s: the work of every rank over the slowest rank's time."""
    return world * flops_per_rank_step * steps / (ms_max * 1e-3) / 1e12


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML reads only; nothing is changed)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x1: "gpu_idle"}

    def __init__(self, index):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception as e:  # pragma: no cover - depends on the box
            self.error = str(e)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append(mhz)
                for b, name in self.REASONS.items():
                    if bits & b and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.02)

    def start(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._ok:
            self._stop.set()
            self._t.join()
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# CPU oracle timing (reported baseline, and the reference arm)
# ---------------------------------------------------------------------------
def oracle_rows_tflops(w, q, k, v, nrows, seed, nthreads, descales=(1.0, 1.0, 1.0)):
    """Time the oracle on `nrows` random rows; returns (seconds, flops)."""
    import numpy as np
    import oracle
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.integers(0, w.B * w.Hq * w.Sq, size=nrows))
    i = rows % w.Sq
    keys = (i + 1) if w.causal else np.full_like(i, w.Sk)
    flops = float(4.0 * w.d * keys.sum())
    t0 = time.perf_counter()
    oracle.sdpa_rows(q, k, v, rows, w.scale, w.causal, descales=descales, nthreads=nthreads)
    return time.perf_counter() - t0, flops


def cpu_inputs(w):
    from sdpa_workloads import make_inputs, make_qkv_fp8
    if w.dtype == "e4m3":
        q8, k8, v8, ds, _ = make_qkv_fp8(w)
        return q8, k8, v8, ds
    q, k, v = (t.contiguous() for t in make_inputs(w))
    return q, k, v, (1.0, 1.0, 1.0)


def cpu_baseline(w, seconds):
    import oracle
    nt = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    q, k, v, ds = cpu_inputs(w)
    t, f = oracle_rows_tflops(w, q, k, v, 64, 1, nt, ds)          # calibrate
    nrows = int(max(64, min(200000, 64 * seconds / max(t, 1e-6))))
    t, f = oracle_rows_tflops(w, q, k, v, nrows, 2, nt, ds)
    return {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": nt, "kind": "oracle",
            "sample": "%d random rows of %s (all batches/heads), fp64 C oracle, OpenMP, %.1f s"
                      % (nrows, w.name, t)}


def arm_config(w, world):
    """The `config` object of the JSON line; both arms print the same one."""
    elt = 1 if w.dtype == "e4m3" else 2
    in_mb = (w.B * w.Hq * w.Sq + 2 * w.B * w.Hkv * w.Sk) * w.d * elt / 1e6
    l2_note = ("inputs %.0f MB per GPU > 126 MB L2; no flush" % in_mb if in_mb > 126
               else "inputs %.0f MB per GPU fit in L2: L2-warm timing" % in_mb)
    return dict(w.describe(), global_batch=w.B * world,
                parallelism="dp%d (independent batches per GPU)" % world, l2=l2_note)


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    nt = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    q, k, v, ds = cpu_inputs(w)
    t, _ = oracle_rows_tflops(w, q, k, v, 32, 7, nt, ds)
    per_row = t / 32
    budget = args.ref_budget_s
    rows_per_step = int(max(1, min(4096, budget / max(1, args.steps + args.warmup) / per_row)))
    for s in range(args.warmup):
        oracle_rows_tflops(w, q, k, v, rows_per_step, 100 + s, nt, ds)
    tot_t, tot_f = 0.0, 0.0
    for s in range(args.steps):
        t, f = oracle_rows_tflops(w, q, k, v, rows_per_step, 1000 + s, nt, ds)
        tot_t += t
        tot_f += f
    value = tot_f / tot_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": arm_config(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": nt, "kind": "oracle",
                         "sample": "%d random rows per step of %s, fp64 C oracle, OpenMP"
                                   % (rows_per_step, w.name)},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_backward(args, w):
    """Device-timed sdpa_bwd on one GPU.  FLOPs are the five contractions of
    the backward (S, dP, dV, dK, dQ: 2.5x the forward's).  Head dims 64 and
    128 run on the tensor cores (roofline: the dense bf16 peak); head dim 32
    on the CUDA cores (roofline: their fp32 FMA rate)."""
    import torch
    import scaled_dot_product_11_b200 as sdpa
    from sdpa_workloads import make_qkv
    dev = torch.device("cuda", 0)
    q, k, v = make_qkv(w, dev)
    g = torch.Generator(device="cpu").manual_seed(w.seed + 1)
    dout = torch.randn(q.shape, generator=g).to(q.dtype).to(dev)
    o, lse = sdpa.attention(q, k, v, causal=w.causal, scale=w.scale)
    run = lambda: sdpa.attention_backward(q, k, v, o, lse, dout, causal=w.causal, scale=w.scale)
    for _ in range(args.warmup):
        run()
    torch.cuda.synchronize()
    st, detail = sdpa.sdpa_device_status(clear=True)
    if st != 0:
        raise SystemExit("device status %d (%#x) after warm-up" % (st, detail))
    clocks = ClockSampler(0)
    clocks.start()
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        run()
    e1.record(stream)
    e1.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1) / args.steps
    flops = 2.5 * w.flops
    value = flops / (ms * 1e-3) / 1e12
    props = torch.cuda.get_device_properties(dev)
    max_mhz = float((clk or {}).get("sm_max_mhz") or 1965.0)
    if w.d == 32:
        # head dim 32 runs on the CUDA cores
        bound = "alu"
        peak = props.multi_processor_count * 128 * 2 * max_mhz * 1e6 / 1e12   # fp32 FMA lanes
        peak_source = "%d SMs x 128 fp32 FMA lanes x 2 flop x %.0f MHz" % (props.multi_processor_count, max_mhz)
    else:
        peaks, src = load_peaks()
        bound, peak = "tensor", float(peaks["bf16_tflops"])
        peak_source = "%s bf16_tflops (burst)" % src
    print(json.dumps({
        "metric": "attention bwd (dQ, dK, dV) TFLOP/s on 1 B200", "value": value, "unit": "TFLOP/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic", "config": dict(w.describe(), pass_="bwd"),
        "roofline": {"bound": bound, "achieved": value, "peak": peak, "unit": "TFLOP/s",
                     "frac": value / peak, "traffic": load_traffic("bwd:" + w.name),
                     "traffic_kernel": "sdpa_bwd_dkdv_pipe_kernel (the larger of the two launches)",
                     "peak_source": peak_source},
        "clocks": clk, "gpu_launches": 2 * args.steps}))


def roofline_of(w, ms, peaks, src, fwd=True):
    """Roofline of one launch of workload w taking `ms`: the tensor peak of
    the inputs' dtype (e4m3: the measured bf16 figure x 2, the nominal ratio)
    when the algorithmic arithmetic intensity is above the ridge, HBM
    otherwise; the backward's five contractions are 2.5x the forward's."""
    fp8 = w.dtype == "e4m3"
    flops = w.flops * (1.0 if fwd else 2.5)
    peak = float(peaks["bf16_tflops"]) * (2.0 if fp8 else 1.0)
    ridge = peak * 1e12 / (float(peaks["hbm_gbs"]) * 1e9)
    ai = flops / w.min_hbm_bytes
    if ai < ridge:
        achieved = w.min_hbm_bytes / (ms * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": achieved, "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                "frac": achieved / float(peaks["hbm_gbs"]), "arithmetic_intensity": ai,
                "peak_source": "%s hbm_gbs (copy)" % src}
    achieved = flops / (ms * 1e-3) / 1e12
    return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "arithmetic_intensity": ai,
            "peak_source": "%s bf16_tflops (burst)%s" % (src, " x 2 (nominal fp8/bf16)" if fp8 else "")}


def median_launch_ms(run, stream, n):
    """Median device time of one launch over n launches, each bracketed by its
    own pair of CUDA events on the launching stream (run outside the timed
    region, after the warm-ups)."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for a, b in evs:
        a.record(stream)
        run()
        b.record(stream)
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in evs)


def graph_launch_ms(run, stream, n):
    """Device time of one launch when n launches replay from one CUDA graph,
    so that no host submission separates them (short kernels otherwise wait
    on the Python binding between launches); None if the capture fails."""
    import torch
    g = torch.cuda.CUDAGraph()
    try:
        with torch.cuda.graph(g):
            for _ in range(n):
                run()
    except Exception:
        torch.cuda.synchronize()
        return None
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g.replay()
    e1.record(stream)
    e1.synchronize()
    del g
    return e0.elapsed_time(e1) / n


def config_sweep(dev, launches=20, warmup=3):
    """Every other workload the pages measure (tiny, ViT, GQA, MQA, FP8, two
    sequence-sweep points), one GPU: device
    time over `launches` launches after `warmup`, TFLOP/s, roofline fraction,
    and the largest |O - O_ref| over sampled rows against the oracle; then the
    backward on the causal LM shape (timing only)."""
    import numpy as np
    import torch
    import oracle
    import scaled_dot_product_11_b200 as sdpa
    from sdpa_workloads import WORKLOADS, make_qkv, make_qkv_fp8, sample_rows, sweep
    peaks, src = load_peaks()
    names = ["tiny", "vit", "gqa", "mqa", "fp8"]
    todo = [WORKLOADS[n] for n in names] + [sweep(False)[5], sweep(True)[0]]
    stream = torch.cuda.current_stream(dev)
    out = []
    for w in todo:
        fp8 = w.dtype == "e4m3"
        if fp8:
            q, k, v, ds, _ = make_qkv_fp8(w, dev)
            run = lambda: sdpa.attention_fp8(q, k, v, ds, causal=w.causal, scale=w.scale, out=o, lse=lse)
            o = torch.empty((w.B, w.Hq, w.Sq, w.d), dtype=torch.bfloat16, device=dev)
        else:
            q, k, v = make_qkv(w, dev)
            ds = (1.0, 1.0, 1.0)
            run = lambda: sdpa.attention(q, k, v, causal=w.causal, scale=w.scale, out=o, lse=lse)
            o = torch.empty_like(q)
        lse = torch.empty((w.B, w.Hq, w.Sq), dtype=torch.float32, device=dev)
        for _ in range(warmup):
            run()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(launches):
            run()
        e1.record(stream)
        e1.synchronize()
        ms = e0.elapsed_time(e1) / launches
        med = median_launch_ms(run, stream, launches)
        gms = graph_launch_ms(run, stream, launches)
        st, detail = sdpa.sdpa_device_status(clear=True)
        rows = sample_rows(w, n_random=32)
        rows = rows[:: max(1, len(rows) // 64)]
        ro, _ = oracle.sdpa_rows(*(t.contiguous().cpu() for t in (q, k, v)), rows, w.scale, w.causal,
                                 descales=ds)
        go = o.reshape(-1, w.d).index_select(0, torch.tensor(rows, device=dev)).double().cpu().numpy()
        # the roofline takes the kernel's own launch time: for launches
        # shorter than 100 us the graph replay's (the binding's host path
        # between eager launches would show in theirs), else the eager loop's
        use_graph = gms is not None and ms < 0.1
        roof = roofline_of(w, gms if use_graph else ms, peaks, src)
        roof["traffic"] = load_traffic(w.name)
        roof["timing"] = ("%d launches from one CUDA graph" if use_graph else
                          "%d back-to-back launches") % launches
        out.append({"workload": w.name, "ms": ms, "tflops": w.flops / (ms * 1e-3) / 1e12,
                    "launches": launches, "median_ms": med, "median_tflops": w.flops / (med * 1e-3) / 1e12,
                    "graph_ms": gms, "graph_tflops": w.flops / (gms * 1e-3) / 1e12 if gms else None,
                    "roofline": roof,
                    "parity": {"rows": len(rows), "max_abs_o": float(np.abs(go - ro).max())},
                    "device_status": st})
        del q, k, v, o, lse
    # backward on the causal LM shape
    w = WORKLOADS["lm_causal"]
    q, k, v = make_qkv(w, dev)
    g = torch.Generator(device="cpu").manual_seed(w.seed + 1)
    dout = torch.randn(q.shape, generator=g).to(q.dtype).to(dev)
    o, lse = sdpa.attention(q, k, v, causal=w.causal, scale=w.scale)
    run = lambda: sdpa.attention_backward(q, k, v, o, lse, dout, causal=w.causal, scale=w.scale)
    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(launches):
        run()
    e1.record(stream)
    e1.synchronize()
    ms = e0.elapsed_time(e1) / launches
    med = median_launch_ms(run, stream, launches)
    st, _ = sdpa.sdpa_device_status(clear=True)
    out.append({"workload": w.name, "pass": "bwd", "ms": ms, "tflops": 2.5 * w.flops / (ms * 1e-3) / 1e12,
                "launches": launches, "median_ms": med, "median_tflops": 2.5 * w.flops / (med * 1e-3) / 1e12,
                "roofline": roofline_of(w, ms, peaks, src, fwd=False),
                "device_status": st})
    return out


def main():
    args = parse()
    from sdpa_workloads import WORKLOADS, make_inputs, make_qkv_fp8, sample_rows, with_shape
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if args.pass_ == "bwd":
        assert args.warmup >= 3, "at least 3 warm-up steps"
        return run_backward(args, w)
    assert args.warmup >= 3, "at least 3 warm-up steps"

    import numpy as np
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE %d" % (args.gpus, world))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    import scaled_dot_product_11_b200 as sdpa
    fp8 = w.dtype == "e4m3"
    # every rank draws its own batch of the same shape (weak scaling)
    w_rank = with_shape(w, seed=w.seed + 1000 * rank)
    if fp8:
        q, k, v, ds, _ = make_qkv_fp8(w_rank, dev)
        run = lambda: sdpa.attention_fp8(q, k, v, ds, causal=w.causal, scale=w.scale, out=o, lse=lse)
    else:
        # "btnh" workloads: [B,S,H,d] data as views, through sdpa_fwd_strided
        q, k, v = make_inputs(w_rank, dev)
        run = lambda: sdpa.attention(q, k, v, causal=w.causal, scale=w.scale, out=o, lse=lse)
    o = torch.empty((w.B, w.Hq, w.Sq, w.d), dtype=torch.bfloat16 if fp8 or w.dtype == "bf16"
                    else torch.float16, device=dev)
    if w.layout == "btnh":
        o = torch.empty_like(q)             # laid out like q: [B,S,H,d] memory
    lse = torch.empty((w.B, w.Hq, w.Sq), dtype=torch.float32, device=dev)

    barrier = lambda: rank_barrier(world)
    max_over_ranks = lambda x: max_over_ranks_value(x, world, dev)

    # warm-up (also the parity spot check of this exact launch configuration)
    for _ in range(args.warmup):
        run()
    torch.cuda.synchronize()
    st, detail = sdpa.sdpa_device_status(clear=True)
    if st != 0:
        raise SystemExit("device status %d (%#x) after warm-up" % (st, detail))
    parity = None
    if rank == 0:
        import oracle
        rows = sample_rows(w, n_random=32)[:: max(1, len(sample_rows(w, n_random=32)) // 96)]
        qc, kc, vc = (t.contiguous().cpu() for t in (q, k, v))
        ro, rl = oracle.sdpa_rows(qc, kc, vc, rows, w.scale, w.causal,
                                  descales=ds if fp8 else (1.0, 1.0, 1.0))
        idx = torch.tensor(rows, device=dev)
        go = o.reshape(-1, w.d).index_select(0, idx).double().cpu().numpy()
        gl = lse.reshape(-1).index_select(0, idx).double().cpu().numpy()
        parity = {"rows": len(rows), "max_abs_o": float(np.abs(go - ro).max()),
                  "max_abs_lse": float(np.abs(gl - rl).max())}

    # timed region: device time with CUDA events on the launching stream
    stream = torch.cuda.current_stream(dev)
    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        run()
    e1.record(stream)
    e1.synchronize()
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms_total = max_over_ranks(e0.elapsed_time(e1))
    st, detail = sdpa.sdpa_device_status(clear=True)
    if st != 0:
        raise SystemExit("device status %d (%#x) after timing" % (st, detail))
    ms_per_step = ms_total / args.steps
    value = job_throughput(world, w.flops, args.steps, ms_total)
    # per-launch device times, after the timed region: the median of up to 50
    # launches, each with its own event pair (max over ranks)
    n_med = min(50, args.steps)
    med_ms = max_over_ranks(median_launch_ms(run, stream, n_med))
    median = {"ms": med_ms, "value": job_throughput(world, w.flops, 1, med_ms), "launches": n_med}

    # end to end through the public API: pinned host inputs -> device -> fused
    # forward -> O and LSE back to pinned host memory, every step's copies and
    # launch inside the region.  Steps are pipelined the way a serving loop
    # would run them: step i+1's host-to-device copies (one stream) and step
    # i-1's device-to-host copies (another) run under step i's forward, on two
    # sets of device buffers; the region ends when the last result is on the
    # host.
    e2e_steps = 0 if args.no_e2e else max(3, min(20, args.steps // 20))
    hq_, hk_, hv_ = (t.cpu().pin_memory() for t in (q, k, v))
    ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    hl = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    bufs = [dict(q=torch.empty_like(q), k=torch.empty_like(k), v=torch.empty_like(v),
                 o=torch.empty_like(o), lse=torch.empty_like(lse)) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    fwd_done = [None, None]   # the forward that last read / wrote buffer set b
    out_done = [None, None]   # the copy that last read set b's O and LSE

    def run_e2e(i):
        b = i % 2
        d = bufs[b]
        with torch.cuda.stream(s_in):
            if fwd_done[b] is not None:
                s_in.wait_event(fwd_done[b])
            d["q"].copy_(hq_, non_blocking=True)
            d["k"].copy_(hk_, non_blocking=True)
            d["v"].copy_(hv_, non_blocking=True)
            in_done = ev()
            in_done.record(s_in)
        stream.wait_event(in_done)
        if out_done[b] is not None:
            stream.wait_event(out_done[b])
        if fp8:
            sdpa.attention_fp8(d["q"], d["k"], d["v"], ds, causal=w.causal, scale=w.scale, out=d["o"], lse=d["lse"])
        else:
            sdpa.attention(d["q"], d["k"], d["v"], causal=w.causal, scale=w.scale, out=d["o"], lse=d["lse"])
        fwd_done[b] = ev()
        fwd_done[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(fwd_done[b])
            ho.copy_(d["o"], non_blocking=True)
            hl.copy_(d["lse"], non_blocking=True)
            out_done[b] = ev()
            out_done[b].record(s_out)

    h2d = sum(t.numel() * t.element_size() for t in (q, k, v))
    d2h = o.numel() * o.element_size() + lse.numel() * lse.element_size()
    e2e_value = None
    if e2e_steps:
        for i in range(2):
            run_e2e(i)
        torch.cuda.synchronize()
        barrier()
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(s_in)
        for i in range(e2e_steps):
            run_e2e(i)
        stream.wait_event(out_done[(e2e_steps - 1) % 2])
        end.record(stream)
        end.synchronize()
        barrier()
        ms_e2e = max_over_ranks(start.elapsed_time(end))
        e2e_value = job_throughput(world, w.flops, e2e_steps, ms_e2e)
        del bufs
        torch.cuda.synchronize()

    if rank == 0:
        peaks, src = load_peaks()
        # a contraction takes the peak of its own dtype: e4m3 is the measured
        # bf16 figure times the nominal dense fp8 / bf16 ratio (2)
        ratio = 2.0 if fp8 else 1.0
        peak = float(peaks["bf16_tflops"]) * ratio
        achieved = w.flops / (ms_per_step * 1e-3) / 1e12
        traffic = load_traffic(w.name)
        # the bound: tensor peak when the arithmetic intensity (algorithmic
        # flops per algorithmic byte) is above the ridge, HBM otherwise
        ridge = peak * 1e12 / (float(peaks["hbm_gbs"]) * 1e9)
        hbm_bound = w.flops / w.min_hbm_bytes < ridge
        if hbm_bound:
            roofline = {"bound": "hbm", "achieved": w.min_hbm_bytes / (ms_per_step * 1e-3) / 1e9,
                        "peak": float(peaks["hbm_gbs"]), "unit": "GB/s", "traffic": traffic,
                        "peak_source": "%s hbm_gbs (copy)" % src,
                        "arithmetic_intensity": w.flops / w.min_hbm_bytes, "ridge": ridge}
            roofline["frac"] = roofline["achieved"] / roofline["peak"]
        else:
            roofline = {"bound": "tensor", "achieved": achieved, "peak": peak,
                        "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                        "peak_source": "%s bf16_tflops (burst)%s; frac of sustained %.3f" % (
                            src, " x 2 (nominal fp8/bf16)" if fp8 else "",
                            achieved / (float(peaks["bf16_tflops_sustained"]) * ratio))}
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3" if fp8 else w.dtype, "data": "synthetic",
            "config": arm_config(w, world),
            "roofline": roofline,
            "clocks": clk,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps},
            "gpu_launches": args.steps * sdpa.sdpa_launches_per_call(),
            "median": median,
            "parity": parity,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
        if world == 1 and not args.no_configs:
            line["configs"] = config_sweep(dev)
        print(json.dumps(line), flush=True)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
