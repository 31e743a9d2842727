#!/usr/bin/env python
"""Benchmark of gated triangle self-attention, forward + backward, on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one forward and one backward call (every kernel of the path) over
one batch of synthetic inputs: N=768 residues, H=4 heads, c=32, bf16, starting
node, no mask, inputs drawn by tri_inputs (seeded). The metric counts
4*N^3*H*c forward and 10*N^3*H*c backward FLOPs per step. Inputs (755 MB of
pair tensors, 5.6 GB of workspace) are larger than the 126 MB L2, so no flush
is needed between steps.

With N > 1 GPUs (torchrun, one process per GPU) every rank runs its own
independent problem (weak scaling); ranks share only a barrier and a max of
the elapsed time. `--impl reference` times the fp64 CPU oracle on this host's
cores instead (rank 0 only), on bounded samples of attention rows.

Other lines (`--op`): `trimul` times the triangle multiplicative update
contraction (N=768, C=128, both directions, forward + backward), `proj` the
LayerNorm and projection stages around the attention (N=768, cz=128), `block`
the whole block LayerNorm -> projections -> attention -> output projection and
its backward. The default line is the attention.

Rank 0 prints one JSON line.
"""

from __future__ import annotations

import argparse
import hashlib
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

import tri_inputs  # noqa: E402

WORKLOAD = "n768_bf16"
METRIC = "triangle-attention fwd+bwd TFLOP/s at N=768 bf16 (% of B200 BF16 peak)"
UNIT = "TFLOP/s"
SPEC_BF16_TFLOPS = 2250.0
SMS = 148
EXP2_PER_CLK_PER_SM = 16     # measured ex2.approx issue rate of one SM


def flops(N: int, H: int, c: int) -> tuple:
    n3 = float(N) ** 3 * H * c
    return 4.0 * n3, 10.0 * n3


def load_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def tensor_peak(peaks: dict, clk: dict) -> tuple:
    """The bf16 matmul peak that matches how the kernel ran: the sustained figure
    when the sampled SM clock sat below 90% of its maximum under load (the
    power cap of a long run), else the burst figure."""
    mhz, mx = clk.get("sm_mhz"), clk.get("sm_max_mhz")
    if mhz and mx and peaks.get("bf16_tflops_sustained") and mhz < 0.9 * mx:
        return peaks["bf16_tflops_sustained"], f"{peaks['source']} bf16 matmul (sustained)"
    return peaks["bf16_tflops"], f"{peaks['source']} bf16 matmul (burst)"


def config_dict(w) -> dict:
    return {"workload": w.name, "N": w.N, "H": w.H, "c": w.c, "dtype": w.dtype,
            "variant": "starting", "mask": w.mask, "seed": w.seed,
            "l2": "inputs larger than L2 (755 MB pair tensors + 5.6 GB workspace per step)",
            "parallelism": "independent replica per GPU"}


# ----------------------------------------------------------------- clocks --

class ClockSampler:
    """SM clock and clock-event reasons sampled DURING the timed region.

    A thread polls NVML (read-only queries) every `period_s` seconds, so even a
    timed region of a few tens of milliseconds gets many samples; nvidia-smi's
    own polling (100 ms at best) would see none. Falls back to `nvidia-smi -lms`
    when NVML is not importable."""

    REASON_BITS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40,
                   "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4}

    def __init__(self, device: int, period_s: float = 0.002):
        self.device = device
        self.period = period_s
        self.samples = []
        self.begin = 0
        self.handle = None
        self.thread = None
        self.source = "nvml"

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.device).uuid)
            return pynvml.nvmlDeviceGetHandleByUUID(
                uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            visible = [v.strip() for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
                       if v.strip()]
            idx = int(visible[self.device]) if self.device < len(visible) and \
                visible[self.device].isdigit() else self.device
            return pynvml.nvmlDeviceGetHandleByIndex(idx)

    def start(self):
        import threading
        try:
            import pynvml
            self.handle = self._nvml_handle()
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle,
                                                                  pynvml.NVML_CLOCK_SM))
        except Exception:
            self.handle = None
            self.source = "unavailable"
            return
        self.running = True

        def poll():
            import pynvml
            while self.running:
                try:
                    mhz = pynvml.nvmlDeviceGetClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
                    rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                    self.samples.append((float(mhz), int(rs)))
                except Exception:
                    pass
                time.sleep(self.period)

        self.thread = threading.Thread(target=poll, daemon=True)
        self.thread.start()
        t_end = time.time() + 2.0
        while not self.samples and time.time() < t_end:
            time.sleep(0.001)

    def mark(self):
        """Index of the first sample taken inside the timed region."""
        self.begin = len(self.samples)

    def stop(self) -> dict:
        if self.handle is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["NVML unavailable"],
                    "samples": 0, "source": self.source}
        end = len(self.samples)
        self.running = False
        self.thread.join(timeout=2)
        window = self.samples[self.begin:end] or self.samples[-1:]
        sm = [m for m, _ in window]
        reasons = sorted(name for name, bit in self.REASON_BITS.items()
                         if any(r & bit for _, r in window))
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(window),
                "source": f"NVML poll every {self.period * 1e3:.0f} ms inside the timed region"}


# ------------------------------------------------------------- distributed --

def dist_setup(backend=None):
    """One process per GPU (torchrun's RANK/LOCAL_RANK/WORLD_SIZE): NCCL over the
    GPUs, or gloo when asked for (the CPU tests of the multi-process path)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = backend or "nccl"
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Slowest rank's time: every rank contributes, every rank gets the maximum."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world: int, flops_per_replica_step: float, ms_max: float) -> float:
    """Whole-job throughput of `world` replicas, each doing one step's FLOPs,
    timed by the slowest rank (weak scaling)."""
    return world * flops_per_replica_step / (ms_max * 1e-3) / 1e12


# --------------------------------------------------------------- CPU oracle --

def oracle_threads() -> int:
    env = os.environ.get("OMP_NUM_THREADS")
    return int(env) if env and env.isdigit() else (os.cpu_count() or 1)


def oracle_inputs(d) -> dict:
    """The workload's tensors widened once to float32 numpy (exact for bf16), so
    the oracle calls below time arithmetic, not conversion."""
    out = {}
    for k, v in d.items():
        if torch.is_tensor(v):
            v = v.to(torch.float32).numpy() if v.is_floating_point() else v.numpy()
        out[k] = v
    return out


def oracle_rows_step(d, rows) -> float:
    """fp64 oracle forward + backward of the listed attention rows; seconds."""
    import oracle
    args = (d["q"], d["k"], d["v"], d["bias"], d["gate"])
    t0 = time.perf_counter()
    oracle.fwd(*args, d["mask"], tri_inputs.STARTING, rows=rows)
    oracle.bwd(*args, d["dout"], d["mask"], tri_inputs.STARTING, rows=rows)
    return time.perf_counter() - t0


def oracle_rows_per_step(d, w, cores: int, step_s: float = 1.0) -> int:
    """Attention rows in one oracle step: a whole number of rounds of the host's
    threads (the oracle spreads (row, head) pairs over them), about step_s long.
    Both CPU legs (cpu_baseline and --impl reference) take steps of this size, so
    they time the same thing and report the same throughput."""
    t_row = oracle_rows_step(d, [0]) + 1e-9     # calibration, also warms the library
    unit = max(1, -(-cores // w.H))             # rows that give every thread one pair
    rounds = max(1, round(step_s / (t_row * unit)))
    return int(min(w.N, unit * rounds))


def oracle_sample(d, w, steps: int, warmup: int, seed: int, budget_s: float = 0.0) -> dict:
    """fp64 oracle forward + backward on random samples of whole attention rows
    (every head, query and key) of the workload, `steps` steps (or, with a
    budget, steps until `budget_s` seconds of oracle time are spent);
    throughput per row."""
    cores = oracle_threads()
    rows_per_step = oracle_rows_per_step(d, w, cores)
    rng = np.random.default_rng(seed)
    for _ in range(warmup):
        oracle_rows_step(d, rng.choice(w.N, rows_per_step, replace=False))
    secs, done = 0.0, 0
    while done < steps or secs < budget_s:
        secs += oracle_rows_step(d, rng.choice(w.N, rows_per_step, replace=False))
        done += 1
    steps = done
    f_fwd, f_bwd = flops(w.N, w.H, w.c)
    unit_flops = (f_fwd + f_bwd) / w.N          # one attention row, all heads
    value = unit_flops * rows_per_step * steps / secs / 1e12
    return {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{steps} steps of {rows_per_step} of {w.N} attention rows (all heads), "
                      f"fp64 forward+backward, {secs:.1f} s",
            "ms_per_step": secs / steps * 1e3}


def cpu_baseline(d, w, budget_s: float = 15.0) -> dict:
    """The oracle as it stands, on this host's cores, on a bounded sample of
    attention rows of the same workload: steps of about a second until the
    budget is spent (the same step shape as the reference arm)."""
    d = oracle_inputs(d)
    res = oracle_sample(d, w, steps=1, warmup=1, seed=2, budget_s=budget_s)
    res.pop("ms_per_step")
    return res


def run_reference(args, rank, world, w):
    """The oracle on host cores, each step a bounded sample of attention rows."""
    if rank != 0:
        return None
    d = oracle_inputs(tri_inputs.workload_inputs(w.name))
    res = oracle_sample(d, w, steps=args.steps, warmup=args.warmup, seed=2)
    value = res["value"]
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": res["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(w),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": res["cores"],
                             "kind": "oracle", "sample": res["sample"]},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------- our arm --

def traffic_record(kernel: str):
    """DRAM bytes per launch of a kernel from the committed ncu summary, or None
    if the kernel's source changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    src = {"fwd_bf16_kernel": "fwd_bf16.cu", "bwd_bf16_kernel": "bwd_bf16.cu"}[kernel]
    h = hashlib.sha256(open(os.path.join(ROOT, "triangle_attention_b200", "csrc", src),
                            "rb").read()).hexdigest()[:16]
    for line in open(path):
        parts = line.split()
        if len(parts) == 3 and parts[0] == kernel and parts[1] == h:
            return float(parts[2])
    return None


def run_ours(args, rank, world, local, w):
    import triangle_attention_b200 as ta

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    d = tri_inputs.workload_inputs(w.name, seed=w.seed + rank)
    g = {k: (v.to(dev).contiguous() if torch.is_tensor(v) else v) for k, v in d.items()}
    q, k, v, bias, gate, dout, mask = (g[n] for n in ("q", "k", "v", "bias", "gate", "dout",
                                                      "mask"))
    prob = ta.problem(q, mask, ta.STARTING)
    ws_f = ta.workspace(ta.fwd_workspace_size(prob), dev)
    ws_b = ta.workspace(ta.bwd_workspace_size(prob), dev)
    out = torch.empty_like(q)
    lse = torch.empty((w.N, w.H, w.N), dtype=torch.float32, device=dev)
    grads = tuple(torch.empty_like(t) for t in (q, k, v, bias, gate))
    stream = torch.cuda.current_stream()
    launches_per_step = (ta.kernel_launches(prob, False, mask is not None) +
                         ta.kernel_launches(prob, True, mask is not None))

    def step(opts_f=None, opts_b=None):
        ta.fwd(q, k, v, bias, gate, mask, ta.STARTING, out=out, lse=lse, ws=ws_f, opts=opts_f)
        ta.bwd(q, k, v, bias, gate, mask, out, lse, dout, ta.STARTING, grads=grads, ws=ws_b,
               opts=opts_b)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if ta.read_status(ws_f) or ta.read_status(ws_b):
        raise RuntimeError("device status reported a failure during warm-up")

    # per-step events around the two main kernels
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    opts = [(ta.launch_opts(e[0], e[1]), ta.launch_opts(e[2], e[3])) for e in ev]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)

    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    clocks.mark()
    t0.record(stream)
    for i in range(args.steps):
        step(*opts[i])
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    status = ta.read_status(ws_f) | ta.read_status(ws_b)
    if status:
        raise RuntimeError(f"device status {status} in the timed region")

    ms_local = t0.elapsed_time(t1) / args.steps
    ms = max_over_ranks(ms_local, world)
    f_fwd, f_bwd = flops(w.N, w.H, w.c)
    value = whole_job_tflops(world, f_fwd + f_bwd, ms)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    bwd_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in ev)
    fwd_med = statistics.median(e[0].elapsed_time(e[1]) for e in ev)
    bwd_med = statistics.median(e[2].elapsed_time(e[3]) for e in ev)
    # Each call resets its status word, so a bounded wait that ran out in an
    # earlier step of the timed region leaves no status behind; it does leave a
    # launch that ran for the wait's whole limit (2 s). Under a profiler (which
    # injects itself into the process) a captured launch is slow by design.
    if "CUDA_INJECTION64_PATH" not in os.environ:
        for name, col, med in (("forward", 0, fwd_med), ("backward", 2, bwd_med)):
            worst = max(e[col].elapsed_time(e[col + 1]) for e in ev)
            if worst > 1900.0:
                raise RuntimeError(f"a {name} launch in the timed region took {worst:.1f} ms "
                                   f"against a median of {med:.3f} ms: a bounded wait ran out")

    # roofline of the dominant kernel: algorithmic FLOPs per launch / launch time
    peaks = load_peaks()
    if bwd_ms >= fwd_ms:
        kname, kms, kflops = "bwd_bf16_kernel", bwd_ms, f_bwd
    else:
        kname, kms, kflops = "fwd_bf16_kernel", fwd_ms, f_fwd
    achieved = kflops / (kms * 1e-3) / 1e12
    traffic = traffic_record(kname)
    tpeak, tsrc = tensor_peak(peaks, clk)
    roofline = {"bound": "tensor", "kernel": kname, "achieved": achieved,
                "peak": tpeak, "unit": UNIT, "frac": achieved / tpeak, "traffic": traffic,
                "peak_source": tsrc}
    # the same kernel against the other two ceilings: HBM (its measured DRAM
    # bytes, when recorded for this source) and the exp2 unit (one exp2 per
    # logit; 16 per clock per SM, at the SM clock sampled during the run)
    sm_mhz = clk.get("sm_mhz") or 1965.0
    exp_peak = EXP2_PER_CLK_PER_SM * SMS * sm_mhz * 1e6
    exps = float(w.N) ** 3 * w.H
    rooflines = {
        "kernel": kname,
        "tensor": {"achieved_tflops": achieved, "peak_tflops": tpeak, "frac": achieved / tpeak},
        "hbm": ({"achieved_gbs": traffic / (kms * 1e-3) / 1e9, "peak_gbs": peaks["hbm_gbs"],
                 "frac": traffic / (kms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
                if traffic else None),
        "exp2": {"achieved_per_s": exps / (kms * 1e-3), "peak_per_s": exp_peak,
                 "frac": exps / (kms * 1e-3) / exp_peak,
                 "peak_source": "16 ex2 per clock per SM (microbenchmark) x 148 SMs x sampled clock"},
        "step_exp2_frac": 2 * exps / (ms_local * 1e-3) / exp_peak,
    }

    # End to end through the public API with pinned host buffers. Every step
    # uploads its inputs, runs forward + backward and downloads all its
    # results; the steps are double-buffered over three streams, so step k's
    # upload and step k-2's download overlap step k-1's kernels (PCIe carries
    # the two directions at once). Events order each buffer set's reuse.
    e2e_steps = max(4, min(args.steps, 12))
    host_in = {n: d[n].pin_memory() for n in ("q", "k", "v", "bias", "gate", "dout")}
    out_names = ("out", "lse", "dq", "dk", "dv", "dbias", "dgate")
    host_out = {n: torch.empty(t.shape, dtype=t.dtype).pin_memory()
                for n, t in zip(out_names, (out, lse) + tuple(grads))}
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    sets = []
    for j in range(2):
        dev_in = {n: (g[n] if j == 0 else torch.empty_like(g[n])) for n in host_in}
        dev_out = ({"out": out, "lse": lse, "grads": grads} if j == 0 else
                   {"out": torch.empty_like(out), "lse": torch.empty_like(lse),
                    "grads": tuple(torch.empty_like(t) for t in grads)})
        ev = {k: torch.cuda.Event() for k in ("in_ready", "in_free", "done", "out_free")}
        sets.append((dev_in, dev_out, ev))
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    s_comp = stream

    def e2e_step(k, first):
        dev_in, dev_out, ev = sets[k % 2]
        with torch.cuda.stream(s_in):
            if not first:
                s_in.wait_event(ev["in_free"])
            for n, t in host_in.items():
                dev_in[n].copy_(t, non_blocking=True)
            ev["in_ready"].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev["in_ready"])
            if not first:
                s_comp.wait_event(ev["out_free"])
            o, l = ta.fwd(dev_in["q"], dev_in["k"], dev_in["v"], dev_in["bias"], dev_in["gate"],
                          mask, ta.STARTING, out=dev_out["out"], lse=dev_out["lse"], ws=ws_f)
            ta.bwd(dev_in["q"], dev_in["k"], dev_in["v"], dev_in["bias"], dev_in["gate"], mask,
                   o, l, dev_in["dout"], ta.STARTING, grads=dev_out["grads"], ws=ws_b)
            ev["in_free"].record(s_comp)
            ev["done"].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["done"])
            for n, t in zip(out_names, (dev_out["out"], dev_out["lse"]) + tuple(dev_out["grads"])):
                host_out[n].copy_(t, non_blocking=True)
            ev["out_free"].record(s_out)

    e2e_step(0, True)
    e2e_step(1, True)
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    s_comp.wait_event(e0)
    s_out.wait_event(e0)
    for k in range(e2e_steps):
        e2e_step(k, False)
    s_out.wait_stream(s_comp)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)
    e2e_value = whole_job_tflops(world, f_fwd + f_bwd, e2e_ms)

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) pair tensors, tri_inputs)",
            "config": config_dict(w),
            "pct_of_spec_bf16_peak": 100.0 * value / world / SPEC_BF16_TFLOPS,
            "pct_of_measured_bf16_peak": 100.0 * value / world / peaks["bf16_tflops"],
            "kernels": {"fwd_bf16_kernel_ms": fwd_ms, "bwd_bf16_kernel_ms": bwd_ms,
                        "fwd_bf16_kernel_median_ms": fwd_med,
                        "bwd_bf16_kernel_median_ms": bwd_med, "step_ms": ms_local},
            "roofline": roofline,
            "rooflines": rooflines,
            "clocks": clk,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "pipelining": "double-buffered: upload of step k and download of step "
                                  "k-2 overlap the kernels of step k-1"},
            "gpu_launches": launches_per_step * args.steps}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(d, w)
    return line


# ---------------------------------------------- triangle multiplication --

TRIMUL_METRIC = "triangle-multiplication fwd+bwd TFLOP/s at N=768, C=128 bf16 (both directions)"


def run_trimul(args, rank, world, local):
    """One step: forward and backward of the outgoing and the incoming
    contraction on channel-major bf16 stacks, N=768 residues, C=128 channels."""
    import triangle_attention_b200 as ta
    N, C = 768, 128
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    gen = np.random.default_rng(11 + rank)
    host = [torch.from_numpy(gen.standard_normal((C, N, N)).astype(np.float32))
            .to(torch.bfloat16) for _ in range(3)]
    a, b, dt = (x.to(dev) for x in host)
    t = torch.empty_like(a)
    da, db = torch.empty_like(a), torch.empty_like(a)
    ws = ta.workspace(256, dev)
    stream = torch.cuda.current_stream()

    def step():
        for d in (ta.OUTGOING, ta.INCOMING):
            ta.mul_fwd(a, b, d, t=t, ws=ws)
            ta.mul_bwd(a, b, dt, d, grads=(da, db), ws=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    clocks.mark()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    if ta.read_status(ws):
        raise RuntimeError("device status set in the timed region")
    ms_local = t0.elapsed_time(t1) / args.steps
    ms = max_over_ranks(ms_local, world)
    flops_step = 2 * 6.0 * N ** 3 * C          # per direction: fwd 2N^3C, bwd 4N^3C
    value = whole_job_tflops(world, flops_step, ms)
    peaks = load_peaks()
    per_gemm_ms = ms_local / 6                 # six GEMMs of 2N^3C each per step
    achieved = 2.0 * N ** 3 * C / (per_gemm_ms * 1e-3) / 1e12
    line = {"metric": TRIMUL_METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) channel-major stacks)",
            "config": {"workload": "trimul_n768_c128", "N": N, "C": C,
                       "directions": ["outgoing", "incoming"],
                       "l2": "inputs larger than L2 (3 x 151 MB stacks)",
                       "parallelism": "independent replica per GPU"},
            "roofline": {"bound": "tensor", "kernel": "gemm_tc_kernel",
                         "achieved": achieved, "peak": tensor_peak(peaks, clk)[0], "unit": UNIT,
                         "frac": achieved / tensor_peak(peaks, clk)[0], "traffic": None,
                         "peak_source": tensor_peak(peaks, clk)[1]},
            "clocks": clk,
            "gpu_launches": 6 * args.steps}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        t_start = time.perf_counter()
        oracle.mul_fwd(host[0][:1], host[1][:1], oracle.OUTGOING)
        oracle.mul_bwd(host[0][:1], host[1][:1], host[2][:1], oracle.OUTGOING)
        secs = time.perf_counter() - t_start
        line["cpu_baseline"] = {"value": 6.0 * N ** 3 / secs / 1e12, "unit": UNIT,
                                "cores": oracle_threads(), "kind": "oracle",
                                "sample": f"1 of {C} channels, outgoing fwd+bwd, fp64, "
                                          f"{secs:.1f} s"}
    return line


UPDATE_METRIC = ("triangle multiplicative update fwd+bwd TFLOP/s at N=768, cz=128, c=128 bf16 "
                 "(both directions; LayerNorms, gated projections, contraction, output)")


def update_flops(N: int, cz: int, c: int) -> float:
    """Matmul FLOPs of one forward + backward of the update (2 per multiply-add):
    the input projection x W_in and its two gradients, the contraction and its
    two, the output projection and its two."""
    R, pgw = N * N, 4 * c + cz
    return 3 * 2.0 * R * cz * pgw + 3 * 2.0 * N ** 3 * c + 3 * 2.0 * R * c * cz


def run_trimul_update(args, rank, world, local):
    """One step: forward and backward of the full triangle multiplicative update,
    outgoing and incoming, N=768, cz=c=128."""
    import triangle_attention_b200 as ta
    N, cz, c = 768, 128, 128
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    d = tri_inputs.make_update_inputs(N, cz=cz, c=c, seed=21 + rank)
    z, dy = d["z"].to(dev), d["dy"].to(dev)
    params = {k: v.to(dev) for k, v in d["params"].items()}
    prob = ta.MulUpdateProblem(N, cz, c, ta.OUTGOING, 1e-5)
    nsaved, nws = ta.mul_update_sizes(prob)
    ws = ta.workspace(nws, dev)
    stream = torch.cuda.current_stream()

    def step():
        for direction in (ta.OUTGOING, ta.INCOMING):
            y, saved = ta.mul_update_fwd(z, params, direction, ws=ws)
            ta.mul_update_bwd(z, params, saved, dy, direction, ws=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    clocks.mark()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    if ta.get_status(ws):
        raise RuntimeError("device status set in the timed region")
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, world)
    flops_step = 2 * update_flops(N, cz, c)
    peaks = load_peaks()
    achieved = flops_step / (ms * 1e-3) / 1e12
    return {"metric": UPDATE_METRIC, "value": whole_job_tflops(world, flops_step, ms),
            "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded inputs and random-init parameters, tri_inputs)",
            "config": {"workload": "trimul_update_n768_cz128_c128", "N": N, "cz": cz, "c": c,
                       "directions": ["outgoing", "incoming"],
                       "l2": "inputs larger than L2 (saved activations 1.7 GB per direction)",
                       "parallelism": "independent replica per GPU"},
            "roofline": {"bound": "tensor", "kernel": "whole step (every kernel of the update)",
                         "achieved": achieved, "peak": tensor_peak(peaks, clk)[0], "unit": UNIT,
                         "frac": achieved / tensor_peak(peaks, clk)[0], "traffic": None,
                         "peak_source": tensor_peak(peaks, clk)[1]},
            "clocks": clk,
            # per direction: forward 8 kernels (2 LayerNorms, 2 products, the
            # contraction, 2 elementwise, a transpose); backward 19 (2 products, 2
            # weight gradients with their sums, 2 contraction products, 2 LayerNorm
            # backwards with their sums, 2 column sums with their sums, 2 elementwise,
            # a transpose)
            "gpu_launches": 2 * (8 + 19) * args.steps}


BLOCK_METRIC = ("triangle-attention block fwd+bwd TFLOP/s at N=768, cz=128, H=4, c=32 bf16 "
                "(LayerNorm, projections, attention, output projection)")


def block_flops(N: int, cz: int, H: int, c: int) -> dict:
    """Matmul FLOPs of each stage of the block (2 per multiply-add)."""
    R, hc = N * N, H * c
    f_fwd, f_bwd = flops(N, H, c)
    return {"proj_in_fwd": 2.0 * R * cz * (4 * hc + H),
            "attention_fwd": f_fwd, "proj_out_fwd": 2.0 * R * hc * cz,
            "proj_out_bwd": 4.0 * R * hc * cz, "attention_bwd": f_bwd,
            "proj_in_bwd": 4.0 * R * cz * (4 * hc + H)}


def block_bytes(N: int, cz: int, H: int, c: int) -> dict:
    """Minimum HBM bytes of the projection stages (each tensor read or written
    once; the attention stages are reported by the attention line)."""
    R, hc = N * N, H * c
    act, pair, bias = R * cz * 2, R * hc * 2, R * H * 2
    return {"proj_in_fwd": act + act + R * 8 + 4 * pair + bias,     # z; x, stats, q|k|v|g, bias
            "proj_out_fwd": pair + act,                             # o; y
            "proj_out_bwd": pair + act + pair,                      # o, dy; do
            "proj_in_bwd": act + act + R * 8 + 4 * pair + bias + act}   # z, x, stats, grads; dz


def run_block(args, rank, world, local):
    """One step: the whole triangle-attention block around the attention,
    forward and backward, N=768 (starting node, no mask), cz=128, H=4, c=32:
    LayerNorm and the q/k/v/gate/bias projections, the attention, the output
    projection, then the backward of each in reverse order."""
    import triangle_attention_b200 as ta
    N, cz, H, c = 768, 128, 4, 32
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    d = tri_inputs.make_block_inputs(N, cz, H, c, None, seed=11 + rank)
    g = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in d.items()}
    stream = torch.cuda.current_stream()
    prob = ta.proj_problem(g["z"], H, c)
    ws_p = ta.workspace(ta.proj_workspace_size(prob), dev)
    x, stats, q, k, v, gate, bias = ta.proj_in_fwd(g["z"], g["gamma"], g["beta"], g["w_qkvg"],
                                                   g["b_g"], g["w_b"], ws=ws_p)
    aprob = ta.problem(q, None, ta.STARTING)
    ws_f = ta.workspace(ta.fwd_workspace_size(aprob), dev)
    ws_b = ta.workspace(ta.bwd_workspace_size(aprob), dev)
    o, lse = ta.fwd(q, k, v, bias, gate, None, ta.STARTING, ws=ws_f)
    y = ta.proj_out_fwd(o, g["w_o"], g["b_o"], ws=ws_p)
    og = ta.proj_out_bwd(o, g["w_o"], g["dy"], ws=ws_p)
    ag = ta.bwd(q, k, v, bias, gate, None, o, lse, og[0], ta.STARTING, ws=ws_b)
    ig = ta.proj_in_bwd(g["z"], g["gamma"], g["w_qkvg"], g["w_b"], x, stats, ag[0], ag[1],
                        ag[2], ag[4], ag[3], grads=None, ws=ws_p)
    stages = {
        "proj_in_fwd": lambda: ta.proj_in_fwd(g["z"], g["gamma"], g["beta"], g["w_qkvg"],
                                              g["b_g"], g["w_b"],
                                              outs=(x, stats, q, k, v, gate, bias), ws=ws_p),
        "attention_fwd": lambda: ta.fwd(q, k, v, bias, gate, None, ta.STARTING, out=o, lse=lse,
                                        ws=ws_f),
        "proj_out_fwd": lambda: ta.proj_out_fwd(o, g["w_o"], g["b_o"], y=y, ws=ws_p),
        "proj_out_bwd": lambda: ta.proj_out_bwd(o, g["w_o"], g["dy"], grads=og, ws=ws_p),
        "attention_bwd": lambda: ta.bwd(q, k, v, bias, gate, None, o, lse, og[0], ta.STARTING,
                                        grads=ag, ws=ws_b),
        "proj_in_bwd": lambda: ta.proj_in_bwd(g["z"], g["gamma"], g["w_qkvg"], g["w_b"], x,
                                              stats, ag[0], ag[1], ag[2], ag[4], ag[3],
                                              grads=ig, ws=ws_p),
    }
    names = list(stages)

    def step(events=None):
        for i, n in enumerate(names):
            if events:
                events[i][0].record(stream)
            stages[n]()
            if events:
                events[i][1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    clocks.mark()
    ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in names]
          for _ in range(args.steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        step(ev[i])
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    for ws in (ws_p, ws_f, ws_b):
        if ta.read_status(ws):
            raise RuntimeError("device status set in the timed region")
    ms_local = t0.elapsed_time(t1) / args.steps
    ms = max_over_ranks(ms_local, world)
    stage_ms = {n: float(np.median([ev[i][j][0].elapsed_time(ev[i][j][1])
                                    for i in range(args.steps)])) for j, n in enumerate(names)}
    fl = block_flops(N, cz, H, c)
    by = block_bytes(N, cz, H, c)
    peaks = load_peaks()
    proj = {n: {"ms": stage_ms[n], "GB/s": by[n] / (stage_ms[n] * 1e-3) / 1e9,
                "frac_hbm": by[n] / (stage_ms[n] * 1e-3) / 1e9 / peaks["hbm_gbs"]}
            for n in by}
    top = max(by, key=lambda n: stage_ms[n])
    launches = {"proj_in_fwd": 2, "attention_fwd": ta.kernel_launches(aprob, False, False),
                "proj_out_fwd": 1, "proj_out_bwd": 4,
                "attention_bwd": ta.kernel_launches(aprob, True, False), "proj_in_bwd": 6}
    return {"metric": BLOCK_METRIC, "value": whole_job_tflops(world, sum(fl.values()), ms),
            "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded, tri_inputs.make_block_inputs)",
            "config": {"workload": "block_n768_cz128", "N": N, "cz": cz, "H": H, "c": c,
                       "variant": "starting", "mask": "none",
                       "l2": "inputs larger than L2 (z 151 MB, q/k/v/g 151 MB each)",
                       "parallelism": "independent replica per GPU"},
            "stage_ms": stage_ms, "projection_stages": proj,
            "roofline": {"bound": "hbm", "kernel": top, "achieved": proj[top]["GB/s"],
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": proj[top]["frac_hbm"], "traffic": None,
                         "note": "algorithmic bytes of the whole stage over its event time"},
            "clocks": clk, "gpu_launches": sum(launches.values()) * args.steps}


PROJ_METRIC = ("LayerNorm + projection stages fwd+bwd GB/s (algorithmic HBM bytes) at N=768, "
               "cz=128, H=4, c=32 bf16")


def run_mma_rate(args, rank, world, local):
    """Cycles per tcgen05.mma instruction (M=128, K=16, bf16, fp32 accumulator) by N
    and operand form, one CTA per SM issuing back to back, and the tensor-pipe floor
    they set for the attention step at N=768, H=4, c=32 (every instruction of the
    forward and backward main kernels issued back to back, nothing else)."""
    import triangle_attention_b200 as ta
    torch.cuda.set_device(local)
    ta.probe_mma(128, 0, instructions=1024)                 # warm-up
    forms = [(32, 0, "K-major A and B (S = Q K^T form)"), (64, 0, "K-major A and B"),
             (128, 0, "K-major A and B"), (256, 0, "K-major A and B"),
             (32, 1, "MN-major A and B (dV = P^T dU, dK = dS^T Q form)"),
             (32, 2, "A from tensor memory (O += P V form)")]
    rows, cyc = [], {}
    for n, layout, form in forms:
        c = ta.probe_mma(n, layout, instructions=16384)
        cyc[(n, layout)] = c
        rows.append({"n": n, "layout": layout, "form": form, "cycles_per_instruction": c,
                     "mac_per_cycle_per_sm": 128 * n * 16 / c,
                     "frac_of_dense": 128 * n * 16 / c / 4096})
    N, H = 768, 4
    nb = N // 128
    # backward, per 128 x 128 block and attention row: S and dP (2 + 2 at N = 128),
    # dV, dK, dQ (8 each at N = 32, K = 128 in steps of 16)
    bwd_block = 4 * cyc[(128, 0)] + 24 * cyc[(32, 1)]
    # forward, per 64-key step of 128 queries: S (2 at N = 64), O += P V (4 at N = 32)
    fwd_step = 2 * cyc[(64, 0)] + 4 * cyc[(32, 2)]
    bwd_units, fwd_units = nb * nb * N * H, nb * (N // 64) * N * H
    ghz = 1.965
    floor = {"backward_cycles_per_block_row": bwd_block, "forward_cycles_per_step": fwd_step,
             "backward_ms": bwd_units / SMS * bwd_block / ghz / 1e6,
             "forward_ms": fwd_units / SMS * fwd_step / ghz / 1e6}
    floor["step_ms"] = floor["backward_ms"] + floor["forward_ms"]
    return {"metric": "tcgen05.mma cycles per instruction (M=128, K=16, bf16, fp32 accumulate)",
            "unit": "cycles", "n_gpus": 1, "rows": rows,
            "tensor_floor_n768_h4_c32_at_1965mhz": floor,
            "config": {"workload": "mma_issue_rate", "ctas": SMS, "instructions": 16384}}


def run_proj(args, rank, world, local):
    """One step: the four projection calls around the attention (input side
    forward and backward, output side forward and backward) at N=768, cz=128,
    H=4, c=32, without the attention itself. HBM-bound work: the value is the
    algorithmic bytes of the four stages over the step time."""
    import triangle_attention_b200 as ta
    N, cz, H, c = 768, 128, 4, 32
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    d = tri_inputs.make_block_inputs(N, cz, H, c, None, seed=11 + rank)
    g = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in d.items()}
    stream = torch.cuda.current_stream()
    ws = ta.workspace(ta.proj_workspace_size(ta.proj_problem(g["z"], H, c)), dev)
    outs = ta.proj_in_fwd(g["z"], g["gamma"], g["beta"], g["w_qkvg"], g["b_g"], g["w_b"], ws=ws)
    ig = ta.proj_in_bwd(g["z"], g["gamma"], g["w_qkvg"], g["w_b"], outs[0], outs[1], g["dq"],
                        g["dk"], g["dv"], g["dg"], g["dbias"], ws=ws)
    o = g["dq"]                                   # stands in for the attention output
    y = ta.proj_out_fwd(o, g["w_o"], g["b_o"], ws=ws)
    og = ta.proj_out_bwd(o, g["w_o"], g["dy"], ws=ws)
    stages = {
        "proj_in_fwd": lambda: ta.proj_in_fwd(g["z"], g["gamma"], g["beta"], g["w_qkvg"],
                                              g["b_g"], g["w_b"], outs=outs, ws=ws),
        "proj_in_bwd": lambda: ta.proj_in_bwd(g["z"], g["gamma"], g["w_qkvg"], g["w_b"], outs[0],
                                              outs[1], g["dq"], g["dk"], g["dv"], g["dg"],
                                              g["dbias"], grads=ig, ws=ws),
        "proj_out_fwd": lambda: ta.proj_out_fwd(o, g["w_o"], g["b_o"], y=y, ws=ws),
        "proj_out_bwd": lambda: ta.proj_out_bwd(o, g["w_o"], g["dy"], grads=og, ws=ws),
    }
    names = list(stages)
    for _ in range(args.warmup):
        for n in names:
            stages[n]()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    clocks.mark()
    ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in names]
          for _ in range(args.steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        for j, n in enumerate(names):
            ev[i][j][0].record(stream)
            stages[n]()
            ev[i][j][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    if ta.read_status(ws):
        raise RuntimeError("device status set in the timed region")
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, world)
    stage_ms = {n: float(np.median([ev[i][j][0].elapsed_time(ev[i][j][1])
                                    for i in range(args.steps)])) for j, n in enumerate(names)}
    by = block_bytes(N, cz, H, c)
    peaks = load_peaks()
    gbs = {n: by[n] / (stage_ms[n] * 1e-3) / 1e9 for n in names}
    top = max(names, key=lambda n: stage_ms[n])
    return {"metric": PROJ_METRIC, "value": world * sum(by.values()) / (ms * 1e-3) / 1e9,
            "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded, tri_inputs.make_block_inputs)",
            "config": {"workload": "proj_n768_cz128", "N": N, "cz": cz, "H": H, "c": c,
                       "l2": "inputs larger than L2 (z 151 MB, q/k/v/g 151 MB each)",
                       "parallelism": "independent replica per GPU"},
            "stage_ms": stage_ms, "stage_gbs": gbs,
            "roofline": {"bound": "hbm", "kernel": top, "achieved": gbs[top],
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs[top] / peaks["hbm_gbs"], "traffic": None,
                         "note": "algorithmic bytes of the whole stage over its event time"},
            "clocks": clk, "gpu_launches": 13 * args.steps}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[1])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--op", choices=["attention", "trimul", "trimul_update", "block", "proj",
                                     "mma_rate"],
                    default="attention",
                    help="attention (the default line), the triangle multiplication "
                         "contraction, the full triangle multiplicative update, the whole "
                         "block around the attention, or its projection stages alone")
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(tri_inputs.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be at least 3")
    w = tri_inputs.WORKLOADS[args.workload]
    if not w.backward:
        ap.error("the benchmark step is forward + backward; pick a workload with a backward")

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        line = run_reference(args, rank, world, w)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    rank, world, local = dist_setup()
    try:
        if args.op == "trimul":
            line = run_trimul(args, rank, world, local)
        elif args.op == "trimul_update":
            line = run_trimul_update(args, rank, world, local)
        elif args.op == "block":
            line = run_block(args, rank, world, local)
        elif args.op == "proj":
            line = run_proj(args, rank, world, local)
        elif args.op == "mma_rate":
            line = run_mma_rate(args, rank, world, local)
        else:
            line = run_ours(args, rank, world, local, w)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
