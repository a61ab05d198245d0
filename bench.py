#!/usr/bin/env python
"""Packed LoRA forward + backward throughput on B200.

One step = one plora_forward + one plora_backward (all eight products of the
packed layer plus the factor packing) over the LLaMA-3-8B up_proj workload
(4096 -> 14336, bf16, 32 adapters, ranks U{8..128}, long-tail token counts
log-uniform in [512, 4096]).  Inputs are seeded synthetic tensors of that
shape, resident in HBM before the timed region (larger than L2, so no flush).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torch.distributed.run, one process per GPU.  By default the
32 adapters are split across the GPUs by plora_partition (longest processing
time first over the per-adapter cost): adapters are independent, so the work
shards with no data-path collective (strong scaling); `--scaling weak` gives
every rank its own 32-adapter set instead.  The step time is the max over ranks.
`--impl reference` times the fp64 CPU oracle on the host cores instead.
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import plora_workloads as wl  # noqa: E402

METRIC = "packed LoRA fwd+bwd tokens/sec on 1 B200 (32 adapters); % HBM / tensor roofline"
UNIT = "tokens/s"
WORKLOAD = "llama3-8b up_proj 4096->14336 bf16, 32 adapters r~U{8,16,32,64,128}, tokens~logU[512,4096]"
WORKLOADS = {
    "llama_up32": WORKLOAD,
    "small": "llama3-8b up_proj 4096->14336 bf16, the first 8 adapters of the 32-adapter mix x 2048 tokens",
    "layer_q": "llama3-8b q_proj 4096->4096 bf16, 16 adapters r~U{16,32,64} x 8192 tokens",
    "llama_up_r16x1": "llama3-8b up_proj 4096->14336 bf16, one rank-16 adapter over the 32-adapter mix's tokens",
}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TC_KINDS = ("base_fwd", "base_dx", "base_dx+wgrad_a")


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--seed", type=int, default=1003)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--unfused", action="store_true",
                    help="run the expand products as separate passes (for comparison with the fused default)")
    ap.add_argument("--base-pair", action="store_true",
                    help="base GEMMs on SM pairs (cta_group::2) instead of single SMs")
    ap.add_argument("--layer-tokens", type=int, default=8192,
                    help="tokens per adapter of the one-layer line (the stated workload has 8192)")
    ap.add_argument("--layer-only", action="store_true",
                    help="only the suite's one-layer line (seven calls, four calls with output blocks, one layer call)")
    ap.add_argument("--suite", action="store_true",
                    help="measure every workload (packed vs per-adapter sequential loop); one JSON line each")
    ap.add_argument("--workload", choices=list(WORKLOADS), default="llama_up32",
                    help="small: 8 adapters of the same mix cut to 2048 tokens each; layer_q: the 4096x4096 q_proj "
                         "of the one-layer workload, 16 adapters x 8192 tokens (both for profiler captures); "
                         "llama_up_r16x1: one rank-16 adapter over the same tokens (base GEMMs with negligible "
                         "low-rank work)")
    ap.add_argument("--scaling", choices=["strong", "weak"], default="strong",
                    help="N > 1: strong = one 32-adapter set split across the GPUs by plora_partition (LPT over "
                         "the per-adapter cost); weak = every GPU runs its own 32-adapter set")
    ap.add_argument("--base-gemm-reference", action="store_true",
                    help="time the workload's two base GEMMs (Y = X W^T, dX = dY W) through torch.matmul "
                         "(cuBLAS) with the same timing, clock and energy records; a context line, not a "
                         "product path")
    return ap.parse_args(argv)


# ----------------------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def algorithmic_work(p):
    """Per-launch algorithmic work of every kernel kind of one step: (flops, bytes)."""
    n = p.counts.astype(np.float64)
    r = p.ranks.astype(np.float64)
    di, do = float(p.d_in), float(p.d_out)
    T = float(p.T)
    rp16 = np.ceil(r / 16) * 16
    w = {
        "base_fwd": (2 * T * di * do, 2 * (T * di + di * do + T * do)),
        "base_dx": (2 * T * di * do, 2 * (T * do + di * do + T * di)),
        "shrink_x": (float(np.sum(2 * n * di * r)), float(np.sum(n * (2 * di + 2 * r) + 2 * r * di))),
        "expand_y": (float(np.sum(2 * n * do * r)), float(np.sum(n * (4 * do + 2 * r) + 2 * r * do))),
        "shrink_dy": (float(np.sum(2 * n * do * r)), float(np.sum(n * (2 * do + 2 * r) + 2 * r * do))),
        "expand_dx": (float(np.sum(2 * n * di * r)), float(np.sum(n * (4 * di + 2 * r) + 2 * r * di))),
        "wgrad_b": (float(np.sum(2 * n * do * r)), float(np.sum(n * (2 * do + 2 * r) + 4 * r * do))),
        "wgrad_a": (float(np.sum(2 * n * di * r)), float(np.sum(n * (2 * di + 2 * r) + 4 * r * di))),
        # one pack per step: reads each factor once, writes A's rows and B's columns up to rp16
        "pack_ab": (0.0, float(np.sum(2 * r * (di + do) + 2 * rp16 * (di + do)))),
    }
    # K7's items share K5's launch; K8's share the dX GEMM's
    w["shrink_dy+wgrad_b"] = (w["shrink_dy"][0] + w["wgrad_b"][0], w["shrink_dy"][1] + w["wgrad_b"][1])
    w["base_dx+wgrad_a"] = (w["base_dx"][0] + w["wgrad_a"][0], w["base_dx"][1] + w["wgrad_a"][1])
    return w


class EnergyMeter:
    """The GPU's cumulative energy counter (NVML, millijoules), read around the timed region."""

    def __init__(self, gpu_uuid: str):
        self.h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByUUID(gpu_uuid)
        except Exception:
            self.h = None

    def read_mj(self):
        if self.h is None:
            return None
        try:
            return float(self.nvml.nvmlDeviceGetTotalEnergyConsumption(self.h))
        except Exception:
            return None

    def start(self):
        self.e0, self.t0 = self.read_mj(), time.time()

    def stop(self):
        e1, t1 = self.read_mj(), time.time()
        if self.e0 is None or e1 is None:
            return None, None
        joules = (e1 - self.e0) / 1e3
        return joules, joules / max(t1 - self.t0, 1e-9)


class ClockSampler:
    """SM clock and clock-event (throttle) reasons during the timed region: NVML (the counters
    nvidia-smi reads) polled every 5 ms from a background thread between start() and stop(), which
    bracket the timed steps, so that a region of a few hundred milliseconds still gets dozens of
    samples and none from the idle GPU around it.  Falls back to nvidia-smi -lms 100 without NVML."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = (("hw_slowdown", 0x8 | 0x80), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))

    def __init__(self, gpu_uuid: str):
        self.gpu_uuid = gpu_uuid
        self.h = None
        self.proc = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByUUID(gpu_uuid)
        except Exception:
            self.h = None

    def _poll(self):
        nv = self.nvml
        while not self.done.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                why = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((float(mhz), int(why)))
            except Exception:
                pass
            self.done.wait(0.005)

    def start(self):
        import threading
        self.samples = []
        if self.h is not None:
            self.done = threading.Event()
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        fd, self.path = tempfile.mkstemp(prefix="plora_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits", "-lms", "100",
                 "--id=" + self.gpu_uuid, "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.h is not None:
            self.done.set()
            self.thread.join(timeout=5)
            try:
                mx = float(self.nvml.nvmlDeviceGetMaxClockInfo(self.h, self.nvml.NVML_CLOCK_SM))
            except Exception:
                mx = None
            sm = [m for m, _ in self.samples]
            reasons = sorted({name for _, why in self.samples for name, bit in self.REASONS if why & bit})
            return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": reasons,
                    "samples": len(sm), "source": "NVML every 5 ms during the timed region"}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "source": "nvidia-smi -lms 100 around the timed region"}


def reduce_max(x: float, dist) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process group)."""
    if dist is None or not dist.is_initialized():
        return float(x)
    import torch
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(x: float, dist) -> float:
    if dist is None or not dist.is_initialized():
        return float(x)
    import torch
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def shard_for_rank(p, world: int, rank: int):
    """This rank's share of one adapter set split across `world` GPUs (plora_partition: longest
    processing time first over the per-adapter cost); adapters are independent, so no rank needs
    another's data."""
    import packed_lora_fine_b200 as pl
    owner, _ = pl.plora_partition(p.counts, p.ranks, p.d_in, p.d_out, world)
    ids, _, _ = pl.shard(owner, p.off, rank)
    if len(ids) == 0:
        raise SystemExit(f"rank {rank}: no adapter left for this GPU ({p.n_adapters} adapters over {world} GPUs)")
    return wl.take_adapters(p, ids)


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def oracle_sample_problem(seed: int, adapters: int, tokens_each: int):
    """A bounded sample of the workload: the first `adapters` adapters of the 32-adapter mix,
    each cut to `tokens_each` tokens, same layer shapes and distributions."""
    ranks, counts, alphas = wl.config3_shape(seed)
    k = adapters
    return wl.make_problem("cfg3_sample", "bf16", 4096, 14336, ranks[:k], [tokens_each] * k, alphas[:k],
                           wl.init_llm(4096), seed + 7777)


def time_oracle(p, nthreads: int) -> float:
    import oracle
    t0 = time.perf_counter()
    oracle.full(p, nthreads=nthreads)
    return time.perf_counter() - t0


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(seed: int) -> dict:
    import oracle
    oracle.build()
    cores = host_cores()
    nt = min(cores, oracle.num_procs())
    p = oracle_sample_problem(seed, 8, 4)
    time_oracle(oracle_sample_problem(seed, 1, 1), nt)  # load / page in
    dt = time_oracle(p, nt)
    return {"value": p.T / dt, "unit": UNIT, "cores": nt, "kind": "oracle", "cpu_model": cpu_model(),
            "sample": f"fp64 oracle fwd+bwd (Y, dX, dA, dB) of {p.T} tokens: the first 8 adapters of the "
                      f"32-adapter LLaMA-3-8B up_proj mix cut to 4 tokens each; {dt:.2f} s"}


# ----------------------------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    cores = host_cores()
    nt = min(cores, oracle.num_procs())
    # Size the per-step sample so the whole run stays within a few minutes.
    probe = oracle_sample_problem(args.seed, 2, 2)
    time_oracle(probe, nt)
    t_tok = time_oracle(probe, nt) / probe.T
    budget = 150.0 / max(1, args.steps + args.warmup)
    tokens_each = int(max(1, min(8, budget / t_tok / 8)))
    p = oracle_sample_problem(args.seed, 8, tokens_each)
    for _ in range(args.warmup):
        time_oracle(p, nt)
    total = 0.0
    for _ in range(args.steps):
        total += time_oracle(p, nt)
    ms = 1000.0 * total / args.steps
    value = p.T / (ms / 1000.0)
    sample = (f"fp64 oracle fwd+bwd of {p.T} tokens per step (first 8 adapters of the 32-adapter mix, "
              f"{tokens_each} tokens each) on {nt} host threads")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "strong" if (args.gpus > 1 and args.scaling == "strong") else "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD, "adapters": 8, "tokens_per_step": p.T, "d_in": 4096,
                       "d_out": 14336},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": nt, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- our arm
def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.layer_only:
        return layer_shared_inputs(args)
    if args.suite:
        return run_suite(args)
    if args.base_gemm_reference:
        return run_base_gemm_reference(args)

    import torch
    import torch.distributed as dist
    import packed_lora_fine_b200 as pl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    else:
        dist = None
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks, peaks_src = load_peaks()

    if args.workload == "small":
        ranks, counts, alphas = wl.config3_shape(args.seed)
        p = wl.make_problem("cfg3_small", "bf16", 4096, 14336, ranks[:8], [2048] * 8, alphas[:8],
                            wl.init_llm(4096), args.seed + 1000 * rank)
    elif args.workload == "layer_q":
        p = wl.config4(seed=1004)[0]
    elif args.workload == "llama_up_r16x1":
        _, counts, _ = wl.config3_shape(args.seed + 1000 * rank)
        p = wl.make_problem("cfg3_r16x1", "bf16", 4096, 14336, np.array([16]), [int(np.sum(counts))], [32.0],
                            wl.init_llm(4096), args.seed + 1000 * rank)
    elif world > 1 and args.scaling == "strong":
        p = shard_for_rank(wl.config3(seed=args.seed), world, rank)
    else:
        p = wl.config3(seed=args.seed + 1000 * rank)
    T = p.T

    def tdev(a):
        return torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).to(dev)

    X, W, dY = tdev(p.X), tdev(p.W), tdev(p.dY)
    A = [tdev(a) for a in p.A]
    B = [tdev(b) for b in p.B]
    Y = torch.empty((T, p.d_out), dtype=torch.bfloat16, device=dev)
    dX = torch.empty((T, p.d_in), dtype=torch.bfloat16, device=dev)
    dA = [torch.empty(a.shape, dtype=torch.float32, device=dev) for a in A]
    dB = [torch.empty(b.shape, dtype=torch.float32, device=dev) for b in B]
    eng = pl.PackedLoRA(p.d_in, p.d_out, "bf16", max_adapters=p.n_adapters, max_rank=int(max(p.ranks)),
                        max_tokens=T, unfused=args.unfused, base_pair=args.base_pair)
    dev_info = pl.plora_device_info(eng.h)
    base_gemm = ("SM-pair 256x256 tiles, %d co-resident pairs of %d SMs" % (dev_info["pairs_fwd"], dev_info["sms"])
                 if args.base_pair else "1-SM %dx256 tiles on %d SMs, %d-row windows" %
                 (dev_info["base_rows"], dev_info["sms"], dev_info["window_rows"]))
    tab_f = eng.table(p.scales, A, B)
    tab_b = eng.table(p.scales, A, B, dA, dB)
    saved = torch.empty(eng.saved_bytes(p.off, tab_f), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    st = stream.cuda_stream
    n = p.n_adapters
    off = np.ascontiguousarray(p.off, dtype=np.int64)

    def step():
        pl.plora_forward(eng.h, X.data_ptr(), W.data_ptr(), Y.data_ptr(), n, off, tab_f, saved.data_ptr(), st)
        pl.plora_backward(eng.h, X.data_ptr(), W.data_ptr(), dY.data_ptr(), dX.data_ptr(), n, off, tab_b,
                          saved.data_ptr(), st)

    def barrier():
        if dist is not None:
            dist.barrier(device_ids=[local])

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    assert pl.plora_check(eng.h, st) == pl.PLORA_OK
    pl.plora_profile_read(eng.h)          # reset the counters
    pl.plora_profile_enable(eng.h, True)

    gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
    if not gpu_uuid.startswith("GPU-"):
        gpu_uuid = "GPU-" + gpu_uuid
    clocks = ClockSampler(gpu_uuid)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    energy = EnergyMeter(gpu_uuid)
    energy.start()
    clocks.start()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    joules, watts = energy.stop()
    barrier()
    ms_local = ev0.elapsed_time(ev1) / args.steps
    prof = pl.plora_profile_read(eng.h)
    pl.plora_profile_enable(eng.h, False)
    assert pl.plora_check(eng.h, st) == pl.PLORA_OK

    # The same steps with L2 flushed before each one (a 256 MB write, twice the L2): each step is
    # timed on its own between events, so the flush stays outside the timed time.
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    k_fl = max(3, min(args.steps, 10))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(k_fl)]
    barrier()
    for a_, b_ in evs:
        flush.fill_(1)
        a_.record(stream)
        step()
        b_.record(stream)
    torch.cuda.synchronize()
    ms_flushed = reduce_max(sum(a_.elapsed_time(b_) for a_, b_ in evs) / k_fl, dist)
    del flush
    assert pl.plora_check(eng.h, st) == pl.PLORA_OK
    ms = reduce_max(ms_local, dist)
    tokens_all = reduce_sum(T, dist)
    # every rank takes part in both sums; a rank without an energy counter turns them into NaN
    j_all = reduce_sum(joules if joules is not None else float("nan"), dist)
    w_all = reduce_sum(watts if watts is not None else float("nan"), dist)
    energy_line = None if math.isnan(j_all) else {
        "joules_per_step": j_all / args.steps, "watts_per_gpu": w_all / world,
        "source": "NVML total-energy counter read around the timed region, summed over ranks"}
    value = tokens_all / (ms / 1000.0)

    # Per-kernel roofline (device time from events bracketing each launch on its stream).
    work = algorithmic_work(p)
    kernels = {}
    launches = 0
    for kind, (cnt, tot) in prof.items():
        launches += cnt
        if cnt == 0:
            continue
        avg_ms = tot / cnt
        if kind not in work:
            # no algorithmic work of its own (the schedule staging copy): latency, not a roofline
            kernels[kind] = {"launches": cnt, "avg_ms": avg_ms, "bound": "latency", "achieved": None,
                             "unit": None, "frac": None}
            continue
        fl, by = work[kind]
        if kind in TC_KINDS:
            ach = fl / (avg_ms / 1e3) / 1e12
            kernels[kind] = {"launches": cnt, "avg_ms": avg_ms, "bound": "tensor", "achieved": ach,
                             "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops_sustained"]}
        else:
            ach = by / (avg_ms / 1e3) / 1e9
            kernels[kind] = {"launches": cnt, "avg_ms": avg_ms, "bound": "hbm", "achieved": ach, "unit": "GB/s",
                             "frac": ach / peaks["hbm_gbs"]}
    # DRAM bytes per launch from the committed ncu captures (the 16384-token case of the LLaMA up_proj
    # mix), scaled by this rank's tokens: X, Y and the passes over W all grow in proportion.  Only for
    # that projection's workloads, and only while the kernel sources still hash to the captures'.
    try:
        with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
            tr = json.load(f)
    except Exception:
        tr = {}
    sha = source_sha()

    def traffic_of(kind):
        e = tr.get(kind)
        if not e or e.get("source_sha") != sha or args.workload not in ("llama_up32", "small"):
            return None
        return int(round(e["captured_bytes"] * T / 16384))
    for kind in kernels:
        kernels[kind]["traffic"] = traffic_of(kind)
    dom = max(kernels, key=lambda k: kernels[k]["avg_ms"] * kernels[k]["launches"])
    kd = kernels[dom]
    traffic = traffic_of(dom)
    peak_key = "bf16_tflops_sustained" if kd["bound"] == "tensor" else "hbm_gbs"
    roofline = {"bound": kd["bound"], "achieved": kd["achieved"], "peak": peaks[peak_key], "unit": kd["unit"],
                "frac": kd["frac"], "traffic": traffic, "kernel": dom,
                "peak_source": f"{peaks_src} {peak_key}"}

    # End to end through the C ABI with host buffers, pipelined like a training loop: every step
    # copies its X and dY in from pinned host memory (copy stream), runs forward + backward (compute
    # stream), and copies every adapter's dA, dB out to pinned host memory (copy-out stream).  Inputs
    # and gradients are double-buffered, so step k+1's inputs stream in while step k computes.
    e2e = None
    if not args.no_e2e:
        hX = torch.empty(X.shape, dtype=X.dtype, pin_memory=True).copy_(X.cpu())
        hdY = torch.empty(dY.shape, dtype=dY.dtype, pin_memory=True).copy_(dY.cpu())
        hdA = [torch.empty(a.shape, dtype=torch.float32, pin_memory=True) for a in dA]
        hdB = [torch.empty(b.shape, dtype=torch.float32, pin_memory=True) for b in dB]
        h2d = hX.numel() * 2 + hdY.numel() * 2
        d2h = sum(a.numel() * 4 for a in hdA) + sum(b.numel() * 4 for b in hdB)
        Xb = [X, torch.empty_like(X)]
        dYb = [dY, torch.empty_like(dY)]
        dAb = [dA, [torch.empty_like(a) for a in dA]]
        dBb = [dB, [torch.empty_like(b) for b in dB]]
        tabs = [tab_b, eng.table(p.scales, A, B, dAb[1], dBb[1])]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()
        in_done = [ev(), ev()]
        used = [ev(), ev()]      # compute of the step that last read / wrote buffer b is done
        out_done = [ev(), ev()]  # copy-out of buffer b's gradients is done
        for e_ in used + out_done:
            e_.record(stream)

        def e2e_step(k):
            b = k % 2
            with torch.cuda.stream(s_in):
                s_in.wait_event(used[b])
                Xb[b].copy_(hX, non_blocking=True)
                dYb[b].copy_(hdY, non_blocking=True)
                in_done[b].record(s_in)
            stream.wait_event(in_done[b])
            stream.wait_event(out_done[b])
            pl.plora_forward(eng.h, Xb[b].data_ptr(), W.data_ptr(), Y.data_ptr(), n, off, tab_f, saved.data_ptr(),
                             st)
            pl.plora_backward(eng.h, Xb[b].data_ptr(), W.data_ptr(), dYb[b].data_ptr(), dX.data_ptr(), n, off,
                              tabs[b], saved.data_ptr(), st)
            used[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(used[b])
                for a, h in zip(dAb[b], hdA):
                    h.copy_(a, non_blocking=True)
                for g_, h in zip(dBb[b], hdB):
                    h.copy_(g_, non_blocking=True)
                out_done[b].record(s_out)

        for k in range(2):
            e2e_step(k)
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        k2 = max(5, min(args.steps, 50))   # the pipeline fill (one uncovered copy) spreads over k2 steps
        e0.record(stream)
        s_in.wait_stream(stream)
        s_out.wait_stream(stream)
        for k in range(k2):
            e2e_step(k)
        stream.wait_stream(s_out)
        stream.wait_stream(s_in)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        ms_e2e = reduce_max(e0.elapsed_time(e1) / k2, dist)
        e2e = {"value": tokens_all / (ms_e2e / 1000.0), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": ms_e2e, "steps": k2,
               "pipeline": "H2D of step k+1 overlaps compute of step k (double-buffered inputs and gradients)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.seed)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": max(3, args.warmup), "ms_per_step": ms, "higher_is_better": True,
                "scaling": "strong" if (world > 1 and args.scaling == "strong" and args.workload == "llama_up32") else "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": WORKLOADS[args.workload], "adapters": n, "tokens_per_gpu": T,
                           "global_tokens": int(tokens_all),
                           "d_in": p.d_in, "d_out": p.d_out,
                           "parallelism": (f"one adapter set split over {world} GPUs (LPT, plora_partition)"
                                           if world > 1 and args.scaling == "strong" else f"adapter-sharded x{world}"),
                           "l2": "inputs larger than L2 (X %.0f MB, dY %.0f MB); no flush" % (
                               X.numel() * 2 / 1e6, dY.numel() * 2 / 1e6),
                           "base_gemm": base_gemm},
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": int(launches),
                "clocks": {"sm_mhz": clk["sm_mhz"], "sm_max_mhz": clk["sm_max_mhz"], "reasons": clk["reasons"],
                           "samples": clk["samples"], "source": clk.get("source")},
                "energy": energy_line,
                "l2_flushed": {"value": tokens_all / (ms_flushed / 1000.0), "unit": UNIT, "ms_per_step": ms_flushed,
                               "steps": k_fl, "how": "256 MB written before each step, outside its timed region; the inputs "
                               "exceed L2 anyway, and the pause for the write lets the power-capped clock recover, so "
                               "this figure can run above the back-to-back one"},
                "kernels": kernels}
        print(json.dumps(line), flush=True)
    eng.close()
    if dist is not None:
        dist.destroy_process_group()
    return 0


def run_base_gemm_reference(args):
    """The benchmark workload's two frozen-base GEMMs, Y = X W^T and dX = dY W, through torch.matmul
    (cuBLAS), timed like a step of our arm: warm-up, CUDA events around `steps` back-to-back pairs,
    clocks and energy sampled during the timed region.  It measures what the library GEMMs reach on
    the same shapes under the same power limit; it runs no low-rank work."""
    import torch
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    _, counts, _ = wl.config3_shape(args.seed)
    T, di, do = int(np.sum(counts)), 4096, 14336
    g = torch.Generator(device=dev)
    g.manual_seed(args.seed)
    X = torch.randn((T, di), generator=g, device=dev).to(torch.bfloat16)
    dY = torch.randn((T, do), generator=g, device=dev).to(torch.bfloat16)
    W = (torch.randn((do, di), generator=g, device=dev) * 0.02).to(torch.bfloat16)
    Y = torch.empty((T, do), dtype=torch.bfloat16, device=dev)
    dX = torch.empty((T, di), dtype=torch.bfloat16, device=dev)

    def step():
        torch.matmul(X, W.t(), out=Y)
        torch.matmul(dY, W, out=dX)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    clocks, energy = ClockSampler(uuid), EnergyMeter(uuid)
    energy.start()
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    joules, watts = energy.stop()
    ms = e0.elapsed_time(e1) / args.steps
    flops = 2 * 2.0 * T * di * do
    print(json.dumps({"impl": "cublas-base-gemms", "what": "torch.matmul Y = X W^T and dX = dY W only (no low-rank work)",
                      "config": {"workload": WORKLOAD, "tokens": T, "d_in": di, "d_out": do},
                      "steps": args.steps, "ms_per_step": ms, "tflops": flops / (ms / 1e3) / 1e12,
                      "energy": None if joules is None else {"joules_per_step": joules / args.steps, "watts": watts},
                      "clocks": {"sm_mhz": clk["sm_mhz"], "sm_max_mhz": clk["sm_max_mhz"], "reasons": clk["reasons"]}}),
          flush=True)
    return 0


def source_sha() -> str:
    """Hash of the kernel sources' code (comments and blank lines left out), to tell whether committed
    ncu counters still describe them."""
    import hashlib
    import re
    h = hashlib.sha256()
    d = os.path.join(ROOT, "packed_lora_fine_b200", "csrc")
    for f in sorted(os.listdir(d)):
        with open(os.path.join(d, f), encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        code = "\n".join(line.rstrip() for line in text.splitlines() if line.strip())
        h.update(f.encode())
        h.update(code.encode())
    return h.hexdigest()[:16]



# ----------------------------------------------------------------------------- measurement suite
def _suite_problem_shapes():
    """(name, [(d_in, d_out), ...], ranks, counts, alphas) of every suite workload."""
    out = []
    r2 = [8, 8, 16, 16, 32, 32, 64, 64]
    out.append(("qwen2.5-7b q_proj 3584x3584, 8 adapters", [(3584, 3584)], r2, [2048] * 8, [2.0 * x for x in r2]))
    r3, c3, a3 = wl.config3_shape(1003)
    out.append(("llama3-8b up_proj 4096x14336, 32 adapters (long tail)", [(4096, 14336)], list(r3), list(c3),
                list(a3)))
    r4 = list(wl.rng_for(1004, 1).choice(np.array([16, 32, 64]), size=16))
    out.append(("llama3-8b layer: 7 projections, 16 adapters x 8192 tokens",
                [(di, do) for _, di, do in wl.LLAMA3_LAYER], r4, [8192] * 16, [2.0 * x for x in r4]))
    for k in (1, 2, 4, 8, 16, 32):
        out.append((f"scaling 4096x4096 r16, {k} adapters x 2048 tokens", [(4096, 4096)], [16] * k, [2048] * k,
                    [32.0] * k))
    for which in ("i", "ii", "iii", "iv"):
        p = wl.config5_mix(which)
        out.append((f"degenerate mix {which} 4096x4096", [(4096, 4096)], [int(x) for x in p.ranks],
                    [int(x) for x in p.counts], [float(x) for x in p.alphas]))
    return out


def run_suite(args):
    """Packed fwd+bwd tokens/s and per-kernel roofline on every workload, next to the same kernels run
    once per adapter (the naive sequential loop).  One JSON line per workload."""
    import torch
    import packed_lora_fine_b200 as pl
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    peaks, _ = load_peaks()
    g = torch.Generator(device=dev)
    g.manual_seed(args.seed)
    st = torch.cuda.current_stream(dev)
    for name, projs, ranks, counts, alphas in _suite_problem_shapes():
        n = len(ranks)
        off = np.zeros(n + 1, np.int64)
        off[1:] = np.cumsum(counts)
        T = int(off[-1])
        scales = [a / r for a, r in zip(alphas, ranks)]
        layers = []
        for di, do in projs:
            X = (torch.randn((T, di), generator=g, device=dev)).to(torch.bfloat16)
            dY = (torch.randn((T, do), generator=g, device=dev)).to(torch.bfloat16)
            W = (torch.randn((do, di), generator=g, device=dev) * 0.02).to(torch.bfloat16)
            bound = math.sqrt(6.0 / di)
            A = [((torch.rand((r, di), generator=g, device=dev) * 2 - 1) * bound).to(torch.bfloat16) for r in ranks]
            B = [(torch.randn((do, r), generator=g, device=dev) * 0.01).to(torch.bfloat16) for r in ranks]
            eng = pl.PackedLoRA(di, do, "bf16", max_adapters=n, max_rank=max(ranks), max_tokens=max(T, 1))
            Y = torch.empty((T, do), dtype=torch.bfloat16, device=dev)
            dX = torch.empty((T, di), dtype=torch.bfloat16, device=dev)
            dA = [torch.empty(a.shape, dtype=torch.float32, device=dev) for a in A]
            dB = [torch.empty(b.shape, dtype=torch.float32, device=dev) for b in B]
            tf = eng.table(scales, A, B)
            tb = eng.table(scales, A, B, dA, dB)
            saved = torch.empty(max(256, eng.saved_bytes(off, tf)), dtype=torch.uint8, device=dev)
            # the sequential loop: one handle call per adapter on its own slice
            seq = []
            for i in range(n):
                a, b = int(off[i]), int(off[i + 1])
                o1 = np.array([0, b - a], np.int64)
                t1f = eng.table([scales[i]], [A[i]], [B[i]])
                t1b = eng.table([scales[i]], [A[i]], [B[i]], [dA[i]], [dB[i]])
                sv = torch.empty(max(256, eng.saved_bytes(o1, t1f)), dtype=torch.uint8, device=dev)
                seq.append((a, b, o1, t1f, t1b, sv))
            layers.append(dict(X=X, dY=dY, W=W, A=A, B=B, eng=eng, Y=Y, dX=dX, tf=tf, tb=tb, saved=saved, seq=seq,
                               di=di, do=do))

        def packed_step():
            for L in layers:
                e = L["eng"]
                pl.plora_forward(e.h, L["X"].data_ptr(), L["W"].data_ptr(), L["Y"].data_ptr(), n, off, L["tf"],
                                 L["saved"].data_ptr(), st.cuda_stream)
                pl.plora_backward(e.h, L["X"].data_ptr(), L["W"].data_ptr(), L["dY"].data_ptr(),
                                  L["dX"].data_ptr(), n, off, L["tb"], L["saved"].data_ptr(), st.cuda_stream)

        def seq_step():
            for L in layers:
                e = L["eng"]
                esz = 2
                for (a, b, o1, t1f, t1b, sv) in L["seq"]:
                    xp = L["X"].data_ptr() + a * L["di"] * esz
                    yp = L["Y"].data_ptr() + a * L["do"] * esz
                    dyp = L["dY"].data_ptr() + a * L["do"] * esz
                    dxp = L["dX"].data_ptr() + a * L["di"] * esz
                    pl.plora_forward(e.h, xp, L["W"].data_ptr(), yp, 1, o1, t1f, sv.data_ptr(), st.cuda_stream)
                    pl.plora_backward(e.h, xp, L["W"].data_ptr(), dyp, dxp, 1, o1, t1b, sv.data_ptr(),
                                      st.cuda_stream)

        def timed(fn, steps, profile=False):
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            for L in layers:
                pl.plora_profile_read(L["eng"].h)
                pl.plora_profile_enable(L["eng"].h, profile)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(st)
            for _ in range(steps):
                fn()
            e1.record(st)
            torch.cuda.synchronize()
            prof = {}
            for L in layers:
                for k, (c, ms) in pl.plora_profile_read(L["eng"].h).items():
                    pc, pm = prof.get(k, (0, 0.0))
                    prof[k] = (pc + c, pm + ms)
                pl.plora_profile_enable(L["eng"].h, False)
            return e0.elapsed_time(e1) / steps, prof

        steps = max(5, min(args.steps, 30))
        # both loops timed without the per-launch profiling events (they cost microseconds per
        # launch, which shows on the small workloads); the kernel breakdown comes from its own pass
        ms_p, _ = timed(packed_step, steps)
        ms_s, _ = timed(seq_step, max(3, steps // 3))
        _, prof = timed(packed_step, steps, profile=True)
        kern = {}
        for k, (c, tot) in prof.items():
            if c:
                kern[k] = {"launches": c, "ms_per_step": tot / steps}
        base_ms = sum(v["ms_per_step"] for k, v in kern.items() if k in TC_KINDS)
        base_flops = sum(4.0 * T * L["di"] * L["do"] for L in layers)
        adamw = None
        if len(layers) == 1:
            # the optimizer step of the same adapters: fp32 masters and moments, grads from the step above
            L = layers[0]
            f32 = lambda t_: torch.zeros(t_.shape, dtype=torch.float32, device=dev)
            Am = [a.float() for a in L["A"]]
            Bm = [b.float() for b in L["B"]]
            mA, vA = [f32(a) for a in L["A"]], [f32(a) for a in L["A"]]
            mB, vB = [f32(b) for b in L["B"]], [f32(b) for b in L["B"]]
            hps = [dict(lr=1e-4, step=1) for _ in range(n)]
            sts = pl.make_adamw_states(hps, [x.data_ptr() for x in Am], [x.data_ptr() for x in Bm],
                                       [x.data_ptr() for x in mA], [x.data_ptr() for x in vA],
                                       [x.data_ptr() for x in mB], [x.data_ptr() for x in vB])
            e = L["eng"]
            for _ in range(3):
                pl.plora_adamw_step(e.h, n, L["tb"], sts, st.cuda_stream)
            torch.cuda.synchronize()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(st)
            for _ in range(20):
                pl.plora_adamw_step(e.h, n, L["tb"], sts, st.cuda_stream)
            a1.record(st)
            torch.cuda.synchronize()
            ms_a = a0.elapsed_time(a1) / 20
            elems = sum(int(r) * (L["di"] + L["do"]) for r in ranks)
            adamw = {"ms": ms_a, "elements": elems, "hbm_frac": elems * 30 / (ms_a / 1e3) / 1e9 / peaks["hbm_gbs"]}
        line = {"suite": name, "tokens": T, "adapters": n, "projections": len(layers), "adamw_step": adamw,
                "packed_ms_per_step": ms_p, "packed_tokens_per_s": T / (ms_p / 1e3),
                "sequential_ms_per_step": ms_s, "sequential_tokens_per_s": T / (ms_s / 1e3),
                "packed_over_sequential": ms_s / ms_p,
                "base_gemm_tflops": base_flops / (base_ms / 1e3) / 1e12 if base_ms else None,
                "base_gemm_frac_of_sustained_peak": (base_flops / (base_ms / 1e3) / 1e12) / peaks["bf16_tflops_sustained"]
                if base_ms else None,
                "kernels_ms_per_step": {k: round(v["ms_per_step"], 4) for k, v in kern.items()}}
        print(json.dumps(line), flush=True)
        for L in layers:
            L["eng"].close()
        del layers
        torch.cuda.empty_cache()
    layer_shared_inputs(args)
    return 0


def layer_shared_inputs(args):
    """One LLaMA-3-8B layer whose LoRA targets read their inputs as in the model: q, k and v share
    one input, gate and up another, o and down have their own.  Timed as seven single-projection
    calls, as four calls with q|k|v and gate|up stacked as output blocks (one base GEMM each), and as
    one layer call over those four (plora_layer_*: one launch set, one persistent launch per product
    kind).  The projections are independent here (no attention or activation between them).
    16 adapters x 8192 tokens (--layer-tokens), r ~ U{16,32,64}, alpha = 2r.  One JSON line."""
    import torch
    import packed_lora_fine_b200 as pl
    dev = torch.device("cuda", 0)
    st = torch.cuda.current_stream(dev)
    g = torch.Generator(device=dev)
    g.manual_seed(args.seed + 7)
    ranks = [int(x) for x in wl.rng_for(1004, 1).choice(np.array([16, 32, 64]), size=16)]
    n = len(ranks)
    off = np.arange(n + 1, dtype=np.int64) * args.layer_tokens
    T = int(off[-1])
    scales = [2.0] * n
    shape = {nm: (di, do) for nm, di, do in wl.LLAMA3_LAYER}
    groups = [("q", "k", "v"), ("o",), ("gate", "up"), ("down",)]
    proj = {}
    for grp in groups:
        X = torch.randn((T, shape[grp[0]][0]), generator=g, device=dev).to(torch.bfloat16)
        for nm in grp:
            di, do = shape[nm]
            bound = math.sqrt(6.0 / di)
            proj[nm] = dict(X=X, dY=torch.randn((T, do), generator=g, device=dev).to(torch.bfloat16),
                            W=(torch.randn((do, di), generator=g, device=dev) * 0.02).to(torch.bfloat16),
                            A=[((torch.rand((r, di), generator=g, device=dev) * 2 - 1) * bound).to(torch.bfloat16)
                               for r in ranks],
                            B=[(torch.randn((do, r), generator=g, device=dev) * 0.01).to(torch.bfloat16)
                               for r in ranks])

    def call(nms):
        """A handle and its buffers for the projections `nms` (stacked as output blocks if several)."""
        di = shape[nms[0]][0]
        widths = [shape[nm][1] for nm in nms]
        cat = lambda ts, dim=0: ts[0] if len(ts) == 1 else torch.cat(ts, dim=dim).contiguous()
        W = cat([proj[nm]["W"] for nm in nms])
        dY = cat([proj[nm]["dY"] for nm in nms], 1)
        A = [cat([proj[nm]["A"][i] for nm in nms]) for i in range(n)]
        B = [cat([proj[nm]["B"][i] for nm in nms]) for i in range(n)]
        eng = pl.PackedLoRA(di, sum(widths), "bf16", max_adapters=n, max_rank=max(ranks), max_tokens=T,
                            out_blocks=widths if len(nms) > 1 else None)
        dA = [torch.empty(a.shape, dtype=torch.float32, device=dev) for a in A]
        dB = [torch.empty(b.shape, dtype=torch.float32, device=dev) for b in B]
        tf, tb = eng.table(scales, A, B), eng.table(scales, A, B, dA, dB)
        return dict(eng=eng, X=proj[nms[0]]["X"], W=W, dY=dY, A=A, B=B, dA=dA, dB=dB, tf=tf, tb=tb,
                    Y=torch.empty((T, sum(widths)), dtype=torch.bfloat16, device=dev),
                    dX=torch.empty((T, di), dtype=torch.bfloat16, device=dev),
                    saved=torch.empty(max(256, eng.saved_bytes(off, tf)), dtype=torch.uint8, device=dev))

    def step(calls):
        for c in calls:
            e = c["eng"]
            pl.plora_forward(e.h, c["X"].data_ptr(), c["W"].data_ptr(), c["Y"].data_ptr(), n, off, c["tf"],
                             c["saved"].data_ptr(), st.cuda_stream)
            pl.plora_backward(e.h, c["X"].data_ptr(), c["W"].data_ptr(), c["dY"].data_ptr(), c["dX"].data_ptr(),
                              n, off, c["tb"], c["saved"].data_ptr(), st.cuda_stream)

    gpu_uuid = str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
    if not gpu_uuid.startswith("GPU-"):
        gpu_uuid = "GPU-" + gpu_uuid
    power = {"fused_calls": [], "layer_call": []}

    def metered(key, run, steps):
        # energy per step and median SM clock over the timed steps of run (after its warm-up)
        energy, clocks = EnergyMeter(gpu_uuid), ClockSampler(gpu_uuid)
        energy.start()
        clocks.start()
        out = run()
        clk = clocks.stop()
        joules, _ = energy.stop()
        power[key].append({"j_per_step": None if joules is None else round(joules / steps, 2),
                           "sm_mhz": clk["sm_mhz"]})
        return out

    def timed(calls, steps, meter=None):
        for _ in range(3):
            step(calls)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def run():
            e0.record(st)
            for _ in range(steps):
                step(calls)
            e1.record(st)
            torch.cuda.synchronize()
        metered(meter, run, steps) if meter else run()
        for c in calls:
            assert pl.plora_check(c["eng"].h, 0) == pl.PLORA_OK
        return e0.elapsed_time(e1) / steps

    steps = max(5, min(args.steps, 20))
    sep = [call((nm,)) for grp in groups for nm in grp]
    ms_sep = timed(sep, steps)
    q_sep = sep[0]["Y"].clone()
    for c in sep:
        c["eng"].close()
    del sep
    torch.cuda.empty_cache()
    fused = [call(grp) for grp in groups]
    ms_fused = timed(fused, steps)
    same_q = bool(torch.equal(fused[0]["Y"][:, :shape["q"][1]], q_sep))
    y_fused = [c["Y"].clone() for c in fused]
    for c in fused:
        c["eng"].close()
    # The same four calls as ONE launch set (plora_layer_*): one persistent launch per product kind over
    # all four projections, on the same buffers.
    layer = pl.PackedLoRALayer([(c["X"].shape[1], c["Y"].shape[1]) + ((list(map(lambda nm: shape[nm][1], grp)),)
                                if len(grp) > 1 else ()) for c, grp in zip(fused, groups)],
                               max_adapters=n, max_rank=max(ranks), max_tokens=T)
    offc = np.ascontiguousarray(off, dtype=np.int64)
    keep = []

    def projs(backward):
        items = []
        for c in fused:
            keep.append(c["tb"] if backward else c["tf"])
            items.append({"X": c["X"].data_ptr(), "W": c["W"].data_ptr(), "Y": c["Y"].data_ptr(),
                          "dY": c["dY"].data_ptr(), "dX": c["dX"].data_ptr(), "tab": keep[-1],
                          "saved": c["saved"].data_ptr()})
        return pl.make_projs(items)
    pf, pb = projs(False), projs(True)
    lib = pl.load()

    def layer_step(_):
        assert lib.plora_layer_forward(layer.L, n, offc.ctypes.data, pf, st.cuda_stream) == pl.PLORA_OK
        assert lib.plora_layer_backward(layer.L, n, offc.ctypes.data, pb, st.cuda_stream) == pl.PLORA_OK

    def timed_layer(steps, profile=False, meter=None):
        for _ in range(3):
            layer_step(None)
        torch.cuda.synchronize()
        pl.plora_profile_read(layer.handle(0))
        pl.plora_profile_enable(layer.handle(0), profile)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def run():
            e0.record(st)
            for _ in range(steps):
                layer_step(None)
            e1.record(st)
            torch.cuda.synchronize()
        metered(meter, run, steps) if meter else run()
        assert layer.check() == pl.PLORA_OK
        prof = pl.plora_profile_read(layer.handle(0))
        pl.plora_profile_enable(layer.handle(0), False)
        return e0.elapsed_time(e1) / steps, prof

    # the four calls again on the same buffers, alternated with the layer call (the power-capped clock
    # drifts over a run), and one profiled pass of each for the per-kernel split
    refused = []
    for c, grp in zip(fused, groups):
        c["eng"] = pl.PackedLoRA(c["X"].shape[1], c["Y"].shape[1], "bf16", max_adapters=n, max_rank=max(ranks),
                                 max_tokens=T, out_blocks=[shape[nm][1] for nm in grp] if len(grp) > 1 else None)
        refused.append(c["eng"])
    ms_layer_runs, ms_fused_runs = [], []
    for _ in range(2):
        ms_fused_runs.append(timed(fused, steps, meter="fused_calls"))
        ms_layer_runs.append(timed_layer(steps, meter="layer_call")[0])
    ms_layer, ms_fused = min(ms_layer_runs), min(ms_fused_runs)

    def kernel_split(prof, steps_):
        return {k: round(v[1] / steps_, 4) for k, v in prof.items() if v[0]}
    _, prof_layer = timed_layer(steps, profile=True)
    launches_layer = sum(v[0] for v in prof_layer.values()) / steps
    for _ in range(3):
        step(fused)
    torch.cuda.synchronize()
    for c in fused:
        pl.plora_profile_read(c["eng"].h)
        pl.plora_profile_enable(c["eng"].h, True)
    for _ in range(steps):
        step(fused)
    torch.cuda.synchronize()
    prof_fused = {}
    for c in fused:
        for k, (cnt, tot) in pl.plora_profile_read(c["eng"].h).items():
            a, b = prof_fused.get(k, (0, 0.0))
            prof_fused[k] = (a + cnt, b + tot)
        pl.plora_profile_enable(c["eng"].h, False)
    same_layer = all(bool(torch.equal(c["Y"], y)) for c, y in zip(fused, y_fused))
    for e in refused:
        e.close()
    layer.close()
    print(json.dumps({"suite": "llama3-8b layer, shared inputs: q|k|v and gate|up as output blocks",
                      "tokens": T, "adapters": n, "projections": 7,
                      "separate_calls": 7, "separate_ms_per_step": ms_sep, "separate_tokens_per_s": T / (ms_sep / 1e3),
                      "fused_calls": len(groups), "fused_ms_per_step": ms_fused,
                      "fused_tokens_per_s": T / (ms_fused / 1e3), "fused_over_separate": ms_sep / ms_fused,
                      "q_output_bit_identical": same_q,
                      "layer_call_ms_per_step": ms_layer, "layer_call_tokens_per_s": T / (ms_layer / 1e3),
                      "layer_call_launches_per_step": launches_layer,
                      "layer_call_over_fused_calls": ms_fused / ms_layer,
                      "alternated_ms": {"fused_calls": ms_fused_runs, "layer_call": ms_layer_runs},
                      "alternated_power": power,
                      "kernels_ms_per_step": {"fused_calls": kernel_split(prof_fused, steps),
                                              "layer_call": kernel_split(prof_layer, steps)},
                      "layer_call_outputs_bit_identical": same_layer}), flush=True)
    torch.cuda.empty_cache()


if __name__ == "__main__":
    sys.exit(main())
