"""Benchmark: dense varlen causal MLA prefill throughput on B200.

One step = one ``mla_prefill_fwd`` call (tile planning, Q/K/V TMA loads,
S = QK^T, masking, online softmax, O += PV, epilogue with LSE) over the
"dense varlen" workload: 8 sequences with lengths uniform in [512, 4096]
(seed 2), 128 heads, qk 192 / v 128, bf16 N(0,1) inputs, scale 1/sqrt(192),
causal, fp32 LSE.  Throughput counts causal-adjusted algorithmic FLOPs:
2 * (192 + 128) * heads * (visible query-key pairs).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Multi-GPU (torchrun): every rank runs its own independent batch of the
same workload (weak scaling, no collective on the data path); the value is
the sum of all ranks' FLOPs over the slowest rank's time.

Timing: CUDA events on the launching stream; inputs (Q+K+V = 2.4 GB) are
larger than the 126 MB L2, so nothing is flushed between steps.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MLA prefill attn TFLOPS (causal-adj) and % of B200 dense BF16 peak, 1 GPU"
UNIT = "TFLOP/s"
WORKLOAD = ("dense varlen causal MLA prefill: 8 sequences, lengths U[512,4096] (seed 2), "
            "128 heads, qk 192 (128 nope + 64 rope) / v 128, bf16 N(0,1), scale 1/sqrt(192), "
            "fp32 LSE")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SPEC_BF16_TFLOPS = 2250.0
KERNEL_SRCS = [os.path.join(ROOT, "mla_prefill_attention_causal_b200", "csrc", f)
               for f in ("dense_fwd.cuh", "ptx.cuh")]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dense_fwd_varlen16k.md")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_sha() -> str:
    """Hash of the dense kernel's sources (the traffic figure is only valid
    for the source it was measured on)."""
    h = hashlib.sha256()
    for path in KERNEL_SRCS:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source (otherwise None)."""
    try:
        text = open(TRAFFIC_FILE).read()
    except OSError:
        return None
    vals = {}
    for line in text.splitlines():
        if ":" in line and line.strip().startswith("- "):
            k, v = line.strip()[2:].split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_sha256_16") != kernel_sha():
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                                 hw=parts[5], hwt=parts[6], swt=parts[7], swpc=parts[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [r for r in rows if r["power"] > 250.0] or rows
        reasons = set()
        for r in loaded:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("swpc", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded),
                "sm_max_mhz": max(r["smax"] for r in rows),
                "power_w_max": max(r["power"] for r in rows),
                "samples": len(rows), "samples_under_load": len(loaded),
                "reasons": sorted(reasons)}


def make_workload(seed: int, heads: int = 128):
    import mla_synth as syn
    return syn.varlen16k_config(seed=seed, num_heads=heads)


def oracle_sample(case, heads=(0, 1)):
    """Time the fp64 oracle on the given heads of the workload (all rows)."""
    import oracle
    h = list(heads)
    t0 = time.perf_counter()
    oracle.dense_prefill(case["q"][:, h], case["k"][:, h], case["v"][:, h], case["cu_q"],
                         case["cu_k"], case["scale"], True)
    dt = time.perf_counter() - t0
    flops = oracle.dense_flops(case["lens_q"], case["lens_k"], len(h), True)
    return flops, dt


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max(int(i.get("num_threads", 1)) for i in threadpool_info()) or 1
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def reference_step(case, i: int):
    """One bounded oracle step: every query row of sequence (i mod B) for
    head (i mod H), through the fp64 oracle as it stands."""
    import oracle
    B, H = len(case["lens_q"]), case["num_heads"]
    b, h = i % B, i % H
    q0, q1 = int(case["cu_q"][b]), int(case["cu_q"][b + 1])
    k0, k1 = int(case["cu_k"][b]), int(case["cu_k"][b + 1])
    t0 = time.perf_counter()
    oracle.dense_prefill(case["q"][q0:q1, h:h + 1], case["k"][k0:k1, h:h + 1],
                         case["v"][k0:k1, h:h + 1], [0, q1 - q0], [0, k1 - k0], case["scale"], True)
    dt = time.perf_counter() - t0
    return oracle.dense_flops([q1 - q0], [k1 - k0], 1, True), dt


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return 0
    import oracle
    case = make_workload(2)
    total_flops = oracle.dense_flops(case["lens_q"], case["lens_k"], case["num_heads"], True)
    for i in range(args.warmup):
        reference_step(case, i)
    flops, secs = 0, 0.0
    for i in range(args.steps):
        f, dt = reference_step(case, i)
        flops += f
        secs += dt
    value = flops / secs / 1e12
    sample = (f"step i = all query rows of sequence (i mod 8) for head (i mod 128); "
              f"{args.steps} steps = {flops:.3e} of the workload's {total_flops:.3e} FLOPs")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": {"workload": WORKLOAD, "sample": sample},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_gpu(args, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    import mla_prefill_attention_causal_b200 as mla
    import oracle

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    case = make_workload(2 if world == 1 else 2 + 1000 * rank, heads=args.heads)
    H = case["num_heads"]
    flops = oracle.dense_flops(case["lens_q"], case["lens_k"], H, True)
    to_t = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.bfloat16)
    hq, hk, hv = to_t(case["q"]).pin_memory(), to_t(case["k"]).pin_memory(), to_t(case["v"]).pin_memory()
    hcu = torch.from_numpy(case["cu_q"]).pin_memory()
    q, k, v = hq.to(dev), hk.to(dev), hv.to(dev)
    cu = hcu.to(dev)
    T = q.shape[0]
    out = torch.empty((T, H, 128), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((H, T), dtype=torch.float32, device=dev)
    max_q = case["max_q"]
    stream = torch.cuda.current_stream()

    def step():
        mla.mla_prefill_fwd(q, k, v, cu, cu, max_q, max_q, case["scale"], causal=True,
                            out=out, lse=lse)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    sampler = ClockSampler(local_rank) if (rank == 0 and not args.kernel_only) else None
    if sampler:
        sampler.start()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    ms_total = ev0.elapsed_time(ev1)
    t = torch.tensor([ms_total], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_step = float(t.item()) / args.steps
    value = flops * world / (ms_step * 1e-3) / 1e12
    status = mla.mla_device_status(reset=True)
    if args.kernel_only:
        if rank == 0:
            print(json.dumps({"kernel_only": True, "heads": H, "ms_per_step": ms_step,
                              "tflops": flops / (ms_step * 1e-3) / 1e12, "device_status": status}),
                  flush=True)
        return 0

    # End to end through the public call with host buffers: H2D of the step's
    # inputs from pinned memory, the kernel, D2H of out and lse.
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    hlse = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    e2e_steps = max(3, min(args.steps, 20))

    def e2e_step():
        q.copy_(hq, non_blocking=True)
        k.copy_(hk, non_blocking=True)
        v.copy_(hv, non_blocking=True)
        cu.copy_(hcu, non_blocking=True)
        step()
        hout.copy_(out, non_blocking=True)
        hlse.copy_(lse, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ev0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    ev1.record(stream)
    torch.cuda.synchronize()
    te = torch.tensor([ev0.elapsed_time(ev1) / e2e_steps], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(te, op=dist.ReduceOp.MAX)
    e2e_ms = float(te.item())
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hcu))
    d2h = hout.numel() * hout.element_size() + hlse.numel() * hlse.element_size()

    if rank != 0:
        return 0
    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    achieved = flops / (ms_step * 1e-3) / 1e12  # one kernel launch per step
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16, lengths U[512,4096])",
        "config": {"workload": WORKLOAD, "batch": len(case["lens_q"]), "total_tokens": T,
                   "heads": H, "seq_lens": case["lens_q"], "flops_per_step": flops,
                   "l2": "inputs larger than L2 (Q+K+V %.2f GB > 126 MB); no flush" %
                         ((q.numel() + k.numel() + v.numel()) * 2 / 1e9),
                   "parallelism": f"replicas x{world} (independent batches)"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                     "frac": achieved / peak, "peak_source": f"{peak_src} bf16_tflops (burst)",
                     "frac_of_spec_2250": achieved / SPEC_BF16_TFLOPS,
                     "frac_of_sustained": achieved / float(peaks.get("bf16_tflops_sustained",
                                                                     peak)),
                     "traffic": recorded_traffic(),
                     "kernel": "mla::dense::dense_fwd_kernel"},
        "e2e": {"value": flops * world / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps,
        "clocks": clocks,
        "device_status": status,
    }
    if world == 1 and not args.no_cpu_baseline:
        f, dt = oracle_sample(case, heads=tuple(range(6)))
        line["cpu_baseline"] = {
            "value": f / dt / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"heads 0-5 of 128, all {T} query rows of the same batch "
                      f"({f:.3e} FLOPs in {dt:.1f} s)"}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel-only", action="store_true",
                    help="time the kernel only (no e2e, clocks or CPU baseline); for profiling")
    ap.add_argument("--heads", type=int, default=128,
                    help="heads of the workload (128 for the bench line; fewer for profiling)")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if world > 1:
        import datetime

        import torch.distributed as dist
        import torch
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        return run_gpu(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
