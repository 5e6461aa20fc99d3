"""Benchmark: dense varlen causal MLA prefill throughput on B200.

One step = one ``mla_prefill_fwd`` call (tile planning, Q/K/V TMA loads,
S = QK^T, masking, online softmax, O += PV, epilogue with LSE) over the
"dense varlen" workload: 8 sequences with lengths uniform in [512, 4096]
(seed 2), 128 heads, qk 192 / v 128, bf16 N(0,1) inputs, scale 1/sqrt(192),
causal, fp32 LSE.  Throughput counts causal-adjusted algorithmic FLOPs:
2 * (192 + 128) * heads * (visible query-key pairs).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                  [--workload dense|long32k|chunked|chunked-context|splitkv|sparse|
                              sparse-padded]

``--workload long32k`` times one 32768-token causal sequence (128 heads);
``--workload chunked`` times the chunked prefill with context (a non-causal
prefix pass, a causal self pass and ``mla_attn_merge``; the merge is also
event-timed on its own against the HBM roofline), ``--workload
chunked-context`` the same in one ``mla_prefill_fwd_context`` call;
``--workload splitkv`` a few-tile shape (16 heads, 129 queries over 8192
keys) through ``mla_prefill_fwd_splitkv``; ``--workload sparse``
times the absorbed top-k path instead: one ``mla_sparse_prefill_fwd`` call
over 4096 tokens x 128 heads (q dim 576), a 32768-row latent cache and
top-k 2048 (``sparse-padded``: the same with the tokens at the start of the
cache, so early lists carry -1 padding); FLOPs count 2 * (576 + 512) *
heads per valid slot.

Multi-GPU (torchrun): every rank runs its own independent batch of the
same workload (weak scaling, no collective on the data path); the value is
the sum of all ranks' FLOPs over the slowest rank's time.

``--gpus N`` without torchrun starts N ranks itself (torch.distributed.run on
127.0.0.1); under torchrun, ``--gpus`` must equal WORLD_SIZE.

Timing: CUDA events on the launching stream; the inputs (Q+K+V = 2.08 GB for
the dense workload) are larger than the 126 MB L2, so nothing is flushed
between steps; the splitkv workload's inputs fit in L2, so a 256 MB buffer is
read before each of its calls and each call is timed alone.  The roofline fraction is given against the measured burst
bf16 peak and, as ``frac_of_sustained``, against the measured sustained one;
the default 30 timed calls match the burst measurement, while a few hundred
back-to-back calls run under the power cap and land near the sustained
figure.
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
L2_FLUSH_BYTES = 256 << 20  # read between timed calls of workloads smaller than the 126 MB L2


class L2Flush:
    """Evicts L2 by reading a buffer twice its size.  The buffer is written
    once, here; each flush only reads it, so the lines it leaves in L2 are
    clean and the kernel timed next pays no write-back for them."""

    def __init__(self, dev):
        import torch
        self.buf = torch.ones(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self()
        torch.cuda.synchronize()

    def __call__(self):
        import torch
        return self.buf.sum(dtype=torch.int32)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


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


LONG_WORKLOAD = ("long single-sequence causal MLA prefill: 1 sequence of 32768 tokens, 128 heads, "
                 "qk 192 (128 nope + 64 rope) / v 128, bf16 N(0,1), scale 1/sqrt(192), fp32 LSE")


def make_workload(seed: int, heads: int = 128, long: bool = False):
    import mla_synth as syn
    if long:
        return syn.long32k_config(seed=seed, num_heads=heads)
    return syn.varlen16k_config(seed=seed, num_heads=heads)


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max(int(i.get("num_threads", 1)) for i in threadpool_info()) or 1
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def source_sha(files) -> str:
    h = hashlib.sha256()
    for name in files:
        with open(os.path.join(ROOT, "mla_prefill_attention_causal_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic_for(profile: str, files):
    """DRAM bytes per launch recorded in a committed ncu summary, if it was
    taken on the current source of the kernel (otherwise None)."""
    try:
        text = open(os.path.join(ROOT, "profiles", profile)).read()
    except OSError:
        return None
    vals = {}
    for line in text.splitlines():
        if ":" in line and line.strip().startswith("- "):
            k, v = line.strip()[2:].split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_sha256_16") != source_sha(files):
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------------------
# Workloads.  Each builds its seeded inputs (pinned host + device copies),
# one step of the hot path through the public API, the end-to-end step with
# host copies, and a bounded oracle sample for the CPU baseline.
# ---------------------------------------------------------------------------

class DenseWorkload:
    """Dense varlen causal prefill (the headline metric's configuration), or
    with ``long`` the single 32768-token sequence."""

    metric = METRIC
    kernel = "mla::dense::dense_fwd_kernel"
    sources = ("dense_fwd.cuh", "ptx.cuh")
    profile = "dense_fwd_varlen16k.md"
    in_attrs = ("q", "k", "v", "cu")  # device inputs, in the order of self.hin
    out_attrs = ("out", "lse")        # device outputs, in the order of self.hout

    def __init__(self, dev, seed, heads, long=False):
        import torch
        import oracle
        self.long = long
        self.name = "long32k" if long else "dense"
        self.profile = "dense_fwd_long32k.md" if long else "dense_fwd_varlen16k.md"
        self.case = case = make_workload(seed, heads=heads, long=long)
        self.H = H = case["num_heads"]
        self.flops = oracle.dense_flops(case["lens_q"], case["lens_k"], H, True)
        to_t = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.bfloat16)
        self.hin = [to_t(case["q"]).pin_memory(), to_t(case["k"]).pin_memory(),
                    to_t(case["v"]).pin_memory(), torch.from_numpy(case["cu_q"]).pin_memory()]
        self.q, self.k, self.v, self.cu = [x.to(dev) for x in self.hin]
        T = self.T = self.q.shape[0]
        self.out = torch.empty((T, H, 128), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((H, T), dtype=torch.float32, device=dev)
        self.hout = [torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory(),
                     torch.empty(self.lse.shape, dtype=self.lse.dtype).pin_memory()]
        self.launches = 2  # planner + attention kernel

    def step(self):
        import mla_prefill_attention_causal_b200 as mla
        c = self.case
        mla.mla_prefill_fwd(self.q, self.k, self.v, self.cu, self.cu, c["max_q"], c["max_q"],
                            c["scale"], causal=True, out=self.out, lse=self.lse)

    def config(self):
        c = self.case
        return {"workload": LONG_WORKLOAD if self.long else WORKLOAD, "batch": len(c["lens_q"]),
                "total_tokens": self.T,
                "heads": self.H, "seq_lens": c["lens_q"], "flops_per_step": self.flops,
                "l2": "inputs larger than L2 (Q+K+V %.2f GB > 126 MB); no flush" %
                      ((self.q.numel() + self.k.numel() + self.v.numel()) * 2 / 1e9)}

    @property
    def data(self):
        return ("synthetic (seeded N(0,1) bf16, one 32768-token sequence)" if self.long else
                "synthetic (seeded N(0,1) bf16, lengths U[512,4096])")

    def oracle_sample(self):
        """The fp64 oracle on heads 0-5 of the workload (all query rows); for
        the long sequence, 2048 evenly spaced query rows of heads 0-1."""
        import oracle
        c = self.case
        if self.long:
            rows = list(range(7, self.T, self.T // 2048))
            h = [0, 1]
            t0 = time.perf_counter()
            oracle.dense_prefill(c["q"][:, h], c["k"][:, h], c["v"][:, h], c["cu_q"], c["cu_k"],
                                 c["scale"], True, rows=rows)
            dt = time.perf_counter() - t0
            f = 2 * (192 + 128) * len(h) * sum(r + 1 for r in rows)
            return f, dt, (f"{len(rows)} evenly spaced query rows of heads 0-1 of the 32768-token "
                           f"sequence ({f:.3e} FLOPs in {dt:.1f} s)")
        h = list(range(6))
        t0 = time.perf_counter()
        oracle.dense_prefill(c["q"][:, h], c["k"][:, h], c["v"][:, h], c["cu_q"], c["cu_k"],
                             c["scale"], True)
        dt = time.perf_counter() - t0
        f = oracle.dense_flops(c["lens_q"], c["lens_k"], len(h), True)
        return f, dt, (f"heads 0-5 of {self.H}, all {self.T} query rows of the same batch "
                       f"({f:.3e} FLOPs in {dt:.1f} s)")

    def reference_step(self, i):
        """All query rows of sequence (i mod B) for head (i mod H) through the
        oracle; for the long sequence, 512 rows of head (i mod H)."""
        import oracle
        c = self.case
        B, H = len(c["lens_q"]), c["num_heads"]
        if self.long:
            h = i % H
            rows = list(range(i % 64, self.T, self.T // 512))
            t0 = time.perf_counter()
            oracle.dense_prefill(c["q"][:, h:h + 1], c["k"][:, h:h + 1], c["v"][:, h:h + 1],
                                 c["cu_q"], c["cu_k"], c["scale"], True, rows=rows)
            return 2 * (192 + 128) * sum(r + 1 for r in rows), time.perf_counter() - t0
        b, h = i % B, i % H
        q0, q1 = int(c["cu_q"][b]), int(c["cu_q"][b + 1])
        k0, k1 = int(c["cu_k"][b]), int(c["cu_k"][b + 1])
        t0 = time.perf_counter()
        oracle.dense_prefill(c["q"][q0:q1, h:h + 1], c["k"][k0:k1, h:h + 1],
                             c["v"][k0:k1, h:h + 1], [0, q1 - q0], [0, k1 - k0], c["scale"], True)
        return oracle.dense_flops([q1 - q0], [k1 - k0], 1, True), time.perf_counter() - t0

    @property
    def reference_sample(self):
        return ("step i = 512 evenly spaced query rows (offset i mod 64) of head (i mod 128)"
                if self.long else
                "step i = all query rows of sequence (i mod 8) for head (i mod 128)")


class SparseWorkload:
    """Absorbed top-k sparse prefill: 4096 tokens x 128 heads, 32768-row latent
    cache, top-k 2048 (``padded``: the tokens sit at cache positions 0..4095,
    so the first 2047 lists carry -1 padding)."""

    metric = ("MLA absorbed sparse prefill attn TFLOPS (valid top-k slots) and % of B200 dense "
              "BF16 peak, 1 GPU")
    kernel = "mla::sparse::sparse_fwd_kernel"
    sources = ("sparse_fwd.cuh", "ptx.cuh")
    profile = "sparse_fwd_4k.md"
    in_attrs = ("q", "kv", "idx")
    out_attrs = ("out", "lse")
    data = "synthetic (seeded N(0,1) bf16 q and latent cache, causal top-k index lists)"
    reference_sample = "step i = all 128 heads of token (i * 997 mod 4096)"

    def __init__(self, dev, seed, heads, padded=False):
        import torch
        import mla_synth as syn
        import oracle
        self.name = "sparse-padded" if padded else "sparse"
        self.padded = padded
        self.case = case = syn.sparse_config(seed=seed, padded=padded)
        self.H = H = case["num_heads"]
        self.flops = oracle.sparse_flops(case["indices"], case["num_rows"], H)
        to_t = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.bfloat16)
        self.hin = [to_t(case["q"]).pin_memory(), to_t(case["kv"]).pin_memory(),
                    torch.from_numpy(case["indices"]).pin_memory()]
        self.q, self.kv, self.idx = [x.to(dev) for x in self.hin]
        T = self.T = self.q.shape[0]
        self.out = torch.empty((T, H, 512), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((H, T), dtype=torch.float32, device=dev)
        self.hout = [torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory(),
                     torch.empty(self.lse.shape, dtype=self.lse.dtype).pin_memory()]
        self.launches = 1

    def step(self):
        import mla_prefill_attention_causal_b200 as mla
        mla.mla_sparse_prefill_fwd(self.q, self.kv, self.idx, self.case["scale"], out=self.out,
                                   lse=self.lse)

    def config(self):
        c = self.case
        return {"workload": ("absorbed sparse MLA prefill: %d tokens x %d heads, q/latent dim 576 "
                             "(V = first 512), %d-row latent cache, top-k %d without replacement "
                             "from the causally visible rows%s, scale 1/sqrt(576), fp32 LSE" %
                             (self.T, self.H, c["num_rows"], c["topk"],
                              " (tokens at positions 0..4095: -1 padding)" if self.padded
                              else " (tokens at the last 4096 positions)")),
                "tokens": self.T, "heads": self.H, "topk": c["topk"], "cache_rows": c["num_rows"],
                "flops_per_step": self.flops,
                "l2": "q + out %.2f GB > 126 MB (the 38 MB cache stays L2-resident); no flush" %
                      ((self.q.numel() + self.out.numel()) * 2 / 1e9)}

    def _oracle_tokens(self, tokens):
        import oracle
        c = self.case
        t0 = time.perf_counter()
        oracle.sparse_prefill(c["q"], c["kv"], c["indices"], c["scale"], tokens=tokens)
        dt = time.perf_counter() - t0
        f = oracle.sparse_flops(c["indices"][tokens], c["num_rows"], self.H)
        return f, dt

    def oracle_sample(self):
        tokens = [int(x) for x in (np.arange(64) * 61) % self.T]
        f, dt = self._oracle_tokens(tokens)
        return f, dt, (f"64 of the {self.T} tokens (all heads; tokens 61*i mod {self.T}); "
                       f"{f:.3e} FLOPs in {dt:.1f} s")

    def reference_step(self, i):
        return self._oracle_tokens([(i * 997) % self.T])


class ChunkedWorkload:
    """Chunked prefill with context: 4 sequences, each a 2048-token query
    chunk attending non-causally to a 16384-token prefix and causally to
    itself, the two partial results combined by ``mla_attn_merge``."""

    name = "chunked"
    metric = ("MLA chunked prefill (prefix pass + causal self pass + LSE merge) attn TFLOPS "
              "(causal-adj) and % of B200 dense BF16 peak, 1 GPU")
    kernel = "mla::dense::dense_fwd_kernel"
    sources = ("dense_fwd.cuh", "ptx.cuh")
    profile = "dense_fwd_chunked.md"  # DRAM bytes of the step's two attention launches
    merge_sources = ("merge.cuh",)
    merge_profile = "merge_chunked.md"
    in_attrs = ("q", "kp", "vp", "ks", "vs", "cu_q", "cu_p")
    out_attrs = ("out", "lse")
    data = "synthetic (seeded N(0,1) bf16 query chunks, prefix and self K/V)"
    reference_sample = ("step i = head (i mod 128) of sequence (i mod 4): prefix pass, self pass "
                        "and merge of that head's 2048 query rows")

    def __init__(self, dev, seed, heads):
        import torch
        import mla_synth as syn
        import oracle
        self.case = c = syn.chunked_config(seed=seed, num_heads=heads)
        self.H = H = c["num_heads"]
        B, L, P = c["batch"], c["chunk"], c["prefix"]
        self.flops = (oracle.dense_flops([L] * B, [P] * B, H, False) +
                      oracle.dense_flops([L] * B, [L] * B, H, True))
        to_t = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.bfloat16)
        self.hin = [to_t(c[k]).pin_memory() for k in ("q", "k_prefix", "v_prefix", "k_self",
                                                      "v_self")]
        self.hin += [torch.from_numpy(c["cu_q"]).pin_memory(),
                     torch.from_numpy(c["cu_prefix"]).pin_memory()]
        (self.q, self.kp, self.vp, self.ks, self.vs, self.cu_q, self.cu_p) = [
            x.to(dev) for x in self.hin]
        T = self.T = self.q.shape[0]
        mk = lambda: (torch.empty((T, H, 128), dtype=torch.bfloat16, device=dev),
                      torch.empty((H, T), dtype=torch.float32, device=dev))
        (self.op, self.lp), (self.os, self.ls), (self.out, self.lse) = mk(), mk(), mk()
        self.hout = [torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory(),
                     torch.empty(self.lse.shape, dtype=self.lse.dtype).pin_memory()]
        self.launches = 5  # 2 x (planner + attention) + merge
        self.merge_bytes = 3 * self.out.numel() * 2 + 3 * self.lse.numel() * 4
        self.merge_events = None

    def step(self):
        import torch
        import mla_prefill_attention_causal_b200 as mla
        c = self.case
        mla.mla_prefill_fwd(self.q, self.kp, self.vp, self.cu_q, self.cu_p, c["chunk"], c["prefix"],
                            c["scale"], causal=False, out=self.op, lse=self.lp)
        mla.mla_prefill_fwd(self.q, self.ks, self.vs, self.cu_q, self.cu_q, c["chunk"], c["chunk"],
                            c["scale"], causal=True, out=self.os, lse=self.ls)
        if self.merge_events is not None:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            mla.mla_attn_merge(self.op, self.lp, self.os, self.ls, out=self.out, lse_out=self.lse)
            e1.record()
            self.merge_events.append((e0, e1))
        else:
            mla.mla_attn_merge(self.op, self.lp, self.os, self.ls, out=self.out, lse_out=self.lse)

    def time_merge_alone(self, steps):
        """Milliseconds per merge launch in a run of `steps` back-to-back
        merges (after 3 untimed ones), CUDA events around the run: the
        kernel's streaming rate on its own, as the copy bandwidth it is
        compared with is measured (its 0.8 GB of operands exceed L2)."""
        import torch
        import mla_prefill_attention_causal_b200 as mla
        merge = lambda: mla.mla_attn_merge(self.op, self.lp, self.os, self.ls, out=self.out,
                                           lse_out=self.lse)
        for _ in range(3):
            merge()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            merge()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    def config(self):
        c = self.case
        return {"workload": ("chunked MLA prefill with context: %d sequences, %d-token query "
                             "chunks, non-causal prefix of %d tokens plus causal self pass, "
                             "merged with mla_attn_merge; %d heads, qk 192 / v 128, bf16 N(0,1), "
                             "scale 1/sqrt(192)" % (c["batch"], c["chunk"], c["prefix"], self.H)),
                "tokens": self.T, "heads": self.H, "flops_per_step": self.flops,
                "merge_bytes_per_step": self.merge_bytes,
                "l2": "prefix K/V %.2f GB > 126 MB; no flush" %
                      ((self.kp.numel() + self.vp.numel()) * 2 / 1e9)}

    def _oracle_head(self, b, h):
        import oracle
        c = self.case
        L, P = c["chunk"], c["prefix"]
        sl = lambda a, n, lo: a[lo * n:(lo + 1) * n, h:h + 1]
        t0 = time.perf_counter()
        o1, l1 = oracle.dense_prefill(sl(c["q"], L, b), sl(c["k_prefix"], P, b),
                                      sl(c["v_prefix"], P, b), [0, L], [0, P], c["scale"], False)
        o2, l2 = oracle.dense_prefill(sl(c["q"], L, b), sl(c["k_self"], L, b),
                                      sl(c["v_self"], L, b), [0, L], [0, L], c["scale"], True)
        oracle.attn_merge(o1, l1, o2, l2)
        dt = time.perf_counter() - t0
        f = oracle.dense_flops([L], [P], 1, False) + oracle.dense_flops([L], [L], 1, True)
        return f, dt

    def oracle_sample(self):
        f, dt = self._oracle_head(0, 0)
        return f, dt, (f"head 0 of sequence 0 (prefix pass, self pass and merge of its "
                       f"{self.case['chunk']} query rows): {f:.3e} FLOPs in {dt:.1f} s")

    def reference_step(self, i):
        return self._oracle_head(i % self.case["batch"], i % self.H)


class ChunkedContextWorkload(ChunkedWorkload):
    """The chunked workload in one pass: ``mla_prefill_fwd_context`` attends
    to the prefix (every key) and to the chunk itself (causal) under one
    softmax -- no partial outputs and no merge."""

    name = "chunked-context"
    metric = ("MLA chunked prefill in one pass (context + causal self keys) attn TFLOPS "
              "(causal-adj) and % of B200 dense BF16 peak, 1 GPU")
    profile = "dense_fwd_chunked_context.md"
    reference_sample = ("step i = head (i mod 128) of sequence (i mod 4): prefix pass, self pass "
                        "and merge of that head's 2048 query rows (the oracle's form of the "
                        "one-pass result)")

    def __init__(self, dev, seed, heads):
        super().__init__(dev, seed, heads)
        self.launches = 2  # planner + attention
        self.merge_events = None

    def step(self):
        import mla_prefill_attention_causal_b200 as mla
        c = self.case
        mla.mla_prefill_fwd_context(self.q, self.ks, self.vs, self.cu_q, self.cu_q, self.kp,
                                    self.vp, self.cu_p, c["chunk"], c["chunk"], c["prefix"],
                                    c["scale"], causal=True, out=self.out, lse=self.lse)

    def config(self):
        cfg = super().config()
        cfg["workload"] = cfg["workload"].replace("merged with mla_attn_merge",
                                                  "in one pass (mla_prefill_fwd_context)")
        cfg.pop("merge_bytes_per_step", None)
        return cfg


class SplitKvWorkload(DenseWorkload):
    """A few-tile shape: 16 heads (a tensor-parallel share of 128), one
    sequence of 129 queries (the vLLM warmup probe) over 8192 keys,
    bottom-right causal, through ``mla_prefill_fwd_splitkv`` with the
    library's choice of splits; the same call without splits is timed
    beside it (``config.unsplit_ms``)."""

    metric = ("MLA prefill attn TFLOPS (causal-adj), split-KV on a few-tile shape, "
              "% of B200 dense BF16 peak, 1 GPU")
    profile = "dense_fwd_splitkv.md"
    in_attrs = ("q", "k", "v", "cu", "cuk")
    flush_l2 = True

    def __init__(self, dev, seed, heads):
        import torch
        import mla_synth as syn
        import oracle
        import mla_prefill_attention_causal_b200 as mla
        self.long = False
        self.name = "splitkv"
        H = 16 if heads == 128 else heads
        self.case = case = syn.dense_case([129], [8192], H, seed)
        self.H = H
        self.flops = oracle.dense_flops(case["lens_q"], case["lens_k"], H, True)
        to_t = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.bfloat16)
        self.hin = [to_t(case["q"]).pin_memory(), to_t(case["k"]).pin_memory(),
                    to_t(case["v"]).pin_memory(), torch.from_numpy(case["cu_q"]).pin_memory(),
                    torch.from_numpy(case["cu_k"]).pin_memory()]
        self.q, self.k, self.v, self.cu, self.cuk = [x.to(dev) for x in self.hin]
        T = self.T = self.q.shape[0]
        self.out = torch.empty((T, H, 128), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((H, T), dtype=torch.float32, device=dev)
        self.hout = [torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory(),
                     torch.empty(self.lse.shape, dtype=self.lse.dtype).pin_memory()]
        self.splits = mla.num_splits_for(1, T, H, case["max_q"], case["max_k"])
        self.ws = torch.empty(mla.splitkv_workspace_size(1, T, H, self.splits), dtype=torch.uint8,
                              device=dev)
        self.launches = 3 if self.splits > 1 else 2
        self.unsplit_ms = None

    def _call(self, splits, ws=None):
        import mla_prefill_attention_causal_b200 as mla
        c = self.case
        mla.mla_prefill_fwd_splitkv(self.q, self.k, self.v, self.cu, self.cuk, c["max_q"],
                                    c["max_k"], c["scale"], causal=True, num_splits=splits,
                                    out=self.out, lse=self.lse, workspace=ws)

    def step(self):
        self._call(self.splits, self.ws)

    def time_unsplit(self, steps, flush):
        import torch
        for _ in range(3):
            self._call(1)
        ms = 0.0
        for _ in range(steps):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            self._call(1)
            e1.record()
            torch.cuda.synchronize()
            ms += e0.elapsed_time(e1)
        self.unsplit_ms = ms / steps

    def config(self):
        c = self.case
        return {"workload": ("split-KV few-tile shape: 1 sequence of 129 queries over 8192 keys, "
                             "bottom-right causal, %d heads, qk 192 / v 128, bf16 N(0,1), scale "
                             "1/sqrt(192)" % self.H),
                "heads": self.H, "num_splits": self.splits, "flops_per_step": self.flops,
                "unsplit_ms": self.unsplit_ms,
                "l2": ("inputs %.1f MB < L2: a %d MB buffer is read before every timed "
                       "call, each call timed alone with CUDA events"
                       % ((self.q.numel() + self.k.numel() + self.v.numel()) * 2 / 1e6,
                          L2_FLUSH_BYTES >> 20))}

    data = "synthetic (seeded N(0,1) bf16)"

    def oracle_sample(self):
        import oracle
        c = self.case
        t0 = time.perf_counter()
        oracle.dense_prefill(c["q"], c["k"], c["v"], c["cu_q"], c["cu_k"], c["scale"], True)
        dt = time.perf_counter() - t0
        return self.flops, dt, f"the whole call ({self.flops:.3e} FLOPs in {dt:.1f} s)"

    def reference_step(self, i):
        import oracle
        c = self.case
        h = i % self.H
        t0 = time.perf_counter()
        oracle.dense_prefill(c["q"][:, h:h + 1], c["k"][:, h:h + 1], c["v"][:, h:h + 1],
                             c["cu_q"], c["cu_k"], c["scale"], True)
        return oracle.dense_flops(c["lens_q"], c["lens_k"], 1, True), time.perf_counter() - t0

    reference_sample = "step i = head (i mod 16) of the whole call"


def time_e2e(w, steps: int) -> float:
    """Milliseconds per step of the end-to-end run: every step copies its
    inputs from pinned host memory, runs the call and reads its outputs back
    to pinned host memory.  Two device buffer sets alternate between steps,
    so step i+1's host-to-device copy (its own stream) overlaps step i's
    kernels and device-to-host copy (two more streams); events order each
    set's reuse.  Timed from before the first copy to after the last one."""
    import torch
    sets = [{a: getattr(w, a) for a in w.in_attrs + w.out_attrs}]
    sets.append({a: torch.empty_like(t) for a, t in sets[0].items()})
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    h2d_done = [torch.cuda.Event(), torch.cuda.Event()]
    run_done = [torch.cuda.Event(), torch.cuda.Event()]
    d2h_done = [torch.cuda.Event(), torch.cuda.Event()]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def one(i):
        b = i % 2
        buf = sets[b]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(run_done[b])       # step i-2's kernels are done with the inputs
            for a, h in zip(w.in_attrs, w.hin):
                buf[a].copy_(h, non_blocking=True)
            h2d_done[b].record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(h2d_done[b])
            if i >= 2:
                s_run.wait_event(d2h_done[b])      # step i-2's outputs have been read back
            for a, t in buf.items():
                setattr(w, a, t)
            w.step()
            run_done[b].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(run_done[b])
            for a, h in zip(w.out_attrs, w.hout):
                h.copy_(buf[a], non_blocking=True)
            d2h_done[b].record(s_out)

    one(0)
    one(1)
    torch.cuda.synchronize()
    t0.record(s_in)
    for i in range(steps):
        one(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_run)
    t1.record(s_out)
    torch.cuda.synchronize()
    for a, t in sets[0].items():
        setattr(w, a, t)
    return t0.elapsed_time(t1) / steps


def rank_seed(base: int, rank: int, world: int) -> int:
    """Seed of a rank's batch: the workload's own seed on one GPU, and a
    distinct batch per rank under weak scaling."""
    return base if world == 1 else base + 1000 * rank


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest of every rank's x (all ranks call it; no-op on one rank)."""
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(flops_per_rank: float, world: int, ms_step: float) -> float:
    """Weak scaling: every rank did flops_per_rank in at most ms_step (TFLOP/s)."""
    return flops_per_rank * world / (ms_step * 1e-3) / 1e12


def make(args, dev, rank, world):
    if args.workload == "dense":
        return DenseWorkload(dev, rank_seed(2, rank, world), args.heads)
    if args.workload == "long32k":
        return DenseWorkload(dev, rank_seed(3, rank, world), args.heads, long=True)
    if args.workload == "chunked":
        return ChunkedWorkload(dev, rank_seed(4, rank, world), args.heads)
    if args.workload == "chunked-context":
        return ChunkedContextWorkload(dev, rank_seed(4, rank, world), args.heads)
    if args.workload == "splitkv":
        return SplitKvWorkload(dev, rank_seed(6, rank, world), args.heads)
    return SparseWorkload(dev, rank_seed(5, rank, world), args.heads,
                          padded=args.workload == "sparse-padded")


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return 0
    # The reference arm runs the oracle on the host only: build the host-side case.
    if args.workload == "splitkv":
        import mla_synth as syn
        w = SplitKvWorkload.__new__(SplitKvWorkload)
        w.H = 16
        w.case = syn.dense_case([129], [8192], w.H, 6)
    elif args.workload in ("dense", "long32k"):
        w = DenseWorkload.__new__(DenseWorkload)
        w.long = args.workload == "long32k"
        w.case = make_workload(3 if w.long else 2, long=w.long)
        w.H, w.T = w.case["num_heads"], w.case["q"].shape[0]
    elif args.workload in ("chunked", "chunked-context"):
        import mla_synth as syn
        cls = ChunkedWorkload if args.workload == "chunked" else ChunkedContextWorkload
        w = cls.__new__(cls)
        w.case = syn.chunked_config(seed=4)
        w.H = w.case["num_heads"]
    else:
        import mla_synth as syn
        w = SparseWorkload.__new__(SparseWorkload)
        w.padded = args.workload == "sparse-padded"
        w.case = syn.sparse_config(seed=5, padded=w.padded)
        w.H, w.T = w.case["num_heads"], w.case["q"].shape[0]
    for i in range(args.warmup):
        w.reference_step(i)
    flops, secs = 0, 0.0
    for i in range(args.steps):
        f, dt = w.reference_step(i)
        flops += f
        secs += dt
    value = flops / secs / 1e12
    sample = f"{w.reference_sample}; {args.steps} steps = {flops:.3e} FLOPs"
    line = {
        "metric": w.metric, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": {"workload": {"dense": WORKLOAD, "long32k": LONG_WORKLOAD}.get(args.workload,
                                                                                  args.workload),
                   "sample": sample},
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

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = make(args, dev, rank, world)
    stream = torch.cuda.current_stream()

    for _ in range(max(args.warmup, 3)):
        w.step()
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
    if hasattr(w, "merge_events"):
        w.merge_events = []
    flush = L2Flush(dev) if getattr(w, "flush_l2", False) else None
    step_events = []
    ev0.record(stream)
    for _ in range(args.steps):
        if flush is None:
            w.step()
            continue
        # Inputs smaller than L2: read a buffer larger than L2 before every
        # call and time the call alone.
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        w.step()
        b.record(stream)
        step_events.append((a, b))
    ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    if hasattr(w, "time_unsplit"):
        w.time_unsplit(args.steps, flush)  # outside the timed region, for comparison
    merge_ms = None
    if getattr(w, "merge_events", None):
        merge_ms = sum(a.elapsed_time(b) for a, b in w.merge_events) / len(w.merge_events)
        w.merge_events = None
    ms_total = (sum(a.elapsed_time(b) for a, b in step_events) if step_events
                else ev0.elapsed_time(ev1))
    del flush
    ms_step = max_over_ranks(ms_total, world, dev) / args.steps
    value = whole_job_value(w.flops, world, ms_step)
    status = mla.mla_device_status(reset=True)
    if args.kernel_only:
        if rank == 0:
            print(json.dumps({"kernel_only": True, "workload": w.name, "heads": w.H,
                              "ms_per_step": ms_step,
                              "tflops": w.flops / (ms_step * 1e-3) / 1e12,
                              "device_status": status}), flush=True)
        return 0

    # End to end through the public call with host buffers: H2D of the step's
    # inputs from pinned memory, the kernel(s), D2H of out and lse.
    e2e_steps = max(3, min(args.steps, 20))
    if world > 1:
        dist.barrier()
    e2e_ms = max_over_ranks(time_e2e(w, e2e_steps), world, dev)
    h2d = sum(x.numel() * x.element_size() for x in w.hin)
    d2h = sum(x.numel() * x.element_size() for x in w.hout)

    if rank != 0:
        return 0
    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    attn_ms = ms_step - (merge_ms or 0.0)  # the attention launches of the step
    achieved = w.flops / (attn_ms * 1e-3) / 1e12
    config = w.config()
    config["parallelism"] = f"replicas x{world} (independent batches)"
    line = {
        "metric": w.metric, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": w.data,
        "config": config,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                     "frac": achieved / peak, "peak_source": f"{peak_src} bf16_tflops (burst)",
                     "frac_of_spec_2250": achieved / SPEC_BF16_TFLOPS,
                     "frac_of_sustained": achieved / float(peaks.get("bf16_tflops_sustained",
                                                                     peak)),
                     "traffic": recorded_traffic_for(w.profile, w.sources),
                     "kernel": w.kernel,
                     "timed": "one public call per step; CUDA events on its stream"},
        "e2e": {"value": whole_job_value(w.flops, world, e2e_ms), "unit": UNIT,
                "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "pipelined": "two device buffer sets: a step's host-to-device copy overlaps the "
                             "previous step's kernels and device-to-host copy"},
        "gpu_launches": args.steps * w.launches,
        "clocks": clocks,
        "device_status": status,
    }
    if merge_ms is not None:
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        gbs = w.merge_bytes / (merge_ms * 1e-3) / 1e9
        line["roofline"]["timed"] = ("attention launches of the step (step time minus the "
                                     "separately event-timed merge)")
        line["merge_roofline"] = {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                                  "frac": gbs / hbm, "ms": merge_ms,
                                  "peak_source": f"{peak_src} hbm_gbs",
                                  "traffic": recorded_traffic_for(w.merge_profile,
                                                                  w.merge_sources),
                                  "kernel": "mla::merge::merge_kernel",
                                  "timed": ("inside the step, right after the two attention "
                                            "passes (whose outputs are still being written "
                                            "back from L2)")}
        alone_ms = w.time_merge_alone(20)
        alone_gbs = w.merge_bytes / (alone_ms * 1e-3) / 1e9
        line["merge_roofline"]["alone"] = {"ms": alone_ms, "achieved": alone_gbs,
                                           "frac": alone_gbs / hbm,
                                           "timed": "20 back-to-back merges after 3 untimed"}
    if world == 1 and not args.no_cpu_baseline:
        f, dt, sample = w.oracle_sample()
        line["cpu_baseline"] = {"value": f / dt / 1e12, "unit": UNIT, "cores": blas_threads(),
                                "kind": "oracle", "sample": sample}
    print(json.dumps(line), flush=True)
    return 0


def relaunch_with_ranks(n: int) -> int:
    """Start n ranks of this script (one per GPU) with torch.distributed.run."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30,
                    help="timed calls (default 30: about 60 ms of back-to-back dense calls, like the "
                         "short matmul bursts the measured burst peak comes from; longer runs "
                         "settle under the power cap, which the sustained fraction covers)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel-only", action="store_true",
                    help="time the kernel only (no e2e, clocks or CPU baseline); for profiling")
    ap.add_argument("--heads", type=int, default=128,
                    help="heads of the dense workload (128 for the bench line; fewer for profiling)")
    ap.add_argument("--workload", default="dense",
                    choices=["dense", "long32k", "chunked", "chunked-context", "splitkv",
                             "sparse", "sparse-padded"],
                    help="dense: the headline configuration; long32k: one 32768-token causal "
                         "sequence; chunked: prefix + self passes and the LSE merge; "
                         "chunked-context: the same in one pass; splitkv: a few-tile shape through "
                         "split-KV; sparse: the absorbed top-k path")
    args = ap.parse_args()
    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        return relaunch_with_ranks(args.gpus)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE is {world}", file=sys.stderr)
        return 2
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
