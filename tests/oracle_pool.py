"""Whole-tensor oracle checks for the GPU parity tests (not collected by pytest).

The fp64 oracle is run as it stands, on independent slices of a problem
(groups of heads for the dense call, groups of tokens for the sparse call),
in a pool of worker processes started with ``spawn`` (a pool forked from a
process that already holds a CUDA context can hang).  Each worker limits its
BLAS to one thread, so the pool uses every host core once.  The slices are
exact: attention for one (token, head) reads nothing of another head, and a
sparse token reads nothing of another token.

Results stream back in order and are compared with the GPU output slice by
slice, so neither side of a large workload is ever held whole in float64.
The errors of every full-tensor check are kept in ``SUMMARY`` and printed at
the end of the pytest run (``conftest.pytest_terminal_summary``).
"""
from __future__ import annotations

import multiprocessing as mp
import os

import numpy as np
import torch

from gpu_util import TOL_LSE, TOL_OUT_MAX, TOL_OUT_MEAN

SUMMARY: list[dict] = []
_POOL = None


def _limit_threads():
    from threadpoolctl import threadpool_limits
    threadpool_limits(1)


def pool():
    global _POOL
    if _POOL is None:
        n = max(1, len(os.sched_getaffinity(0)))
        _POOL = mp.get_context("spawn").Pool(n, initializer=_limit_threads)
    return _POOL


def close_pool():
    global _POOL
    if _POOL is not None:
        _POOL.close()
        _POOL.join()
        _POOL = None


def _dense_job(args):
    import oracle
    q, k, v, cu_q, cu_k, scale, causal = args
    return oracle.dense_prefill(q, k, v, cu_q, cu_k, scale, causal)


def _sparse_job(args):
    import oracle
    q, kv, idx, scale = args
    return oracle.sparse_prefill(q, kv, idx, scale)


class ErrorTally:
    """Running max / mean absolute error of outputs and max LSE error."""

    def __init__(self, name: str):
        self.name = name
        self.out_max = 0.0
        self.out_sum = 0.0
        self.out_n = 0
        self.lse_max = 0.0
        self.inf_mismatch = 0
        self.nonfinite = 0

    def add(self, got_o: np.ndarray, ref_o: np.ndarray, got_l: np.ndarray, ref_l: np.ndarray):
        assert got_o.shape == ref_o.shape and got_l.shape == ref_l.shape
        self.nonfinite += int(np.count_nonzero(~np.isfinite(got_o)))
        err = np.abs(got_o - ref_o)
        if err.size:
            self.out_max = max(self.out_max, float(np.nanmax(err)))
            self.out_sum += float(np.nansum(err))
            self.out_n += err.size
        inf_ref = np.isneginf(ref_l)
        self.inf_mismatch += int(np.count_nonzero(np.isneginf(got_l) != inf_ref))
        fin = ~inf_ref
        if np.any(fin):
            self.lse_max = max(self.lse_max, float(np.abs(got_l[fin] - ref_l[fin]).max()))

    @property
    def out_mean(self) -> float:
        return self.out_sum / self.out_n if self.out_n else 0.0

    def check(self):
        SUMMARY.append(dict(name=self.name, values=self.out_n, out_max=self.out_max,
                            out_mean=self.out_mean, lse_max=self.lse_max))
        assert self.nonfinite == 0, f"{self.name}: {self.nonfinite} non-finite outputs"
        assert self.inf_mismatch == 0, f"{self.name}: -inf LSE pattern differs at {self.inf_mismatch}"
        assert self.out_max <= TOL_OUT_MAX and self.out_mean <= TOL_OUT_MEAN, \
            f"{self.name}: out max {self.out_max:.3g} mean {self.out_mean:.3g}"
        assert self.lse_max <= TOL_LSE, f"{self.name}: lse max {self.lse_max:.3g}"


def check_dense_full(name, q, k, v, cu_q, cu_k, scale, causal, out, lse, heads=None,
                     heads_per_job: int = 2):
    """Compare every query row of the GPU ``out``/``lse`` with the oracle.

    ``q``/``k``/``v`` are host bf16 bit arrays; ``heads`` (default: all) names
    the heads to check, taken ``heads_per_job`` at a time."""
    H = q.shape[1]
    heads = list(range(H)) if heads is None else sorted(heads)
    groups = [heads[i:i + heads_per_job] for i in range(0, len(heads), heads_per_job)]
    jobs = ((np.ascontiguousarray(q[:, g]), np.ascontiguousarray(k[:, g]),
             np.ascontiguousarray(v[:, g]), cu_q, cu_k, scale, causal) for g in groups)
    tally = ErrorTally(name)
    for g, (ref_o, ref_l) in zip(groups, pool().imap(_dense_job, jobs)):
        sel = torch.as_tensor(g, device=out.device)
        got_o = out.index_select(1, sel).float().cpu().numpy().astype(np.float64)
        got_l = lse.index_select(0, sel).cpu().numpy().astype(np.float64)
        tally.add(got_o, ref_o, got_l, ref_l)
    tally.check()
    return tally


def check_sparse_full(name, q, kv, indices, scale, out, lse, tokens_per_job: int = 128):
    """Compare every token and head of the GPU sparse ``out``/``lse`` with the oracle."""
    T = q.shape[0]
    spans = [(t, min(T, t + tokens_per_job)) for t in range(0, T, tokens_per_job)]
    jobs = ((np.ascontiguousarray(q[a:b]), kv, np.ascontiguousarray(indices[a:b]), scale)
            for a, b in spans)
    tally = ErrorTally(name)
    for (a, b), (ref_o, ref_l) in zip(spans, pool().imap(_sparse_job, jobs)):
        got_o = out[a:b].float().cpu().numpy().astype(np.float64)
        got_l = lse[:, a:b].cpu().numpy().astype(np.float64)
        tally.add(got_o, ref_o, got_l, ref_l)
    tally.check()
    return tally
