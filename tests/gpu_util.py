"""Shared helpers for the GPU parity tests (not collected by pytest)."""
import numpy as np
import torch

import mla_synth as syn
import oracle

# Tolerances against the fp64 oracle for bf16 outputs and fp32 LSE.
TOL_OUT_MAX = 2e-2
TOL_OUT_MEAN = 2e-3
TOL_LSE = 1e-3


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev_i32(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_out_close(got: np.ndarray, ref: np.ndarray, what: str = "out"):
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - ref)
    mx, mean = float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0
    assert mx <= TOL_OUT_MAX and mean <= TOL_OUT_MEAN, f"{what}: max {mx:.3g} mean {mean:.3g}"
    return mx, mean


def assert_lse_close(got: np.ndarray, ref: np.ndarray, what: str = "lse"):
    assert got.shape == ref.shape, (got.shape, ref.shape)
    inf_ref = np.isneginf(ref)
    assert np.array_equal(np.isneginf(got), inf_ref), f"{what}: -inf pattern differs"
    fin = ~inf_ref
    err = np.abs(got[fin] - ref[fin])
    mx = float(err.max()) if err.size else 0.0
    assert mx <= TOL_LSE, f"{what}: max abs err {mx:.3g}"
    return mx


def sample_rows(lens, seed: int, per_seq: int = 24):
    """Global rows to check: tile edges, sequence ends and random rows."""
    g = np.random.Generator(np.random.PCG64(seed))
    cu = syn.cu_seqlens(lens)
    rows = []
    for b, L in enumerate(lens):
        if L == 0:
            continue
        cand = {0, 1, 2, 127, 128, 129, 255, 256, 257, L - 2, L - 1, L // 2}
        cand |= set(int(x) for x in g.integers(0, L, size=per_seq))
        rows += [int(cu[b]) + i for i in sorted(cand) if 0 <= i < L]
    return rows


def run_dense(case: dict, causal=None, want_lse=True):
    import mla_prefill_attention_causal_b200 as mla
    q, k, v = dev_bf16(case["q"]), dev_bf16(case["k"]), dev_bf16(case["v"])
    cq, ck = dev_i32(case["cu_q"]), dev_i32(case["cu_k"])
    c = case["causal"] if causal is None else causal
    out, lse = mla.mla_prefill_fwd(q, k, v, cq, ck, case["max_q"], case["max_k"], case["scale"],
                                   causal=c, return_lse=want_lse)
    torch.cuda.synchronize()
    return out, lse


def check_dense(case: dict, rows=None, causal=None):
    """Run the CUDA path and compare (sampled) rows with the oracle."""
    c = case["causal"] if causal is None else causal
    out, lse = run_dense(case, causal=c)
    ref_o, ref_l = oracle.dense_prefill(case["q"], case["k"], case["v"], case["cu_q"],
                                        case["cu_k"], case["scale"], c, rows=rows)
    if rows is None:
        got_o, got_l = to_f64(out), lse.cpu().numpy().astype(np.float64)
    else:
        idx = torch.as_tensor(rows, device=out.device)
        got_o = to_f64(out.index_select(0, idx))
        got_l = lse.index_select(1, idx).cpu().numpy().astype(np.float64)
    e1 = assert_out_close(got_o, ref_o)
    e2 = assert_lse_close(got_l, ref_l)
    return e1, e2
