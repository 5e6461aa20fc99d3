"""Parity of the CUDA LSE merge with the oracle, plus the bounded-wait probe."""
import numpy as np
import pytest
import torch

import mla_synth as syn
import oracle

pytestmark = pytest.mark.gpu

from gpu_util import TOL_LSE, dev_bf16, to_f64  # noqa: E402


def _partials(T, H, D, seed, empty_frac=0.1):
    g = np.random.Generator(np.random.PCG64(seed))
    oa = syn.normal_bf16(seed * 10 + 1, (T, H, D))
    ob = syn.normal_bf16(seed * 10 + 2, (T, H, D))
    la = (g.standard_normal((H, T)) * 4).astype(np.float32)
    lb = (g.standard_normal((H, T)) * 4).astype(np.float32)
    la[g.random((H, T)) < empty_frac] = -np.inf
    lb[g.random((H, T)) < empty_frac] = -np.inf
    return oa, la, ob, lb


def _check(T, H, D, seed, alias=False):
    import mla_prefill_attention_causal_b200 as mla
    oa, la, ob, lb = _partials(T, H, D, seed)
    ta, tb = dev_bf16(oa), dev_bf16(ob)
    tla, tlb = torch.from_numpy(la).cuda(), torch.from_numpy(lb).cuda()
    out, lse = mla.mla_attn_merge(ta, tla, tb, tlb, out=ta if alias else None)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.attn_merge(oa, la, ob, lb)
    got = to_f64(out)
    err = np.abs(got - ref_o)
    # inputs are bf16 in [-5, 5]: bf16 output rounding is <= 2^-8 relative
    assert err.max() <= 2e-2 and err.mean() <= 2e-3, (err.max(), err.mean())
    gl = lse.cpu().numpy().astype(np.float64)
    assert np.array_equal(np.isneginf(gl), np.isneginf(ref_l))
    fin = np.isfinite(ref_l)
    assert np.abs(gl[fin] - ref_l[fin]).max() <= TOL_LSE
    both = np.isneginf(la) & np.isneginf(lb)
    assert np.all(got.transpose(1, 0, 2)[both] == 0)


@pytest.fixture(autouse=True)
def _need_gpu(cuda_ok):
    yield


@pytest.mark.parametrize("T,H,D", [(1, 1, 128), (37, 5, 128), (1000, 16, 128), (300, 3, 8),
                                   (129, 7, 512)])
def test_merge_matches_oracle(T, H, D):
    _check(T, H, D, seed=T + H + D)


def test_merge_in_place_output():
    _check(513, 4, 128, seed=9, alias=True)


def test_merge_large():
    _check(8192, 128, 128, seed=10)


def test_bounded_wait_gives_up_and_reports():
    import mla_prefill_attention_causal_b200 as mla
    mla.mla_device_status(reset=True)
    mla.mla_debug_wait_timeout(20000)  # 20 ms
    torch.cuda.synchronize()
    st = mla.mla_device_status(reset=True)
    assert st & mla._lib.DEVSTAT_WAIT_TIMEOUT_TEST
    assert mla.mla_device_status(reset=True) == 0
    # the context is still usable afterwards
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0
