"""mla_prefill_fwd_noalloc: the dense prefill for callers that cannot allocate.

Some callers have no way to hand the library a workspace (they may not call
cudaMalloc at all, or have no allocator of their own), so this entry point
keeps the work list in a fixed scratch array inside the library.  These
tests call it through the C ABI and check it against mla_prefill_fwd (which
takes a caller workspace) on two calls in a row with different batches, so
a stale work list left in the shared scratch would show up, and on a call
that fills the scratch exactly.  (The refusal of larger calls is checked
on the CPU, in test_abi.py.)  The file is named so that pytest collects it
last.
"""
import ctypes

import pytest
import torch

import mla_synth as syn

pytestmark = pytest.mark.gpu

from gpu_util import dev_bf16, dev_i32  # noqa: E402


def _inputs(case):
    return dict(q=dev_bf16(case["q"]), k=dev_bf16(case["k"]), v=dev_bf16(case["v"]),
                cq=dev_i32(case["cu_q"]), ck=dev_i32(case["cu_k"]))


def _run(case, t, noalloc):
    from mla_prefill_attention_causal_b200 import _lib
    lib = _lib.load()
    T, H = t["q"].shape[0], t["q"].shape[1]
    out = torch.empty((T, H, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((H, T), dtype=torch.float32, device="cuda")
    P = lambda x: ctypes.c_void_p(x.data_ptr())
    args = [P(t["q"]), P(t["k"]), P(t["v"]), P(t["cq"]), P(t["ck"]), case["max_q"], case["max_k"],
            case["scale"], 1 if case["causal"] else 0, P(out), P(lse),
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream),
            len(case["lens_q"]), H, T, t["k"].shape[0]]
    if noalloc:
        st = lib.mla_prefill_fwd_noalloc(*args)
    else:
        nbytes = lib.mla_prefill_workspace_size(len(case["lens_q"]), T)
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        st = lib.mla_prefill_fwd(*args, P(ws), nbytes)
    assert st == 0, _lib.status_string(st)
    torch.cuda.synchronize()
    return out, lse


def test_noalloc_matches_workspace_entry_point_on_two_calls(cuda_ok):
    """Both entry points run the same kernels on the same work list, so the
    results must be bitwise equal; the second call has another work list."""
    from mla_prefill_attention_causal_b200 import _lib
    _lib.mla_device_status(reset=True)
    cases = [syn.dense_case([700, 129, 1300, 1], [700, 129, 1300, 1], 8, seed=31),
             syn.dense_case([64, 2000], [300, 2000], 4, seed=32, causal=False)]
    for case in cases:  # two calls in a row; the second has a different work list
        t = _inputs(case)
        ref_o, ref_l = _run(case, t, noalloc=False)
        got_o, got_l = _run(case, t, noalloc=True)
        assert torch.equal(got_o, ref_o) and torch.equal(got_l, ref_l)
    assert _lib.mla_device_status(reset=True) == 0


def test_noalloc_at_the_scratch_limit(cuda_ok):
    """8144 one-token sequences: ceil(8144/512) + 8144 = 8160 work-list
    entries, exactly what the scratch holds."""
    from mla_prefill_attention_causal_b200 import _lib
    lens = [1] * 8144
    case = syn.dense_case(lens, lens, 1, seed=33)
    t = _inputs(case)
    ref_o, ref_l = _run(case, t, noalloc=False)
    got_o, got_l = _run(case, t, noalloc=True)
    assert torch.equal(got_o, ref_o) and torch.equal(got_l, ref_l)
    # a single key per row: O is that key's V row (bf16 of the exact value)
    assert torch.equal(got_o, t["v"])
    assert _lib.mla_device_status(reset=True) == 0
