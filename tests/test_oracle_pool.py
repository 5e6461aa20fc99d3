"""The whole-tensor check helpers (tests/oracle_pool.py) on the CPU.

The helpers cut a problem into head groups (dense) or token spans (sparse),
run the oracle on each in spawned workers and compare slice by slice.  Here
the "GPU output" is the oracle's own whole-tensor result on CPU tensors, so
a correct cut gives zero error; a value planted in one slice must be caught.
"""
import numpy as np
import pytest
import torch

import mla_synth as syn
import oracle
from oracle_pool import check_dense_full, check_sparse_full


def _as_tensors(o, l):
    return torch.from_numpy(o.astype(np.float32)).to(torch.bfloat16), torch.from_numpy(
        l.astype(np.float32))


def test_dense_head_groups_reassemble_the_whole_tensor():
    case = syn.dense_case([70, 1, 130], [70, 1, 130], 5, seed=91)
    o, l = oracle.dense_prefill(case["q"], case["k"], case["v"], case["cu_q"], case["cu_k"],
                                case["scale"], True)
    out, lse = _as_tensors(o, l)
    t = check_dense_full("cpu dense", case["q"], case["k"], case["v"], case["cu_q"],
                         case["cu_k"], case["scale"], True, out, lse, heads_per_job=2)
    assert t.out_n == o.size and t.lse_max < 1e-5 and t.out_max < 1e-2
    bad = out.clone()
    bad[150, 4, 17] += 0.5                     # one value in the last head group
    with pytest.raises(AssertionError, match="out max"):
        check_dense_full("cpu dense planted", case["q"], case["k"], case["v"], case["cu_q"],
                         case["cu_k"], case["scale"], True, bad, lse, heads_per_job=2)
    sub = check_dense_full("cpu dense heads", case["q"], case["k"], case["v"], case["cu_q"],
                           case["cu_k"], case["scale"], True, bad, lse, heads=[0, 2, 3])
    assert sub.out_n == o.size // 5 * 3        # head 4 not checked: the planted value is unseen


def test_sparse_token_spans_reassemble_the_whole_tensor():
    case = syn.sparse_case(num_tokens=10, num_heads=3, num_rows=90, topk=40, first_pos=20,
                           seed=92)
    o, l = oracle.sparse_prefill(case["q"], case["kv"], case["indices"], case["scale"])
    out, lse = _as_tensors(o, l)
    t = check_sparse_full("cpu sparse", case["q"], case["kv"], case["indices"], case["scale"],
                          out, lse, tokens_per_job=3)
    assert t.out_n == o.size and t.lse_max < 1e-5
    bad = lse.clone()
    bad[1, 9] = -float("inf")                  # last span: -inf where the oracle has a value
    with pytest.raises(AssertionError, match="-inf"):
        check_sparse_full("cpu sparse planted", case["q"], case["kv"], case["indices"],
                          case["scale"], out, bad, tokens_per_job=3)
