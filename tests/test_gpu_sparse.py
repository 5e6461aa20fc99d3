"""GPU parity: absorbed top-k sparse MLA prefill against the fp64 oracle.

The kernel handles a token with two CTAs (value dims 0-255 and 256-511),
64 selected rows per chunk, 128 heads as the MMA rows.  The cases cover a
ragged last chunk, fewer heads than 128, -1 padding, out-of-range indices,
a token with no valid index, duplicates, topk = 1, and the 4096-token
workload (with and without padding) on every token.
"""
import numpy as np
import pytest
import torch

import mla_synth as syn
import oracle

pytestmark = pytest.mark.gpu

from gpu_util import assert_lse_close, assert_out_close, dev_bf16, dev_i32, to_f64  # noqa: E402
from oracle_pool import check_sparse_full  # noqa: E402


def run_sparse(case, indices=None, want_lse=True):
    import mla_prefill_attention_causal_b200 as mla
    idx = case["indices"] if indices is None else indices
    out, lse = mla.mla_sparse_prefill_fwd(dev_bf16(case["q"]), dev_bf16(case["kv"]), dev_i32(idx),
                                          case["scale"], return_lse=want_lse)
    torch.cuda.synchronize()
    return out, lse


def check_sparse(case, indices=None, tokens=None):
    idx = case["indices"] if indices is None else indices
    out, lse = run_sparse(case, idx)
    ref_o, ref_l = oracle.sparse_prefill(case["q"], case["kv"], idx, case["scale"], tokens=tokens)
    if tokens is None:
        got_o, got_l = to_f64(out), lse.cpu().numpy().astype(np.float64)
    else:
        sel = torch.as_tensor(list(tokens), device=out.device)
        got_o = to_f64(out.index_select(0, sel))
        got_l = lse.index_select(1, sel).cpu().numpy().astype(np.float64)
    assert_out_close(got_o, ref_o, "sparse out")
    assert_lse_close(got_l, ref_l, "sparse lse")
    return out, lse


def test_small_full_check_ragged_chunk(cuda_ok):
    # topk 200 = 3 full chunks of 64 + 8; early tokens padded with -1
    case = syn.sparse_case(num_tokens=9, num_heads=128, num_rows=260, topk=200, first_pos=190,
                           seed=41)
    assert (case["indices"] < 0).any()
    check_sparse(case)


@pytest.mark.parametrize("heads", [1, 16, 50, 127])
def test_fewer_heads_than_mma_rows(cuda_ok, heads):
    case = syn.sparse_case(num_tokens=6, num_heads=heads, num_rows=500, topk=130, first_pos=400,
                           seed=42 + heads)
    check_sparse(case)


def test_topk_one_and_single_valid_index(cuda_ok):
    case = syn.sparse_case(num_tokens=4, num_heads=128, num_rows=64, topk=1, first_pos=10,
                           seed=43)
    check_sparse(case)
    case = syn.sparse_case(num_tokens=4, num_heads=128, num_rows=64, topk=96, first_pos=0,
                           seed=44)
    idx = np.full_like(case["indices"], -1)
    idx[:, 77] = [3, 0, 63, 31]  # one valid slot per token, in the second chunk
    check_sparse(case, idx)


def test_all_padding_and_out_of_range_rows(cuda_ok):
    case = syn.sparse_case(num_tokens=5, num_heads=128, num_rows=100, topk=128, first_pos=99,
                           seed=45)
    idx = case["indices"].copy()
    idx[0, :] = -1                      # no valid slot: O = 0, LSE = -inf
    idx[1, ::3] = 100                   # == num_rows: padding
    idx[2, 5:40] = -7                   # other negatives: padding
    idx[3, :] = np.iinfo(np.int32).max  # all out of range
    out, lse = check_sparse(case, idx)
    assert torch.count_nonzero(out[0]).item() == 0 and torch.count_nonzero(out[3]).item() == 0
    assert torch.isneginf(lse[:, 0]).all() and torch.isneginf(lse[:, 3]).all()


def test_padded_chunks_and_late_valid_slots(cuda_ok):
    # Whole chunks of padding (zero-filled, never read from the cache) before
    # and between valid slots, and padding scattered through every chunk.
    case = syn.sparse_case(num_tokens=4, num_heads=128, num_rows=5000, topk=320, first_pos=4999,
                           seed=50)
    idx = case["indices"].copy()
    idx[0, :] = -1                       # five chunks, nothing valid
    idx[1, :300] = -1                    # valid slots only in the last chunk
    idx[2, 64:256] = -1                  # whole chunks 1-3 padded between valid ones
    idx[3, 4:320:8] = -1                 # a padded slot in every other group
    out, lse = check_sparse(case, idx)
    assert torch.count_nonzero(out[0]).item() == 0 and torch.isneginf(lse[:, 0]).all()


def test_duplicate_indices_count_twice(cuda_ok):
    case = syn.sparse_case(num_tokens=3, num_heads=64, num_rows=40, topk=192, first_pos=39,
                           seed=46)
    g = np.random.Generator(np.random.PCG64(460))
    idx = g.integers(0, 40, size=(3, 192)).astype(np.int32)  # many repeats
    check_sparse(case, idx)


def test_lse_optional_and_deterministic(cuda_ok):
    case = syn.sparse_case(num_tokens=8, num_heads=128, num_rows=1000, topk=256, first_pos=900,
                           seed=47)
    a, la = run_sparse(case)
    b, _ = run_sparse(case, want_lse=False)
    c, lc = run_sparse(case)
    assert torch.equal(a, b) and torch.equal(a, c) and torch.equal(la, lc)


def test_large_values_do_not_overflow(cuda_ok):
    # q x 32: scores with a standard deviation of 32 (natural-log units) make the
    # running maximum jump between chunks and the weights nearly one-hot
    case = syn.sparse_case(num_tokens=3, num_heads=128, num_rows=300, topk=256, first_pos=299,
                           seed=48)
    q = case["q"].copy()
    widened = (q[1].astype(np.uint32) << np.uint32(16)).view(np.float32)
    q[1] = syn.f32_to_bf16_bits(widened * np.float32(32.0))  # exact: a power of two
    case = dict(case, q=q)
    check_sparse(case)


@pytest.mark.parametrize("padded", [False, True])
def test_workload_4096_tokens_full(cuda_ok, padded):
    """4096 tokens x 128 heads, top-k 2048 over a 32768-row cache: every
    token and head against the oracle (padded: tokens at positions 0..4095,
    so the first 2047 carry -1 fill)."""
    case = syn.sparse_config(seed=5, padded=padded)
    out, lse = run_sparse(case)
    check_sparse_full(f"sparse 4096 x 128, top-k 2048{' padded' if padded else ''}",
                      case["q"], case["kv"], case["indices"], case["scale"], out, lse)


def test_output_only_16_byte_aligned_gives_the_same_bits(cuda_ok):
    """The epilogue stores 32-byte pieces when the output is 32-byte aligned
    and 16-byte pieces otherwise; both give the same bits."""
    import mla_prefill_attention_causal_b200 as mla
    case = syn.sparse_case(num_tokens=9, num_heads=128, num_rows=700, topk=320, first_pos=600,
                           seed=48)
    q, kv = dev_bf16(case["q"]), dev_bf16(case["kv"])
    idx = torch.from_numpy(case["indices"]).cuda()
    a, la = mla.mla_sparse_prefill_fwd(q, kv, idx, case["scale"])
    T, H = q.shape[0], q.shape[1]
    n = T * H * 512
    buf = torch.empty(n + 32, dtype=torch.bfloat16, device="cuda")
    base = (-buf.data_ptr()) % 32 // 2 + 8  # 16 bytes past a 32-byte boundary
    out = buf[base:base + n].view(T, H, 512)
    assert out.data_ptr() % 32 == 16
    b, lb = mla.mla_sparse_prefill_fwd(q, kv, idx, case["scale"], out=out)
    torch.cuda.synchronize()
    assert torch.equal(b, a) and torch.equal(lb, la)
