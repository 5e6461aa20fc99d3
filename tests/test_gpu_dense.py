"""Parity of the CUDA dense MLA prefill (through the C ABI) with the fp64 oracle."""
import numpy as np
import pytest
import torch

import mla_synth as syn
import oracle

pytestmark = pytest.mark.gpu

from gpu_util import (assert_lse_close, assert_out_close, check_dense, dev_bf16, dev_i32,  # noqa: E402
                      run_dense, sample_rows, to_f64)
from oracle_pool import check_dense_full  # noqa: E402


@pytest.fixture(autouse=True)
def _device_status_clean(cuda_ok):
    import mla_prefill_attention_causal_b200 as mla
    mla.mla_device_status(reset=True)
    yield
    assert mla.mla_device_status(reset=True) == 0, "a kernel wait gave up"


def test_tiny_config_full():
    """2 ragged sequences (64, 100), 4 heads, causal: every row and head."""
    check_dense(syn.tiny_config())


@pytest.mark.parametrize("lens", [[1, 127, 128, 129], [255, 256, 257, 300], [511, 513, 1]])
def test_tile_edge_lengths_causal(lens):
    check_dense(syn.dense_case(lens, lens, 3, seed=sum(lens)))


def test_noncausal_ragged_lq_ne_lk():
    check_dense(syn.dense_case([1, 129, 200, 64], [128, 512, 77, 1], 2, seed=11, causal=False))


def test_causal_bottom_right_lq_lt_lk():
    check_dense(syn.dense_case([100, 300, 1], [400, 333, 700], 2, seed=12, causal=True))


def test_causal_lq_gt_lk_rows_without_keys():
    """Bottom-right causal with Lq > Lk: the first Lq-Lk rows see no key."""
    case = syn.dense_case([200, 150], [50, 150], 2, seed=13, causal=True)
    out, lse = run_dense(case)
    check_dense(case)
    o = to_f64(out)
    assert np.all(o[:150] == 0) and np.all(np.isneginf(lse[:, :150].cpu().numpy()))


def test_empty_key_sequence():
    case = syn.dense_case([40, 70], [0, 90], 2, seed=14, causal=False)
    out, lse = run_dense(case)
    check_dense(case)
    assert np.all(to_f64(out)[:40] == 0)


@pytest.mark.parametrize("max_q,max_k", [(1, 128), (129, 512), (1, 4096), (129, 4096)])
@pytest.mark.parametrize("causal", [False, True])
def test_warmup_probe_shapes(max_q, max_k, causal):
    """The (max_seqlen_q, max_seqlen_k) shape probes of vLLM's FA4 MLA warmup."""
    case = syn.dense_case([max_q], [max_k], 2, seed=max_q + max_k, causal=causal)
    check_dense(case)


@pytest.mark.parametrize("causal", [True, False])
def test_large_scores_rescale_the_running_max(causal):
    """q x 32 (exact: a power of two): scores with a standard deviation of 32
    make rows' running maxima jump by more than the lazy threshold in later
    KV blocks, so the O rescale path runs (N(0,1) data almost never takes it)."""
    lens_q = [700, 300, 129]
    lens_k = lens_q if causal else [900, 300, 400]
    case = syn.dense_case(lens_q, lens_k, 4, seed=71, causal=causal)
    widened = (case["q"].astype(np.uint32) << np.uint32(16)).view(np.float32)
    case = dict(case, q=syn.f32_to_bf16_bits(widened * np.float32(32.0)))
    check_dense(case)


def test_tile_handoff_across_alternating_launches():
    """The persistent clusters hand each tile's coordinates from the leader
    CTA to both CTAs through a ring in shared memory.  Alternating a call
    whose clusters run several tiles with one whose clusters end after an
    empty-key tile leaves different contents in the ring slots of the SMs;
    a consumer that read a slot before its new contents landed would act on
    the previous launch's tile (and give up waiting, or compute another
    tile).  200 alternating calls: bitwise-stable outputs, no wait given up."""
    import mla_prefill_attention_causal_b200 as mla
    a = syn.dense_case([300, 1000, 129, 2000], [300, 1000, 129, 2000], 64, seed=21)
    b = syn.dense_case([40, 70], [0, 90], 2, seed=14, causal=False)
    ins = []
    for c in (a, b):
        ins.append((dev_bf16(c["q"]), dev_bf16(c["k"]), dev_bf16(c["v"]), dev_i32(c["cu_q"]),
                    dev_i32(c["cu_k"]), c["max_q"], c["max_k"], c["scale"]))
    ref = [mla.mla_prefill_fwd(*x, causal=c["causal"]) for x, c in zip(ins, (a, b))]
    outs = [(torch.empty_like(o), torch.empty_like(l)) for o, l in ref]
    for _ in range(100):
        for x, c, (o, l) in zip(ins, (a, b), outs):
            mla.mla_prefill_fwd(*x, causal=c["causal"], out=o, lse=l)
    torch.cuda.synchronize()
    for (ro, rl), (o, l) in zip(ref, outs):
        assert torch.equal(ro, o) and torch.equal(rl, l)


def test_lse_optional_and_out_identical():
    case = syn.dense_case([300, 77], [300, 77], 2, seed=15)
    o1, l1 = run_dense(case, want_lse=True)
    o2, l2 = run_dense(case, want_lse=False)
    assert l2 is None
    assert torch.equal(o1, o2)


def test_bitwise_deterministic():
    case = syn.dense_case([700, 1300, 257], [700, 1300, 257], 8, seed=16)
    o1, l1 = run_dense(case)
    o2, l2 = run_dense(case)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_batch_invariant():
    """A sequence gives identical bits alone and inside a batch."""
    lens = [300, 1000, 129]
    case = syn.dense_case(lens, lens, 4, seed=17)
    o_all, l_all = run_dense(case)
    s0, s1 = int(case["cu_q"][1]), int(case["cu_q"][2])
    alone = dict(case)
    alone.update(q=case["q"][s0:s1], k=case["k"][s0:s1], v=case["v"][s0:s1],
                 cu_q=syn.cu_seqlens([lens[1]]), cu_k=syn.cu_seqlens([lens[1]]),
                 max_q=lens[1], max_k=lens[1])
    o1, l1 = run_dense(alone)
    assert torch.equal(o1, o_all[s0:s1])
    assert torch.equal(l1, l_all[:, s0:s1])


@pytest.mark.parametrize("causal", [False, True])
def test_strided_views_match_packed_inputs(causal):
    """q, k, v as views into wider buffers (v interleaved with k_nope per head,
    as in vLLM's MLA prefill backend) give the packed call's result exactly."""
    import mla_prefill_attention_causal_b200 as mla
    case = syn.dense_case([300, 129, 1], [300, 129, 1] if causal else [513, 64, 200], 4, seed=77,
                          causal=causal)
    q, k, v = dev_bf16(case["q"]), dev_bf16(case["k"]), dev_bf16(case["v"])
    cq, ck = dev_i32(case["cu_q"]), dev_i32(case["cu_k"])
    T, H = q.shape[0], q.shape[1]
    Tk = k.shape[0]
    qbuf = torch.zeros((T, H, 256), dtype=torch.bfloat16, device="cuda")
    qbuf[..., :192] = q                       # head stride 256
    kbuf = torch.zeros((Tk, H + 1, 192), dtype=torch.bfloat16, device="cuda")
    kbuf[:, :H] = k                           # row stride (H + 1) * 192
    kv = torch.zeros((Tk, H, 256), dtype=torch.bfloat16, device="cuda")
    kv[..., 128:] = v                         # v = kv[..., 128:]: head stride 256, offset 256 B
    qs, ks, vs = qbuf[..., :192], kbuf[:, :H], kv[..., 128:]
    assert not (qs.is_contiguous() or ks.is_contiguous() or vs.is_contiguous())
    a = mla.mla_prefill_fwd(q, k, v, cq, ck, case["max_q"], case["max_k"], case["scale"],
                            causal=causal)
    b = mla.mla_prefill_fwd(qs, ks, vs, cq, ck, case["max_q"], case["max_k"], case["scale"],
                            causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    ref_o, ref_l = oracle.dense_prefill(case["q"], case["k"], case["v"], case["cu_q"],
                                        case["cu_k"], case["scale"], causal)
    assert_out_close(to_f64(b[0]), ref_o)
    assert_lse_close(b[1].cpu().numpy().astype(np.float64), ref_l)


def test_many_heads_small():
    lens = [383, 129]
    check_dense(syn.dense_case(lens, lens, 128, seed=18))


def test_thousands_of_heads_on_tiny_sequences():
    """4096 heads (tensor-parallel layouts keep fewer, but the head is the
    slowest index of the work list and of the tensor maps' middle dimension)
    over sequences of 3, 1 and 130 tokens: 12 288 tiles of mostly empty rows."""
    lens = [3, 1, 130]
    check_dense(syn.dense_case(lens, lens, 4096, seed=19))


def test_varlen16k_config_full():
    """8 sequences, lengths U[512,4096] (15843 tokens), 128 heads, causal:
    every query row and head against the oracle."""
    case = syn.varlen16k_config()
    out, lse = run_dense(case)
    check_dense_full("varlen16k (8 x U[512,4096], 128 heads, causal)", case["q"], case["k"],
                     case["v"], case["cu_q"], case["cu_k"], case["scale"], True, out, lse)


def test_long32k_config_sampled():
    """One 32768-token sequence, 128 heads: 300+ sampled rows, all heads."""
    case = syn.long32k_config()
    rows = sample_rows(case["lens_q"], seed=3, per_seq=300)
    rows += [r for r in range(4095, 32768, 4096)]
    check_dense(case, rows=sorted(set(rows)))


# heads of the chunked workload checked on every row (0 and the last included)
CHUNKED_HEADS = sorted(set(range(0, 128, 4)) | {127})


def test_chunked_prefill_with_context_merge():
    """Prefix pass (unmasked, LSE) + self pass (causal) + merge equals one
    bottom-right causal pass over [prefix, chunk]: every query row of the
    4 x 2048-token chunks, on 33 of the 128 heads."""
    import mla_prefill_attention_causal_b200 as mla
    d = syn.chunked_config()
    q = dev_bf16(d["q"])
    kp, vp = dev_bf16(d["k_prefix"]), dev_bf16(d["v_prefix"])
    ks, vs = dev_bf16(d["k_self"]), dev_bf16(d["v_self"])
    cq, cp = dev_i32(d["cu_q"]), dev_i32(d["cu_prefix"])
    o1, l1 = mla.mla_prefill_fwd(q, kp, vp, cq, cp, d["chunk"], d["prefix"], d["scale"], causal=False)
    o2, l2 = mla.mla_prefill_fwd(q, ks, vs, cq, cq, d["chunk"], d["chunk"], d["scale"], causal=True)
    om, lm = mla.mla_attn_merge(o1, l1, o2, l2)
    torch.cuda.synchronize()
    k_cat, v_cat, cu_cat = chunked_concat(d)
    check_dense_full("chunked (4 x 2048 over 16384 prefix, prefix + self + merge, 33 heads)",
                     d["q"], k_cat, v_cat, d["cu_q"], cu_cat, d["scale"], True, om, lm,
                     heads=CHUNKED_HEADS, heads_per_job=1)


def chunked_concat(d):
    """Each sequence's prefix keys followed by its own chunk's keys: the key
    set that one bottom-right causal call over [prefix, chunk] sees."""
    B, C, P = d["batch"], d["chunk"], d["prefix"]
    k_cat = np.concatenate([np.concatenate([d["k_prefix"][b * P:(b + 1) * P],
                                            d["k_self"][b * C:(b + 1) * C]]) for b in range(B)])
    v_cat = np.concatenate([np.concatenate([d["v_prefix"][b * P:(b + 1) * P],
                                            d["v_self"][b * C:(b + 1) * C]]) for b in range(B)])
    return k_cat, v_cat, syn.cu_seqlens([P + C] * B)


# ----------------------------------------------------------------- context pass
def _context_call(q, k, v, cu_q, cu_k, kc, vc, cu_c, scale, causal):
    import mla_prefill_attention_causal_b200 as mla
    lq, lk, lc = np.diff(cu_q), np.diff(cu_k), np.diff(cu_c)
    out, lse = mla.mla_prefill_fwd_context(
        dev_bf16(q), dev_bf16(k), dev_bf16(v), dev_i32(cu_q), dev_i32(cu_k), dev_bf16(kc),
        dev_bf16(vc), dev_i32(cu_c), int(lq.max()), int(lk.max()), int(lc.max()), scale,
        causal=causal)
    torch.cuda.synchronize()
    return out, lse


@pytest.mark.parametrize("causal", [True, False])
def test_context_pass_matches_merge_of_context_and_own_keys(causal):
    """The one-pass chunked prefill equals the oracle's merge of an unmasked
    pass over the context and a pass over the sequence's own keys, on a
    ragged batch: contexts of 700, 0, 129, 1, 128 and 127 keys, a sequence
    with more queries than keys and one without keys of its own."""
    lens_q = [300, 129, 1, 513, 200, 64]
    lens_k = [300, 129, 1, 513, 150, 0] if causal else [256, 40, 7, 600, 150, 0]
    lens_c = [700, 0, 129, 1, 128, 127]
    H = 4
    case = syn.dense_case(lens_q, lens_k, H, seed=81, causal=causal)
    ctx = syn.dense_case(lens_c, lens_c, H, seed=82)
    out, lse = _context_call(case["q"], case["k"], case["v"], case["cu_q"], case["cu_k"],
                             ctx["k"], ctx["v"], ctx["cu_k"], case["scale"], causal)
    o_c, l_c = oracle.dense_prefill(case["q"], ctx["k"], ctx["v"], case["cu_q"], ctx["cu_k"],
                                    case["scale"], False)
    o_s, l_s = oracle.dense_prefill(case["q"], case["k"], case["v"], case["cu_q"], case["cu_k"],
                                    case["scale"], causal)
    ref_o, ref_l = oracle.attn_merge(o_c, l_c, o_s, l_s)
    assert_out_close(to_f64(out), ref_o, "context out")
    assert_lse_close(lse.cpu().numpy().astype(np.float64), ref_l, "context lse")


def test_context_pass_without_context_is_the_plain_call():
    """Empty contexts: bit for bit the result of mla_prefill_fwd."""
    lens = [700, 129, 300]
    case = syn.dense_case(lens, lens, 4, seed=83)
    kc = np.zeros((1, 4, 192), dtype=case["k"].dtype)  # a real (unread) buffer
    vc = np.zeros((1, 4, 128), dtype=case["v"].dtype)
    out, lse = _context_call(case["q"], case["k"], case["v"], case["cu_q"], case["cu_k"], kc, vc,
                             syn.cu_seqlens([0, 0, 0]), case["scale"], True)
    o_p, l_p = run_dense(case)
    assert torch.equal(out, o_p) and torch.equal(lse, l_p)


def test_context_pass_chunked_workload_full():
    """The chunked workload (4 x 2048 new tokens over 16384-token contexts,
    128 heads) in one pass: every row of 33 heads against one bottom-right
    causal oracle call over each sequence's [context, chunk] keys."""
    d = syn.chunked_config()
    out, lse = _context_call(d["q"], d["k_self"], d["v_self"], d["cu_q"], d["cu_q"],
                             d["k_prefix"], d["v_prefix"], d["cu_prefix"], d["scale"], True)
    k_cat, v_cat, cu_cat = chunked_concat(d)
    check_dense_full("chunked in one pass (mla_prefill_fwd_context, 33 heads)", d["q"], k_cat,
                     v_cat, d["cu_q"], cu_cat, d["scale"], True, out, lse,
                     heads=CHUNKED_HEADS, heads_per_job=1)


# ------------------------------------------------------- sinks and e4m3 output
def _run_ex(case, sinks=None, output_scale=None):
    import mla_prefill_attention_causal_b200 as mla
    s = None if sinks is None else torch.tensor(sinks, dtype=torch.float32, device="cuda")
    o_s = None if output_scale is None else torch.tensor([output_scale], dtype=torch.float32,
                                                         device="cuda")
    out, lse = mla.mla_prefill_fwd_ex(dev_bf16(case["q"]), dev_bf16(case["k"]), dev_bf16(case["v"]),
                                      dev_i32(case["cu_q"]), dev_i32(case["cu_k"]), case["max_q"],
                                      case["max_k"], case["scale"], causal=case["causal"], sinks=s,
                                      output_scale=o_s)
    torch.cuda.synchronize()
    return out, lse


def test_ex_without_options_is_the_plain_call():
    case = syn.dense_case([700, 129, 300], [700, 129, 300], 4, seed=95)
    o, l = _run_ex(case)
    o_p, l_p = run_dense(case)
    assert torch.equal(o, o_p) and torch.equal(l, l_p)


@pytest.mark.parametrize("causal", [True, False])
def test_sinks_match_oracle(causal):
    """One sink logit per head (two of them far above every score) on a
    ragged batch that has rows without any key (O = 0, LSE = the sink)."""
    lens_q = [300, 129, 1, 200]
    lens_k = [300, 129, 1, 150] if causal else [256, 40, 7, 0]
    case = syn.dense_case(lens_q, lens_k, 4, seed=96, causal=causal)
    sinks = np.array([0.5, -1.5, 12.0, 3.0], dtype=np.float32)
    out, lse = _run_ex(case, sinks=sinks)
    ref_o, ref_l = oracle.dense_prefill_sinks(case["q"], case["k"], case["v"], case["cu_q"],
                                              case["cu_k"], case["scale"], causal,
                                              sinks.astype(np.float64))
    assert_out_close(to_f64(out), ref_o, "sink out")
    assert_lse_close(lse.cpu().numpy().astype(np.float64), ref_l, "sink lse")


def _e4m3_step(y):
    """Spacing of the e4m3 grid around |y| (2^-9 below the normal range)."""
    a = np.minimum(np.abs(y), 448.0)
    return np.exp2(np.floor(np.log2(np.maximum(a, 2.0 ** -6))) - 3.0)


@pytest.mark.parametrize("scale", [0.01, 0.25, 1e-4])
def test_fp8_output_is_the_e4m3_of_the_same_output(scale):
    """e4m3 output of O / scale.  The kernel rounds the same fp32 O that its
    bf16 output rounds, so each code lies within one e4m3 step of that bf16
    value / scale (the bf16 rounding is far finer than the e4m3 grid), and
    within the bf16 tolerance plus one step of the oracle.  The LSE is the
    plain call's, bit for bit.  Scale 1e-4 saturates most outputs at 448."""
    case = syn.dense_case([513, 130, 1], [513, 130, 1], 4, seed=97)
    out, lse = _run_ex(case, output_scale=scale)
    assert out.dtype == torch.float8_e4m3fn
    got = oracle.e4m3_decode(out.view(torch.uint8).cpu().numpy())
    o_p, l_p = run_dense(case)
    assert torch.equal(lse, l_p)
    y_b = np.clip(to_f64(o_p) / np.float64(scale), -448.0, 448.0)
    assert np.all(np.abs(got - y_b) <= _e4m3_step(y_b) * 1.0001)
    ref_o, _ = oracle.dense_prefill(case["q"], case["k"], case["v"], case["cu_q"], case["cu_k"],
                                    case["scale"], True)
    y = ref_o / np.float64(scale)
    err = np.abs(got - np.clip(y, -448.0, 448.0))
    assert np.all(err <= 2e-2 / scale + _e4m3_step(y) * 1.0001)
    # saturated where the exact value is clearly out of range
    sat = np.abs(y) > 448.0 * 1.01
    assert np.all(np.abs(got[sat]) == 448.0)
    # the bulk of the codes are the oracle's own rounding
    assert np.mean(oracle.e4m3_quantize(ref_o, scale) ==
                   out.view(torch.uint8).cpu().numpy()) > 0.9


def test_sinks_with_fp8_output():
    """Both options at once: the e4m3 codes of the sink-weighted output."""
    case = syn.dense_case([257, 64], [257, 64], 2, seed=98)
    sinks = np.array([1.0, -0.5], dtype=np.float32)
    out, lse = _run_ex(case, sinks=sinks, output_scale=0.02)
    o_b, l_b = _run_ex(case, sinks=sinks)
    assert torch.equal(lse, l_b)
    got = oracle.e4m3_decode(out.view(torch.uint8).cpu().numpy())
    y_b = np.clip(to_f64(o_b) / 0.02, -448.0, 448.0)
    assert np.all(np.abs(got - y_b) <= _e4m3_step(y_b) * 1.0001)


# -------------------------------------------------------------------- split-KV
def _run_split(case, num_splits):
    import mla_prefill_attention_causal_b200 as mla
    out, lse = mla.mla_prefill_fwd_splitkv(
        dev_bf16(case["q"]), dev_bf16(case["k"]), dev_bf16(case["v"]), dev_i32(case["cu_q"]),
        dev_i32(case["cu_k"]), case["max_q"], case["max_k"], case["scale"], causal=case["causal"],
        num_splits=num_splits)
    torch.cuda.synchronize()
    return out, lse


@pytest.mark.parametrize("max_q,max_k", [(1, 4096), (1, 8192), (129, 4096), (129, 512)])
@pytest.mark.parametrize("causal", [False, True])
def test_splitkv_on_the_warmup_probe_shapes(max_q, max_k, causal):
    """vLLM's MLA warmup probes with few heads (a tensor-parallel share):
    fewer tiles than CTA pairs, so the library splits the KV blocks."""
    import mla_prefill_attention_causal_b200 as mla
    case = syn.dense_case([max_q], [max_k], 4, seed=max_q + max_k + 7, causal=causal)
    ns = mla.num_splits_for(1, max_q, 4, max_q, max_k)
    assert ns > 1
    out, lse = _run_split(case, None)
    ref_o, ref_l = oracle.dense_prefill(case["q"], case["k"], case["v"], case["cu_q"],
                                        case["cu_k"], case["scale"], causal)
    assert_out_close(to_f64(out), ref_o, f"split-KV ({ns} splits) out")
    assert_lse_close(lse.cpu().numpy().astype(np.float64), ref_l, f"split-KV ({ns} splits) lse")


@pytest.mark.parametrize("splits", [2, 3, 7, 64])
def test_splitkv_ragged_batch(splits):
    """A ragged causal batch with rows without keys (Lq > Lk) and an empty
    key sequence; 64 splits leave most ranges of the short tiles empty."""
    lens_q = [300, 129, 1, 200, 40]
    lens_k = [900, 129, 700, 150, 0]
    case = syn.dense_case(lens_q, lens_k, 2, seed=101 + splits, causal=True)
    out, lse = _run_split(case, splits)
    ref_o, ref_l = oracle.dense_prefill(case["q"], case["k"], case["v"], case["cu_q"],
                                        case["cu_k"], case["scale"], True)
    assert_out_close(to_f64(out), ref_o, "split-KV ragged out")
    assert_lse_close(lse.cpu().numpy().astype(np.float64), ref_l, "split-KV ragged lse")
    assert np.all(to_f64(out)[sum(lens_q[:4]):] == 0)


def test_splitkv_with_one_split_is_the_plain_call():
    case = syn.dense_case([700, 129, 1300], [700, 129, 1300], 4, seed=102)
    o, l = _run_split(case, 1)
    o_p, l_p = run_dense(case)
    assert torch.equal(o, o_p) and torch.equal(l, l_p)


def test_splitkv_is_deterministic_and_close_to_unsplit():
    case = syn.dense_case([1], [8192], 8, seed=103, causal=False)
    a, la = _run_split(case, 9)
    b, lb = _run_split(case, 9)
    assert torch.equal(a, b) and torch.equal(la, lb)
    o_p, l_p = run_dense(case)
    assert (a.float() - o_p.float()).abs().max().item() <= 2 ** -7
    assert (la - l_p).abs().max().item() <= 1e-4


# ------------------------------------------------------ other MLA head geometries
@pytest.mark.parametrize("qk,v", [(256, 256), (128, 128), (256, 128), (128, 256)])
@pytest.mark.parametrize("causal", [True, False])
def test_other_head_geometries(qk, v, causal):
    """vLLM's supports_mla_dimensions rows (192+64, 256), (64+64, 128),
    (256+0, 256), and the mixed widths, on a ragged batch with tile edges
    and rows without keys."""
    import mla_prefill_attention_causal_b200 as mla
    lens_q = [300, 129, 1, 513]
    lens_k = [300, 129, 1, 513] if causal else [256, 40, 7, 600]
    case = syn.dense_case(lens_q, lens_k, 3, seed=qk + v + causal, causal=causal, qk_dim=qk,
                          v_dim=v)
    out, lse = mla.mla_prefill_fwd_dims(dev_bf16(case["q"]), dev_bf16(case["k"]),
                                        dev_bf16(case["v"]), dev_i32(case["cu_q"]),
                                        dev_i32(case["cu_k"]), case["max_q"], case["max_k"],
                                        case["scale"], causal=causal)
    torch.cuda.synchronize()
    assert out.shape == (sum(lens_q), 3, v)
    ref_o, ref_l = oracle.dense_prefill(case["q"], case["k"], case["v"], case["cu_q"],
                                        case["cu_k"], case["scale"], causal)
    assert_out_close(to_f64(out), ref_o, f"qk {qk} v {v} out")
    assert_lse_close(lse.cpu().numpy().astype(np.float64), ref_l, f"qk {qk} v {v} lse")


def test_dims_call_with_the_default_geometry_is_the_plain_call():
    import mla_prefill_attention_causal_b200 as mla
    case = syn.dense_case([700, 129], [700, 129], 4, seed=104)
    out, lse = mla.mla_prefill_fwd_dims(dev_bf16(case["q"]), dev_bf16(case["k"]),
                                        dev_bf16(case["v"]), dev_i32(case["cu_q"]),
                                        dev_i32(case["cu_k"]), case["max_q"], case["max_k"],
                                        case["scale"], causal=True)
    o_p, l_p = run_dense(case)
    assert torch.equal(out, o_p) and torch.equal(lse, l_p)


# -------------------------------------------------- output alignment (16 vs 32 bytes)
def test_outputs_only_16_byte_aligned_give_the_same_bits():
    """The epilogue stores 32-byte pieces where every output row is 32-byte
    aligned and 16-byte pieces otherwise; outputs (bf16 and e4m3) and a
    split-KV workspace that start 16 bytes past a 32-byte boundary must give
    the bits of aligned ones."""
    import mla_prefill_attention_causal_b200 as mla
    case = syn.dense_case([513, 130, 1, 700], [513, 130, 1, 700], 4, seed=131)
    q, k, v = dev_bf16(case["q"]), dev_bf16(case["k"]), dev_bf16(case["v"])
    cq, ck = dev_i32(case["cu_q"]), dev_i32(case["cu_k"])
    T, H = q.shape[0], q.shape[1]
    args = (q, k, v, cq, ck, case["max_q"], case["max_k"], case["scale"])

    def shifted(n_elems, dtype, shift_bytes):
        esz = torch.empty((), dtype=dtype).element_size()
        buf = torch.empty(n_elems + 64 // esz, dtype=dtype, device="cuda")
        base = (-buf.data_ptr()) % 32 // esz + shift_bytes // esz  # 32-byte boundary + shift
        return buf[base:base + n_elems]

    o_a, l_a = mla.mla_prefill_fwd(*args, causal=True)
    o_s = shifted(T * H * 128, torch.bfloat16, 16).view(T, H, 128)
    assert o_s.data_ptr() % 32 == 16
    mla.mla_prefill_fwd(*args, causal=True, out=o_s)
    torch.cuda.synchronize()
    assert torch.equal(o_s, o_a)

    sc = torch.tensor([0.05], dtype=torch.float32, device="cuda")
    f_a, _ = mla.mla_prefill_fwd_ex(*args, causal=True, output_scale=sc)
    f_s = shifted(T * H * 128, torch.uint8, 16).view(torch.float8_e4m3fn).view(T, H, 128)
    assert f_s.data_ptr() % 32 == 16
    mla.mla_prefill_fwd_ex(*args, causal=True, output_scale=sc, out=f_s)
    torch.cuda.synchronize()
    assert torch.equal(f_s.view(torch.uint8), f_a.view(torch.uint8))

    ns = 3
    wbytes = mla.splitkv_workspace_size(len(case["lens_q"]), T, H, ns)
    s_a, sl_a = mla.mla_prefill_fwd_splitkv(*args, causal=True, num_splits=ns)
    ws = shifted(wbytes, torch.uint8, 16)
    assert ws.data_ptr() % 32 == 16
    s_s, sl_s = mla.mla_prefill_fwd_splitkv(*args, causal=True, num_splits=ns, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(s_s, s_a) and torch.equal(sl_s, sl_a)
