"""Pins for the fp64 oracle, independent of the oracle's own code.

Each pin checks the oracle against something fixed from outside it: the
bfloat16 format, a library routine that computes the same special case
(PyTorch's fp64 ``scaled_dot_product_attention`` and ``logsumexp``),
closed forms, and invariants of softmax attention.  The mutation tests at
the bottom plant plausible mistakes in the oracle (on the CPU) and check
that at least one pin fails for each.
"""
import math

import numpy as np
import pytest
import torch

import mla_synth as syn
import oracle
import oracle.attention as oa

torch.set_num_threads(max(1, min(8, torch.get_num_threads())))


def _rand(seed, shape):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape)


def _sdpa(q, k, v, scale, is_causal=False):
    """Library attention for one sequence: q [Lq,H,D], k [Lk,H,D], v [Lk,H,Dv]."""
    tq = torch.from_numpy(np.ascontiguousarray(q.transpose(1, 0, 2)))[None]
    tk = torch.from_numpy(np.ascontiguousarray(k.transpose(1, 0, 2)))[None]
    tv = torch.from_numpy(np.ascontiguousarray(v.transpose(1, 0, 2)))[None]
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=is_causal,
                                                         scale=scale)
    return o[0].numpy().transpose(1, 0, 2)


def _logsumexp(q, k, scale):
    """Library LSE per (head, query): ``[H, Lq]``."""
    s = torch.einsum("qhd,khd->hqk", torch.from_numpy(q), torch.from_numpy(k)) * scale
    return torch.logsumexp(s, dim=-1).numpy()


# ---------------------------------------------------------------------------
# Pins.  Each takes the oracle module so the mutation tests can re-run them.
# ---------------------------------------------------------------------------

def pin_dense_noncausal_vs_library(o=oracle):
    lens_q, lens_k = [7, 33, 1], [12, 5, 40]
    H, scale = 3, 0.37
    q = _rand(1, (sum(lens_q), H, 192))
    k = _rand(2, (sum(lens_k), H, 192))
    v = _rand(3, (sum(lens_k), H, 128))
    cq, ck = syn.cu_seqlens(lens_q), syn.cu_seqlens(lens_k)
    out, lse = o.dense_prefill(q, k, v, cq, ck, scale, causal=False)
    for b in range(3):
        qs, ks = slice(cq[b], cq[b + 1]), slice(ck[b], ck[b + 1])
        ref = _sdpa(q[qs], k[ks], v[ks], scale)
        np.testing.assert_allclose(out[qs], ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[:, qs], _logsumexp(q[qs], k[ks], scale), rtol=0, atol=1e-12)


def pin_dense_causal_square_vs_library(o=oracle):
    lens = [1, 17, 64, 100]
    H, scale = 2, 1.0 / math.sqrt(192)
    q = _rand(4, (sum(lens), H, 192))
    k = _rand(5, (sum(lens), H, 192))
    v = _rand(6, (sum(lens), H, 128))
    cu = syn.cu_seqlens(lens)
    out, lse = o.dense_prefill(q, k, v, cu, cu, scale, causal=True)
    for b in range(len(lens)):
        s = slice(cu[b], cu[b + 1])
        ref = _sdpa(q[s], k[s], v[s], scale, is_causal=True)
        np.testing.assert_allclose(out[s], ref, rtol=0, atol=1e-12)
        for i in range(lens[b]):  # row i sees keys 0..i
            ls = _logsumexp(q[s][i:i + 1], k[s][: i + 1], scale)
            np.testing.assert_allclose(lse[:, cu[b] + i], ls[:, 0], rtol=0, atol=1e-12)


def pin_dense_causal_bottom_right(o=oracle):
    """Lq < Lk: row i equals non-causal attention over keys 0..i+(Lk-Lq)."""
    lq, lk, H, scale = 9, 30, 2, 0.25
    q = _rand(7, (lq, H, 192))
    k = _rand(8, (lk, H, 192))
    v = _rand(9, (lk, H, 128))
    out, lse = o.dense_prefill(q, k, v, [0, lq], [0, lk], scale, causal=True)
    for i in range(lq):
        n = i + (lk - lq) + 1
        ref = _sdpa(q[i:i + 1], k[:n], v[:n], scale)
        np.testing.assert_allclose(out[i:i + 1], ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[:, i], _logsumexp(q[i:i + 1], k[:n], scale)[:, 0],
                                   rtol=0, atol=1e-12)


def pin_causal_first_row_single_key(o=oracle):
    """Causal, Lq == Lk: row 0 sees only key 0 -> O = V[0], LSE = scale q0.k0."""
    L, H, scale = 5, 3, 0.11
    q, k, v = _rand(10, (L, H, 192)), _rand(11, (L, H, 192)), _rand(12, (L, H, 128))
    out, lse = o.dense_prefill(q, k, v, [0, L], [0, L], scale, causal=True)
    np.testing.assert_allclose(out[0], v[0], rtol=0, atol=1e-14)
    for h in range(H):
        s = scale * math.fsum(q[0, h] * k[0, h])
        assert abs(lse[h, 0] - s) < 1e-12


def pin_constant_v(o=oracle):
    """Every visible V row equal to c -> O = c for every row (weights sum to 1)."""
    lens, H = [6, 40], 2
    q, k = _rand(13, (46, H, 192)), _rand(14, (46, H, 192))
    c = _rand(15, (H, 128))
    v = np.broadcast_to(c, (46, H, 128)).copy()
    cu = syn.cu_seqlens(lens)
    out, _ = o.dense_prefill(q, k, v, cu, cu, 0.3, causal=True)
    np.testing.assert_allclose(out, np.broadcast_to(c, out.shape), rtol=0, atol=1e-13)


def pin_zero_q_uniform(o=oracle):
    """Q = 0 -> all scores 0 -> O = mean of visible V rows, LSE = ln(count)."""
    L, H = 20, 2
    q = np.zeros((L, H, 192))
    k, v = _rand(16, (L, H, 192)), _rand(17, (L, H, 128))
    out, lse = o.dense_prefill(q, k, v, [0, L], [0, L], 0.5, causal=True)
    for i in range(L):
        np.testing.assert_allclose(out[i], v[: i + 1].mean(axis=0), rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[:, i], math.log(i + 1), rtol=0, atol=1e-13)


def pin_identical_keys(o=oracle):
    """All keys equal -> LSE = s + ln(n), O = mean(V)."""
    lk, H, scale = 11, 2, 0.2
    q = _rand(18, (3, H, 192))
    k = np.broadcast_to(_rand(19, (1, H, 192)), (lk, H, 192)).copy()
    v = _rand(20, (lk, H, 128))
    out, lse = o.dense_prefill(q, k, v, [0, 3], [0, lk], scale, causal=False)
    for i in range(3):
        for h in range(H):
            s = scale * math.fsum(q[i, h] * k[0, h])
            assert abs(lse[h, i] - (s + math.log(lk))) < 1e-12
        np.testing.assert_allclose(out[i], v.mean(axis=0), rtol=0, atol=1e-13)


def pin_two_key_hand_case(o=oracle):
    """s0 = 0, s1 = ln 3 -> weights 1/4, 3/4 and LSE = ln 4 (scale 1)."""
    q = np.zeros((1, 1, 192)); q[0, 0, 0] = math.log(3.0)
    k = np.zeros((2, 1, 192)); k[1, 0, 0] = 1.0
    v = np.zeros((2, 1, 128)); v[0, 0, :] = 4.0; v[1, 0, :] = -8.0
    out, lse = o.dense_prefill(q, k, v, [0, 1], [0, 2], 1.0, causal=False)
    np.testing.assert_allclose(out[0, 0], np.full(128, 0.25 * 4.0 + 0.75 * -8.0), atol=1e-14)
    assert abs(lse[0, 0] - math.log(4.0)) < 1e-14


def pin_empty_rows(o=oracle):
    """No visible key -> O = 0, LSE = -inf (Lk = 0, and Lq > Lk causal)."""
    H = 2
    q = _rand(21, (4 + 6, H, 192))
    k = _rand(22, (3, H, 192))
    v = _rand(23, (3, H, 128))
    # sequence 0: Lq=4, Lk=0; sequence 1: Lq=6, Lk=3 (rows 0..2 see nothing)
    out, lse = o.dense_prefill(q, k, v, [0, 4, 10], [0, 0, 3], 0.5, causal=True)
    assert np.all(out[:4] == 0) and np.all(np.isneginf(lse[:, :4]))
    assert np.all(out[4:7] == 0) and np.all(np.isneginf(lse[:, 4:7]))
    assert np.all(np.isfinite(lse[:, 7:]))
    np.testing.assert_allclose(out[7], v[0], atol=1e-14)  # row 3 sees key 0 only


def pin_lse_layout_heads_by_tokens(o=oracle):
    """lse is [H, total_q]: lse[h, t] is head h of token t (H != T)."""
    T, H, scale = 5, 3, 0.4
    q, k, v = _rand(24, (T, H, 192)), _rand(25, (7, H, 192)), _rand(26, (7, H, 128))
    _, lse = o.dense_prefill(q, k, v, [0, T], [0, 7], scale, causal=False)
    assert lse.shape == (H, T)
    np.testing.assert_allclose(lse, _logsumexp(q, k, scale), rtol=0, atol=1e-12)


def pin_merge_equals_union(o=oracle):
    """merge(attn over A, attn over B) = attn over A u B."""
    H, scale, lq = 3, 0.3, 8
    q = _rand(27, (lq, H, 192))
    ka, va = _rand(28, (13, H, 192)), _rand(29, (13, H, 128))
    kb, vb = _rand(30, (21, H, 192)), _rand(31, (21, H, 128))
    oa_, la = o.dense_prefill(q, ka, va, [0, lq], [0, 13], scale, causal=False)
    ob_, lb = o.dense_prefill(q, kb, vb, [0, lq], [0, 21], scale, causal=False)
    om, lm = o.attn_merge(oa_, la, ob_, lb)
    ku, vu = np.concatenate([ka, kb]), np.concatenate([va, vb])
    ref = _sdpa(q, ku, vu, scale)
    np.testing.assert_allclose(om, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lm, _logsumexp(q, ku, scale), rtol=0, atol=1e-12)


def pin_chunked_prefix_plus_self(o=oracle):
    """Unmasked prefix pass + causal self pass, merged, = one bottom-right call.

    This is the context-chunk use of the vLLM backend: the merged result
    equals causal attention of the chunk over [prefix, chunk] with Lq < Lk.
    """
    H, scale, lq, lp = 2, 0.2, 10, 25
    q = _rand(32, (lq, H, 192))
    kp, vp = _rand(33, (lp, H, 192)), _rand(34, (lp, H, 128))
    ks, vs = _rand(35, (lq, H, 192)), _rand(36, (lq, H, 128))
    o1, l1 = o.dense_prefill(q, kp, vp, [0, lq], [0, lp], scale, causal=False)
    o2, l2 = o.dense_prefill(q, ks, vs, [0, lq], [0, lq], scale, causal=True)
    om, lm = o.attn_merge(o1, l1, o2, l2)
    ku, vu = np.concatenate([kp, ks]), np.concatenate([vp, vs])
    for i in range(lq):
        n = lp + i + 1
        np.testing.assert_allclose(om[i:i + 1], _sdpa(q[i:i + 1], ku[:n], vu[:n], scale),
                                   rtol=0, atol=1e-12)
        np.testing.assert_allclose(lm[:, i], _logsumexp(q[i:i + 1], ku[:n], scale)[:, 0],
                                   rtol=0, atol=1e-12)


def pin_merge_closed_forms(o=oracle):
    T, H, D = 3, 2, 128
    a, b = _rand(37, (T, H, D)), _rand(38, (T, H, D))
    la = np.array([[0.0, -np.inf, 5.0], [1.0, -np.inf, -np.inf]])
    lb = np.array([[math.log(3.0), 2.0, -np.inf], [-np.inf, -np.inf, 0.5]])
    out, lse = o.attn_merge(a, la, b, lb)
    np.testing.assert_allclose(out[0, 0], 0.25 * a[0, 0] + 0.75 * b[0, 0], atol=1e-14)
    assert abs(lse[0, 0] - math.log(4.0)) < 1e-14
    np.testing.assert_allclose(out[1, 0], b[1, 0], atol=0)      # a side empty
    np.testing.assert_allclose(out[2, 0], a[2, 0], atol=0)      # b side empty
    assert lse[0, 1] == 2.0 and lse[0, 2] == 5.0
    assert np.all(out[1, 1] == 0) and np.isneginf(lse[1, 1])     # both empty


def _sparse_small(seed=40, T=6, H=4, N=50, K=16, first=3):
    d = syn.sparse_case(T, H, N, K, first, seed)
    return d


def pin_sparse_vs_library(o=oracle):
    d = _sparse_small()
    q = oa.bf16_bits_to_f64(d["q"]); kv = oa.bf16_bits_to_f64(d["kv"])
    out, lse = o.sparse_prefill(q, kv, d["indices"], d["scale"])
    for t in range(q.shape[0]):
        ids = d["indices"][t]; ids = ids[ids >= 0]
        sel = kv[ids]
        kk = np.broadcast_to(sel[:, None, :], (len(ids), q.shape[1], 576)).copy()
        vv = np.ascontiguousarray(kk[:, :, :512])
        ref = _sdpa(q[t:t + 1], kk, vv, d["scale"])
        np.testing.assert_allclose(out[t:t + 1], ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[:, t], _logsumexp(q[t:t + 1], kk, d["scale"])[:, 0],
                                   rtol=0, atol=1e-12)


def pin_sparse_single_index(o=oracle):
    """Only one valid slot -> O = that row's first 512 dims, LSE = scale q.kv."""
    T, H, N, K = 3, 2, 9, 8
    q, kv = _rand(41, (T, H, 576)), _rand(42, (N, 576))
    idx = np.full((T, K), -1, dtype=np.int32)
    idx[0, 0] = 4          # left-aligned
    idx[1, 5] = 7          # valid slot in the middle, -1 around it
    idx[2, :] = -1; idx[2, 3] = 0; idx[2, 6] = N + 3   # out-of-range index is padding
    out, lse = o.sparse_prefill(q, kv, idx, 0.7)
    for t, r in [(0, 4), (1, 7), (2, 0)]:
        np.testing.assert_allclose(out[t], np.broadcast_to(kv[r, :512], (H, 512)), atol=1e-14)
        for h in range(H):
            assert abs(lse[h, t] - 0.7 * math.fsum(q[t, h] * kv[r])) < 1e-12


def pin_sparse_all_padding(o=oracle):
    q, kv = _rand(43, (2, 3, 576)), _rand(44, (5, 576))
    idx = np.full((2, 4), -1, dtype=np.int32)
    out, lse = o.sparse_prefill(q, kv, idx, 0.5)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def pin_sparse_permutation_invariant(o=oracle):
    d = _sparse_small(seed=45, first=30)
    q = oa.bf16_bits_to_f64(d["q"]); kv = oa.bf16_bits_to_f64(d["kv"])
    o1, l1 = o.sparse_prefill(q, kv, d["indices"], d["scale"])
    perm = d["indices"][:, ::-1].copy()
    o2, l2 = o.sparse_prefill(q, kv, perm, d["scale"])
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


def pin_sparse_all_visible_equals_dense(o=oracle):
    """Indices = every causally visible row -> dense causal attention with
    K = kv (one head broadcast) and V = kv[:, :512]."""
    N, H, scale = 24, 2, 0.15
    q, kv = _rand(46, (N, H, 576)), _rand(47, (N, 576))
    idx = np.full((N, N), -1, dtype=np.int32)
    for t in range(N):
        idx[t, : t + 1] = np.arange(t + 1)
    out_s, lse_s = o.sparse_prefill(q, kv, idx, scale)
    k = np.broadcast_to(kv[:, None, :], (N, H, 576)).copy()
    v = np.ascontiguousarray(k[:, :, :512])
    ref = _sdpa(q, k, v, scale, is_causal=True)
    np.testing.assert_allclose(out_s, ref, rtol=0, atol=1e-12)


PINS = [pin_dense_noncausal_vs_library, pin_dense_causal_square_vs_library,
        pin_dense_causal_bottom_right, pin_causal_first_row_single_key, pin_constant_v,
        pin_zero_q_uniform, pin_identical_keys, pin_two_key_hand_case, pin_empty_rows,
        pin_lse_layout_heads_by_tokens, pin_merge_equals_union, pin_chunked_prefix_plus_self,
        pin_merge_closed_forms, pin_sparse_vs_library, pin_sparse_single_index,
        pin_sparse_all_padding, pin_sparse_permutation_invariant,
        pin_sparse_all_visible_equals_dense]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


# ---------------------------------------------------------------------------
# bf16 decoding and the generator
# ---------------------------------------------------------------------------

def test_bf16_decode_fixed_by_format():
    bits = np.array([0x3F80, 0xC000, 0x4049, 0x3F81, 0x0001, 0x7F7F, 0x0000, 0x8000],
                    dtype=np.uint16)
    want = [1.0, -2.0, 3.140625, 1.0078125, 2.0 ** -133, (2 - 2 ** -7) * 2.0 ** 127, 0.0, -0.0]
    got = oa.bf16_bits_to_f64(bits)
    assert list(got) == want


def test_generator_rounding_matches_torch():
    x = np.random.Generator(np.random.PCG64(0)).standard_normal(100000).astype(np.float32)
    x[:4] = [1.00390625, 1.01171875, -1.00390625, 3.0e-39]  # ties and a subnormal
    ours = syn.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_generator_deterministic_and_normal():
    a = syn.normal_bf16(7, (3, 1 << 21))
    b = syn.normal_bf16(7, (3, 1 << 21))
    assert np.array_equal(a, b)
    v = oa.bf16_bits_to_f64(a)
    assert abs(v.mean()) < 5e-3 and abs(v.std() - 1.0) < 5e-3


def test_generator_topk_indices():
    idx = syn.topk_indices(3, 40, 64, 16, first_pos=0)
    for t in range(40):
        vis = min(64, t + 1)
        row = idx[t]
        n_valid = min(vis, 16)
        assert np.all(row[:n_valid] >= 0) and np.all(row[:n_valid] < vis)
        assert np.all(row[n_valid:] == -1)
        assert len(set(row[:n_valid].tolist())) == n_valid


def test_generator_lengths_and_cu():
    lens = syn.uniform_lengths(2, 8, 512, 4096)
    assert len(lens) == 8 and all(512 <= x <= 4096 for x in lens)
    cu = syn.cu_seqlens(lens)
    assert cu.dtype == np.int32 and cu[0] == 0 and np.all(np.diff(cu) == lens)


def test_flop_counts():
    assert oracle.dense_flops([4], [4], 1, True) == 2 * 320 * 10
    assert oracle.dense_flops([3], [5], 2, True) == 2 * 320 * 2 * (3 + 4 + 5)
    assert oracle.dense_flops([3], [5], 2, False) == 2 * 320 * 2 * 15
    idx = np.array([[0, 1, -1], [2, -1, -1]])
    assert oracle.sparse_flops(idx, 10, 4) == 2 * (576 + 512) * 4 * 3


def test_flop_counts_match_the_counted_mask():
    """The FLOP numerator of every TFLOP/s figure: visible (query, key) pairs
    counted on an explicit bottom-right mask matrix (numpy's tril with the
    diagonal offset Lk - Lq) for square and ragged shapes."""
    g = np.random.Generator(np.random.PCG64(11))
    shapes = [(1, 1), (1, 300), (300, 1), (128, 128), (129, 127), (512, 4096), (4096, 512)]
    shapes += [tuple(int(x) for x in g.integers(0, 700, size=2)) for _ in range(20)]
    for lq, lk in shapes:
        mask = np.tril(np.ones((lq, lk), dtype=np.int64), k=lk - lq)
        assert oracle.dense_flops([lq], [lk], 3, True) == 2 * 320 * 3 * int(mask.sum()), (lq, lk)
        assert oracle.dense_flops([lq], [lk], 3, False) == 2 * 320 * 3 * lq * lk


# ---------------------------------------------------------------------------
# Attention sinks and the e4m3 output encoding
# ---------------------------------------------------------------------------

def _sink_case(seed=61, lens=(5, 1, 9), heads=3, causal=True):
    g = np.random.Generator(np.random.PCG64(seed))
    lens = list(lens)
    tq = sum(lens)
    q = g.standard_normal((tq, heads, 192))
    k = g.standard_normal((tq, heads, 192))
    v = g.standard_normal((tq, heads, 128))
    cu = np.concatenate([[0], np.cumsum(lens)])
    sinks = g.standard_normal(heads) * 2.0
    return q, k, v, cu, 1.0 / np.sqrt(192), causal, sinks


def pin_sinks_minus_inf_is_no_sink():
    q, k, v, cu, sc, causal, _ = _sink_case()
    o, l = oracle.dense_prefill_sinks(q, k, v, cu, cu, sc, causal, np.full(3, -np.inf))
    o0, l0 = oracle.dense_prefill(q, k, v, cu, cu, sc, causal)
    assert np.allclose(o, o0, atol=1e-12) and np.allclose(l, l0, atol=1e-12)


def pin_sinks_single_key_closed_form():
    # causal row 0 of each sequence sees one key: O = v0 e^x0 / (e^x0 + e^s)
    q, k, v, cu, sc, causal, sinks = _sink_case()
    o, l = oracle.dense_prefill_sinks(q, k, v, cu, cu, sc, True, sinks)
    for b in range(len(cu) - 1):
        r = int(cu[b])
        for h in range(3):
            x = sc * float(q[r, h] @ k[r, h])
            w = np.exp(x) / (np.exp(x) + np.exp(sinks[h]))
            assert np.allclose(o[r, h], w * v[r, h], atol=1e-12)
            assert abs(l[h, r] - np.log(np.exp(x) + np.exp(sinks[h]))) < 1e-12


def pin_sinks_row_without_keys():
    q, k, v, _, sc, _, sinks = _sink_case()
    cu_q, cu_k = np.array([0, 4]), np.array([0, 0])  # no keys at all
    o, l = oracle.dense_prefill_sinks(q[:4], k[:0], v[:0], cu_q, cu_k, sc, True, sinks)
    assert np.all(o == 0) and np.allclose(l, sinks[:, None].repeat(4, axis=1))


def pin_sinks_are_a_zero_valued_extra_key():
    # the sink merges like a partial result with O = 0 and LSE = s_h
    q, k, v, cu, sc, causal, sinks = _sink_case(causal=False)
    o, l = oracle.dense_prefill_sinks(q, k, v, cu, cu, sc, False, sinks)
    o0, l0 = oracle.dense_prefill(q, k, v, cu, cu, sc, False)
    om, lm = oracle.attn_merge(o0, l0, np.zeros_like(o0), np.repeat(sinks[:, None], o0.shape[0], 1))
    assert np.allclose(o, om, atol=1e-12) and np.allclose(l, lm, atol=1e-12)


SINK_PINS = [pin_sinks_minus_inf_is_no_sink, pin_sinks_single_key_closed_form,
             pin_sinks_row_without_keys, pin_sinks_are_a_zero_valued_extra_key]


@pytest.mark.parametrize("pin", SINK_PINS, ids=lambda f: f.__name__)
def test_sink_pin(pin):
    pin()


def test_e4m3_every_finite_code_round_trips():
    codes = np.arange(256)
    vals = oracle.e4m3_decode(codes)
    finite = ~np.isnan(vals)
    assert finite.sum() == 254  # 0x7F and 0xFF are NaN
    assert np.array_equal(oracle.e4m3_decode(oracle.e4m3_quantize(vals[finite], 1.0)), vals[finite])
    assert vals[finite].max() == 448.0 and oracle.e4m3_decode([0x01])[0] == 2.0 ** -9


def test_e4m3_matches_torch_inside_the_range():
    """torch's float8_e4m3fn cast (round to nearest even) on a dense sweep,
    the subnormal range and exact midpoints; torch turns values past the
    range into NaN, so the sweep stops below 464."""
    import torch
    g = np.random.Generator(np.random.PCG64(62))
    x = np.concatenate([np.linspace(-463.9, 463.9, 100001), g.standard_normal(20000) * 1e-2,
                        (np.arange(1, 64) + 0.5) * 2.0 ** -9])
    ref = torch.tensor(x, dtype=torch.float64).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_quantize(x, 1.0)
    assert np.array_equal(oracle.e4m3_decode(got), oracle.e4m3_decode(ref))


def test_e4m3_saturates_and_divides_by_the_scale():
    assert list(oracle.e4m3_decode(oracle.e4m3_quantize([464.0, 1e6, -1e9, 500.0], 1.0))) == \
        [448.0, 448.0, -448.0, 448.0]
    x = np.linspace(-30, 30, 997)
    assert np.array_equal(oracle.e4m3_quantize(x, 0.25), oracle.e4m3_quantize(x / 0.25, 1.0))


# ---------------------------------------------------------------------------
# Mutation tests: plant a mistake in the oracle; some pin must fail.
# ---------------------------------------------------------------------------

def _fails_some_pin(pins):
    for p in pins:
        try:
            p()
        except AssertionError:
            return True
    return False


def test_mutant_causal_off_by_one(monkeypatch):
    real = oa.visible_key_count
    monkeypatch.setattr(oa, "visible_key_count",
                        lambda i, lq, lk, c: real(i, lq, lk, c) - 1 if c else lk)
    assert _fails_some_pin([pin_causal_first_row_single_key, pin_dense_causal_square_vs_library])


def test_mutant_top_left_causal(monkeypatch):
    monkeypatch.setattr(oa, "visible_key_count",
                        lambda i, lq, lk, c: max(0, min(lk, i + 1)) if c else lk)
    assert _fails_some_pin([pin_dense_causal_bottom_right])


def test_mutant_lse_without_max(monkeypatch):
    real = oa._softmax_rows

    def bad(scores, counts):
        e, row_max, z = real(scores, counts)
        return e, np.zeros_like(row_max), z  # drops the max from the LSE
    monkeypatch.setattr(oa, "_softmax_rows", bad)
    assert _fails_some_pin([pin_dense_noncausal_vs_library])


def test_mutant_dropped_scale(monkeypatch):
    real = oa.dense_prefill
    monkeypatch.setattr(oracle, "dense_prefill",
                        lambda q, k, v, cq, ck, s, causal, **kw: real(q, k, v, cq, ck, 1.0, causal, **kw))
    assert _fails_some_pin([lambda: pin_dense_noncausal_vs_library(oracle)])


def test_mutant_merge_sign(monkeypatch):
    def bad(o_a, lse_a, o_b, lse_b):
        return oa.attn_merge(o_a, -np.asarray(lse_a), o_b, -np.asarray(lse_b))
    monkeypatch.setattr(oracle, "attn_merge", bad)
    assert _fails_some_pin([pin_merge_equals_union])


def test_mutant_sparse_negative_index_wraps(monkeypatch):
    """Python's kv[-1] is the last row: forgetting to drop -1 must be caught."""
    real = oa.sparse_prefill

    def bad(q, kv, indices, scale, v_dim=512, tokens=None):
        idx = np.asarray(indices).copy()
        idx[idx < 0] += np.asarray(kv).shape[0]
        return real(q, kv, idx, scale, v_dim, tokens)
    monkeypatch.setattr(oracle, "sparse_prefill", bad)
    assert _fails_some_pin([pin_sparse_single_index])


def test_mutant_sparse_value_dims(monkeypatch):
    """Taking V from the last 512 latent dims instead of the first 512."""
    real = oa.sparse_prefill

    def bad(q, kv, indices, scale, v_dim=512, tokens=None):
        kv = np.asarray(kv)
        shifted = np.concatenate([kv[:, 64:], kv[:, :64]], axis=1)
        o, _ = real(q, shifted, indices, scale, v_dim, tokens)
        _, l = real(q, kv, indices, scale, v_dim, tokens)
        return o, l
    monkeypatch.setattr(oracle, "sparse_prefill", bad)
    assert _fails_some_pin([pin_sparse_single_index])


def test_row_subsets_match_full_evaluation():
    """Evaluating a subset of rows/tokens gives the same values as the full run."""
    lens = [5, 130, 64]
    d = syn.dense_case(lens, lens, 2, seed=50)
    full_o, full_l = oracle.dense_prefill(d["q"], d["k"], d["v"], d["cu_q"], d["cu_k"],
                                          d["scale"], True)
    rows = [134, 0, 7, 198, 4]
    o, l = oracle.dense_prefill(d["q"], d["k"], d["v"], d["cu_q"], d["cu_k"], d["scale"], True,
                                rows=rows, row_group=3)
    # BLAS may sum in another order for another matrix shape: equal to ~1 ulp.
    np.testing.assert_allclose(o, full_o[rows], rtol=0, atol=1e-13)
    np.testing.assert_allclose(l, full_l[:, rows], rtol=0, atol=1e-13)
    s = _sparse_small(seed=51)
    so, sl = oracle.sparse_prefill(s["q"], s["kv"], s["indices"], s["scale"])
    to, tl = oracle.sparse_prefill(s["q"], s["kv"], s["indices"], s["scale"], tokens=[5, 2])
    np.testing.assert_allclose(to, so[[5, 2]], rtol=0, atol=1e-13)
    np.testing.assert_allclose(tl, sl[:, [5, 2]], rtol=0, atol=1e-13)


def test_exp2_polynomial_constants_error_bound():
    """The cubic used by the kernel's FMA-pipe exp2 (Cody-Waite reduction to
    f in [-1/2, 1/2], 2^rint(t) folded into the exponent) stays within 1e-4
    relative error over t in [-125, 8], emulated step by step in float32."""
    import re
    src = open(ROOT_PTX).read()
    block = src[src.index("Exp2PolyConsts exp2_poly_consts()"):]
    c = [np.float32(float(v)) for v in re.findall(r"splat_f32x2\(([0-9.e+-]+)f\)", block)[1:5]]
    x = np.linspace(-125, 8, 400001).astype(np.float32)
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic).astype(np.float32)).astype(np.float32)
    p = c[3]
    for k in (2, 1, 0):
        p = (p * f + c[k]).astype(np.float32)
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23))
    res = (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32).astype(np.float64)
    rel = np.abs(res / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1e-4


ROOT_PTX = __import__("os").path.join(__import__("os").path.dirname(__import__("os").path.dirname(
    __import__("os").path.abspath(__file__))), "mla_prefill_attention_causal_b200", "csrc", "ptx.cuh")


def test_mutant_sink_scaled_like_a_score(monkeypatch):
    # the sink is already in score units: scaling it again must be caught
    real = oracle.dense_prefill_sinks

    def mutant(q, k, v, cu_q, cu_k, sc, causal, sinks, rows=None):
        return real(q, k, v, cu_q, cu_k, sc, causal, np.asarray(sinks) * sc, rows=rows)
    monkeypatch.setattr(oracle, "dense_prefill_sinks", mutant)
    assert _fails_some_pin(SINK_PINS)


def test_mutant_sink_left_out_of_the_lse(monkeypatch):
    real = oracle.dense_prefill_sinks

    def mutant(q, k, v, cu_q, cu_k, sc, causal, sinks, rows=None):
        o, _ = real(q, k, v, cu_q, cu_k, sc, causal, sinks, rows=rows)
        _, l = oracle.dense_prefill(q, k, v, cu_q, cu_k, sc, causal, rows=rows)
        return o, l
    monkeypatch.setattr(oracle, "dense_prefill_sinks", mutant)
    assert _fails_some_pin(SINK_PINS)
