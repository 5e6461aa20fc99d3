"""fp64 oracle for MLA prefill attention (test infrastructure only).

Sources, by page and section:

* SparseFlashMla README (ops-transformer ``attention/sparse_flash_mla``),
  "Description -- Formula": ``O = softmax(Q @ K~^T * softmax_scale) @ V~``
  where ``K~ = V~`` are the rows that actually take part.  This is the only
  formula the pages print; it fixes the dense and the sparse computation.
* vLLM ``vllm/v1/attention/backends/mla/prefill/flash_attn.py``,
  ``FA4MLAPrefillKernel.dispatch``: packed shapes q ``(tokens, heads,
  nope+rope)``, k the same, v ``(tokens, heads, v_head_dim)``; K/V are already
  expanded to every head (module comment on ``qhead_per_kvhead=1``);
  ``FlashAttnPrefillBackend.run_prefill_new_tokens``: causal, same
  cu_seqlens for q and k; ``run_prefill_context_chunk``: the context chunk is
  unmasked and returns the LSE for a later merge.
* Sgl project Sglang FA4 Interface, "I/O Contract": ``cu_seqlens_*`` int32
  ``(batch+1,)``; output has ``head_dim_v``; ``lse`` is float32.
* SparseFlashMla README, "Parameters": sparse index ``-1`` is an invalid or
  padded slot; "Constraints": index shape ``[Q_T, KV_N=1, K]`` (one list per
  token shared by all heads), ``cu_seqlens`` starts at 0 and never decreases;
  "ori_mask_mode": mode 3 is *RightDownCausal*.
* Mojo ``mla_prefill_branch_sparse_fp8``: the absorbed sparse prefill runs
  over the BF16 latent cache with the indices already mapped to physical
  rows.

Readings where the pages are silent (each one is listed with its reason in
the repository's design notes):

* causal alignment: bottom-right (RightDownCausal) -- query ``i`` of a
  sequence with ``Lq`` queries and ``Lk`` keys sees key ``j`` iff
  ``j <= i + (Lk - Lq)``; identical to ``j <= i`` when ``Lq == Lk``;
* LSE: natural log of ``sum_j exp(scale * q.k_j)``, stored ``[heads, tokens]``;
* a row that sees no key: output 0, LSE ``-inf``;
* sparse: any index ``< 0`` or ``>= num_rows`` is padding; each slot counts
  once; V is the first 512 of the 576 latent dims;
* merge: the log-sum-exp identity; a ``-inf`` side has weight 0.
* attention sinks (FA4 interface feature list: "learnable sink tokens";
  SparseFlashMla "sinks"; Mojo ``attn_sink_ptr``; the arithmetic is not
  given): one logit ``s_h`` per head, in the units of the scaled scores,
  that joins each row's softmax with a zero value -- ``O = sum_j e^x_j v_j /
  (e^s_h + sum_j e^x_j)`` -- and counts in the LSE; a row with no visible
  key gets ``O = 0`` and ``LSE = s_h``;
* FP8 static output scale (vLLM ``supports_quant_output``:
  ``kFp8StaticTensorSym``; ``output_scale``): the output is
  ``e4m3(O / output_scale)``, rounded to nearest even and saturated to the
  largest finite e4m3 value, 448 (the static symmetric scheme clamps to
  the format's range).

Everything is computed in float64 from the exact bf16 inputs.  There is no
tiling and no online softmax: each row takes its maximum, then its sum.
Rows are independent, so they may be evaluated in groups to bound memory.
"""
from __future__ import annotations

import numpy as np


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen raw bfloat16 bit patterns exactly to float64.

    bfloat16 is the top half of an IEEE-754 binary32, so shifting the bits
    left by 16 gives the float32 with the same value.
    """
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def _as_f64(x: np.ndarray) -> np.ndarray:
    if x.dtype == np.uint16:
        return bf16_bits_to_f64(x)
    return np.asarray(x, dtype=np.float64)


def visible_key_count(i: int, lq: int, lk: int, causal: bool) -> int:
    """Number of keys query ``i`` may attend to; they are keys ``[0, count)``.

    Non-causal: all ``lk`` keys.  Causal (bottom-right): keys
    ``j <= i + (lk - lq)``, clipped to ``[0, lk]``.
    """
    if not causal:
        return lk
    return max(0, min(lk, i + (lk - lq) + 1))


def _softmax_rows(scores: np.ndarray, counts: np.ndarray):
    """Row-wise softmax of ``scores[r, :counts[r]]`` (the rest is masked).

    Returns the weights (0 on masked entries), the row maxima and the row
    sums ``Z = sum exp(s - max)``; rows with ``count == 0`` get weight 0,
    max ``-inf`` and ``Z = 0``.
    """
    n_rows, n_cols = scores.shape
    cols = np.arange(n_cols)[None, :]
    masked = np.where(cols < counts[:, None], scores, -np.inf)
    row_max = masked.max(axis=1) if n_cols else np.full(n_rows, -np.inf)
    safe_max = np.where(np.isfinite(row_max), row_max, 0.0)
    e = np.exp(masked - safe_max[:, None])
    z = e.sum(axis=1)
    return e, row_max, z


def dense_prefill(q, k, v, cu_seqlens_q, cu_seqlens_k, softmax_scale: float,
                  causal: bool, rows=None, row_group: int = 2048):
    """Dense varlen MLA prefill: ``O = softmax(scale * Q K^T [+mask]) V``.

    Args:
      q: ``[total_q, H, Dqk]`` (bf16 bits as uint16, or real values).
      k: ``[total_k, H, Dqk]``;  v: ``[total_k, H, Dv]``.
      cu_seqlens_q / cu_seqlens_k: ``[B+1]`` prefix sums.
      softmax_scale: the scale applied to every ``q . k`` product.
      causal: bottom-right causal mask when true.
      rows: optional sequence of global query rows to evaluate.

    Returns ``(out, lse)`` in float64: ``out [R, H, Dv]`` and ``lse [H, R]``
    where R runs over all query rows in order (``rows=None``) or over the
    given rows in the given order.  bf16 inputs are widened one
    (sequence, head) slice at a time.
    """
    cu_q = np.asarray(cu_seqlens_q, dtype=np.int64)
    cu_k = np.asarray(cu_seqlens_k, dtype=np.int64)
    total_q, num_heads, _ = q.shape
    dv = v.shape[2]
    sel_rows = np.arange(total_q) if rows is None else np.asarray(list(rows), dtype=np.int64)
    out = np.zeros((sel_rows.size, num_heads, dv))
    lse = np.zeros((num_heads, sel_rows.size))
    seq_of = np.searchsorted(cu_q, sel_rows, side="right") - 1
    scale = float(softmax_scale)

    for b in np.unique(seq_of):
        q0, q1 = int(cu_q[b]), int(cu_q[b + 1])
        k0, k1 = int(cu_k[b]), int(cu_k[b + 1])
        lq, lk = q1 - q0, k1 - k0
        pos = np.nonzero(seq_of == b)[0]          # positions in the output
        local = sel_rows[pos] - q0                # rows within the sequence
        counts_all = np.array([visible_key_count(int(i), lq, lk, causal)
                               for i in local], dtype=np.int64)
        for h in range(num_heads):
            kb = _as_f64(k[k0:k1, h, :])
            vb = _as_f64(v[k0:k1, h, :])
            for g in range(0, local.size, row_group):
                sel = local[g:g + row_group]
                dst = pos[g:g + row_group]
                counts = counts_all[g:g + row_group]
                scores = scale * (_as_f64(q[q0 + sel, h, :]) @ kb.T)
                e, row_max, z = _softmax_rows(scores, counts)
                has = z > 0
                o = np.zeros((sel.size, dv))
                o[has] = (e[has] @ vb) / z[has, None]
                out[dst, h, :] = o
                with np.errstate(divide="ignore"):
                    lse[h, dst] = np.where(has, row_max + np.log(np.where(has, z, 1.0)),
                                           -np.inf)
    return out, lse


def dense_prefill_sinks(q, k, v, cu_seqlens_q, cu_seqlens_k, softmax_scale: float,
                        causal: bool, sinks, rows=None):
    """``dense_prefill`` with one attention-sink logit per head.

    Each row's softmax runs over its visible keys' scaled scores and the
    head's sink logit ``sinks[h]``; the sink has no value.  Returns ``(out,
    lse)`` like ``dense_prefill``: ``lse = log(e^s_h + sum_j e^x_j)``, and a
    row without visible keys gets ``out = 0``, ``lse = s_h``.
    """
    cu_q = np.asarray(cu_seqlens_q, dtype=np.int64)
    cu_k = np.asarray(cu_seqlens_k, dtype=np.int64)
    sk = np.asarray(sinks, dtype=np.float64)
    total_q, num_heads, _ = q.shape
    dv = v.shape[2]
    sel_rows = np.arange(total_q) if rows is None else np.asarray(list(rows), dtype=np.int64)
    out = np.zeros((sel_rows.size, num_heads, dv))
    lse = np.zeros((num_heads, sel_rows.size))
    seq_of = np.searchsorted(cu_q, sel_rows, side="right") - 1
    for n, (r, b) in enumerate(zip(sel_rows, seq_of)):
        q0, k0, k1 = int(cu_q[b]), int(cu_k[b]), int(cu_k[b + 1])
        lq, lk = int(cu_q[b + 1]) - q0, k1 - k0
        cnt = visible_key_count(int(r) - q0, lq, lk, causal)
        for h in range(num_heads):
            x = float(softmax_scale) * (_as_f64(k[k0:k0 + cnt, h, :]) @ _as_f64(q[r, h, :]))
            m = max(float(x.max()) if cnt else -np.inf, sk[h])
            e = np.exp(x - m)
            z = float(e.sum()) + np.exp(sk[h] - m)
            out[n, h, :] = (e @ _as_f64(v[k0:k0 + cnt, h, :])) / z if cnt else 0.0
            lse[h, n] = m + np.log(z)
    return out, lse


def e4m3_decode(codes):
    """Values of e4m3 codes (1 sign, 4 exponent bits with bias 7, 3 mantissa
    bits; exponent 0 is subnormal, m * 2^-9; 0x7F and 0xFF are NaN, there is
    no infinity)."""
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((c & 0x7F) == 0x7F, np.nan, val)
    return sign * val


def e4m3_quantize(x, scale: float):
    """e4m3 codes of ``x / scale``: round to nearest (ties to an even
    mantissa) on the format's grid -- spacing 2^(e - 3) in binade
    [2^e, 2^(e+1)), e >= -6, and 2^-9 below 2^-6 -- and saturate at +-448."""
    y = np.asarray(x, dtype=np.float64) / float(scale)
    a = np.minimum(np.abs(y), 448.0)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -6.0)
    quantum = np.exp2(e - 3.0)
    steps = np.round(a / quantum)          # numpy rounds halves to even
    v = np.minimum(steps * quantum, 448.0)
    # code of v: normal values as (exponent, mantissa), subnormals below 2^-6
    ev = np.floor(np.log2(np.where(v > 0, v, 1.0)))
    normal = v >= 2.0 ** -6
    mant = np.where(normal, np.round(v / np.exp2(ev) * 8.0) - 8.0, np.round(v / 2.0 ** -9))
    expo = np.where(normal, ev + 7.0, 0.0)
    code = (expo.astype(np.int64) << 3) | mant.astype(np.int64)
    return np.where(y < 0, code | 0x80, code).astype(np.uint8)


def attn_merge(o_a, lse_a, o_b, lse_b):
    """Merge two partial attention results over disjoint key sets A and B.

    With ``M = max(lse_a, lse_b)`` (per token and head):
    ``lse = M + ln(exp(lse_a - M) + exp(lse_b - M))`` and
    ``out = exp(lse_a - lse) * o_a + exp(lse_b - lse) * o_b``.
    A side whose LSE is ``-inf`` (no visible key) has weight 0; when both
    are ``-inf`` the result is ``out = 0``, ``lse = -inf``.

    Shapes: ``o_* [T, H, D]``, ``lse_* [H, T]``.
    """
    o_a = _as_f64(o_a)
    o_b = _as_f64(o_b)
    la = np.asarray(lse_a, dtype=np.float64).T  # [T, H]
    lb = np.asarray(lse_b, dtype=np.float64).T
    m = np.maximum(la, lb)
    both_empty = ~np.isfinite(m)
    m_safe = np.where(both_empty, 0.0, m)
    wa = np.exp(la - m_safe)
    wb = np.exp(lb - m_safe)
    zsum = wa + wb
    with np.errstate(divide="ignore", invalid="ignore"):
        lse = np.where(both_empty, -np.inf, m_safe + np.log(np.where(both_empty, 1.0, zsum)))
        fa = np.where(both_empty, 0.0, wa / np.where(both_empty, 1.0, zsum))
        fb = np.where(both_empty, 0.0, wb / np.where(both_empty, 1.0, zsum))
    out = fa[:, :, None] * o_a + fb[:, :, None] * o_b
    return out, lse.T.copy()


def sparse_prefill(q, kv, indices, softmax_scale: float, v_dim: int = 512,
                   tokens=None):
    """Absorbed top-k sparse MLA prefill over a shared latent cache.

    For token ``t`` the keys are the cache rows ``kv[indices[t, r]]`` for
    every slot ``r`` whose index is a valid row (``0 <= idx < num_rows``);
    all heads share the list.  K~ = V~ are the same rows; the value is their
    first ``v_dim`` dims.  ``O[t, h] = softmax_r(scale * q[t,h] . kv_r) @
    kv_r[:v_dim]``; ``lse[h, t]`` is the natural log-sum-exp of the scores.

    Shapes: ``q [T, H, Dl]``, ``kv [N, Dl]``, ``indices [T, K]`` int.
    Returns float64 ``out [R, H, v_dim]`` and ``lse [H, R]`` with R running
    over all tokens (``tokens=None``) or over the given tokens in order.
    """
    kv = _as_f64(kv)
    idx = np.asarray(indices, dtype=np.int64)
    num_tokens, num_heads, _ = q.shape
    num_rows = kv.shape[0]
    todo = np.arange(num_tokens) if tokens is None else np.asarray(list(tokens), dtype=np.int64)
    out = np.zeros((todo.size, num_heads, v_dim))
    lse = np.zeros((num_heads, todo.size))
    scale = float(softmax_scale)
    for pos, t in enumerate(todo):
        t = int(t)
        row_ids = idx[t]
        row_ids = row_ids[(row_ids >= 0) & (row_ids < num_rows)]
        if row_ids.size == 0:
            out[pos] = 0.0
            lse[:, pos] = -np.inf
            continue
        sel = kv[row_ids]                             # [n, Dl]
        scores = scale * (_as_f64(q[t]) @ sel.T)      # [H, n]
        counts = np.full(num_heads, row_ids.size, dtype=np.int64)
        e, row_max, z = _softmax_rows(scores, counts)
        out[pos] = (e @ sel[:, :v_dim]) / z[:, None]
        lse[:, pos] = row_max + np.log(z)
    return out, lse


def dense_flops(lens_q, lens_k, num_heads: int, causal: bool,
                qk_dim: int = 192, v_dim: int = 128) -> int:
    """Algorithmic FLOPs: ``2 * (Dqk + Dv) * H * (visible query-key pairs)``."""
    pairs = 0
    for lq, lk in zip(lens_q, lens_k):
        if not causal:
            pairs += lq * lk
        else:
            pairs += sum(visible_key_count(i, lq, lk, True) for i in range(lq)) \
                if lq != lk else lq * (lq + 1) // 2
    return 2 * (qk_dim + v_dim) * num_heads * pairs


def sparse_flops(indices, num_rows: int, num_heads: int,
                 qk_dim: int = 576, v_dim: int = 512) -> int:
    """Algorithmic FLOPs of the sparse path: ``2 * (Dl + Dv) * H * valid slots``."""
    idx = np.asarray(indices)
    valid = int(np.count_nonzero((idx >= 0) & (idx < num_rows)))
    return 2 * (qk_dim + v_dim) * num_heads * valid


__all__ = ["bf16_bits_to_f64", "visible_key_count", "dense_prefill", "attn_merge",
           "sparse_prefill", "dense_flops", "sparse_flops"]
