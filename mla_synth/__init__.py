"""Seeded synthetic inputs for MLA prefill attention.

This module only draws random numbers and lays them out; it holds none of
the attention arithmetic.  Both the CPU oracle (``oracle/``) and the CUDA
path (tests, ``bench.py``) take their inputs from here, so both sides see
exactly the same bits.

Recipe (every draw is reproducible from an integer seed):

* Real-valued tensors are i.i.d. N(0, 1) drawn as float32 from numpy's
  PCG64 generator and rounded to bfloat16 with round-to-nearest-even.  The
  tensor is cut into fixed 4 Mi-element pieces; piece ``p`` uses the stream
  ``SeedSequence(seed).spawn(...)[p]``, so the result does not depend on how
  many threads generate it.  Values are returned as raw bf16 bit patterns
  (``uint16``).
* Sequence lengths are uniform integers in ``[lo, hi]`` (inclusive).
* ``cu_seqlens`` is the int32 exclusive prefix sum with a leading 0, the
  layout of the varlen interface (FA4 interface page, I/O Contract:
  ``cu_seqlens_q``/``cu_seqlens_k`` of shape ``(batch_size+1,)``, int32;
  SparseFlashMla README, Constraints: first element 0, non-decreasing).
* Sparse top-k indices: query token ``t`` sits at cache position
  ``first_pos + t`` and may see cache rows ``[0, first_pos + t]``.  When at
  least ``topk`` rows are visible, ``topk`` distinct rows are drawn without
  replacement in random order; otherwise every visible row is used, in
  random order, left-aligned, and the rest of the list is ``-1``
  (SparseFlashMla README, Parameters: ``-1`` marks an invalid or padded
  slot; Constraints: valid entries left-aligned, ``-1`` fill recommended).
"""
from __future__ import annotations

import concurrent.futures as _cf
import os

import numpy as np

_PIECE = 1 << 22  # elements per independently seeded piece


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return bits.

    NaN/Inf never occur in the drawn data, so no special cases are needed.
    """
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1)))
            >> np.uint32(16)).astype(np.uint16)


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def normal_bf16(seed: int, shape) -> np.ndarray:
    """i.i.d. N(0,1) samples rounded to bf16, as a uint16 bit array."""
    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape)) if shape else 1
    out = np.empty(n, dtype=np.uint16)
    npieces = (n + _PIECE - 1) // _PIECE
    seqs = np.random.SeedSequence(seed).spawn(max(npieces, 1))

    def fill(p: int) -> None:
        lo = p * _PIECE
        hi = min(n, lo + _PIECE)
        g = np.random.Generator(np.random.PCG64(seqs[p]))
        out[lo:hi] = f32_to_bf16_bits(g.standard_normal(hi - lo, dtype=np.float32))

    if npieces <= 1:
        if n:
            fill(0)
    else:
        with _cf.ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(fill, range(npieces)))
    return out.reshape(shape)


def constant_bf16(value: float, shape) -> np.ndarray:
    """A tensor filled with one bf16 value (for closed-form cases)."""
    return np.full(shape, f32_to_bf16_bits(np.float32(value)), dtype=np.uint16)


def uniform_lengths(seed: int, n: int, lo: int, hi: int) -> list[int]:
    """``n`` integers uniform in ``[lo, hi]``."""
    g = np.random.Generator(np.random.PCG64(seed))
    return [int(x) for x in g.integers(lo, hi + 1, size=n)]


def cu_seqlens(lengths) -> np.ndarray:
    """int32 ``[B+1]`` prefix sums with a leading zero."""
    cu = np.zeros(len(lengths) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    if cu[-1] > np.iinfo(np.int32).max:
        raise ValueError("total length does not fit int32")
    return cu.astype(np.int32)


def topk_indices(seed: int, num_tokens: int, num_rows: int, topk: int,
                 first_pos: int) -> np.ndarray:
    """int32 ``[num_tokens, topk]`` causal top-k row lists with -1 padding."""
    g = np.random.Generator(np.random.PCG64(seed))
    idx = np.full((num_tokens, topk), -1, dtype=np.int32)
    for t in range(num_tokens):
        visible = min(num_rows, first_pos + t + 1)
        if visible <= 0:
            continue
        if visible >= topk:
            idx[t] = g.choice(visible, size=topk, replace=False)
        else:
            idx[t, :visible] = g.permutation(visible)
    return idx


# ---------------------------------------------------------------------------
# Workload recipes.  Each returns host arrays (bf16 as uint16 bits, int32
# index arrays) plus the scalar parameters; nothing here computes attention.
# ---------------------------------------------------------------------------

QK_DIM = 192   # 128 nope + 64 rope
V_DIM = 128
LATENT_DIM = 576  # 512 latent + 64 rope
LATENT_V_DIM = 512


def dense_case(lens_q, lens_k, num_heads: int, seed: int, causal: bool = True,
               qk_dim: int = QK_DIM, v_dim: int = V_DIM) -> dict:
    """Packed varlen Q/K/V for a dense MLA prefill call."""
    lens_q = [int(x) for x in lens_q]
    lens_k = [int(x) for x in lens_k]
    tq, tk = sum(lens_q), sum(lens_k)
    return dict(
        q=normal_bf16(seed * 1000 + 1, (tq, num_heads, qk_dim)),
        k=normal_bf16(seed * 1000 + 2, (tk, num_heads, qk_dim)),
        v=normal_bf16(seed * 1000 + 3, (tk, num_heads, v_dim)),
        cu_q=cu_seqlens(lens_q), cu_k=cu_seqlens(lens_k),
        max_q=max(lens_q) if lens_q else 0, max_k=max(lens_k) if lens_k else 0,
        scale=float(np.float32(1.0 / np.sqrt(qk_dim))), causal=bool(causal),
        num_heads=num_heads, lens_q=lens_q, lens_k=lens_k,
    )


def tiny_config(seed: int = 1) -> dict:
    """2 ragged sequences (64 and 100 tokens), 4 heads, causal."""
    return dense_case([64, 100], [64, 100], 4, seed)


def varlen16k_config(seed: int = 2, num_heads: int = 128) -> dict:
    """8 sequences with lengths uniform in [512, 4096], 128 heads, causal."""
    lens = uniform_lengths(seed, 8, 512, 4096)
    return dense_case(lens, lens, num_heads, seed)


def long32k_config(seed: int = 3, num_heads: int = 128, length: int = 32768) -> dict:
    """One 32768-token sequence, 128 heads, causal."""
    return dense_case([length], [length], num_heads, seed)


def chunked_config(seed: int = 4, num_heads: int = 128, batch: int = 4,
                   chunk: int = 2048, prefix: int = 16384) -> dict:
    """Query chunks attending to a prefix (non-causal) and to themselves (causal).

    Returns the query chunk ``q``, the prefix ``k_prefix``/``v_prefix`` and
    the chunk's own ``k_self``/``v_self`` with their cu_seqlens.
    """
    tq, tp = batch * chunk, batch * prefix
    return dict(
        q=normal_bf16(seed * 1000 + 1, (tq, num_heads, QK_DIM)),
        k_prefix=normal_bf16(seed * 1000 + 2, (tp, num_heads, QK_DIM)),
        v_prefix=normal_bf16(seed * 1000 + 3, (tp, num_heads, V_DIM)),
        k_self=normal_bf16(seed * 1000 + 4, (tq, num_heads, QK_DIM)),
        v_self=normal_bf16(seed * 1000 + 5, (tq, num_heads, V_DIM)),
        cu_q=cu_seqlens([chunk] * batch), cu_prefix=cu_seqlens([prefix] * batch),
        chunk=chunk, prefix=prefix, batch=batch, num_heads=num_heads,
        scale=float(np.float32(1.0 / np.sqrt(QK_DIM))),
    )


def sparse_case(num_tokens: int, num_heads: int, num_rows: int, topk: int,
                first_pos: int, seed: int) -> dict:
    """Absorbed sparse prefill inputs: q, shared latent cache, top-k lists."""
    return dict(
        q=normal_bf16(seed * 1000 + 1, (num_tokens, num_heads, LATENT_DIM)),
        kv=normal_bf16(seed * 1000 + 2, (num_rows, LATENT_DIM)),
        indices=topk_indices(seed * 1000 + 3, num_tokens, num_rows, topk, first_pos),
        topk=topk, num_heads=num_heads, num_rows=num_rows, first_pos=first_pos,
        scale=float(np.float32(1.0 / np.sqrt(LATENT_DIM))),
    )


def sparse_config(seed: int = 5, padded: bool = False) -> dict:
    """4096 tokens x 128 heads, 32768-row cache, top-k 2048.

    The query tokens are the last 4096 positions of the cache (every token
    sees at least 28673 rows, so no padding).  ``padded=True`` puts them at
    positions 0..4095 instead, so the first 2047 tokens get -1 padding.
    """
    rows, tokens = 32768, 4096
    first = 0 if padded else rows - tokens
    return sparse_case(tokens, 128, rows, 2048, first, seed)
