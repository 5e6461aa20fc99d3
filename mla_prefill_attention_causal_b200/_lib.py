"""ctypes binding of libmla.so (argument marshalling only).

Every function here checks tensor dtypes/shapes/devices, allocates outputs
with PyTorch when the caller passes none, and calls the C entry point of
the same name on the current CUDA stream.  All computation happens in the
library's CUDA kernels; if the library is missing or fails to load, every
call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG_DIR, "libmla.so")

MLA_OK = 0
MLA_ERR_INVALID_ARG = 1
MLA_ERR_UNSUPPORTED = 2
MLA_ERR_CUDA = 3
MLA_ERR_SCRATCH_TOO_SMALL = 4
NOALLOC_SCRATCH_BYTES = 65536
DEVSTAT_WAIT_TIMEOUT_LOAD = 0x1
DEVSTAT_WAIT_TIMEOUT_MMA = 0x2
DEVSTAT_WAIT_TIMEOUT_SOFTMAX = 0x4
DEVSTAT_WAIT_TIMEOUT_TEST = 0x100

QK_DIM, V_DIM = 192, 128
LATENT_DIM, LATENT_V_DIM = 576, 512

# name -> (restype, argtypes), mirroring include/mla.h
_P, _I, _F, _S, _L = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_int64
SIGNATURES = {
    "mla_status_string": (ctypes.c_char_p, [_I]),
    "mla_version": (_I, []),
    "mla_prefill_workspace_size": (_S, [_I, _I]),
    "mla_prefill_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _F, _I, _P, _P, _P, _I, _I, _I, _I, _P,
                             _S]),
    "mla_prefill_fwd_strided": (_I, [_P, _L, _L, _P, _L, _L, _P, _L, _L, _P, _P, _I, _I, _F, _I,
                                     _P, _P, _P, _I, _I, _I, _I, _P, _S]),
    "mla_prefill_fwd_context": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _F, _I, _P, _P,
                                     _P, _I, _I, _I, _I, _I, _P, _S]),
    "mla_prefill_fwd_ex": (_I, [_P, _P, _P, _P, _P, _I, _I, _F, _I, _P, _P, _P, _P, _P, _I, _I, _I,
                                _I, _P, _S]),
    "mla_prefill_fwd_dims": (_I, [_P, _P, _P, _P, _P, _I, _I, _F, _I, _P, _P, _P, _I, _I, _I, _I,
                                  _I, _I, _P, _S]),
    "mla_prefill_splitkv_workspace_size": (_S, [_I, _I, _I, _I]),
    "mla_prefill_num_splits": (_I, [_I, _I, _I, _I, _I]),
    "mla_prefill_fwd_splitkv": (_I, [_P, _P, _P, _P, _P, _I, _I, _F, _I, _I, _P, _P, _P, _I, _I,
                                     _I, _I, _P, _S]),
    "mla_prefill_fwd_noalloc": (_I, [_P, _P, _P, _P, _P, _I, _I, _F, _I, _P, _P, _P, _I, _I, _I,
                                     _I]),
    "mla_attn_merge": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _P]),
    "mla_sparse_prefill_fwd": (_I, [_P, _P, _P, _I, _F, _P, _P, _P, _I, _I, _I]),
    "mla_device_status": (_I, [ctypes.POINTER(ctypes.c_uint), _I]),
    "mla_debug_wait_timeout": (_I, [_I, _P]),
}


class MlaError(RuntimeError):
    """A libmla call returned an error status."""

    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status_string(status)}")


_lib: Optional[ctypes.CDLL] = None


def load() -> ctypes.CDLL:
    """Load libmla.so (once).  Raises if it is missing: there is no fallback."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libmla.so not built ({LIB_PATH}); run "
                               "`python -m mla_prefill_attention_causal_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().mla_status_string(int(status)).decode()


def _check(fn: str, status: int) -> None:
    if status != MLA_OK:
        raise MlaError(fn, status)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need(t: torch.Tensor, name: str, dtype, ndim: int, contiguous: bool = True) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if not contiguous and (t.stride(-1) != 1 or any(x % 8 for x in t.stride()[:-1])
                           or t.data_ptr() % 16):
        raise ValueError(f"{name} needs a contiguous last dim, other strides that are multiples "
                         f"of 8 elements and a 16-byte aligned start; got strides {t.stride()}")


def _same_device(ref: torch.Tensor, **tensors) -> None:
    for name, t in tensors.items():
        if t is not None and t.device != ref.device:
            raise ValueError(f"{name} is on {t.device}, the inputs on {ref.device}")


def mla_prefill_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                    cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor,
                    max_seqlen_q: int, max_seqlen_k: int,
                    softmax_scale: Optional[float] = None, causal: bool = True,
                    out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                    return_lse: bool = True, workspace: Optional[torch.Tensor] = None):
    """Dense varlen MLA prefill forward (``mla_prefill_fwd`` in ``mla.h``).

    q ``[total_q, H, 192]``, k ``[total_k, H, 192]``, v ``[total_k, H, 128]``
    (bf16, CUDA; contiguous, or views whose last dim is contiguous and whose
    other strides are multiples of 8 elements, which go through
    ``mla_prefill_fwd_strided``); cu_seqlens int32 ``[B+1]`` on the same
    device.
    ``workspace`` (uint8, >= ``prefill_workspace_size(B, total_q)`` bytes) is
    allocated from PyTorch's stream-ordered allocator when not given.
    Returns ``(out [total_q, H, 128] bf16, lse [H, total_q] fp32 or None)``.
    """
    _need(q, "q", torch.bfloat16, 3, contiguous=False)
    _need(k, "k", torch.bfloat16, 3, contiguous=False)
    _need(v, "v", torch.bfloat16, 3, contiguous=False)
    _need(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32, 1)
    total_q, num_heads, dq = q.shape
    total_k = k.shape[0]
    if dq != QK_DIM or k.shape[1:] != (num_heads, QK_DIM) or v.shape != (total_k, num_heads, V_DIM):
        raise ValueError(f"MLA dims must be q/k [*, H, {QK_DIM}], v [*, H, {V_DIM}]; got "
                         f"{tuple(q.shape)}, {tuple(k.shape)}, {tuple(v.shape)}")
    batch = cu_seqlens_q.numel() - 1
    if batch < 1 or cu_seqlens_k.numel() != batch + 1:
        raise ValueError("cu_seqlens_q/k must both have batch+1 >= 2 entries")
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(QK_DIM)
    if out is None:
        out = torch.empty((total_q, num_heads, V_DIM), dtype=torch.bfloat16, device=q.device)
    else:
        _need(out, "out", torch.bfloat16, 3)
        if out.shape != (total_q, num_heads, V_DIM):
            raise ValueError("out has the wrong shape")
    if lse is None and return_lse:
        lse = torch.empty((num_heads, total_q), dtype=torch.float32, device=q.device)
    elif lse is not None:
        _need(lse, "lse", torch.float32, 2)
        if lse.shape != (num_heads, total_q):
            raise ValueError("lse must be [num_heads, total_q]")
    ws_bytes = prefill_workspace_size(batch, total_q)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    elif workspace.numel() * workspace.element_size() < ws_bytes or not workspace.is_cuda:
        raise ValueError(f"workspace must be a CUDA buffer of >= {ws_bytes} bytes")
    _same_device(q, k=k, v=v, cu_seqlens_q=cu_seqlens_q, cu_seqlens_k=cu_seqlens_k, out=out,
                 lse=lse, workspace=workspace)
    with torch.cuda.device(q.device):
        return _prefill_call(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                             softmax_scale, causal, out, lse, batch, num_heads, total_q, total_k,
                             workspace)


def _prefill_call(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, softmax_scale,
                  causal, out, lse, batch, num_heads, total_q, total_k, workspace):
    rest = (_ptr(cu_seqlens_q), _ptr(cu_seqlens_k), int(max_seqlen_q), int(max_seqlen_k),
            float(softmax_scale), 1 if causal else 0, _ptr(out), _ptr(lse), _stream(), batch,
            num_heads, total_q, total_k, _ptr(workspace),
            workspace.numel() * workspace.element_size())
    if q.is_contiguous() and k.is_contiguous() and v.is_contiguous():
        st = load().mla_prefill_fwd(_ptr(q), _ptr(k), _ptr(v), *rest)
        _check("mla_prefill_fwd", st)
    else:
        st = load().mla_prefill_fwd_strided(_ptr(q), q.stride(0), q.stride(1), _ptr(k), k.stride(0),
                                            k.stride(1), _ptr(v), v.stride(0), v.stride(1), *rest)
        _check("mla_prefill_fwd_strided", st)
    return out, lse


def _packed_dense_args(q, k, v, cu_seqlens_q, cu_seqlens_k, softmax_scale, out, lse,
                       return_lse, workspace, out_dtype=torch.bfloat16):
    """Checks shared by the packed dense calls; allocates what is missing."""
    for t, n, d in ((q, "q", QK_DIM), (k, "k", QK_DIM), (v, "v", V_DIM)):
        _need(t, n, torch.bfloat16, 3)
        if t.shape[2] != d:
            raise ValueError(f"{n} must be [*, H, {d}], got {tuple(t.shape)}")
    _need(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32, 1)
    total_q, num_heads, _ = q.shape
    total_k = k.shape[0]
    if k.shape[1] != num_heads or v.shape[:2] != (total_k, num_heads):
        raise ValueError("q, k and v must agree on heads, k and v on rows")
    batch = cu_seqlens_q.numel() - 1
    if batch < 1 or cu_seqlens_k.numel() != batch + 1:
        raise ValueError("cu_seqlens_q/k must both have batch+1 >= 2 entries")
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(QK_DIM)
    if out is None:
        out = torch.empty((total_q, num_heads, V_DIM), dtype=out_dtype, device=q.device)
    else:
        _need(out, "out", out_dtype, 3)
        if out.shape != (total_q, num_heads, V_DIM):
            raise ValueError("out has the wrong shape")
    if lse is None and return_lse:
        lse = torch.empty((num_heads, total_q), dtype=torch.float32, device=q.device)
    elif lse is not None:
        _need(lse, "lse", torch.float32, 2)
        if lse.shape != (num_heads, total_q):
            raise ValueError("lse must be [num_heads, total_q]")
    ws_bytes = prefill_workspace_size(batch, total_q)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    elif workspace.numel() * workspace.element_size() < ws_bytes or not workspace.is_cuda:
        raise ValueError(f"workspace must be a CUDA buffer of >= {ws_bytes} bytes")
    return (float(softmax_scale), out, lse, workspace, batch, num_heads, total_q, total_k)


def mla_prefill_fwd_context(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                            cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor,
                            k_ctx: torch.Tensor, v_ctx: torch.Tensor, cu_seqlens_ctx: torch.Tensor,
                            max_seqlen_q: int, max_seqlen_k: int, max_seqlen_ctx: int,
                            softmax_scale: Optional[float] = None, causal: bool = True,
                            out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                            return_lse: bool = True, workspace: Optional[torch.Tensor] = None):
    """Chunked prefill in one pass (``mla_prefill_fwd_context`` in ``mla.h``).

    The queries attend to all of their sequence's context keys (``k_ctx`` /
    ``v_ctx`` rows given by ``cu_seqlens_ctx``) and to their own keys (``k``
    / ``v``, causal when ``causal``) under one softmax: the merged result of
    a context pass and a new-token pass.  All tensors packed, bf16
    ``[*, H, 192]`` / ``[*, H, 128]``; cu_seqlens int32 ``[B+1]``.
    Returns ``(out [total_q, H, 128] bf16, lse [H, total_q] fp32 or None)``.
    """
    scale, out, lse, workspace, batch, num_heads, total_q, total_k = _packed_dense_args(
        q, k, v, cu_seqlens_q, cu_seqlens_k, softmax_scale, out, lse, return_lse, workspace)
    for t, n, d in ((k_ctx, "k_ctx", QK_DIM), (v_ctx, "v_ctx", V_DIM)):
        _need(t, n, torch.bfloat16, 3)
        if t.shape[1:] != (num_heads, d):
            raise ValueError(f"{n} must be [*, {num_heads}, {d}], got {tuple(t.shape)}")
    _need(cu_seqlens_ctx, "cu_seqlens_ctx", torch.int32, 1)
    total_ctx = k_ctx.shape[0]
    if v_ctx.shape[0] != total_ctx or cu_seqlens_ctx.numel() != batch + 1:
        raise ValueError("k_ctx / v_ctx rows or cu_seqlens_ctx entries do not match")
    _same_device(q, k=k, v=v, k_ctx=k_ctx, v_ctx=v_ctx, cu_seqlens_q=cu_seqlens_q,
                 cu_seqlens_k=cu_seqlens_k, cu_seqlens_ctx=cu_seqlens_ctx, out=out, lse=lse,
                 workspace=workspace)
    with torch.cuda.device(q.device):
        st = load().mla_prefill_fwd_context(
            _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), _ptr(k_ctx),
            _ptr(v_ctx), _ptr(cu_seqlens_ctx), int(max_seqlen_q), int(max_seqlen_k),
            int(max_seqlen_ctx), scale, 1 if causal else 0, _ptr(out), _ptr(lse), _stream(),
            batch, num_heads, total_q, total_k, total_ctx, _ptr(workspace),
            workspace.numel() * workspace.element_size())
    _check("mla_prefill_fwd_context", st)
    return out, lse


def mla_prefill_fwd_ex(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                       cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor,
                       max_seqlen_q: int, max_seqlen_k: int,
                       softmax_scale: Optional[float] = None, causal: bool = True,
                       sinks: Optional[torch.Tensor] = None,
                       output_scale: Optional[torch.Tensor] = None,
                       out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                       return_lse: bool = True, workspace: Optional[torch.Tensor] = None):
    """Dense prefill with attention sinks and/or an FP8 output (``mla_prefill_fwd_ex``).

    ``sinks``: float32 ``[H]`` (one logit per head) or None.  ``output_scale``:
    a float32 one-element CUDA tensor or None; when given, ``out`` is
    ``torch.float8_e4m3fn`` holding O / scale (round to nearest even,
    saturated at 448).  Returns ``(out, lse)``.
    """
    fp8 = output_scale is not None
    scale, out, lse, workspace, batch, num_heads, total_q, total_k = _packed_dense_args(
        q, k, v, cu_seqlens_q, cu_seqlens_k, softmax_scale, out, lse, return_lse, workspace,
        out_dtype=torch.float8_e4m3fn if fp8 else torch.bfloat16)
    if sinks is not None:
        _need(sinks, "sinks", torch.float32, 1)
        if sinks.numel() != num_heads:
            raise ValueError("sinks must hold one value per head")
    if fp8:
        _need(output_scale, "output_scale", torch.float32, 1)
        if output_scale.numel() != 1:
            raise ValueError("output_scale must be a one-element tensor")
    _same_device(q, k=k, v=v, cu_seqlens_q=cu_seqlens_q, cu_seqlens_k=cu_seqlens_k, sinks=sinks,
                 output_scale=output_scale, out=out, lse=lse, workspace=workspace)
    with torch.cuda.device(q.device):
        st = load().mla_prefill_fwd_ex(
            _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), int(max_seqlen_q),
            int(max_seqlen_k), scale, 1 if causal else 0, _ptr(sinks), _ptr(output_scale),
            _ptr(out), _ptr(lse), _stream(), batch, num_heads, total_q, total_k, _ptr(workspace),
            workspace.numel() * workspace.element_size())
    _check("mla_prefill_fwd_ex", st)
    return out, lse


def mla_prefill_fwd_dims(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                         cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor,
                         max_seqlen_q: int, max_seqlen_k: int,
                         softmax_scale: Optional[float] = None, causal: bool = True,
                         out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                         return_lse: bool = True, workspace: Optional[torch.Tensor] = None):
    """Dense prefill for the other MLA head geometries (``mla_prefill_fwd_dims``).

    q/k ``[*, H, qk_dim]`` with qk_dim in {128, 192, 256}, v ``[*, H, v_dim]``
    with v_dim in {128, 256}; packed bf16.  Returns ``(out [total_q, H,
    v_dim] bf16, lse [H, total_q] fp32 or None)``.
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, torch.bfloat16, 3)
    _need(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32, 1)
    total_q, num_heads, qk_dim = q.shape
    total_k, v_dim = k.shape[0], v.shape[2]
    if qk_dim not in (128, 192, 256) or v_dim not in (128, 256):
        raise ValueError(f"unsupported MLA dims: qk {qk_dim}, v {v_dim}")
    if k.shape[1:] != (num_heads, qk_dim) or v.shape[:2] != (total_k, num_heads):
        raise ValueError("q, k and v must agree on heads and dims, k and v on rows")
    batch = cu_seqlens_q.numel() - 1
    if batch < 1 or cu_seqlens_k.numel() != batch + 1:
        raise ValueError("cu_seqlens_q/k must both have batch+1 >= 2 entries")
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(qk_dim)
    if out is None:
        out = torch.empty((total_q, num_heads, v_dim), dtype=torch.bfloat16, device=q.device)
    else:
        _need(out, "out", torch.bfloat16, 3)
        if out.shape != (total_q, num_heads, v_dim):
            raise ValueError("out has the wrong shape")
    if lse is None and return_lse:
        lse = torch.empty((num_heads, total_q), dtype=torch.float32, device=q.device)
    elif lse is not None:
        _need(lse, "lse", torch.float32, 2)
        if lse.shape != (num_heads, total_q):
            raise ValueError("lse must be [num_heads, total_q]")
    ws_bytes = prefill_workspace_size(batch, total_q)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    elif workspace.numel() * workspace.element_size() < ws_bytes or not workspace.is_cuda:
        raise ValueError(f"workspace must be a CUDA buffer of >= {ws_bytes} bytes")
    _same_device(q, k=k, v=v, cu_seqlens_q=cu_seqlens_q, cu_seqlens_k=cu_seqlens_k, out=out,
                 lse=lse, workspace=workspace)
    with torch.cuda.device(q.device):
        st = load().mla_prefill_fwd_dims(
            _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), int(max_seqlen_q),
            int(max_seqlen_k), float(softmax_scale), 1 if causal else 0, _ptr(out), _ptr(lse),
            _stream(), batch, num_heads, total_q, total_k, qk_dim, v_dim, _ptr(workspace),
            workspace.numel() * workspace.element_size())
    _check("mla_prefill_fwd_dims", st)
    return out, lse


def num_splits_for(batch: int, total_q: int, num_heads: int, max_seqlen_q: int,
                   max_seqlen_k: int) -> int:
    """The library's split-KV choice for these sizes (``mla_prefill_num_splits``)."""
    return int(load().mla_prefill_num_splits(int(batch), int(total_q), int(num_heads),
                                             int(max_seqlen_q), int(max_seqlen_k)))


def splitkv_workspace_size(batch: int, total_q: int, num_heads: int, num_splits: int) -> int:
    """Workspace bytes of ``mla_prefill_fwd_splitkv``."""
    return int(load().mla_prefill_splitkv_workspace_size(int(batch), int(total_q),
                                                         int(num_heads), int(num_splits)))


def mla_prefill_fwd_splitkv(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                            cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor,
                            max_seqlen_q: int, max_seqlen_k: int,
                            softmax_scale: Optional[float] = None, causal: bool = True,
                            num_splits: Optional[int] = None,
                            out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                            return_lse: bool = True, workspace: Optional[torch.Tensor] = None):
    """Dense prefill with split-KV (``mla_prefill_fwd_splitkv`` in ``mla.h``).

    ``num_splits``: KV splits per tile (1 .. 64), or None for the library's
    choice (``num_splits_for``).  Packed tensors as ``mla_prefill_fwd``.
    Returns ``(out [total_q, H, 128] bf16, lse [H, total_q] fp32 or None)``.
    """
    batch = cu_seqlens_q.numel() - 1
    total_q, num_heads = q.shape[0], q.shape[1]
    if num_splits is None:
        num_splits = num_splits_for(batch, total_q, num_heads, max_seqlen_q, max_seqlen_k)
    ws_bytes = splitkv_workspace_size(batch, total_q, num_heads, num_splits)
    if ws_bytes == 0:
        raise ValueError(f"invalid split-KV sizes (num_splits={num_splits})")
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    scale, out, lse, workspace, batch, num_heads, total_q, total_k = _packed_dense_args(
        q, k, v, cu_seqlens_q, cu_seqlens_k, softmax_scale, out, lse, return_lse, workspace)
    if workspace.numel() * workspace.element_size() < ws_bytes:
        raise ValueError(f"workspace must hold >= {ws_bytes} bytes")
    _same_device(q, k=k, v=v, cu_seqlens_q=cu_seqlens_q, cu_seqlens_k=cu_seqlens_k, out=out,
                 lse=lse, workspace=workspace)
    with torch.cuda.device(q.device):
        st = load().mla_prefill_fwd_splitkv(
            _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), int(max_seqlen_q),
            int(max_seqlen_k), scale, 1 if causal else 0, int(num_splits), _ptr(out), _ptr(lse),
            _stream(), batch, num_heads, total_q, total_k, _ptr(workspace),
            workspace.numel() * workspace.element_size())
    _check("mla_prefill_fwd_splitkv", st)
    return out, lse


def prefill_workspace_size(batch: int, total_q: int) -> int:
    """Workspace bytes ``mla_prefill_fwd`` needs (``mla_prefill_workspace_size``)."""
    return int(load().mla_prefill_workspace_size(int(batch), int(total_q)))


def mla_attn_merge(o_a: torch.Tensor, lse_a: torch.Tensor, o_b: torch.Tensor,
                   lse_b: torch.Tensor, out: Optional[torch.Tensor] = None,
                   lse_out: Optional[torch.Tensor] = None, return_lse: bool = True):
    """LSE merge of two partial results (``mla_attn_merge`` in ``mla.h``).

    o ``[T, H, D]`` bf16, lse ``[H, T]`` fp32.  ``out`` may be ``o_a`` or
    ``o_b``; ``lse_out`` must be a separate buffer.
    """
    for t, n in ((o_a, "o_a"), (o_b, "o_b")):
        _need(t, n, torch.bfloat16, 3)
    for t, n in ((lse_a, "lse_a"), (lse_b, "lse_b")):
        _need(t, n, torch.float32, 2)
    T, H, D = o_a.shape
    if o_b.shape != o_a.shape or lse_a.shape != (H, T) or lse_b.shape != (H, T):
        raise ValueError("shape mismatch between partial results")
    if out is None:
        out = torch.empty_like(o_a)
    else:
        _need(out, "out", torch.bfloat16, 3)
        if out.shape != o_a.shape:
            raise ValueError("out must have the partial results' shape")
    if lse_out is None and return_lse:
        lse_out = torch.empty_like(lse_a)
    elif lse_out is not None:
        _need(lse_out, "lse_out", torch.float32, 2)
        if lse_out.shape != (H, T):
            raise ValueError("lse_out must be [num_heads, num_tokens]")
    _same_device(o_a, o_b=o_b, lse_a=lse_a, lse_b=lse_b, out=out, lse_out=lse_out)
    with torch.cuda.device(o_a.device):
        st = load().mla_attn_merge(_ptr(o_a), _ptr(lse_a), _ptr(o_b), _ptr(lse_b), _ptr(out),
                                   _ptr(lse_out), T, H, D, _stream())
    _check("mla_attn_merge", st)
    return out, lse_out


def mla_sparse_prefill_fwd(q: torch.Tensor, kv_latent: torch.Tensor, indices: torch.Tensor,
                           softmax_scale: Optional[float] = None,
                           out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                           return_lse: bool = True):
    """Absorbed top-k sparse MLA prefill (``mla_sparse_prefill_fwd``).

    q ``[T, H, 576]`` bf16, kv_latent ``[N, 576]`` bf16, indices ``[T, topk]``
    int32 (values outside ``[0, N)`` are padding).  Returns
    ``(out [T, H, 512] bf16, lse [H, T] fp32 or None)``.
    """
    _need(q, "q", torch.bfloat16, 3)
    _need(kv_latent, "kv_latent", torch.bfloat16, 2)
    _need(indices, "indices", torch.int32, 2)
    T, H, D = q.shape
    N = kv_latent.shape[0]
    if D != LATENT_DIM or kv_latent.shape[1] != LATENT_DIM or indices.shape[0] != T:
        raise ValueError("sparse shapes must be q [T, H, 576], kv [N, 576], indices [T, topk]")
    topk = indices.shape[1]
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(LATENT_DIM)
    if out is None:
        out = torch.empty((T, H, LATENT_V_DIM), dtype=torch.bfloat16, device=q.device)
    else:
        _need(out, "out", torch.bfloat16, 3)
        if out.shape != (T, H, LATENT_V_DIM):
            raise ValueError(f"out must be [T, H, {LATENT_V_DIM}]")
    if lse is None and return_lse:
        lse = torch.empty((H, T), dtype=torch.float32, device=q.device)
    elif lse is not None:
        _need(lse, "lse", torch.float32, 2)
        if lse.shape != (H, T):
            raise ValueError("lse must be [num_heads, num_tokens]")
    _same_device(q, kv_latent=kv_latent, indices=indices, out=out, lse=lse)
    with torch.cuda.device(q.device):
        st = _sparse_call(q, kv_latent, indices, topk, softmax_scale, out, lse, T, H, N)
    _check("mla_sparse_prefill_fwd", st)
    return out, lse


def _sparse_call(q, kv_latent, indices, topk, softmax_scale, out, lse, T, H, N):
    return load().mla_sparse_prefill_fwd(_ptr(q), _ptr(kv_latent), _ptr(indices), topk,
                                       float(softmax_scale), _ptr(out), _ptr(lse), _stream(),
                                       T, H, N)


def mla_device_status(reset: bool = True) -> int:
    """OR of the device status bits set by kernels whose waits gave up."""
    v = ctypes.c_uint(0)
    _check("mla_device_status", load().mla_device_status(ctypes.byref(v), 1 if reset else 0))
    return int(v.value)


def mla_debug_wait_timeout(timeout_us: int) -> None:
    """Launch the bounded-wait probe kernel (see ``mla.h``)."""
    _check("mla_debug_wait_timeout", load().mla_debug_wait_timeout(int(timeout_us), _stream()))
