"""The C-ABI library: it loads, exports every declared symbol, and rejects
bad arguments on the host before touching a GPU (no compute calls here)."""
import ctypes
import os
import re

import pytest

import mla_prefill_attention_causal_b200 as mla
from mla_prefill_attention_causal_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mla.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\**(mla_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("mla_prefill_fwd", "mla_attn_merge", "mla_sparse_prefill_fwd",
                 "mla_status_string", "mla_device_status"):
        assert want in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(_lib.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) == set(_lib.SIGNATURES)


def test_status_strings_and_version():
    assert mla.status_string(0) == "MLA_OK"
    assert "INVALID_ARG" in mla.status_string(1)
    assert "UNSUPPORTED" in mla.status_string(2)
    assert mla.load().mla_version() >= 100


def _call_dense(**over):
    a = dict(q=16, k=16, v=16, cq=16, ck=16, mq=4, mk=4, scale=0.1, causal=1, out=16, lse=None,
             stream=None, batch=1, H=1, tq=4, tk=4, ws=64, wsb=4096)
    a.update(over)
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    return mla.load().mla_prefill_fwd(P(a["q"]), P(a["k"]), P(a["v"]), P(a["cq"]), P(a["ck"]),
                                      a["mq"], a["mk"], a["scale"], a["causal"], P(a["out"]),
                                      P(a["lse"]), None, a["batch"], a["H"], a["tq"], a["tk"],
                                      P(a["ws"]), a["wsb"])


def test_workspace_size():
    f = mla.prefill_workspace_size
    assert f(1, 0) == 256 + 8 * 1  # header + one entry per (sequence, 512-row block)
    assert f(8, 15843) == 256 + 8 * (31 + 8)
    assert mla.load().mla_prefill_workspace_size(0, 10) == 0


@pytest.mark.parametrize("over", [dict(q=None), dict(out=None), dict(cq=None), dict(q=24),
                                  dict(out=8), dict(cq=2), dict(batch=0), dict(H=0),
                                  dict(tq=-1), dict(causal=2), dict(scale=0.0),
                                  dict(scale=float("nan")), dict(scale=-1.0), dict(lse=2),
                                  dict(ws=None), dict(ws=8), dict(wsb=100)])
def test_dense_rejects_bad_arguments(over):
    assert _call_dense(**over) == _lib.MLA_ERR_INVALID_ARG


def test_dense_rejects_tile_counts_beyond_int():
    # 2^31 - 1 query rows x 65535 heads: the workspace is big enough, but the
    # number of (512-row block, head) tiles does not fit the kernels' int
    tq, H = 2**31 - 1, 65535
    need = mla.prefill_workspace_size(1, tq)
    assert need > 0
    assert _call_dense(tq=tq, H=H, wsb=need) == _lib.MLA_ERR_INVALID_ARG


def test_merge_rejects_bad_arguments():
    f = mla.load().mla_attn_merge
    P = ctypes.c_void_p
    ok = dict(oa=16, la=16, ob=16, lb=16, out=16, lo=32, T=4, H=2, D=128)

    def call(**over):
        a = dict(ok)
        a.update(over)
        p = lambda x: None if x is None else P(x)
        return f(p(a["oa"]), p(a["la"]), p(a["ob"]), p(a["lb"]), p(a["out"]), p(a["lo"]),
                 a["T"], a["H"], a["D"], None)
    assert call(oa=None) == _lib.MLA_ERR_INVALID_ARG
    assert call(D=12) == _lib.MLA_ERR_INVALID_ARG
    assert call(lo=16) == _lib.MLA_ERR_INVALID_ARG      # lse_out aliases lse_a
    assert call(out=40) == _lib.MLA_ERR_INVALID_ARG     # misaligned
    assert call(T=-1) == _lib.MLA_ERR_INVALID_ARG


def test_sparse_rejects_bad_arguments():
    f = mla.load().mla_sparse_prefill_fwd
    P = ctypes.c_void_p
    assert f(None, P(16), P(16), 8, 0.1, P(16), None, None, 4, 128, 10) == _lib.MLA_ERR_INVALID_ARG
    assert f(P(16), P(16), P(16), 0, 0.1, P(16), None, None, 4, 128, 10) == _lib.MLA_ERR_INVALID_ARG
    assert f(P(16), P(16), P(16), 8, 0.1, P(16), None, None, 4, 129, 10) == _lib.MLA_ERR_INVALID_ARG
    # two CTAs per token: 2^30 tokens would make a grid of 2^31 CTAs
    assert f(P(16), P(16), P(16), 8, 0.1, P(16), None, None, 1 << 30, 1, 10) == \
        _lib.MLA_ERR_INVALID_ARG


def _call_noalloc(batch, total_q):
    P = ctypes.c_void_p
    return mla.load().mla_prefill_fwd_noalloc(P(16), P(16), P(16), P(16), P(16), 1, 1, 0.1, 1,
                                              P(16), None, None, batch, 1, total_q, total_q)


def test_noalloc_scratch_limit_at_its_edge():
    """The fixed scratch holds ceil(total_q/512) + batch <= 8160 work-list
    entries; one more is refused before the device is touched."""
    assert mla.prefill_workspace_size(8144, 8144) == 65536       # 16 + 8144 = 8160 entries
    assert mla.prefill_workspace_size(8145, 8145) == 65536 + 8   # 8161 entries
    assert _call_noalloc(8145, 8145) == _lib.MLA_ERR_SCRATCH_TOO_SMALL
    assert _call_noalloc(1, 8161 * 512) == _lib.MLA_ERR_SCRATCH_TOO_SMALL
    # at the limit the size check passes (what follows needs a GPU)
    assert _call_noalloc(8144, 8144) != _lib.MLA_ERR_SCRATCH_TOO_SMALL
    assert "scratch" in _lib.status_string(_lib.MLA_ERR_SCRATCH_TOO_SMALL)


def test_python_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", "/nonexistent/libmla.so")
    with pytest.raises(RuntimeError, match="not built"):
        _lib.load()


def _call_strided(qs=(64, 32), ks=(64, 32), vs=(64, 32)):
    P = ctypes.c_void_p
    return mla.load().mla_prefill_fwd_strided(
        P(16), qs[0], qs[1], P(16), ks[0], ks[1], P(16), vs[0], vs[1], P(16), P(16), 4, 4, 0.1, 1,
        P(16), None, None, 1, 1, 4, 4, P(64), 4096)


@pytest.mark.parametrize("bad", [dict(qs=(0, 32)), dict(ks=(64, -8)), dict(vs=(60, 32)),
                                 dict(qs=(64, 12)), dict(vs=(1 << 40, 32))])
def test_strided_rejects_bad_strides(bad):
    # checked on the host before the device is touched
    assert _call_strided(**bad) == _lib.MLA_ERR_INVALID_ARG


def test_python_binding_checks_arguments_before_any_launch():
    import torch
    q = torch.zeros((4, 2, 192), dtype=torch.bfloat16)
    k = torch.zeros((4, 2, 192), dtype=torch.bfloat16)
    v = torch.zeros((4, 2, 128), dtype=torch.bfloat16)
    cu = torch.tensor([0, 4], dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA device"):
        mla.mla_prefill_fwd(q, k, v, cu, cu, 4, 4)
    with pytest.raises(TypeError, match="bfloat16"):
        mla.mla_prefill_fwd(q.float(), k, v, cu, cu, 4, 4)
    with pytest.raises(ValueError, match="3 dims"):
        mla.mla_prefill_fwd(q[0], k, v, cu, cu, 4, 4)
    kv = torch.zeros((4, 576), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA device"):
        mla.mla_sparse_prefill_fwd(torch.zeros((4, 8, 576), dtype=torch.bfloat16), kv,
                                   torch.zeros((4, 16), dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA device"):
        mla.mla_attn_merge(v, torch.zeros((2, 4)), v, torch.zeros((2, 4)))


def _call_context(**over):
    a = dict(q=16, k=16, v=16, cq=16, ck=16, kc=32, vc=32, cc=16, mq=4, mk=4, mc=4, scale=0.1,
             causal=1, out=16, lse=None, batch=1, H=1, tq=4, tk=4, tc=4, ws=64, wsb=4096)
    a.update(over)
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    return mla.load().mla_prefill_fwd_context(
        P(a["q"]), P(a["k"]), P(a["v"]), P(a["cq"]), P(a["ck"]), P(a["kc"]), P(a["vc"]),
        P(a["cc"]), a["mq"], a["mk"], a["mc"], a["scale"], a["causal"], P(a["out"]), P(a["lse"]),
        None, a["batch"], a["H"], a["tq"], a["tk"], a["tc"], P(a["ws"]), a["wsb"])


@pytest.mark.parametrize("over", [dict(kc=None), dict(vc=None), dict(cc=None), dict(kc=40),
                                  dict(vc=24), dict(cc=2), dict(tc=-1), dict(mc=-1), dict(q=None),
                                  dict(wsb=100), dict(causal=3)])
def test_context_call_rejects_bad_arguments(over):
    assert _call_context(**over) == _lib.MLA_ERR_INVALID_ARG


def _call_ex(**over):
    a = dict(q=16, k=16, v=16, cq=16, ck=16, mq=4, mk=4, scale=0.1, causal=1, sinks=None,
             osc=None, out=16, lse=None, batch=1, H=1, tq=4, tk=4, ws=64, wsb=4096)
    a.update(over)
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    return mla.load().mla_prefill_fwd_ex(
        P(a["q"]), P(a["k"]), P(a["v"]), P(a["cq"]), P(a["ck"]), a["mq"], a["mk"], a["scale"],
        a["causal"], P(a["sinks"]), P(a["osc"]), P(a["out"]), P(a["lse"]), None, a["batch"],
        a["H"], a["tq"], a["tk"], P(a["ws"]), a["wsb"])


@pytest.mark.parametrize("over", [dict(sinks=2), dict(osc=6), dict(out=None), dict(out=8),
                                  dict(scale=0.0), dict(H=0)])
def test_ex_call_rejects_bad_arguments(over):
    assert _call_ex(**over) == _lib.MLA_ERR_INVALID_ARG


def test_splitkv_sizes_and_choice():
    f = mla.splitkv_workspace_size
    base = mla.prefill_workspace_size(2, 100)
    assert f(2, 100, 8, 1) == base                       # no partials without splits
    parts = ((base + 255) // 256) * 256
    assert f(2, 100, 8, 3) == parts + 3 * 100 * 8 * 129 * 4
    assert f(2, 100, 8, 0) == 0 and f(2, 100, 8, 65) == 0 and f(2, 100, 0, 2) == 0
    # no GPU here: the choice assumes 74 CTA pairs
    assert mla.num_splits_for(1, 1, 16, 1, 8192) == 4     # 64 split tiles: one wave on 74 pairs
    assert mla.num_splits_for(1, 1, 2, 1, 8192) == 32     # 2 x 32 tiles of 2 blocks
    assert mla.num_splits_for(1, 1, 128, 1, 8192) == 1    # a tile for every pair already
    assert mla.num_splits_for(1, 1, 4, 1, 512) == 2       # at least two KV blocks a split
    assert mla.num_splits_for(1, 1, 1, 1, 1 << 20) == 64  # at most MLA_MAX_SPLITS
    assert mla.num_splits_for(8, 16384, 128, 4096, 4096) == 1


def _call_split(**over):
    a = dict(q=16, k=16, v=16, cq=16, ck=16, mq=4, mk=4, scale=0.1, causal=1, ns=2, out=16,
             lse=None, batch=1, H=1, tq=4, tk=4, ws=64, wsb=1 << 20)
    a.update(over)
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    return mla.load().mla_prefill_fwd_splitkv(
        P(a["q"]), P(a["k"]), P(a["v"]), P(a["cq"]), P(a["ck"]), a["mq"], a["mk"], a["scale"],
        a["causal"], a["ns"], P(a["out"]), P(a["lse"]), None, a["batch"], a["H"], a["tq"],
        a["tk"], P(a["ws"]), a["wsb"])


@pytest.mark.parametrize("over", [dict(ns=0), dict(ns=65), dict(wsb=300), dict(q=None),
                                  dict(out=8), dict(causal=2)])
def test_splitkv_call_rejects_bad_arguments(over):
    assert _call_split(**over) == _lib.MLA_ERR_INVALID_ARG


def test_dims_call_rejects_unsupported_geometries():
    P = ctypes.c_void_p
    f = mla.load().mla_prefill_fwd_dims
    for qk, v in ((64, 128), (192, 64), (320, 128), (192, 512)):
        assert f(P(16), P(16), P(16), P(16), P(16), 4, 4, 0.1, 1, P(16), None, None, 1, 1, 4, 4,
                 qk, v, P(64), 4096) == _lib.MLA_ERR_INVALID_ARG
