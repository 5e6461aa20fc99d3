"""The Python binding's checks of caller-provided outputs (no kernel runs:
every call here raises before the library is reached)."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def _bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16, device="cuda")


def _f32(*shape):
    return torch.zeros(shape, dtype=torch.float32, device="cuda")


def test_merge_rejects_outputs_of_the_wrong_shape(cuda_ok):
    import mla_prefill_attention_causal_b200 as mla
    o, lse = _bf16(5, 2, 128), _f32(2, 5)
    with pytest.raises(ValueError, match="shape"):
        mla.mla_attn_merge(o, lse, o.clone(), lse.clone(), out=_bf16(4, 2, 128))
    with pytest.raises(ValueError, match="lse_out"):
        mla.mla_attn_merge(o, lse, o.clone(), lse.clone(), lse_out=_f32(5, 2))
    with pytest.raises(TypeError, match="lse_out"):
        mla.mla_attn_merge(o, lse, o.clone(), lse.clone(), lse_out=_bf16(2, 5))


def test_sparse_rejects_outputs_of_the_wrong_shape(cuda_ok):
    import mla_prefill_attention_causal_b200 as mla
    q, kv = _bf16(3, 4, 576), _bf16(10, 576)
    idx = torch.zeros((3, 8), dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError, match="out"):
        mla.mla_sparse_prefill_fwd(q, kv, idx, out=_bf16(3, 4, 576))
    with pytest.raises(ValueError, match="lse"):
        mla.mla_sparse_prefill_fwd(q, kv, idx, lse=_f32(3, 4))
    with pytest.raises(ValueError, match="CUDA device"):
        mla.mla_sparse_prefill_fwd(q, kv, idx, lse=torch.zeros((4, 3)))


def test_dense_rejects_outputs_of_the_wrong_shape(cuda_ok):
    import mla_prefill_attention_causal_b200 as mla
    q, k, v = _bf16(6, 2, 192), _bf16(6, 2, 192), _bf16(6, 2, 128)
    cu = torch.tensor([0, 6], dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError, match="out"):
        mla.mla_prefill_fwd(q, k, v, cu, cu, 6, 6, out=_bf16(6, 2, 192))
    with pytest.raises(ValueError, match="lse"):
        mla.mla_prefill_fwd(q, k, v, cu, cu, 6, 6, lse=_f32(6, 2))
    with pytest.raises(ValueError, match="workspace"):
        mla.mla_prefill_fwd(q, k, v, cu, cu, 6, 6, workspace=torch.zeros(8, dtype=torch.uint8,
                                                                           device="cuda"))
