"""The Python binding's argument checks on the CPU: layouts the C structs
cannot express are refused before anything reaches the library."""
import pytest
import torch

from attention_online_softmax_fmha_b200 import binding as B


def _bf16(*shape):
    return torch.zeros(*shape, dtype=torch.bfloat16)


def test_varlen_refuses_strided_last_axis_and_mixed_dtypes():
    q, k, v = _bf16(2, 16, 4, 64), _bf16(2, 16, 2, 64), _bf16(2, 16, 2, 64)
    B.varlen_args(q, k, v)  # accepted
    with pytest.raises(ValueError, match="last axis"):
        B.varlen_args(_bf16(2, 16, 64, 4).transpose(2, 3), k, v)
    with pytest.raises(ValueError, match="dtype"):
        B.varlen_args(q, k.half(), v)
    cu = torch.tensor([0, 16, 32], dtype=torch.int64)
    with pytest.raises(ValueError, match="int32"):
        B.varlen_args(q.view(32, 4, 64), k.view(32, 2, 64), v.view(32, 2, 64), cu_seqlens_q=cu,
                      cu_seqlens_k=cu, max_seqlen_q=16, max_seqlen_k=16)


def test_paged_refuses_bad_layouts():
    q = _bf16(2, 1, 4, 64)
    kc, vc = _bf16(6, 16, 2, 64), _bf16(6, 16, 2, 64)
    bt = torch.zeros(2, 3, dtype=torch.int32)
    cs = torch.tensor([20, 30], dtype=torch.int32)
    B.paged_args(q, kc, vc, bt, cs)  # accepted
    with pytest.raises(ValueError, match="dtype"):
        B.paged_args(q, kc.half(), vc, bt, cs)
    with pytest.raises(ValueError, match="int32"):
        B.paged_args(q, kc, vc, bt.long(), cs)
    with pytest.raises(ValueError, match="together"):
        B.paged_args(q, kc, vc, bt, cs, k_new=_bf16(2, 1, 2, 64))
    with pytest.raises(ValueError, match="last axis"):
        B.paged_args(q, kc, vc, bt, cs, k_new=_bf16(2, 1, 64, 2).transpose(2, 3),
                     v_new=_bf16(2, 1, 2, 64))
    with pytest.raises(ValueError, match="contiguous"):
        B.paged_args(q, kc, vc, bt, torch.tensor([20, 0, 30, 0], dtype=torch.int32)[::2])


def test_mla_refuses_mixed_dtypes():
    q = _bf16(1, 2, 128, 576)
    kv = torch.zeros(4, 64, 1, 576, dtype=torch.float16)
    bt = torch.zeros(1, 4, dtype=torch.int32)
    cs = torch.tensor([100], dtype=torch.int32)
    with pytest.raises(ValueError, match="dtype"):
        B.mla_args(q, kv, bt, cs)
