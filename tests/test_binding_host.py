"""Argument checks of the tensor helpers in long_context_attention_la_b200/la.py that run on the
host before any device pointer is taken (CPU tensors; no kernel is launched)."""
import pytest
import torch

from long_context_attention_la_b200 import la

T, H, D = 300, 2, 128
CU = [0, 100, 300]


def operands(dtype=torch.bfloat16):
    q = torch.zeros((T, H, D), dtype=dtype)
    return q, q.clone(), q.clone(), torch.ones(H), torch.ones(D), torch.ones(D), \
        torch.arange(T, dtype=torch.int64)


def test_prefill_varlen_qk_rejects_bad_shapes_and_types():
    q, k, v, sl, gq, gk, pos = operands()
    with pytest.raises(ValueError, match="positions"):
        la.prefill_varlen_qk(q, k, v, sl, CU, gq, gk, pos.to(torch.int32))
    with pytest.raises(ValueError, match="positions"):
        la.prefill_varlen_qk(q, k, v, sl, CU, gq, gk, pos[:-1])
    with pytest.raises(ValueError, match="gamma_q"):
        la.prefill_varlen_qk(q, k, v, sl, CU, gq[:64], gk, pos)
    with pytest.raises(ValueError, match="gamma_k"):
        la.prefill_varlen_qk(q, k, v, sl, CU, gq, gk.double(), pos)
    with pytest.raises(ValueError, match="shape"):
        la.prefill_varlen_qk(q, k[:-1], v, sl, CU, gq, gk, pos)
    with pytest.raises(ValueError, match="slopes"):
        la.prefill_varlen_qk(q, k, v, sl[:1], CU, gq, gk, pos)
    with pytest.raises(ValueError, match="cu_seqlens"):
        la.prefill_varlen_qk(q, k, v, sl, [0], gq, gk, pos)


def test_prefill_varlen_qk_needs_device_tensors():
    """Well-formed host tensors pass the shape checks and stop at the first device pointer."""
    q, k, v, sl, gq, gk, pos = operands()
    with pytest.raises(ValueError, match="CUDA"):
        la.prefill_varlen_qk(q, k, v, sl, CU, gq, gk, pos)


def test_prefill_varlen_shares_the_operand_checks():
    q, k, v, sl, _, _, _ = operands()
    with pytest.raises(ValueError, match="shape"):
        la.prefill_varlen(q, k, v[:, :1], sl, CU)
    with pytest.raises(ValueError, match="bfloat16 or all float32"):
        la.prefill_varlen(q, k, v.half(), sl, CU)
    with pytest.raises(ValueError, match="state_in"):
        la.prefill_varlen(q, k, v, sl, CU, state_in=torch.zeros((3, H, D, D)))
