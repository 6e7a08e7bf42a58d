"""The Python binding checks shapes, dtypes and contiguity before it hands raw
pointers to the C ABI (CPU tensors; nothing reaches a GPU)."""
import pytest
import torch

import bit_quantized_lora_02_b200 as Q


def _weight(d=64, k=128):
    return Q.NF4Weight(d, k, 1, torch.zeros(d * k // 2, dtype=torch.uint8), None, torch.zeros(d * k // 64, dtype=torch.int8),
                       torch.ones(1, dtype=torch.float32), torch.zeros(1, dtype=torch.float32))


def bf16(*shape):
    return torch.zeros(*shape, dtype=torch.bfloat16)


def test_forward_rejects_mismatched_tensors():
    q = _weight()
    M, r = 8, 4
    with pytest.raises(ValueError, match="X: shape"):
        Q.qlora_linear_fwd(bf16(M, 64), q, bf16(r, 128), bf16(64, r), 16.0)            # X is M x d, not M x k
    with pytest.raises(ValueError, match="B: shape"):
        Q.qlora_linear_fwd(bf16(M, 128), q, bf16(r, 128), bf16(r, 64), 16.0)            # B transposed
    with pytest.raises(ValueError, match="X: dtype"):
        Q.qlora_linear_fwd(torch.zeros(M, 128), q, bf16(r, 128), bf16(64, r), 16.0)
    with pytest.raises(ValueError, match="contiguous"):
        Q.qlora_linear_fwd(bf16(128, M).t(), q, bf16(r, 128), bf16(64, r), 16.0)
    with pytest.raises(ValueError, match="T_save: shape"):
        Q.qlora_linear_fwd(bf16(M, 128), q, bf16(r, 128), bf16(64, r), 16.0, T_save=bf16(M, r))


def test_backward_rejects_mismatched_tensors():
    q = _weight()
    M, r = 8, 4
    with pytest.raises(ValueError, match="dY: shape"):
        Q.qlora_linear_bwd(bf16(M, 128), bf16(M, 128), q, bf16(r, 128), bf16(64, r), 16.0)
    with pytest.raises(ValueError, match="dA: dtype"):
        Q.qlora_linear_bwd(bf16(M, 64), bf16(M, 128), q, bf16(r, 128), bf16(64, r), 16.0, dA=bf16(r, 128))


def test_merge_and_dequantize_reject_mismatched_tensors():
    q = _weight()
    with pytest.raises(ValueError, match="A: shape"):
        Q.qlora_lora_merge(q, bf16(4, 64), bf16(64, 4), 16.0)
    with pytest.raises(ValueError, match="out: shape"):
        Q.qlora_lora_merge(q, bf16(4, 128), bf16(64, 4), 16.0, out=bf16(128, 64))
    with pytest.raises(ValueError, match="out: shape"):
        Q.nf4_dequantize(q, out=bf16(128, 64))
