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


def test_backward_requires_X():
    q = _weight()
    M, r = 8, 4
    with pytest.raises(ValueError, match="X is required"):
        Q.qlora_linear_bwd(bf16(M, 64), None, q, bf16(r, 128), bf16(64, r), 16.0)


def test_weight_buffers_checked_against_the_library_sizes():
    """Every NF4Weight buffer is compared with qlora_nf4_sizes(d, k) for its
    mode: an undersized, mistyped or missing buffer raises before any pointer
    reaches the library."""
    M, r = 8, 4
    args = (bf16(M, 128), None, bf16(r, 128), bf16(64, r), 16.0)

    def fwd(q):
        Q.qlora_linear_fwd(args[0], q, *args[2:])
    q = _weight()
    q.codes = q.codes[:-1]
    with pytest.raises(ValueError, match="codes: .* needs"):
        fwd(q)
    q = _weight()
    q.c2 = torch.zeros(64 * 128 // 64 - 1, dtype=torch.int8)
    with pytest.raises(ValueError, match="c2: .* needs"):
        fwd(q)
    q = _weight()
    q.c2 = q.c2.view(torch.uint8)
    with pytest.raises(ValueError, match="c2: dtype"):
        fwd(q)
    q = _weight()
    q.mean = None
    with pytest.raises(ValueError, match="mean is required"):
        fwd(q)
    q = _weight()
    q.double_quant = 0                 # absmax buffer missing for single-level constants
    with pytest.raises(ValueError, match="absmax is required"):
        fwd(q)
    q = _weight()
    q.double_quant = 2                 # E4M3 constants are bytes, not int8
    with pytest.raises(ValueError, match="c2: dtype"):
        fwd(q)


def test_weight_buffers_must_share_the_activations_device():
    q = _weight()
    q.c1 = torch.ones(1, dtype=torch.float32, device="meta")
    with pytest.raises(ValueError, match="c1 is on meta"):
        Q.qlora_linear_fwd(bf16(8, 128), q, bf16(4, 128), bf16(64, 4), 16.0)


def test_noalloc_rejects_a_mismatched_output_descriptor():
    W0 = bf16(64, 128)
    with pytest.raises(ValueError, match="out describes a 32x128 weight"):
        Q.nf4_quantize_noalloc(W0, True, out=_weight(32, 128))
    with pytest.raises(ValueError, match="double_quant=1 buffers"):
        Q.nf4_quantize_noalloc(W0, 2, out=_weight(64, 128))
    with pytest.raises(ValueError, match="out describes a 32x128 weight"):
        Q.nf4_quantize(W0, True, out=_weight(32, 128))
