"""GPU parity at the full sizes the benchmark times, against the CPU oracle.

Shapes ("LoRA and QLoRA" (chkda), "Double quantization and double
dequantization", the QLoRA expression, applied to the projection shapes of the
synthetic workloads):
  * the 7B-style set's gate/up (11008 x 4096) and down (4096 x 11008)
    projections at M = 4096 tokens, r = 64, alpha = 16;
  * the 65B-style block's q/k/v/o (8192 x 8192), gate/up (22016 x 8192) and
    down (8192 x 22016) projections at M = 8192 tokens, r = 64, alpha = 16;
  * the decode-like forward on 28672 x 8192 and 8192 x 28672 weights with
    M in {1, 8, 32, 128}, r = 16, alpha = 32.

Each training-shape case runs exactly what one bench step runs for that
projection (quantise, forward with T_save, backward), on the bench's seeded
inputs (projection index as seed).  The oracle quantises and reconstructs the
whole weight, then computes Y and dX on 64 sampled token rows and dA, dB in
full; the decode cases compare every element of Y.  Tolerance: relative
Frobenius error <= 1e-2 and element max-abs <= 2e-2 * max|ref|."""
import numpy as np
import pytest
import torch

from bit_quantized_lora_02_b200 import synth
from oracle import qlora_oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import bit_quantized_lora_02_b200 as Q
    from gpu_util import assert_close, dev_bf16, host_f32

_CACHE = {}


def _oracle_weight(d, k, seed):
    """Oracle reconstruction W^ of the seeded weight (bf16 bits), cached for
    the shape last used so the decode cases quantise each weight once."""
    key = (d, k, seed)
    if key not in _CACHE:
        _CACHE.clear()
        W0 = synth.weight(d, k, seed=seed)
        q = O.quantize_tensor(W0.reshape(-1), double_quant=True)
        _CACHE[key] = (W0, O.dequantize_tensor(q).reshape(d, k))
    return _CACHE[key]


def _training_case(M, d, k, seed, r=64, alpha=16.0):
    W0, Wh = _oracle_weight(d, k, seed)
    A, B = synth.lora_a(r, k, seed=seed), synth.lora_b(d, r, seed=seed)
    X, dY = synth.activations(M, k, seed=seed), synth.grad_output(M, d, seed=seed)

    q = Q.nf4_quantize(dev_bf16(W0), double_quant=True)
    Xg, Ag, Bg, dYg = dev_bf16(X), dev_bf16(A), dev_bf16(B), dev_bf16(dY)
    Y, T = Q.qlora_linear_fwd(Xg, q, Ag, Bg, alpha)
    dX, dA, dB = Q.qlora_linear_bwd(dYg, Xg, q, Ag, Bg, alpha, T_save=T)
    torch.cuda.synchronize()
    assert Q.qlora_device_status() == 0
    del Xg, dYg, q

    rows = np.sort(np.random.default_rng(seed).choice(M, 64, replace=False))
    Y_ref, T_ref = O.qlora_forward(X[rows], Wh, A, B, alpha, r)
    assert_close(host_f32(Y[rows]), Y_ref, f"Y rows {d}x{k}")
    s = float(O.lora_scale(alpha, r))
    assert_close(host_f32(T[rows])[:, :r], s * T_ref, f"T_save rows {d}x{k}")
    dX_ref, _, _ = O.qlora_backward(dY[rows], X[rows], Wh, A, B, alpha, r)
    assert_close(host_f32(dX[rows]), dX_ref, f"dX rows {d}x{k}")
    dA_ref, dB_ref = O.qlora_adapter_grads(dY, X, A, B, alpha, r)
    assert_close(host_f32(dA), dA_ref, f"dA {d}x{k}")
    assert_close(host_f32(dB), dB_ref, f"dB {d}x{k}")


@pytest.mark.parametrize("name,d,k,seed", [("gate", 11008, 4096, 4), ("down", 4096, 11008, 6)])
def test_llama7b_projection_full_size(name, d, k, seed):
    """The 7B-style set's K = 11008 and d = 11008 projections (ragged K steps,
    the K-split reduction and the column-pair-first cluster order)."""
    _training_case(4096, d, k, seed)


@pytest.mark.parametrize("name,d,k,seed", [("q", 8192, 8192, 0), ("gate", 22016, 8192, 4),
                                           ("down", 8192, 22016, 6)])
def test_llama65b_projection_full_size(name, d, k, seed):
    """The 65B-style block at M = 8192 tokens."""
    _training_case(8192, d, k, seed)


@pytest.mark.parametrize("M", [1, 8, 32, 128])
@pytest.mark.parametrize("d,k,seed", [(28672, 8192, 0), (8192, 28672, 1)])
def test_decode_full_size(d, k, seed, M):
    """The decode-like forward on its full weights, every element of Y."""
    r, alpha = 16, 32.0
    W0, Wh = _oracle_weight(d, k, seed)
    A, B = synth.lora_a(r, k, seed=seed), synth.lora_b(d, r, seed=seed)
    X = synth.activations(M, k, seed=seed)
    q = _device_weight(W0, d, k, seed)
    Y, T = Q.qlora_linear_fwd(dev_bf16(X), q, dev_bf16(A), dev_bf16(B), alpha)
    torch.cuda.synchronize()
    assert Q.qlora_device_status() == 0
    Y_ref, T_ref = O.qlora_forward(X, Wh, A, B, alpha, r)
    assert_close(host_f32(Y), Y_ref, f"Y {d}x{k} M={M}")
    s = float(O.lora_scale(alpha, r))
    assert_close(host_f32(T)[:, :r], s * T_ref, f"T_save {d}x{k} M={M}")


_DEV = {}


def _device_weight(W0, d, k, seed):
    key = (d, k, seed)
    if key not in _DEV:
        _DEV.clear()
        _DEV[key] = Q.nf4_quantize(dev_bf16(W0), double_quant=True)
    return _DEV[key]
