"""GPU parity for grouped projections ("LoRA and QLoRA: Efficient Fine-Tuning
of Large Language Models" (fromzero2ai.dev), "4. Define LoRA Target Modules
and Config": q, k, v read the same input, as gate and up do) against the CPU
oracle, projection by projection.

Each W_i is quantised on its own into the group's stacked buffers, so its
codes and constants must equal the oracle's quantisation of W_i alone, bit
for bit.  The grouped layer must give, for every projection i,
Y_i = X W^_i^T + s (X A_i^T) B_i^T, T_i, dA_i and dB_i of the oracle's
single layer, and dX = the sum of the projections' dX, at the layer
tolerance (relative Frobenius <= 1e-2, element max-abs <= 2e-2 max|ref|)."""
import numpy as np
import pytest
import torch

from bit_quantized_lora_02_b200 import synth
from oracle import qlora_oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import bit_quantized_lora_02_b200 as Q
    from gpu_util import assert_close, dev_bf16, host_f32


def _group_inputs(M, ds, k, r, seed):
    Ws = [synth.weight(d, k, seed=seed + i) for i, d in enumerate(ds)]
    As = [synth.lora_a(r, k, seed=seed + i) for i in range(len(ds))]
    Bs = [synth.lora_b(d, r, seed=seed + i) for i, d in enumerate(ds)]
    X = synth.activations(M, k, seed=seed)
    dY = synth.grad_output(M, sum(ds), seed=seed)
    return Ws, As, Bs, X, dY


def _oracle_q(W, dq):
    return O.quantize_tensor(W.reshape(-1), double_quant=bool(dq), dq_fp8=(dq == 2))


@pytest.mark.parametrize("M,ds,k,r,dq", [
    (300, (256, 256, 520), 512, 16, 1),    # paired GEMMs, ragged last projection
    (600, (512, 256), 704, 64, 1),         # two projections (gate, up), ragged K
    (200, (256, 256, 256), 256, 8, 0),     # single-level constants
    (300, (256, 256), 512, 16, 2),         # E4M3 second-level constants
    (64, (256, 512, 256), 1024, 16, 1),    # swapped forward (33..128 tokens)
    (8, (256, 256, 256), 512, 16, 1),      # few-token forward (<= 32 tokens)
    (8, (256, 512, 256), 1024, 16, 1),     # few-token forward, c2 through TMA, one mean per projection
    (24, (256, 256, 512), 1024, 16, 1),    # few-token forward with 17..32 tokens (128-row items)
    (1, (512, 256), 256, 8, 1),            # a single token
    (130, (256, 256, 256, 256), 512, 64, 1),   # four projections, n r = 256
])
def test_grouped_layer(M, ds, k, r, dq):
    n = len(ds)
    alpha = 16.0
    Ws, As, Bs, X, dY = _group_inputs(M, ds, k, r, seed=10 * M + n)
    g = Q.nf4_quantize_group([dev_bf16(W) for W in Ws], double_quant=dq)
    A = dev_bf16(np.concatenate(As, axis=0))
    B = dev_bf16(np.concatenate(Bs, axis=0))
    Xg, dYg = dev_bf16(X), dev_bf16(dY)
    Y, T = Q.qlora_linear_fwd_grouped(Xg, g, A, B, alpha)
    dX, dA, dB = Q.qlora_linear_bwd_grouped(dYg, Xg, g, A, B, alpha, T_save=T)
    torch.cuda.synchronize()
    assert Q.qlora_device_status() == 0

    s = float(O.lora_scale(alpha, r))
    Yh, Th, dAh, dBh, dXh = host_f32(Y), host_f32(T), host_f32(dA), host_f32(dB), host_f32(dX)
    dX_ref = np.zeros((M, k))
    row = 0
    for i, d in enumerate(ds):
        qo = _oracle_q(Ws[i], dq)
        part = g.parts[i]
        nb = d * k // 64
        assert np.array_equal(part.codes[: d * k // 2].cpu().numpy(), qo["packed"]), i
        if dq:
            assert np.array_equal(part.c2[:nb].cpu().numpy().view(np.uint8), qo["c2"].view(np.uint8)), i
            assert np.array_equal(part.c1[: -(-nb // 256)].cpu().numpy(), qo["c1"]), i
            assert part.mean.cpu().numpy()[0] == qo["mean"], i
        Wh = O.dequantize_tensor(qo).reshape(d, k)
        Y_ref, T_ref = O.qlora_forward(X, Wh, As[i], Bs[i], alpha, r)
        assert_close(Yh[:, row:row + d], Y_ref, f"Y_{i}")
        assert_close(Th[:, i * r:(i + 1) * r], s * T_ref, f"T_{i}")
        dXi, dAi, dBi = O.qlora_backward(dY[:, row:row + d], X, Wh, As[i], Bs[i], alpha, r)
        dX_ref += dXi
        assert_close(dAh[i * r:(i + 1) * r], dAi, f"dA_{i}")
        assert_close(dBh[row:row + d], dBi, f"dB_{i}")
        row += d
    assert np.all(Th[:, n * r:] == 0)
    assert_close(dXh, dX_ref, "dX")


def test_grouped_equals_separate_calls_on_the_gemm_path():
    """The grouped launch and n single-layer launches on the same buffers
    accumulate in the same order on the paired GEMMs: Y agrees bit for bit."""
    M, ds, k, r = 512, (256, 512), 1024, 16
    Ws, As, Bs, X, _ = _group_inputs(M, ds, k, r, seed=5)
    g = Q.nf4_quantize_group([dev_bf16(W) for W in Ws])
    Xg = dev_bf16(X)
    Y, _ = Q.qlora_linear_fwd_grouped(Xg, g, dev_bf16(np.concatenate(As)), dev_bf16(np.concatenate(Bs)), 16.0)
    row = 0
    for i, d in enumerate(ds):
        Yi, _ = Q.qlora_linear_fwd(Xg, g.parts[i], dev_bf16(As[i]), dev_bf16(Bs[i]), 16.0)
        torch.cuda.synchronize()
        assert torch.equal(Y[:, row:row + d], Yi), i
        row += d
