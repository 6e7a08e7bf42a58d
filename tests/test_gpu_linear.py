"""GPU parity: QLoRA linear forward and backward against the CPU oracle.

Tolerances: relative Frobenius error <= 1e-2 and element max-abs error
<= 2e-2 * max|ref| for Y, dX, dA, dB (fp32 accumulation, bf16 outputs and a
bf16 copy of s*X*A^T / s*dY*B inside the layer)."""
import numpy as np
import pytest
import torch

from bit_quantized_lora_02_b200 import synth
from oracle import qlora_oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import bit_quantized_lora_02_b200 as Q
    from gpu_util import assert_close, dev_bf16, host_bits, host_f32


def _layer(M, d, k, r, seed=0, a_std=None, b_zero=False, outliers=False):
    L = synth.layer(M, d, k, r, seed=seed, a_std=a_std, outliers=outliers)
    if b_zero:
        L["B"] = np.zeros_like(L["B"])
    return L


def _oracle_what(W0_bits, dq=True):
    q = O.quantize_tensor(W0_bits.reshape(-1), double_quant=bool(dq), dq_fp8=(dq == 2))
    d, k = W0_bits.shape
    return O.dequantize_tensor(q).reshape(d, k)


def _run(L, alpha, dq=True, bwd=True, save_T=True):
    d, k = L["W0"].shape
    W = dev_bf16(L["W0"])
    q = Q.nf4_quantize(W, double_quant=dq)
    X, A, B, dY = (dev_bf16(L[n]) for n in ("X", "A", "B", "dY"))
    Y, T = Q.qlora_linear_fwd(X, q, A, B, alpha, save_T=save_T)
    out = {"Y": Y, "T": T}
    if bwd:
        dX, dA, dB = Q.qlora_linear_bwd(dY, X, q, A, B, alpha, T_save=T)
        out.update(dX=dX, dA=dA, dB=dB)
    torch.cuda.synchronize()
    assert Q.qlora_device_status() == 0
    return out


def _check(L, out, alpha, dq=True, bwd=True):
    r = L["A"].shape[0]
    Wh = _oracle_what(L["W0"], dq)
    Y_ref, T_ref = O.qlora_forward(L["X"], Wh, L["A"], L["B"], alpha, r)
    assert_close(host_f32(out["Y"]), Y_ref, "Y")
    if out["T"] is not None:
        s = float(O.lora_scale(alpha, r))
        Tg = host_f32(out["T"])
        assert_close(Tg[:, :r], s * T_ref, "T_save")
        assert np.all(Tg[:, r:] == 0)
    if bwd:
        dX_ref, dA_ref, dB_ref = O.qlora_backward(L["dY"], L["X"], Wh, L["A"], L["B"], alpha, r)
        assert_close(host_f32(out["dX"]), dX_ref, "dX")
        assert_close(host_f32(out["dA"]), dA_ref, "dA")
        assert_close(host_f32(out["dB"]), dB_ref, "dB")


def test_tiny_layer_fwd_bwd():
    """The tiny layer: W0 512x512, r=8, alpha=16, A ~ N(0, 1/8), B ~ N(0, 0.01),
    X 16x512, dY ~ N(0,1); seed 0."""
    L = _layer(16, 512, 512, 8, seed=0, a_std=1.0 / 8)
    out = _run(L, 16.0)
    _check(L, out, 16.0)


@pytest.mark.parametrize("M,d,k,r", [
    (200, 520, 704, 16),     # ragged in every tiled dimension
    (256, 512, 1024, 64),
    (130, 264, 192, 5),      # r not a multiple of 8
    (64, 256, 256, 72),      # r > 64: two LoRA K steps
    (128, 384, 512, 256),    # largest rank
    (1, 512, 256, 8),        # single token
    (33, 1024, 2048, 16),    # swapped small-M forward with split K
])
def test_shapes(M, d, k, r):
    L = _layer(M, d, k, r, seed=M + r)
    out = _run(L, 16.0)
    _check(L, out, 16.0)


def test_dq_off():
    L = _layer(96, 320, 448, 16, seed=4)
    out = _run(L, 32.0, dq=False)
    _check(L, out, 32.0, dq=False)


def test_zero_adapter_is_exact_base():
    """B = 0 makes the adapter contribute exact zeros: Y equals the alpha = 0 run
    bit for bit, and dA is exactly zero."""
    L = _layer(150, 512, 512, 16, seed=9, b_zero=True)
    out0 = _run(L, 16.0)
    L2 = dict(L)
    L2["B"] = synth.lora_b(512, 16, seed=99)
    outa = _run(L2, 0.0, bwd=False)
    assert np.array_equal(host_bits(out0["Y"]), host_bits(outa["Y"]))
    assert np.all(host_f32(out0["dA"]) == 0)
    _check(L, out0, 16.0)


def test_backward_recomputes_T():
    L = _layer(70, 256, 320, 8, seed=12)
    d, k = L["W0"].shape
    q = Q.nf4_quantize(dev_bf16(L["W0"]))
    X, A, B, dY = (dev_bf16(L[n]) for n in ("X", "A", "B", "dY"))
    dX, dA, dB = Q.qlora_linear_bwd(dY, X, q, A, B, 16.0, T_save=None)
    torch.cuda.synchronize()
    Wh = _oracle_what(L["W0"])
    dX_ref, dA_ref, dB_ref = O.qlora_backward(L["dY"], L["X"], Wh, L["A"], L["B"], 16.0, 8)
    assert_close(host_f32(dX), dX_ref, "dX")
    assert_close(host_f32(dA), dA_ref, "dA")
    assert_close(host_f32(dB), dB_ref, "dB")


@pytest.mark.parametrize("M", [1, 8, 32, 128])
def test_decode_like_forward(M):
    """Weight-bound forward shape family (r=16, alpha=32) at a reduced size."""
    L = _layer(M, 2048, 4096, 16, seed=M)
    out = _run(L, 32.0, bwd=False)
    _check(L, out, 32.0, bwd=False)


def test_projection_full_size_sampled():
    """One 4096x4096 projection at M=4096, r=64 (the 7B-style set), checked on
    a sample of 64 token rows: the oracle builds all of W-hat and computes
    those rows of Y and dX, plus dA and dB in full."""
    M, d, k, r, alpha = 4096, 4096, 4096, 64, 16.0
    L = _layer(M, d, k, r, seed=1)
    out = _run(L, alpha)
    rows = np.random.default_rng(0).choice(M, 64, replace=False)
    Wh = _oracle_what(L["W0"])
    Ls = {n: L[n][rows] for n in ("X", "dY")}
    Y_ref, _ = O.qlora_forward(Ls["X"], Wh, L["A"], L["B"], alpha, r)
    assert_close(host_f32(out["Y"])[rows], Y_ref, "Y rows")
    dX_ref, _, _ = O.qlora_backward(Ls["dY"], Ls["X"], Wh, L["A"], L["B"], alpha, r)
    assert_close(host_f32(out["dX"])[rows], dX_ref, "dX rows")
    _, dA_ref, dB_ref = O.qlora_backward(L["dY"], L["X"], Wh, L["A"], L["B"], alpha, r)
    assert_close(host_f32(out["dA"]), dA_ref, "dA")
    assert_close(host_f32(out["dB"]), dB_ref, "dB")


@pytest.mark.parametrize("M,d,k,r", [(200, 520, 704, 16), (4, 1024, 2048, 16), (64, 768, 1024, 32)])
def test_e4m3_constants(M, d, k, r):
    """E4M3 second-level constants through every fused path: the paired GEMMs
    (M > 128), the few-token path (M <= 16) and the swapped forward."""
    L = _layer(M, d, k, r, seed=40 + M)
    out = _run(L, 16.0, dq=2)
    _check(L, out, 16.0, dq=2)
