"""GPU parity of the LoRA merge against the CPU oracle.

"LoRA and QLoRA" (chkda.github.io/posts/lora_qlora), "Merging LoRA weights for
inference": W_merged = W0 + (alpha/r) B A, with the reconstructed NF4 weight as
the base.  The kernel accumulates B A in fp32 and rounds fma(s, acc, W^) once to
bf16, so every element must lie within one bf16 ulp of the fp64 oracle value,
plus an allowance for the fp32 accumulation of s B A (2^-20 of the magnitudes
involved, far below a bf16 ulp of 2^-8 relative).  With B = 0 the result must
equal the reconstructed weight bit for bit, and X W_merged^T must match the
two-path forward within the layer tolerance (the page's equivalence claim)."""
import numpy as np
import pytest
import torch

from bit_quantized_lora_02_b200 import synth
from oracle import qlora_oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import bit_quantized_lora_02_b200 as Q
    from gpu_util import assert_close, dev_bf16, host_bits, host_f32


def _bf16_ulp(x: np.ndarray) -> np.ndarray:
    a = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def _check_merge(got_bits, W_hat_bits, A, B, alpha, r, what):
    ref = O.lora_merge(W_hat_bits, A, B, alpha, r)
    got = O.bf16_bits_to_f32(got_bits).astype(np.float64)
    s = float(O.lora_scale(alpha, r))
    mag = np.abs(O.bf16_bits_to_f32(W_hat_bits)) + s * (np.abs(O.bf16_bits_to_f32(B).astype(np.float64))
                                                        @ np.abs(O.bf16_bits_to_f32(A).astype(np.float64)))
    bound = _bf16_ulp(ref) + 2.0 ** -20 * mag
    err = np.abs(got - ref)
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} elements off, worst {np.max(err - bound):.3e}"


@pytest.mark.parametrize("d,k,r,dq,b_std", [
    (8, 64, 1, True, 0.01),          # smallest shape, rank 1
    (72, 320, 5, True, 0.5),         # ragged rows and columns, odd rank, large adapter
    (256, 512, 64, True, 0.5),
    (136, 1088, 72, True, 0.5),      # rank above one 64-wide chunk, with a remainder
    (64, 256, 256, True, 0.2),       # largest rank
    (520, 704, 16, False, 0.5),      # DQ off
])
def test_merge_shapes(d, k, r, dq, b_std):
    L = synth.layer(4, d, k, r, seed=300 + r)
    B = synth.lora_b(d, r, seed=301 + r, std=b_std)
    q = Q.nf4_quantize(dev_bf16(L["W0"]), double_quant=dq)
    Wm = Q.qlora_lora_merge(q, dev_bf16(L["A"]), dev_bf16(B), 16.0)
    torch.cuda.synchronize()
    qo = O.quantize_tensor(L["W0"].reshape(-1), double_quant=dq)
    Wh = O.dequantize_tensor(qo).reshape(d, k)
    _check_merge(host_bits(Wm), Wh, L["A"], B, 16.0, r, f"merge {d}x{k} r={r}")


def test_merge_zero_adapter_is_the_reconstructed_weight():
    d, k, r = 200, 576, 16
    L = synth.layer(4, d, k, r, seed=9)
    q = Q.nf4_quantize(dev_bf16(L["W0"]), double_quant=True)
    Wm = Q.qlora_lora_merge(q, dev_bf16(L["A"]), dev_bf16(np.zeros((d, r), np.uint16)), 16.0)
    torch.cuda.synchronize()
    Wh = O.dequantize_tensor(O.quantize_tensor(L["W0"].reshape(-1), double_quant=True)).reshape(d, k)
    assert np.array_equal(host_bits(Wm), Wh)


def test_merged_forward_matches_two_path():
    M, d, k, r = 24, 384, 768, 32
    L = synth.layer(M, d, k, r, seed=10)
    B = synth.lora_b(d, r, seed=11, std=0.3)
    q = Q.nf4_quantize(dev_bf16(L["W0"]), double_quant=True)
    Wm = Q.qlora_lora_merge(q, dev_bf16(L["A"]), dev_bf16(B), 16.0)
    torch.cuda.synchronize()
    Wh = O.dequantize_tensor(O.quantize_tensor(L["W0"].reshape(-1), double_quant=True)).reshape(d, k)
    Y_two, _ = O.qlora_forward(L["X"], Wh, L["A"], B, 16.0, r)
    Y_merged = O.bf16_bits_to_f32(L["X"]).astype(np.float64) @ host_f32(Wm).astype(np.float64).T
    assert_close(Y_merged, Y_two, "X W_merged^T vs two-path forward")


def test_merge_full_size_sampled_rows():
    """4096 x 4096, r = 64 (the projection the bench times), DQ off so that the
    oracle can quantise the sampled rows alone (every block lies in one row)."""
    d, k, r = 4096, 4096, 64
    W0 = synth.weight(d, k, seed=12)
    A = synth.lora_a(r, k, seed=12)
    B = synth.lora_b(d, r, seed=12, std=0.5)
    q = Q.nf4_quantize(dev_bf16(W0), double_quant=False)
    Wm = Q.qlora_lora_merge(q, dev_bf16(A), dev_bf16(B), 16.0)
    torch.cuda.synchronize()
    rows = np.random.default_rng(12).choice(d, size=48, replace=False)
    rows = np.concatenate([rows, [0, d - 1]])
    got = host_bits(Wm)[rows]
    qo = O.quantize_tensor(W0[rows].reshape(-1), double_quant=False)
    Wh = O.dequantize_tensor(qo).reshape(len(rows), k)
    _check_merge(got, Wh, A, B[rows], 16.0, r, "merge 4096x4096 sampled rows")


def test_merge_e4m3_constants():
    d, k, r = 136, 576, 16
    L = synth.layer(4, d, k, r, seed=31)
    B = synth.lora_b(d, r, seed=32, std=0.5)
    q = Q.nf4_quantize(dev_bf16(L["W0"]), double_quant=2)
    Wm = Q.qlora_lora_merge(q, dev_bf16(L["A"]), dev_bf16(B), 16.0)
    torch.cuda.synchronize()
    Wh = O.dequantize_tensor(O.quantize_tensor(L["W0"].reshape(-1), double_quant=True, dq_fp8=True)).reshape(d, k)
    _check_merge(host_bits(Wm), Wh, L["A"], B, 16.0, r, "merge with E4M3 constants")
