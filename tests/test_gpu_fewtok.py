"""GPU parity of the few-token forward (M <= 32 tokens) against the CPU oracle.

This path streams the packed codes through a TMA ring, expands them with a
code-byte table and multiplies with register-resident tensor-core fragments;
the block scale is applied to each block's partial sum, row blocks shared by
several CTAs are combined by a finish kernel, and T_s = BF16(s X A^T) comes
from partial sums that sixteen CTAs of the main kernel compute.  The shapes below
cover ragged rows (d not a multiple of the 256-row item), ragged K (k not a
multiple of the 256-column item), odd and large ranks, double quantisation
off, row blocks split over many CTAs and a single item.

Tolerances as for every linear-layer output: relative Frobenius error <= 1e-2
and element max-abs error <= 2e-2 * max|ref|."""
import numpy as np
import pytest
import torch

from bit_quantized_lora_02_b200 import synth
from oracle import qlora_oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import bit_quantized_lora_02_b200 as Q
    from gpu_util import assert_close, dev_bf16, host_bits, host_f32


def _fwd(L, alpha, dq=True, save_T=True):
    W = dev_bf16(L["W0"])
    q = Q.nf4_quantize(W, double_quant=dq)
    X, A, B = (dev_bf16(L[n]) for n in ("X", "A", "B"))
    Y, T = Q.qlora_linear_fwd(X, q, A, B, alpha, save_T=save_T)
    torch.cuda.synchronize()
    assert Q.qlora_device_status() == 0
    return q, Y, T


def _check(L, Y, T, alpha, dq=True):
    r = L["A"].shape[0]
    qo = O.quantize_tensor(L["W0"].reshape(-1), double_quant=bool(dq), dq_fp8=(dq == 2))
    Wh = O.dequantize_tensor(qo).reshape(L["W0"].shape)
    Y_ref, T_ref = O.qlora_forward(L["X"], Wh, L["A"], L["B"], alpha, r)
    assert_close(host_f32(Y), Y_ref, "Y")
    if T is not None:
        Tg = host_f32(T)
        assert_close(Tg[:, :r], float(O.lora_scale(alpha, r)) * T_ref, "T_save")
        assert np.all(Tg[:, r:] == 0)


@pytest.mark.parametrize("M,d,k,r", [
    (1, 296, 320, 5),        # ragged rows and K, odd rank
    (3, 776, 1088, 16),
    (8, 256, 256, 8),        # one item
    (9, 520, 704, 72),       # 16-token tile, two rank groups of 64
    (16, 1000, 2048, 64),
    (16, 64, 64, 256),       # one NF4 block per row, largest rank
    (4, 1024, 16384, 16),    # each row block shared by ~37 CTAs
    (2, 4096, 576, 16),      # many row blocks, two items each
    (5, 776, 3072, 16),      # c2 through TMA with c1 groups changing inside rows (48 blocks per row)
    # 17..32 tokens: items of 128 rows, each warp 32 rows of 32 token slots
    (17, 392, 320, 5),       # ragged rows (not a multiple of 128) and K, odd rank
    (24, 776, 3072, 16),     # c2 through TMA, c1 groups changing inside rows
    (32, 1000, 2048, 64),
    (32, 128, 64, 256),      # one NF4 block per row, largest rank
    (20, 4096, 576, 16),     # many row blocks
    (29, 1024, 16384, 16),   # each row block shared by many CTAs
])
def test_fewtok_shapes(M, d, k, r):
    L = synth.layer(M, d, k, r, seed=100 + M + r)
    _, Y, T = _fwd(L, 16.0)
    _check(L, Y, T, 16.0)


def test_fewtok_dq_off():
    L = synth.layer(5, 600, 960, 16, seed=7)
    _, Y, T = _fwd(L, 32.0, dq=False)
    _check(L, Y, T, 32.0, dq=False)


def test_fewtok_32_tokens_dq_off_and_e4m3():
    """17..32 tokens with single-level constants (loaded one item ahead) and
    with E4M3 second-level constants through TMA."""
    L = synth.layer(25, 600, 960, 16, seed=17)
    _, Y, T = _fwd(L, 32.0, dq=False)
    _check(L, Y, T, 32.0, dq=False)
    L = synth.layer(30, 520, 3072, 8, seed=19)
    _, Y, T = _fwd(L, 16.0, dq=2)
    _check(L, Y, T, 16.0, dq=2)


def test_fewtok_e4m3_groups_inside_rows():
    """E4M3 second-level constants through TMA, with c1 groups of 256 blocks
    starting inside rows (48 blocks per row) and ragged rows."""
    L = synth.layer(3, 520, 3072, 8, seed=9)
    _, Y, T = _fwd(L, 16.0, dq=2)
    _check(L, Y, T, 16.0, dq=2)


def test_fewtok_without_saved_T():
    L = synth.layer(7, 512, 1024, 16, seed=8)
    _, Y, T = _fwd(L, 16.0, save_T=False)
    assert T is None
    _check(L, Y, None, 16.0)


@pytest.mark.parametrize("M", [6, 32])
def test_fewtok_zero_adapter_and_repeat(M):
    """B = 0: Y equals the alpha = 0 run bit for bit.  A second identical call
    gives identical bits (the partial sums of W^ X and of X A^T are added in a
    fixed order)."""
    d, k, r = 1024, 4096, 16
    L = synth.layer(M, d, k, r, seed=11)
    L["B"] = np.zeros_like(L["B"])
    q, Y0, _ = _fwd(L, 16.0)
    X, A = dev_bf16(L["X"]), dev_bf16(L["A"])
    B2 = dev_bf16(synth.lora_b(d, r, seed=12))
    Ya, _ = Q.qlora_linear_fwd(X, q, A, B2, 0.0)
    B0 = dev_bf16(L["B"])
    Yb, _ = Q.qlora_linear_fwd(X, q, A, B0, 16.0)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(Y0), host_bits(Ya))
    assert np.array_equal(host_bits(Y0), host_bits(Yb))
    _check(L, Y0, None, 16.0)
