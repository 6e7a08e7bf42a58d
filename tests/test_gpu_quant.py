"""GPU parity: NF4 quantisation, double quantisation and dequantisation are
bit-exact against the CPU oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

from bit_quantized_lora_02_b200 import synth
from oracle import qlora_oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import bit_quantized_lora_02_b200 as Q
    from gpu_util import dev_bf16, gpu_quantized_arrays, host_bits


def _roundtrip(bits: np.ndarray, dq):
    """GPU quantize + dequantize vs the oracle; all outputs bit-exact.
    dq: False (fp32 absmax), True (Int8 constants) or 2 (E4M3 constants)."""
    d, k = bits.shape if bits.ndim == 2 else (1, bits.size)
    W = dev_bf16(bits.reshape(d, k))
    q = Q.nf4_quantize(W, double_quant=dq)
    Wh = Q.nf4_dequantize(q)
    torch.cuda.synchronize()
    ref = O.quantize_tensor(bits.reshape(-1), double_quant=bool(dq), dq_fp8=(dq == 2))
    got = gpu_quantized_arrays(q, ref["n"])
    assert np.array_equal(got["packed"], ref["packed"]), "packed codes"
    if dq:
        assert np.array_equal(got["mean"].view(np.uint32), np.array([ref["mean"]], np.float32).view(np.uint32)), "mean"
        assert np.array_equal(got["c1"].view(np.uint32), ref["c1"].view(np.uint32)), "c1"
        assert np.array_equal(got["c2"].view(np.uint8), ref["c2"].view(np.uint8)), "c2"
    else:
        assert np.array_equal(got["absmax"].view(np.uint32), ref["absmax"].view(np.uint32)), "absmax"
    ref_w = O.dequantize_tensor(ref)
    assert np.array_equal(host_bits(Wh).reshape(-1), ref_w), "dequantized bf16"
    assert Q.qlora_device_status() == 0
    return q


@pytest.mark.parametrize("dq", [True, False, 2])
def test_tiny_layer_weight(dq):
    """The tiny layer: W0 512 x 512 ~ N(0, 0.02), blocksize 64, DQ groups of 256."""
    _roundtrip(synth.weight(512, 512, seed=0), dq)


@pytest.mark.parametrize("shape", [(3, 37), (5, 200), (1, 64 * 257 + 9), (7, 1000), (2, 8), (1, 1), (130, 64)])
@pytest.mark.parametrize("dq", [True, False, 2])
def test_ragged_sizes(shape, dq):
    """N not a multiple of 8 or 64, partial last DQ group, single element."""
    d, k = shape
    _roundtrip(synth.weight(d, k, seed=11, outliers=True), dq)


def test_zero_blocks_and_signs():
    bits = synth.weight(8, 512, seed=3)
    w = O.bf16_bits_to_f32(bits).copy()
    w[0, :64] = 0.0                  # all-zero block -> code 7, absmax 0
    w[1, 64:128] = -0.0              # negative zeros
    w[2, 128:192] = -np.abs(w[2, 128:192])
    w[3, :] = 0.0                    # whole rows of zeros
    w[4, 5] = 3.0                    # large outlier
    for dq in (True, False, 2):
        _roundtrip(O.bf16_round_bits(w), dq)


@pytest.mark.parametrize("dq", [True, 2])
def test_all_zero_tensor(dq):
    bits = np.zeros((4, 256), np.uint16)
    q = _roundtrip(bits, dq)
    assert float(q.mean[0]) == 0.0


def _pairs_matrix(scale_exp: int):
    """Blocks that pair every bf16 significand of the block scale s (exponent
    `scale_exp`) with a sweep of bf16 weights |w| <= s of both signs."""
    svals = ((0x3F80 + np.arange(128)) << 16).astype(np.uint32).view(np.float32) * np.float32(2.0 ** scale_exp)
    rows = []
    for s in svals:
        sb = int(np.array([s], np.float32).view(np.uint32)[0] >> 16)
        lo = max(sb - 16 * 128, 0x0080)      # 16 binades below s, normal values
        pos = np.arange(lo, sb + 1, dtype=np.uint32)
        ws = np.concatenate([pos, pos | 0x8000]).astype(np.uint16)
        nblk = -(-ws.size // 63)
        blocks = np.zeros((nblk, 64), np.uint16)
        flat = np.zeros(nblk * 63, np.uint16)
        flat[:ws.size] = ws
        blocks[:, 1:] = flat.reshape(nblk, 63)
        blocks[:, 0] = sb                    # the absmax element
        rows.append(blocks.reshape(-1))
    return np.concatenate(rows)


@pytest.mark.parametrize("scale_exp", [0, -7, 40, -60, 61, -100, 100])
def test_code_search_exhaustive_over_significand_pairs(scale_exp):
    """Every bf16 significand of the scale against weights spanning 16
    binades below it: the GPU code search equals the oracle's fp32-distance
    argmin (inside and outside the fast-division range)."""
    bits = _pairs_matrix(scale_exp)
    n = bits.size
    W = dev_bf16(bits.reshape(1, n))
    q = Q.nf4_quantize(W, double_quant=False)
    torch.cuda.synchronize()
    codes, absmax = O.nf4_quantize(O.bf16_bits_to_f32(bits))
    got = q.codes[: (n + 1) // 2].cpu().numpy()
    assert np.array_equal(got, O.pack_codes(codes))


def test_subnormal_scales():
    """Blocks whose absmax is a bf16 subnormal or tiny normal."""
    rng = np.random.default_rng(5)
    sub = rng.integers(1, 0x80, size=64 * 40, dtype=np.uint16)        # positive subnormals
    sub[::3] |= 0x8000
    tiny = rng.integers(0x0080, 0x0400, size=64 * 40, dtype=np.uint16)
    bits = np.concatenate([sub, tiny])
    _roundtrip(bits.reshape(1, -1), False)
    _roundtrip(bits.reshape(1, -1), True)


@pytest.mark.parametrize("shape", [(4096, 4096), (4096, 11008)])
@pytest.mark.parametrize("dq", [True, False, 2])
def test_quant_sweep_full_size(shape, dq):
    """Quantisation sweep: W0 ~ N(0, 0.02) with 1% N(0, 0.2) outliers."""
    d, k = shape
    _roundtrip(synth.weight(d, k, seed=0, outliers=True), dq)


def test_status_clean():
    assert Q.qlora_device_status() == 0
