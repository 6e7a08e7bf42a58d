"""GPU parity for adapter dropout ("LoRA and QLoRA: Efficient Fine-Tuning of
Large Language Models" (fromzero2ai.dev), "Python Implementation: Fine-Tuning
with PEFT and BitsAndBytes", step 4, lora_dropout) against the CPU oracle.

The keep decisions (Philox4x32-10 keyed by seed and offset, one 32-bit word
per element) are integer work: the library's mask must equal the oracle's bit
for bit.  Y, T_save, dX, dA and dB are compared with the oracle's dropout
forward and backward on the oracle's own mask, at the layer tolerance
(relative Frobenius <= 1e-2, element max-abs <= 2e-2 max|ref|)."""
import numpy as np
import pytest
import torch

from bit_quantized_lora_02_b200 import synth
from oracle import qlora_oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import bit_quantized_lora_02_b200 as Q
    from gpu_util import assert_close, dev_bf16, host_bits, host_f32


def _unpack(words: torch.Tensor, n: int) -> np.ndarray:
    w = words.cpu().numpy().view(np.uint32)
    bits = (w[:, None] >> np.arange(32, dtype=np.uint32)[None, :]) & 1
    return bits.reshape(-1).astype(bool), bits.reshape(-1)[n:]


@pytest.mark.parametrize("M,k,p,seed,offset", [
    (1, 1, 0.05, 0, 0),
    (3, 37, 0.3, 7, 1),                        # ragged: 111 elements, the last word part-filled
    (7, 1000, 0.05, 2 ** 40 + 3, 2 ** 33 + 5),  # seed and offset above 32 bits
    (1024, 1024, 0.05, 1234, 0),
    (64, 4096, 0.5, 99, 17),
    (16, 64, 0.0, 5, 5),                       # p = 0 keeps everything
])
def test_mask_bit_exact(M, k, p, seed, offset):
    n = M * k
    words = Q.qlora_dropout_mask(M, k, p, seed, offset)
    torch.cuda.synchronize()
    got, tail = _unpack(words, n)
    want = O.dropout_keep(M, k, p, seed, offset).reshape(-1)
    assert np.array_equal(got[:n], want)
    assert not tail.any()                       # bits past M k are zero


def _layer(M, d, k, r, seed):
    return synth.layer(M, d, k, r, seed=seed)


def _run(L, alpha, drop, T_saved=True):
    q = Q.nf4_quantize(dev_bf16(L["W0"]), double_quant=True)
    X, A, B, dY = (dev_bf16(L[n]) for n in ("X", "A", "B", "dY"))
    Y, T = Q.qlora_linear_fwd(X, q, A, B, alpha, dropout=drop)
    dX, dA, dB = Q.qlora_linear_bwd(dY, X, q, A, B, alpha, T_save=T if T_saved else None, dropout=drop)
    torch.cuda.synchronize()
    assert Q.qlora_device_status() == 0
    return {"Y": Y, "T": T, "dX": dX, "dA": dA, "dB": dB}


def _check(L, out, alpha, drop):
    p, seed, offset = drop
    M, k = L["X"].shape
    r = L["A"].shape[0]
    keep = O.dropout_keep(M, k, p, seed, offset)
    Wh = O.dequantize_tensor(O.quantize_tensor(L["W0"].reshape(-1), True)).reshape(L["W0"].shape)
    Y_ref, T_ref = O.qlora_forward_dropout(L["X"], Wh, L["A"], L["B"], alpha, r, keep, p)
    assert_close(host_f32(out["Y"]), Y_ref, "Y")
    s = float(O.lora_scale(alpha, r))
    Tg = host_f32(out["T"])
    assert_close(Tg[:, :r], s * T_ref, "T_save")
    assert np.all(Tg[:, r:] == 0)
    dX_ref, dA_ref, dB_ref = O.qlora_backward_dropout(L["dY"], L["X"], Wh, L["A"], L["B"], alpha, r, keep, p)
    assert_close(host_f32(out["dX"]), dX_ref, "dX")
    assert_close(host_f32(out["dA"]), dA_ref, "dA")
    assert_close(host_f32(out["dB"]), dB_ref, "dB")


@pytest.mark.parametrize("M,d,k,r,p", [
    (200, 520, 704, 16, 0.05),     # paired GEMMs, ragged tiles
    (256, 512, 1024, 64, 0.5),     # a large p: the mask decides much of the adapter term
    (130, 264, 192, 5, 0.3),       # r not a multiple of 8
    (128, 384, 512, 256, 0.1),     # largest rank (four K chunks of the adapter term)
    (33, 1024, 2048, 16, 0.05),    # swapped forward (33..128 tokens)
    (8, 1024, 2048, 16, 0.2),      # few-token forward (<= 32 tokens)
    (20, 520, 1024, 16, 0.1),      # few-token forward with 17..32 tokens
    (1, 512, 256, 8, 0.4),         # a single token
])
def test_dropout_layer(M, d, k, r, p):
    L = _layer(M, d, k, r, seed=60 + M)
    drop = (p, 1000 + M, 3)
    out = _run(L, 16.0, drop)
    _check(L, out, 16.0, drop)


def test_dropout_recomputed_T_matches_saved():
    L = _layer(150, 256, 320, 8, seed=71)
    drop = (0.25, 5, 9)
    a = _run(L, 16.0, drop, T_saved=True)
    b = _run(L, 16.0, drop, T_saved=False)
    for key in ("dX", "dA", "dB"):
        assert torch.equal(a[key], b[key]), key
    _check(L, b, 16.0, drop)


def test_dropout_mask_seen_through_T():
    """X = 1 and A = the identity make T_save = BF16(s / (1 - p)) exactly where
    the oracle keeps an element and 0 where it drops it: the mask the layer
    applied, read back bit for bit (few-token and many-token paths)."""
    k = r = 64
    for M in (8, 300):
        p, seed, offset = 0.3, 77 + M, 11
        X = np.full((M, k), 0x3F80, np.uint16)                        # 1.0
        A = np.where(np.eye(r, k, dtype=bool), np.uint16(0x3F80), np.uint16(0))
        B = synth.lora_b(64, r, seed=1)
        q = Q.nf4_quantize(dev_bf16(synth.weight(64, k, seed=2)), double_quant=True)
        Y, T = Q.qlora_linear_fwd(dev_bf16(X), q, dev_bf16(A), dev_bf16(B), 16.0, dropout=(p, seed, offset))
        torch.cuda.synchronize()
        keep = O.dropout_keep(M, k, p, seed, offset)
        val = O.bf16_round_bits(np.array([float(O.lora_scale(16.0, r)) * float(O.dropout_scale(p))], np.float32))[0]
        want = np.where(keep, val, np.uint16(0))
        assert np.array_equal(host_bits(T)[:, :r], want), M


def test_dropout_p0_is_the_plain_layer_bitwise():
    L = _layer(200, 520, 704, 16, seed=81)
    q = Q.nf4_quantize(dev_bf16(L["W0"]), double_quant=True)
    X, A, B, dY = (dev_bf16(L[n]) for n in ("X", "A", "B", "dY"))
    plain = Q.qlora_linear_fwd(X, q, A, B, 16.0) + Q.qlora_linear_bwd(dY, X, q, A, B, 16.0)
    zero = (Q.qlora_linear_fwd(X, q, A, B, 16.0, dropout=(0.0, 3, 4)) +
            Q.qlora_linear_bwd(dY, X, q, A, B, 16.0, dropout=(0.0, 3, 4)))
    torch.cuda.synchronize()
    for a, b in zip(plain, zero):
        assert torch.equal(a, b)


def test_dropout_depends_on_seed_and_offset_only():
    L = _layer(130, 256, 512, 16, seed=91)
    q = Q.nf4_quantize(dev_bf16(L["W0"]), double_quant=True)
    X, A, B = (dev_bf16(L[n]) for n in ("X", "A", "B"))
    _, T1 = Q.qlora_linear_fwd(X, q, A, B, 16.0, dropout=(0.1, 5, 6))
    _, T2 = Q.qlora_linear_fwd(X, q, A, B, 16.0, dropout=(0.1, 5, 6))
    _, T3 = Q.qlora_linear_fwd(X, q, A, B, 16.0, dropout=(0.1, 5, 7))
    torch.cuda.synchronize()
    assert torch.equal(T1, T2)
    assert not torch.equal(T1, T3)
    assert Q.qlora_device_status() == 0
