"""CPU oracle for the QLoRA linear layer (blockwise NF4 + double quantisation +
LoRA forward/backward).

TEST INFRASTRUCTURE ONLY.  This is a plain, slow, obviously correct numpy
restatement of what the layer computes.  It shares no code with the CUDA
library and imports nothing from it.  Only the test suite, the smoke check in
``__graft_entry__.smoke()`` and the ``cpu_baseline`` leg of ``bench.py`` may
import it; the product path never calls it.

Sources, cited by page title and section:

* [QLoRA-chkda] "LoRA and QLoRA" (chkda.github.io/posts/lora_qlora) -- the
  most precise page; it wins every conflict.
* [FromZero2AI] "LoRA and QLoRA: Efficient Fine-Tuning of Large Language
  Models" (fromzero2ai.dev).
* [CodeThePapers] "Democratizing LLM Finetuning: A Deep Dive into QLoRA".

Precision: the pages fix bf16 storage for W-hat, X, A, B (section "Double
quantization and double dequantization", QLoRA expression) and an fp32 scale
per block (section "First, how does k-bit quantization work?").  Quantisation
arithmetic is therefore carried out in fp32 with IEEE round-to-nearest, each
operation rounded once, exactly as written.  Matrix products, whose
accumulation precision the pages leave open, are done in fp64 on the exact
fp32 images of the bf16 inputs.

Readings of passages that are silent or ambiguous:

R1  Codebook: C = {Phi^-1(p_i)/Phi^-1(p*)} with 8 positive p_i evenly spaced on
    (1/2, p*] and 7 negative values mirrored from 7 evenly spaced p on
    (1/2, p*], plus an exact 0.  The tail cutoff p* is the midpoint of the
    interval of cutoffs that reproduces all 16 printed 4-decimal values.
R2  Nearest code: distances |RN32(xn - C[j])| in fp32, first minimum wins
    (the page's "choose the smaller index").
R3  xn = RN32(w / s) with IEEE division; codes use the exact block absmax.
R4  Packing: byte t = code[2t] | code[2t+1] << 4, an odd tail padded with 0.
R5  Double quantisation: the page's only spelled-out 8-bit scheme (symmetric
    Int8 absmax, Q = 127) with c1 = RN32(127 / absmax) stored in fp32,
    "round" = round half to even, an all-zero group stored as zeros with
    c1 = 1.  One mean per tensor, mu = RN32(RN64(RN64(sum s_j) / M_b)).
R6  Scale reconstruction s^_j = RN32(RN32(c2_j / c1_g) + mu);
    weight reconstruction w^ = BF16_RNE(RN32(C[q] * s^)).
R7  Forward Y = X W^T + (alpha/r) (X A^T) B^T with W^ the reconstructed bf16
    weights; backward derived by calculus (the pages print no formulas):
    U = dY B, dX = dY W^ + s U A, dA = s U^T X, dB = s dY^T T, T = X A^T.
R8  Merge ([QLoRA-chkda] "Merging LoRA weights for inference"): the base is
    the reconstructed W^, W_merged = W^ + s B A.
R9  FP8 second-level constants (the page's "c2_FP8" label): OCP E4M3 bytes,
    c1 = RN32(448 / max|v|) per group, c2 = E4M3(RN32(c1 v)) nearest even,
    saturating at 448; s^ = RN32(RN32(decode(c2) / c1) + mean).
R10 Adapter dropout ([FromZero2AI] lora_dropout): on the adapter input only,
    keep decisions from Philox4x32-10 keyed by (seed, offset) and the flat
    element index, kept values scaled by RN32(1 / RN32(1 - p)); the backward
    reuses the same decisions.
"""
from __future__ import annotations

import math
from statistics import NormalDist

import numpy as np

__all__ = [
    "TAIL_CUTOFF", "codebook_values", "nf4_codebook", "bf16_round_bits", "bf16_bits_to_f32",
    "nearest_code", "nf4_quantize", "pack_codes", "unpack_codes", "int8_absmax_quantize",
    "int8_dequantize", "exact_mean_f32", "double_quantize", "double_dequantize_scales",
    "nf4_dequantize", "quantize_tensor", "dequantize_tensor", "storage_bits_per_weight",
    "lora_trainable_params", "qlora_forward", "qlora_backward", "qlora_adapter_grads", "lora_scale", "lora_merge",
    "FP8_MAX", "fp8_e4m3_encode", "fp8_e4m3_decode", "double_quantize_fp8", "double_dequantize_scales_fp8",
    "philox4x32_10", "dropout_keep", "dropout_scale", "qlora_forward_dropout", "qlora_backward_dropout",
]

BLOCK = 64          # weights per NF4 block ([QLoRA-chkda] "QLoRA uses blocks of 64 weights")
DQ_GROUP = 256      # block scales per second-level group ([QLoRA-chkda] double quantization)
INT8_Q = 127        # symmetric Int8 range [-127, 127] ([QLoRA-chkda] k-bit quantization)

# Interval of tail cutoffs p* that reproduce every printed 4-decimal NF4 value
# ([QLoRA-chkda] "NF4: Choose the codebook to fit the distribution"); found by
# bisection on codebook_values(p) against the printed table.  Entry 4 (-0.2844)
# binds the lower end, entry 6 (-0.0911) the upper end.
TAIL_CUTOFF_INTERVAL = (0.9677023838639995, 0.9677082837944422)
TAIL_CUTOFF = 0.9677053338292209  # midpoint (reading R1)


# ----------------------------------------------------------------------------
# bf16 helpers (storage rounding written out on the bit pattern)
# ----------------------------------------------------------------------------
def bf16_round_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bits, round to nearest, ties to even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    return ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------
# NF4 codebook  ([QLoRA-chkda] "NF4: Choose the codebook to fit the
# distribution" and "Building the NF4 codebook")
# ----------------------------------------------------------------------------
def codebook_values(p_star: float = TAIL_CUTOFF) -> list[float]:
    """The 16 NF4 values in float64 for a given tail cutoff p* (reading R1).

    Evenly spaced probabilities on (1/2, p*] become normal quantiles; the
    largest is normalised to 1.  Eight positive and seven negative values plus
    an exact zero, as the page requires.
    """
    inv = NormalDist().inv_cdf
    top = inv(p_star)
    pos = [inv(0.5 + (p_star - 0.5) * i / 8) / top for i in range(1, 9)]
    neg = [-inv(0.5 + (p_star - 0.5) * i / 7) / top for i in range(1, 8)]
    return sorted(neg) + [0.0] + pos


def nf4_codebook() -> np.ndarray:
    """The frozen fp32 NF4 table C[0..15], ascending."""
    return np.array(codebook_values(TAIL_CUTOFF), dtype=np.float64).astype(np.float32)


# ----------------------------------------------------------------------------
# NF4 blockwise quantisation  ([QLoRA-chkda] "Quantizing and dequantizing with
# the codebook")
# ----------------------------------------------------------------------------
def nearest_code(xn: np.ndarray, C: np.ndarray) -> np.ndarray:
    """argmin_j |xn - C[j]| with fp32 distances; the first minimum wins (R2)."""
    xn = np.asarray(xn, dtype=np.float32)
    dist = np.abs(xn[..., None] - C.astype(np.float32))          # fp32 subtract, exact abs
    return np.argmin(dist, axis=-1).astype(np.uint8)             # argmin returns the first minimum


def nf4_quantize(w: np.ndarray, blocksize: int = BLOCK, C: np.ndarray | None = None):
    """Blockwise NF4 quantisation of a flat fp32 array (values exact in bf16).

    Per block: scale = |w[argmax |w|]|; if scale == 0 every code is the
    argmin of |C| (the exact zero); otherwise code = nearest(w / scale).
    The last block may be shorter.  Returns (codes uint8[N], absmax f32[M_b]).
    """
    C = nf4_codebook() if C is None else C
    w = np.asarray(w, dtype=np.float32).ravel()
    n = w.size
    nblk = -(-n // blocksize)
    codes = np.empty(n, dtype=np.uint8)
    absmax = np.empty(nblk, dtype=np.float32)
    zero_code = int(np.argmin(np.abs(C)))
    step = 4096 * blocksize                     # chunk only to bound memory
    for c0 in range(0, n, step):
        seg = w[c0:c0 + step]
        nb = -(-seg.size // blocksize)
        padded = np.zeros(nb * blocksize, dtype=np.float32)
        padded[:seg.size] = seg
        blocks = padded.reshape(nb, blocksize)
        s = np.max(np.abs(blocks), axis=1)      # |w[argmax]| equals the max magnitude
        absmax[c0 // blocksize:c0 // blocksize + nb] = s
        safe = np.where(s == 0, np.float32(1), s)
        xn = (blocks / safe[:, None]).astype(np.float32)   # IEEE fp32 division (R3)
        q = nearest_code(xn, C)
        q[s == 0, :] = zero_code
        codes[c0:c0 + seg.size] = q.ravel()[:seg.size]
    return codes, absmax


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """Two 4-bit codes per byte, element 2t in the low nibble (reading R4)."""
    codes = np.asarray(codes, dtype=np.uint8).ravel()
    if codes.size % 2:
        codes = np.concatenate([codes, np.zeros(1, np.uint8)])
    return (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)


def unpack_codes(packed: np.ndarray, n: int) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty(packed.size * 2, dtype=np.uint8)
    out[0::2] = packed & 0x0F
    out[1::2] = packed >> 4
    return out[:n]


# ----------------------------------------------------------------------------
# Symmetric Int8 absmax quantisation  ([QLoRA-chkda] "First, how does k-bit
# quantization work?")
# ----------------------------------------------------------------------------
def int8_absmax_quantize(x: np.ndarray):
    """c = 127 / absmax(x) in fp32; q = round(c * x) with round-half-even.

    An all-zero input is stored as zeros with the nonzero scale c = 1.
    Returns (q int8, c float32).
    """
    x = np.asarray(x, dtype=np.float32)
    a = np.float32(np.max(np.abs(x))) if x.size else np.float32(0)
    if a == 0:
        return np.zeros(x.shape, np.int8), np.float32(1.0)
    c = np.float32(INT8_Q) / a                                   # fp32 division
    q = np.rint((c * x).astype(np.float32))                      # fp32 product, ties to even
    q = np.clip(q, -INT8_Q, INT8_Q).astype(np.int8)
    return q, np.float32(c)


def int8_dequantize(q: np.ndarray, c) -> np.ndarray:
    """x^ = q / c in fp32."""
    return (np.asarray(q).astype(np.float32) / np.float32(c)).astype(np.float32)


# ----------------------------------------------------------------------------
# Double quantisation  ([QLoRA-chkda] "Double quantization and double
# dequantization")
# ----------------------------------------------------------------------------
def exact_mean_f32(s: np.ndarray) -> np.float32:
    """mu = RN32(RN64(RN64(sum s) / M)), the sum correctly rounded (math.fsum)."""
    s = np.asarray(s, dtype=np.float32)
    total = math.fsum(float(v) for v in s.tolist())
    return np.float32(total / s.size)


def double_quantize(absmax: np.ndarray, group: int = DQ_GROUP):
    """Quantise the block scales: subtract the tensor mean, then Int8 absmax per
    group of 256 scales.  Returns (c2 int8[M_b], c1 f32[G], mean f32)."""
    absmax = np.asarray(absmax, dtype=np.float32)
    mu = exact_mean_f32(absmax)
    v = (absmax - mu).astype(np.float32)
    ng = -(-absmax.size // group)
    c2 = np.empty(absmax.size, np.int8)
    c1 = np.empty(ng, np.float32)
    for g in range(ng):
        q, c = int8_absmax_quantize(v[g * group:(g + 1) * group])
        c2[g * group:(g + 1) * group] = q
        c1[g] = c
    return c2, c1, mu


def double_dequantize_scales(c2: np.ndarray, c1: np.ndarray, mean, group: int = DQ_GROUP) -> np.ndarray:
    """scales[j] = dequantize(c2[j], c1[j // 256]) + mean, each op rounded to fp32."""
    c2 = np.asarray(c2, dtype=np.int8)
    g = np.arange(c2.size) // group
    deq = (c2.astype(np.float32) / np.asarray(c1, np.float32)[g]).astype(np.float32)
    return (deq + np.float32(mean)).astype(np.float32)


# ----------------------------------------------------------------------------
# FP8 (E4M3) second-level constants: the page's "c2_FP8" label ([QLoRA-chkda]
# "Double quantization and double dequantization") read literally.  E4M3 is
# 1 sign, 4 exponent (bias 7) and 3 mantissa bits; exponent field 15 with
# mantissa 7 is NaN, so the largest finite value is 448, and exponent field 0
# holds the subnormals m * 2^-9.  The group scale maps max|v| to 448 the way
# the Int8 reading maps it to 127: c1 = RN32(448 / max|v|).
# ----------------------------------------------------------------------------
FP8_MAX = 448.0


def fp8_e4m3_encode(x: np.ndarray) -> np.ndarray:
    """fp32 -> E4M3 bits, round to nearest even; magnitudes past 448 saturate
    to 448 (c1 * v never exceeds 448 by more than an fp32 rounding)."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64).ravel()
    out = np.empty(x.size, np.uint8)
    for i, v in enumerate(x.tolist()):
        sign = 0x80 if math.copysign(1.0, v) < 0 else 0
        a = abs(v)
        if a >= 2.0 ** -6:
            e = math.floor(math.log2(a))
            if 2.0 ** e > a:          # guard log2 rounding
                e -= 1
            elif 2.0 ** (e + 1) <= a:
                e += 1
            q = round((a / 2.0 ** e - 1.0) * 8.0)   # round() is half-to-even on the exact value
            if q == 8:
                e, q = e + 1, 0
            if e > 8 or (e == 8 and q > 6):
                e, q = 8, 6
            out[i] = sign | ((e + 7) << 3) | q
        else:
            q = round(a / 2.0 ** -9)                # subnormal step 2^-9; q = 8 is the smallest normal
            out[i] = sign | q
    return out


def fp8_e4m3_decode(b: np.ndarray) -> np.ndarray:
    """E4M3 bits -> fp32 (exact)."""
    b = np.asarray(b, dtype=np.uint8).ravel()
    out = np.empty(b.size, np.float32)
    for i, v in enumerate(b.tolist()):
        sign = -1.0 if v & 0x80 else 1.0
        e, m = (v >> 3) & 15, v & 7
        if e == 15 and m == 7:
            out[i] = np.nan
        elif e == 0:
            out[i] = sign * m * 2.0 ** -9
        else:
            out[i] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return out


def double_quantize_fp8(absmax: np.ndarray, group: int = DQ_GROUP):
    """Second-level quantisation with E4M3 constants: v = RN32(s - mean), per
    group c1 = RN32(448 / max|v|) (1 for an all-zero group) and
    c2 = E4M3(RN32(c1 * v)).  Returns (c2 uint8[M_b], c1 f32[G], mean f32)."""
    absmax = np.asarray(absmax, dtype=np.float32)
    mu = exact_mean_f32(absmax)
    v = (absmax - mu).astype(np.float32)
    ng = -(-absmax.size // group)
    c2 = np.empty(absmax.size, np.uint8)
    c1 = np.empty(ng, np.float32)
    for g in range(ng):
        vg = v[g * group:(g + 1) * group]
        m = np.float32(np.max(np.abs(vg))) if vg.size else np.float32(0)
        c = np.float32(1.0) if m == 0 else np.float32(np.float32(FP8_MAX) / m)
        c1[g] = c
        c2[g * group:(g + 1) * group] = fp8_e4m3_encode((c * vg).astype(np.float32))
    return c2, c1, mu


def double_dequantize_scales_fp8(c2: np.ndarray, c1: np.ndarray, mean, group: int = DQ_GROUP) -> np.ndarray:
    """scales[j] = RN32(RN32(decode(c2[j]) / c1[j // 256]) + mean)."""
    c2 = np.asarray(c2, dtype=np.uint8)
    g = np.arange(c2.size) // group
    deq = (fp8_e4m3_decode(c2) / np.asarray(c1, np.float32)[g]).astype(np.float32)
    return (deq + np.float32(mean)).astype(np.float32)


def nf4_dequantize(codes: np.ndarray, scales: np.ndarray, blocksize: int = BLOCK,
                   C: np.ndarray | None = None) -> np.ndarray:
    """weights[i] = BF16(C[codes[i]] * scales[i // 64]); returns bf16 bits."""
    C = nf4_codebook() if C is None else C
    codes = np.asarray(codes, dtype=np.uint8).ravel()
    blk = np.arange(codes.size) // blocksize
    prod = (C[codes].astype(np.float32) * np.asarray(scales, np.float32)[blk]).astype(np.float32)
    return bf16_round_bits(prod)


def quantize_tensor(w_bits: np.ndarray, double_quant: bool = True, blocksize: int = BLOCK,
                    dq_fp8: bool = False) -> dict:
    """Full quantisation of a bf16 weight (bits): codes, packed bytes and constants.
    dq_fp8 selects E4M3 second-level constants instead of Int8."""
    w = bf16_bits_to_f32(np.asarray(w_bits).ravel())
    codes, absmax = nf4_quantize(w, blocksize)
    out = {"n": w.size, "codes": codes, "packed": pack_codes(codes), "absmax": absmax,
           "double_quant": bool(double_quant), "dq_fp8": bool(double_quant and dq_fp8)}
    if double_quant:
        c2, c1, mu = double_quantize_fp8(absmax) if dq_fp8 else double_quantize(absmax)
        out.update(c2=c2, c1=c1, mean=mu)
    return out


def dequantize_tensor(q: dict, blocksize: int = BLOCK) -> np.ndarray:
    """doubleDequant (or single dequant when DQ is off); returns bf16 bits."""
    if q["double_quant"] and q.get("dq_fp8"):
        scales = double_dequantize_scales_fp8(q["c2"], q["c1"], q["mean"])
    elif q["double_quant"]:
        scales = double_dequantize_scales(q["c2"], q["c1"], q["mean"])
    else:
        scales = q["absmax"]
    codes = unpack_codes(q["packed"], q["n"])
    return nf4_dequantize(codes, scales, blocksize)


def storage_bits_per_weight(double_quant: bool, blocksize: int = BLOCK, group: int = DQ_GROUP) -> float:
    """Scale overhead in bits per weight ([QLoRA-chkda] 0.373-bit accounting)."""
    if not double_quant:
        return 32.0 / blocksize
    return 8.0 / blocksize + 32.0 / (group * blocksize)


# ----------------------------------------------------------------------------
# LoRA / QLoRA linear layer  ([QLoRA-chkda] "How does it work?", "How does
# alpha/r control adapter strength?", QLoRA expression; [FromZero2AI] "Low-Rank
# Matrix Factorization")
# ----------------------------------------------------------------------------
def lora_trainable_params(d: int, k: int, r: int) -> int:
    """(r x k) + (d x r) trainable entries for one adapted matrix."""
    return r * k + d * r


def lora_scale(alpha: float, r: int) -> np.float32:
    return np.float32(np.float32(alpha) / np.float32(r))


def _f64(a):
    a = np.asarray(a)
    if a.dtype == np.uint16:
        a = bf16_bits_to_f32(a)
    return a.astype(np.float64)


def qlora_forward(X, W_hat, A, B, alpha: float, r: int):
    """Y = X W^T + s (X A^T) B^T, s = alpha / r; returns (Y, T) in fp64.

    X (M x k), W_hat (d x k), A (r x k), B (d x r); bf16-bit arrays or floats.
    """
    X, W_hat, A, B = map(_f64, (X, W_hat, A, B))
    s = float(lora_scale(alpha, r))
    T = X @ A.T
    return X @ W_hat.T + s * (T @ B.T), T


def qlora_adapter_grads(dY, X, A, B, alpha: float, r: int):
    """The adapter gradients alone (no base weight involved):
    dA = s (dY B)^T X and dB = s dY^T (X A^T); returns (dA, dB) in fp64."""
    dY, X, A, B = map(_f64, (dY, X, A, B))
    s = float(lora_scale(alpha, r))
    T = X @ A.T
    U = dY @ B
    return s * (U.T @ X), s * (dY.T @ T)


def qlora_backward(dY, X, W_hat, A, B, alpha: float, r: int):
    """Gradients of the forward for the frozen base (no dW0): returns dX, dA, dB."""
    dY, X, W_hat, A, B = map(_f64, (dY, X, W_hat, A, B))
    s = float(lora_scale(alpha, r))
    U = dY @ B
    dX = dY @ W_hat + s * (U @ A)
    dA, dB = qlora_adapter_grads(dY, X, A, B, alpha, r)
    return dX, dA, dB


# ----------------------------------------------------------------------------
# LoRA merge  ([QLoRA-chkda] "Merging LoRA weights for inference")
# ----------------------------------------------------------------------------
def lora_merge(W_hat, A, B, alpha: float, r: int):
    """W_merged = W + (alpha/r) B A in fp64: the adapter folded into the (here
    reconstructed NF4) base weight, d x k.  Then X W_merged^T equals the
    two-path forward up to rounding (the page's equivalence claim).

    W_hat (d x k), A (r x k), B (d x r); bf16-bit arrays or floats.
    """
    W_hat, A, B = map(_f64, (W_hat, A, B))
    s = float(lora_scale(alpha, r))
    return W_hat + s * (B @ A)


# ----------------------------------------------------------------------------
# Adapter dropout  ([FromZero2AI] LoRA configuration, lora_dropout = 0.05):
# dropout on the adapter's input only, h = W x + s B A drop(x), as a PEFT-style
# LoRA layer applies it.  The pages name no random-number generator; the keep
# decisions come from the counter-based Philox4x32-10 generator (Salmon, Moraes,
# Dror and Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC 2011), so a
# kernel can regenerate the decision for any element from (seed, offset, flat
# index) and the backward needs no stored mask.
# ----------------------------------------------------------------------------
PHILOX_MUL = (0xD2511F53, 0xCD9E8D57)
PHILOX_WEYL = (0x9E3779B9, 0xBB67AE85)


def philox4x32_10(ctr: np.ndarray, key) -> np.ndarray:
    """Philox4x32 with 10 rounds: ctr (N, 4) uint32, key (2,) -> (N, 4) uint32."""
    c = [np.asarray(ctr, np.uint64)[:, i].copy() for i in range(4)]
    k0, k1 = np.uint64(int(key[0]) & 0xFFFFFFFF), np.uint64(int(key[1]) & 0xFFFFFFFF)
    m0, m1 = np.uint64(PHILOX_MUL[0]), np.uint64(PHILOX_MUL[1])
    mask = np.uint64(0xFFFFFFFF)
    for rnd in range(10):
        p0, p1 = m0 * c[0], m1 * c[2]                 # exact 64-bit products of 32-bit words
        hi0, lo0 = p0 >> np.uint64(32), p0 & mask
        hi1, lo1 = p1 >> np.uint64(32), p1 & mask
        c = [(hi1 ^ c[1] ^ k0) & mask, lo1, (hi0 ^ c[3] ^ k1) & mask, lo0]
        if rnd < 9:
            k0 = (k0 + np.uint64(PHILOX_WEYL[0])) & mask
            k1 = (k1 + np.uint64(PHILOX_WEYL[1])) & mask
    return np.stack(c, axis=1).astype(np.uint32)


def dropout_keep(M: int, k: int, p: float, seed: int, offset: int = 0) -> np.ndarray:
    """Keep mask (M x k, bool) for dropout probability p.  Element i = m k + j
    uses word i % 4 of Philox4x32-10 at counter (i // 4 low and high 32 bits,
    offset low and high 32 bits) under key (seed low and high 32 bits); with
    u = (word >> 8) 2^-24 (uniform on [0, 1) with 24 bits, exact in fp32) the
    element is kept when u >= RN32(p)."""
    n = M * k
    q = np.arange((n + 3) // 4, dtype=np.uint64)
    ctr = np.stack([q & np.uint64(0xFFFFFFFF), q >> np.uint64(32),
                    np.full_like(q, offset & 0xFFFFFFFF), np.full_like(q, (offset >> 32) & 0xFFFFFFFF)], axis=1)
    words = philox4x32_10(ctr, (seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)).reshape(-1)[:n]
    u = (words >> np.uint32(8)).astype(np.float64) * 2.0 ** -24
    return (u >= float(np.float32(p))).reshape(M, k)


def dropout_scale(p: float) -> np.float32:
    """Scale of the kept activations: RN32(1 / RN32(1 - p))."""
    return np.float32(np.float32(1.0) / np.float32(np.float32(1.0) - np.float32(p)))


def qlora_forward_dropout(X, W_hat, A, B, alpha: float, r: int, keep: np.ndarray, p: float):
    """Y = X W^T + s (drop(X) A^T) B^T with drop(X) = X * keep * scale; returns
    (Y, T) in fp64, T = drop(X) A^T."""
    X, W_hat, A, B = map(_f64, (X, W_hat, A, B))
    s = float(lora_scale(alpha, r))
    Xd = X * keep * float(dropout_scale(p))
    T = Xd @ A.T
    return X @ W_hat.T + s * (T @ B.T), T


def qlora_backward_dropout(dY, X, W_hat, A, B, alpha: float, r: int, keep: np.ndarray, p: float):
    """Gradients of qlora_forward_dropout for a fixed mask: dX, dA, dB."""
    dY, X, W_hat, A, B = map(_f64, (dY, X, W_hat, A, B))
    s = float(lora_scale(alpha, r))
    g = keep * float(dropout_scale(p))
    Xd = X * g
    T = Xd @ A.T
    U = dY @ B
    dX = dY @ W_hat + s * (U @ A) * g
    dA = s * (U.T @ Xd)
    dB = s * (dY.T @ T)
    return dX, dA, dB
