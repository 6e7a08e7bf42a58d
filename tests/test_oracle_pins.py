"""Pins for the CPU oracle: checks against what the pages and the mathematics fix.

Each test ties an oracle function to something other than itself: values the
pages print, closed forms, invariants, brute force with exact rationals, or
finite differences.  No GPU needed.
"""
from fractions import Fraction

import numpy as np
import pytest

from oracle import qlora_oracle as O


# ---------------------------------------------------------------------------
# exact helpers used only by the brute-force checks
# ---------------------------------------------------------------------------
def rn32(fr: Fraction) -> np.float32:
    """Correctly rounded (ties-to-even) fp32 of an exact rational."""
    cand = np.float32(float(fr))
    best = None
    for c in (np.nextafter(cand, np.float32(-np.inf)), cand, np.nextafter(cand, np.float32(np.inf))):
        err = abs(Fraction(float(c)) - fr)
        even = (int(np.array(c, np.float32).view(np.uint32)) & 1) == 0
        key = (err, not even)
        if best is None or key < best[0]:
            best = (key, c)
    return np.float32(best[1])


def brute_nearest(x: np.float32, C) -> int:
    """argmin over j of RN32(|x - C[j]|), first minimum: exact-rational restatement."""
    best_j, best_d = None, None
    for j, c in enumerate(C):
        d = abs(rn32(Fraction(float(x)) - Fraction(float(c))))
        if best_d is None or d < best_d:
            best_j, best_d = j, d
    return best_j


def ulps_around(x, n):
    x = np.float32(x)
    lo = [x]
    for _ in range(n):
        lo.append(np.nextafter(lo[-1], np.float32(-2)))
    hi = [x]
    for _ in range(n):
        hi.append(np.nextafter(hi[-1], np.float32(2)))
    return lo[1:] + hi


# ---------------------------------------------------------------------------
# codebook
# ---------------------------------------------------------------------------
def test_codebook_matches_printed_table(golden):
    g = golden("nf4_printed_table.json")
    C = O.nf4_codebook()
    assert np.max(np.abs(C.astype(np.float64) - np.array(g["values"]))) <= 0.5 * 10 ** -g["decimals"]


def test_codebook_invariants(golden):
    g = golden("nf4_printed_table.json")
    C = O.nf4_codebook()
    assert C.dtype == np.float32 and C.size == 16
    assert np.all(np.diff(C) > 0)
    assert C[0] == -1.0 and C[15] == 1.0 and C[7] == 0.0
    assert int(np.sum(C < 0)) == g["n_negative"] and int(np.sum(C > 0)) == g["n_positive"]


def test_codebook_cutoff_interval(golden):
    """The chosen cutoff sits inside the set of cutoffs that reproduce the printed
    table, and cutoffs just outside that set do not reproduce it."""
    printed = np.array(golden("nf4_printed_table.json")["values"])

    def ok(p):
        return np.max(np.abs(np.array(O.codebook_values(p)) - printed)) <= 5e-5
    lo, hi = O.TAIL_CUTOFF_INTERVAL
    assert ok(lo) and ok(hi) and ok(O.TAIL_CUTOFF)
    assert lo < O.TAIL_CUTOFF < hi
    assert not ok(lo - 1e-9) and not ok(hi + 1e-9)


def test_codebook_independent_quantile_routine():
    """scipy's normal quantile (a different implementation) yields the same fp32 table."""
    from scipy.stats import norm
    p = O.TAIL_CUTOFF
    top = norm.ppf(p)
    pos = [norm.ppf(0.5 + (p - 0.5) * i / 8) / top for i in range(1, 9)]
    neg = [-norm.ppf(0.5 + (p - 0.5) * i / 7) / top for i in range(1, 8)]
    other = np.array(sorted(neg) + [0.0] + pos).astype(np.float32)
    assert np.array_equal(other.view(np.uint32), O.nf4_codebook().view(np.uint32))


# ---------------------------------------------------------------------------
# NF4 quantisation
# ---------------------------------------------------------------------------
def test_worked_nf4_example(golden):
    g = golden("nf4_worked_example.json")
    C = O.nf4_codebook()
    w_bf16 = O.bf16_bits_to_f32(O.bf16_round_bits(np.array([g["weight"]], np.float32)))[0]
    block = np.zeros(64, np.float32)
    block[0] = g["scale"]
    block[1] = w_bf16
    codes, absmax = O.nf4_quantize(block)
    assert absmax[0] == g["scale"]
    assert codes[1] == g["code"] == int(g["code_binary"], 2)
    assert round(float(C[g["code"]]), 5) == g["nearest_value"]
    assert round(g["weight"] / g["scale"], 2) == g["normalized"]
    recon = O.bf16_bits_to_f32(O.nf4_dequantize(codes, absmax))[1]
    # the page multiplies its 5-decimal C[9] by the scale; the exact product is
    # within one unit of the 5th decimal of that
    assert round(g["nearest_value"] * g["scale"], 5) == g["reconstructed"]
    assert abs(float(np.float32(C[9]) * np.float32(g["scale"])) - g["reconstructed"]) <= 1e-5
    assert abs(float(recon) - g["reconstructed"]) <= 2 ** -8 * g["reconstructed"]
    # the absmax element maps to the top code
    assert codes[0] == 15


def test_nearest_code_bruteforce_near_boundaries():
    """Every fp32 value within 48 ulps of each code midpoint, each code value and a
    random sample: the oracle equals an exact-rational restatement of R2."""
    C = O.nf4_codebook()
    xs = []
    for j in range(15):
        xs += ulps_around((np.float64(C[j]) + np.float64(C[j + 1])) / 2, 48)
    xs += list(C) + [np.float32(-0.0), np.float32(1e-30), np.float32(-1e-30)]
    xs += list(np.random.default_rng(7).uniform(-1, 1, 300).astype(np.float32))
    xs = np.array(xs, np.float32)
    got = O.nearest_code(xs, C)
    want = np.array([brute_nearest(x, C) for x in xs])
    assert np.array_equal(got, want)


def test_tie_breaks_to_smaller_index():
    """Where the two fp32 distances are equal, the smaller code index is chosen."""
    C = O.nf4_codebook()
    ties = 0
    for j in range(15):
        m = np.float32((np.float64(C[j]) + np.float64(C[j + 1])) / 2)
        for x in [m] + ulps_around(m, 3):
            da = np.abs(np.float32(x - C[j]))
            db = np.abs(np.float32(x - C[j + 1]))
            if da == db:
                ties += 1
                assert O.nearest_code(np.array([x], np.float32), C)[0] == j
    assert ties >= 4   # ties do occur for this table (the rule is exercised)


def test_quantize_bruteforce_blocks():
    """Per-block loop written from the page's algorithm with exact-rational
    distances, on blocks that include an all-zero block, -0.0, a negative absmax
    and a ragged last block."""
    rng = np.random.default_rng(3)
    w = rng.standard_normal(64 * 5 + 23).astype(np.float32) * np.float32(0.02)
    w = O.bf16_bits_to_f32(O.bf16_round_bits(w))
    w[64:128] = 0.0
    w[130] = -0.0
    w[200] = -0.5      # negative absmax element
    C = O.nf4_codebook()
    codes, absmax = O.nf4_quantize(w)
    for b in range(-(-w.size // 64)):
        blk = w[64 * b:64 * (b + 1)]
        m = int(np.argmax(np.abs(blk)))
        scale = np.float32(abs(blk[m]))
        assert absmax[b] == scale
        for i, x in enumerate(blk):
            if scale == 0:
                want = int(np.argmin(np.abs(C)))
            else:
                want = brute_nearest(rn32(Fraction(float(x)) / Fraction(float(scale))), C)
            assert codes[64 * b + i] == want


def test_nonzero_blocks_hold_an_extreme_code():
    w = O.bf16_bits_to_f32(O.bf16_round_bits(np.random.default_rng(1).standard_normal(64 * 200).astype(np.float32)))
    codes, absmax = O.nf4_quantize(w)
    blocks = codes.reshape(-1, 64)
    assert np.all((blocks == 0).any(axis=1) | (blocks == 15).any(axis=1))


def test_roundtrip_error_bound():
    """|w - w^| <= s * (half gap of the chosen code's interval) + fp32 slack
    + half a bf16 ulp of w^ (DQ off)."""
    C = O.nf4_codebook().astype(np.float64)
    rng = np.random.default_rng(5)
    w = O.bf16_bits_to_f32(O.bf16_round_bits(rng.standard_normal(64 * 500).astype(np.float32) * np.float32(0.02)))
    codes, absmax = O.nf4_quantize(w)
    what = O.bf16_bits_to_f32(O.nf4_dequantize(codes, absmax)).astype(np.float64)
    s = np.repeat(absmax.astype(np.float64), 64)
    gaps = np.diff(C) / 2
    half = np.maximum(np.concatenate([[0], gaps]), np.concatenate([gaps, [0]]))[codes]
    ulp_half = np.abs(what) * 2.0 ** -8
    assert np.all(np.abs(w - what) <= s * (half + 2 ** -22) + ulp_half + 1e-30)
    assert np.max(half) == pytest.approx(0.15190, abs=5e-5)


def _bf16_rational(bits32: int) -> int:
    """Nearest bf16 (ties to even) of one finite fp32 bit pattern, decided on
    exact rationals between the two bf16 neighbours of the magnitude."""
    sign, mag = bits32 & 0x80000000, bits32 & 0x7FFFFFFF
    x = Fraction(float(np.array(mag, np.uint32).view(np.float32)))
    lo = mag >> 16
    hi = lo + 1

    def val(b):
        if b >= 0x7F80:
            return None                       # rounding up past the largest finite value overflows
        return Fraction(float(np.array(b << 16, np.uint32).view(np.float32)))
    vlo, vhi = val(lo), val(hi)
    if vhi is None:
        # beyond the largest finite bf16: round to nearest with the overflow
        # threshold halfway to 2^128
        vhi = Fraction(2) ** 128
    dlo, dhi = x - vlo, vhi - x
    pick = lo if (dlo < dhi or (dlo == dhi and lo % 2 == 0)) else hi
    return (sign >> 16) | pick


def test_bf16_rounding_ties_and_carries():
    """Every tie pattern (low 16 bits exactly 0x8000) at every finite exponent,
    both parities of the kept last bit, with and without a carry into the
    exponent, both signs; plus the patterns one step off the tie.  Checked
    against exact-rational rounding and against PyTorch's fp32 -> bf16."""
    import torch
    pats = []
    for e in range(0, 255):
        for m_hi in (0x00, 0x01, 0x3E, 0x3F, 0x40, 0x7E, 0x7F):
            for low in (0x8000, 0x7FFF, 0x8001, 0x0000, 0xFFFF):
                for sign in (0, 0x80000000):
                    pats.append(sign | (e << 23) | (m_hi << 16) | low)
    u = np.array(pats, np.uint32)
    x = u.view(np.float32)
    got = O.bf16_round_bits(x)
    want = np.array([_bf16_rational(int(b)) for b in pats], np.uint16)
    assert np.array_equal(got, want)
    ref = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)
    # a tie with an odd kept bit rounds up and one with an even kept bit down
    assert O.bf16_round_bits(np.array([0x3F818000], np.uint32).view(np.float32))[0] == 0x3F82
    assert O.bf16_round_bits(np.array([0x3F808000], np.uint32).view(np.float32))[0] == 0x3F80
    # the carry out of the mantissa moves into the exponent
    assert O.bf16_round_bits(np.array([0x3FFF8000], np.uint32).view(np.float32))[0] == 0x4000


def test_bf16_rounding_wide_sample():
    import torch
    rng = np.random.default_rng(17)
    u = rng.integers(0, 1 << 32, size=1 << 20, dtype=np.uint64).astype(np.uint32)
    u = u[(u & 0x7F800000) != 0x7F800000]            # finite inputs only
    x = u.view(np.float32)
    ref = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.bf16_round_bits(x), ref)
    for b in u[:2000].tolist():
        assert O.bf16_round_bits(np.array([b], np.uint32).view(np.float32))[0] == _bf16_rational(b)


def test_nf4_beats_uniform_codebook_on_gaussian_blocks():
    """Contrast from the page: finer spacing near zero lowers the error on
    bell-shaped blocks compared with 16 evenly spaced values."""
    rng = np.random.default_rng(11)
    w = rng.standard_normal(64 * 2000).astype(np.float32)
    C_nf4 = O.nf4_codebook()
    C_uni = np.linspace(-1, 1, 16).astype(np.float32)
    errs = []
    for C in (C_nf4, C_uni):
        codes, absmax = O.nf4_quantize(w, C=C)
        what = C[codes] * np.repeat(absmax, 64)
        errs.append(np.mean((w - what) ** 2))
    assert errs[0] < errs[1]


def test_pack_layout_and_roundtrip():
    assert list(O.pack_codes(np.array([1, 2, 3], np.uint8))) == [0x21, 0x03]
    c = np.random.default_rng(2).integers(0, 16, 1001).astype(np.uint8)
    assert np.array_equal(O.unpack_codes(O.pack_codes(c), c.size), c)


# ---------------------------------------------------------------------------
# Int8 absmax and double quantisation
# ---------------------------------------------------------------------------
def test_int8_worked_example(golden):
    g = golden("int8_worked_example.json")
    q, c = O.int8_absmax_quantize(np.array(g["x"], np.float32))
    assert float(c) == g["c"]
    assert q.tolist() == g["q"]
    xh = O.int8_dequantize(q, c)
    assert [round(float(v), g["x_hat_decimals"]) for v in xh] == g["x_hat"]
    assert float(xh[1]) == float(np.float32(38) / np.float32(127))


def test_int8_all_zero_uses_nonzero_scale():
    q, c = O.int8_absmax_quantize(np.zeros(7, np.float32))
    assert np.all(q == 0) and c != 0


def test_exact_mean_against_rationals():
    """Values whose naive fp32 running sum is wrong; the mean must be the
    correctly rounded exact rational (via fp64 division as read)."""
    s = np.array([2.0 ** 20] + [2.0 ** -4] * 1000 + [3.0, 2.0 ** -30], np.float32)
    exact = sum(Fraction(float(v)) for v in s)
    want = np.float32(float(Fraction(float(exact)) / len(s)))
    assert O.exact_mean_f32(s) == want


def test_double_quant_scale_error_bound():
    rng = np.random.default_rng(9)
    w = O.bf16_bits_to_f32(O.bf16_round_bits(rng.standard_normal(64 * 256 * 3 + 64 * 17).astype(np.float32) * np.float32(0.02)))
    codes, absmax = O.nf4_quantize(w)
    c2, c1, mu = O.double_quantize(absmax)
    assert c1.size == 4 and c2.size == absmax.size
    sh = O.double_dequantize_scales(c2, c1, mu)
    v = (absmax - mu).astype(np.float32)
    for g in range(c1.size):
        sl = slice(256 * g, 256 * (g + 1))
        a = float(np.max(np.abs(v[sl])))
        tol = a / 254 * (1 + 2 ** -22) + float(np.spacing(np.float32(mu))) + np.spacing(np.abs(sh[sl])).astype(np.float64)
        assert np.all(np.abs(absmax[sl].astype(np.float64) - sh[sl]) <= tol)
    assert np.all(np.abs(c2.astype(int)) <= 127)
    # every group uses the full range at its absmax element
    for g in range(c1.size):
        assert np.max(np.abs(c2[256 * g:256 * (g + 1)].astype(int))) == 127


def test_double_quant_zero_group():
    absmax = np.full(300, 0.5, np.float32)       # mean 0.5 -> every deviation is zero
    c2, c1, mu = O.double_quantize(absmax)
    assert mu == np.float32(0.5) and np.all(c2 == 0) and np.all(c1 == 1.0)
    assert np.array_equal(O.double_dequantize_scales(c2, c1, mu), absmax)


def test_dq_off_reduces_to_single_level():
    w = np.random.default_rng(4).standard_normal((8, 128)).astype(np.float32) * np.float32(0.02)
    bits = O.bf16_round_bits(w)
    q = O.quantize_tensor(bits, double_quant=False)
    codes, absmax = O.nf4_quantize(O.bf16_bits_to_f32(bits))
    assert np.array_equal(O.dequantize_tensor(q), O.nf4_dequantize(codes, absmax))


def _torch_e4m3_bits(x):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_fp8_encode_matches_library_conversion():
    # every finite bf16 value with |x| <= 464 (past 464 the library gives NaN and
    # the oracle saturates; c1 * v never gets there), then a wide fp32 sample
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    x = O.bf16_bits_to_f32(bits)
    x = x[np.isfinite(x) & (np.abs(x) <= 464.0)]
    assert np.array_equal(O.fp8_e4m3_encode(x), _torch_e4m3_bits(x))
    rng = np.random.default_rng(7)
    y = (rng.uniform(-1, 1, 20000) * 2.0 ** rng.integers(-12, 9, 20000)).astype(np.float32)
    y = y[np.abs(y) <= 464.0]
    assert np.array_equal(O.fp8_e4m3_encode(y), _torch_e4m3_bits(y))


def test_fp8_ties_round_to_even():
    vals = O.fp8_e4m3_decode(np.arange(0x7F, dtype=np.uint8)).astype(np.float64)   # 0 .. 448, ascending
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (vals[:-1] + vals[1:]) / 2)      # exact in fp32
    got = O.fp8_e4m3_encode(mids)
    even = np.where(np.arange(1, 0x7F) % 2 == 0, np.arange(1, 0x7F), np.arange(0, 0x7E))
    assert np.array_equal(got, even.astype(np.uint8))


def test_fp8_decode_all_codes():
    import torch
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    got = O.fp8_e4m3_decode(np.arange(256, dtype=np.uint8))
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[~np.isnan(got)], ref[~np.isnan(ref)])
    assert O.fp8_e4m3_decode(np.array([0x7E, 0x01, 0x08, 0x38, 0xC0], np.uint8)).tolist() == [448.0, 2.0 ** -9,
                                                                                             2.0 ** -6, 1.0, -2.0]


def test_double_quant_fp8_group_max_and_error_bound():
    rng = np.random.default_rng(8)
    s = np.abs(rng.standard_normal(1000) * 0.02 + 0.05).astype(np.float32)
    c2, c1, mu = O.double_quantize_fp8(s)
    v = (s - mu).astype(np.float32)
    for g in range(len(c1)):
        dec = O.fp8_e4m3_decode(c2[g * 256:(g + 1) * 256])
        assert np.max(np.abs(dec)) == 448.0          # the group's largest |v| lands on the top code
        assert c1[g] == np.float32(np.float32(448.0) / np.max(np.abs(v[g * 256:(g + 1) * 256])))
    sh = O.double_dequantize_scales_fp8(c2, c1, mu).astype(np.float64)
    g = np.arange(s.size) // 256
    bound = 2.0 ** -4 * np.abs(v) + 2.0 ** -10 / c1[g] + 4 * 2.0 ** -24 * (np.abs(s) + np.abs(v))
    assert np.all(np.abs(sh - s) <= bound)


def test_double_quant_fp8_zero_group():
    s = np.full(300, 0.25, np.float32)
    c2, c1, mu = O.double_quantize_fp8(s)
    assert mu == np.float32(0.25) and np.all(c2 == 0) and np.all(c1 == 1.0)
    assert np.array_equal(O.double_dequantize_scales_fp8(c2, c1, mu), s)


# Known-answer vectors of Philox4x32-10, as published with the generator's
# reference implementation (Salmon, Moraes, Dror and Shaw, "Parallel Random
# Numbers: As Easy as 1, 2, 3", SC 2011): (counter, key) -> output.
PHILOX_KAT = [
    ((0x00000000, 0x00000000, 0x00000000, 0x00000000), (0x00000000, 0x00000000),
     (0x6627e8d5, 0xe169c58d, 0xbc57ac4c, 0x9b00dbd8)),
    ((0xffffffff, 0xffffffff, 0xffffffff, 0xffffffff), (0xffffffff, 0xffffffff),
     (0x408f276d, 0x41c83b0e, 0xa20bc7c6, 0x6d5451fd)),
    ((0x243f6a88, 0x85a308d3, 0x13198a2e, 0x03707344), (0xa4093822, 0x299f31d0),
     (0xd16cfe09, 0x94fdcceb, 0x5001e420, 0x24126ea1)),
]


def test_philox_known_answers():
    for ctr, key, want in PHILOX_KAT:
        got = O.philox4x32_10(np.array([ctr], np.uint32), key)[0]
        assert [int(v) for v in got] == list(want)


def test_dropout_keep_fraction():
    n, p = 1 << 20, 0.05
    keep = O.dropout_keep(1024, 1024, p, seed=77)
    assert keep.shape == (1024, 1024)
    assert abs(keep.mean() - (1 - p)) <= 5 * np.sqrt(p * (1 - p) / n)


def test_dropout_keep_structure():
    a = O.dropout_keep(12, 40, 0.3, seed=5)
    assert np.array_equal(a, O.dropout_keep(1, 480, 0.3, seed=5).reshape(12, 40))   # flat index only
    assert not np.array_equal(a, O.dropout_keep(12, 40, 0.3, seed=6))
    assert not np.array_equal(a, O.dropout_keep(12, 40, 0.3, seed=5, offset=1))
    assert O.dropout_keep(7, 9, 0.0, seed=1).all()
    assert not O.dropout_keep(7, 9, 1.0, seed=1).any()
    # a larger p keeps a subset of what a smaller p keeps (same draws)
    assert not (O.dropout_keep(12, 40, 0.6, seed=5) & ~a).any()


def test_dropout_p0_is_the_plain_layer():
    X, W, A, B, dY = _tiny(11)
    keep = np.ones(X.shape, bool)
    Y, T = O.qlora_forward_dropout(X, W, A, B, 16.0, 3, keep, 0.0)
    Y0, T0 = O.qlora_forward(X, W, A, B, 16.0, 3)
    assert np.array_equal(Y, Y0) and np.array_equal(T, T0)
    for g, g0 in zip(O.qlora_backward_dropout(dY, X, W, A, B, 16.0, 3, keep, 0.0),
                     O.qlora_backward(dY, X, W, A, B, 16.0, 3)):
        assert np.array_equal(g, g0)


def test_dropout_backward_finite_differences():
    X, W, A, B, dY = _tiny(12)
    keep = O.dropout_keep(*X.shape, 0.4, seed=3)
    assert keep.any() and not keep.all()
    dX, dA, dB = O.qlora_backward_dropout(dY, X, W, A, B, 16.0, 3, keep, 0.4)

    def loss(X_, A_, B_):
        Y, _ = O.qlora_forward_dropout(X_, W, A_, B_, 16.0, 3, keep, 0.4)
        return float(np.sum(Y * dY))

    h = 1e-6
    for arr, grad in ((X, dX), (A, dA), (B, dB)):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            old = arr[idx]
            arr[idx] = old + h
            lp = loss(X, A, B)
            arr[idx] = old - h
            lm = loss(X, A, B)
            arr[idx] = old
            num[idx] = (lp - lm) / (2 * h)
        assert np.allclose(num, grad, rtol=1e-6, atol=1e-6)


def test_dropout_scale_against_exact_rationals():
    """RN32(1 / RN32(1 - p)): both roundings taken on exact rationals; a scale
    of (1 - p) instead of its reciprocal, or a missing rounding, fails."""
    for p in (0.05, 0.1, 0.5, 0.3, 0.9):
        p32 = Fraction(float(np.float32(p)))
        one_minus = rn32(Fraction(1) - p32)
        want = rn32(Fraction(1) / Fraction(float(one_minus)))
        got = O.dropout_scale(p)
        assert got.dtype == np.float32
        assert got.view(np.uint32) == want.view(np.uint32), p
    assert O.dropout_scale(0.0) == np.float32(1.0)
    assert O.dropout_scale(0.5) == np.float32(2.0)


def test_dropout_preserves_the_mean():
    """Inverted dropout keeps E[drop(x)] = x: over 2^20 elements the mean of
    keep * scale is 1 within 5 sigma (sigma = scale sqrt(p (1 - p) / n))."""
    n, p = 1 << 20, 0.05
    keep = O.dropout_keep(1024, 1024, p, seed=123)
    scale = float(O.dropout_scale(p))
    m = float(np.mean(keep * scale))
    assert abs(m - 1.0) <= 5 * scale * np.sqrt(p * (1 - p) / n)


def test_storage_accounting(golden):
    g = golden("storage_accounting.json")
    before = O.storage_bits_per_weight(False)
    after = O.storage_bits_per_weight(True)
    assert before == g["bits_per_weight_before"]
    assert after == g["bits_per_weight_after"]
    assert before - after == g["saved"]
    assert 4 + before == g["total_before"]
    assert round(4 + after, 3) == g["total_after_approx"]
    # context: a 65e9-parameter model saves about 3 GB
    assert round(65e9 * (before - after) / 8 / 1e9) == g["context_65b_saving_gb_approx"]


# ---------------------------------------------------------------------------
# LoRA forward / backward
# ---------------------------------------------------------------------------
def test_param_count(golden):
    g = golden("lora_param_count.json")
    assert O.lora_trainable_params(g["d"], g["k"], g["r"]) == g["trainable"]
    assert g["d"] * g["k"] == g["full_params"] == g["ratio"] * g["trainable"]


def test_forward_hand_example():
    # d=3, k=2, r=1, alpha=2 -> s=2.  T = X A^T = 1*1 + 2*1 = 3.
    # base = X W^T = [1, 2, 1+2];  adapter = s * T * B^T = 6 * [1, 0, 2].
    X = np.array([[1.0, 2.0]])
    W = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]])
    A = np.array([[1.0, 1.0]])
    B = np.array([[1.0], [0.0], [2.0]])
    Y, T = O.qlora_forward(X, W, A, B, alpha=2.0, r=1)
    assert T.tolist() == [[3.0]]
    assert Y.tolist() == [[7.0, 2.0, 15.0]]


def _tiny(seed, m=5, d=7, k=6, r=3):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((m, k)), rng.standard_normal((d, k)), rng.standard_normal((r, k)),
            rng.standard_normal((d, r)), rng.standard_normal((m, d)))


def test_forward_zero_adapter_and_zero_scale():
    X, W, A, B, _ = _tiny(0)
    base = X @ W.T
    Y0, _ = O.qlora_forward(X, W, A, np.zeros_like(B), alpha=16.0, r=3)
    assert np.array_equal(Y0, base)
    Ya, _ = O.qlora_forward(X, W, A, B, alpha=0.0, r=3)
    assert np.array_equal(Ya, base)


def test_forward_merged_equivalence():
    X, W, A, B, _ = _tiny(1)
    s = float(O.lora_scale(16.0, 3))
    Y, _ = O.qlora_forward(X, W, A, B, alpha=16.0, r=3)
    merged = X @ (W + s * (B @ A)).T
    assert np.allclose(Y, merged, rtol=1e-12, atol=1e-12)


def test_merge_hand_example():
    # d=3, k=2, r=1, alpha=2 -> s=2.  B A = [[1, 1], [0, 0], [2, 2]], so
    # W + 2 B A = [[3, 2], [0, 1], [5, 5]] ([QLoRA-chkda] "Merging LoRA weights
    # for inference": W_merged = W0 + (alpha/r) B A).
    W = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]])
    A = np.array([[1.0, 1.0]])
    B = np.array([[1.0], [0.0], [2.0]])
    assert O.lora_merge(W, A, B, alpha=2.0, r=1).tolist() == [[3.0, 2.0], [0.0, 1.0], [5.0, 5.0]]


def test_merge_bruteforce_sum():
    _, W, A, B, _ = _tiny(3, d=4, k=5, r=3)
    s = float(O.lora_scale(8.0, 3))
    got = O.lora_merge(W, A, B, alpha=8.0, r=3)
    for n in range(4):
        for c in range(5):
            ref = W[n, c]
            acc = 0.0
            for j in range(3):
                acc += B[n, j] * A[j, c]
            assert abs(got[n, c] - (ref + s * acc)) <= 1e-12 * (abs(ref) + abs(s * acc) + 1.0)


def test_merge_matches_two_path_forward():
    # the page's equivalence: before merging h = W0 x + (alpha/r) B (A x),
    # after merging h = W_merged x
    X, W, A, B, _ = _tiny(4)
    Y, _ = O.qlora_forward(X, W, A, B, alpha=16.0, r=3)
    Ym = X @ O.lora_merge(W, A, B, alpha=16.0, r=3).T
    assert np.allclose(Y, Ym, rtol=1e-12, atol=1e-12)


def test_merge_zero_adapter_or_scale_is_identity():
    _, W, A, B, _ = _tiny(5)
    assert np.array_equal(O.lora_merge(W, A, np.zeros_like(B), alpha=16.0, r=3), W)
    assert np.array_equal(O.lora_merge(W, A, B, alpha=0.0, r=3), W)


@pytest.mark.parametrize("shape", [(1, 1, 1, 1), (4, 6, 5, 2), (3, 8, 16, 4)])
def test_backward_finite_differences(shape):
    m, d, k, r = shape
    X, W, A, B, G = _tiny(2 + r, m, d, k, r)
    alpha = 3.0

    def loss(X_, A_, B_):
        return float(np.sum(O.qlora_forward(X_, W, A_, B_, alpha, r)[0] * G))
    dX, dA, dB = O.qlora_backward(G, X, W, A, B, alpha, r)
    h = 1e-6
    for name, P, grad in (("X", X, dX), ("A", A, dA), ("B", B, dB)):
        num = np.zeros_like(P)
        for idx in np.ndindex(P.shape):
            Pp, Pm = P.copy(), P.copy()
            Pp[idx] += h
            Pm[idx] -= h
            args = {"X": (X, A, B), "A": (X, A, B), "B": (X, A, B)}[name]
            ap = list(args)
            am = list(args)
            pos = {"X": 0, "A": 1, "B": 2}[name]
            ap[pos], am[pos] = Pp, Pm
            num[idx] = (loss(*ap) - loss(*am)) / (2 * h)
        err = np.linalg.norm(num - grad) / max(np.linalg.norm(grad), 1e-30)
        assert err <= 1e-6, (name, err)


def test_backward_zero_B_gives_zero_dA():
    X, W, A, B, G = _tiny(3)
    dX, dA, dB = O.qlora_backward(G, X, W, A, np.zeros_like(B), 16.0, 3)
    assert np.all(dA == 0)
    assert np.allclose(dX, G @ W)
