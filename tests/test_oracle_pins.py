"""Pins of the oracle against what the pages and the mathematics fix.

Nothing here retypes the oracle's formulas: each test checks a worked case
from the pages (tests/golden/, with citations), a closed form, an invariant,
a brute-force float64 evaluation, or a library routine (numpy matmul,
np.packbits, math.fsum, math.tanh, torch's bf16 cast).  The cases are chosen so
that a dropped term, a wrong sign or index, a transposed operand, the wrong
tie rule or the wrong scale fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from binary_weight_transformer_b200 import workloads as wls

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


def _golden(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# integer dot: add / subtract / skip
# --------------------------------------------------------------------------

def test_add_sub_skip_hand_worked(golden_dir):
    g = _golden(golden_dir, "add_sub_skip_4x4.json")
    q = np.array(g["q"], np.int8)
    c = np.array(g["codes"], np.int8)
    acc = oracle.int_dot(q, c, oracle.TERNARY2)
    assert acc.tolist() == g["acc"]


@pytest.mark.parametrize("fmt,lo,hi", [(oracle.TERNARY2, -1, 1), (oracle.BINARY1, -1, 1),
                                       (oracle.INT4, -7, 7)])
def test_int_dot_equals_numpy_int64_matmul(fmt, lo, hi):
    rng = np.random.default_rng(7)
    M, N, K = 13, 29, 211
    q = rng.integers(-128, 128, size=(M, K)).astype(np.int8)
    c = rng.integers(lo, hi + 1, size=(N, K)).astype(np.int8)
    if fmt == oracle.BINARY1:
        c[c == 0] = 1
    ref = q.astype(np.int64) @ c.astype(np.int64).T
    assert np.array_equal(oracle.int_dot(q, c, fmt), ref)
    assert np.array_equal(oracle.int_dot(q, c, fmt, nthreads=4), ref)


def test_degenerate_weights():
    rng = np.random.default_rng(3)
    q = rng.integers(-128, 128, size=(7, 96)).astype(np.int8)
    rowsum = q.astype(np.int64).sum(axis=1)
    zeros = np.zeros((5, 96), np.int8)
    assert not oracle.int_dot(q, zeros, oracle.TERNARY2).any()
    plus = np.ones((5, 96), np.int8)
    acc = oracle.int_dot(q, plus, oracle.TERNARY2)
    assert np.array_equal(acc, np.repeat(rowsum[:, None], 5, axis=1))
    acc = oracle.int_dot(q, -plus, oracle.BINARY1)
    assert np.array_equal(acc, -np.repeat(rowsum[:, None], 5, axis=1))


def test_int32_overflow_bound_rejected():
    # M8.8 §0x09C: a worst-case dot product beyond INT32 is rejected.
    K = 2147483647 // 128 + 1
    q = np.zeros((1, K), np.int8)
    c = np.zeros((1, K), np.int8)
    with pytest.raises(oracle.OracleError) as e:
        oracle.int_dot(q, c, oracle.TERNARY2)
    assert e.value.status == oracle.EOVERFLOW
    K4 = 2147483647 // (128 * 7) + 1
    with pytest.raises(oracle.OracleError):
        oracle.int_dot(np.zeros((1, K4), np.int8), np.zeros((1, K4), np.int8), oracle.INT4)
    # one below the 4-bit bound is accepted
    K4 -= 1
    acc = oracle.int_dot(np.zeros((1, K4), np.int8), np.zeros((1, K4), np.int8), oracle.INT4)
    assert acc[0, 0] == 0


# --------------------------------------------------------------------------
# ternary absmean codes
# --------------------------------------------------------------------------

def test_ternary_worked_rows(golden_dir):
    g = _golden(golden_dir, "ternary_absmean_rows.json")
    codes, gamma = oracle.ternary_codes(np.array(g["w"], np.float32), g["eps"])
    assert codes.tolist() == g["codes"]
    assert gamma[0] == pytest.approx(g["gamma"], rel=1e-6)


def test_ternary_tie_is_nearest_even(golden_dir):
    g = _golden(golden_dir, "ternary_tie.json")
    codes, gamma = oracle.ternary_codes(np.array(g["w"], np.float32), g["eps"])
    assert gamma[0] == g["gamma"]
    assert codes.tolist() == g["codes"]


def _exact_mean_f32(w):
    """fp32 rounding of the fp64-rounded exact mean of |w| (math.fsum is
    correctly rounded)."""
    s = math.fsum(abs(float(v)) for v in w.ravel())
    return np.float32(s / w.size)


@pytest.mark.parametrize("seed,N,K", [(11, 37, 101), (12, 300, 257), (13, 1, 4096)])
def test_ternary_gamma_is_the_mean_abs(seed, N, K):
    w = wls.normal_weights(seed, N, K)
    _, gamma = oracle.ternary_codes(w)
    assert gamma[0] == _exact_mean_f32(w)


def test_ternary_alphabet_and_zero_fraction_closed_form():
    # For W ~ N(0, s^2): gamma -> s*sqrt(2/pi); code 0 iff |w| < (gamma+eps)/2,
    # so P(0) = erf(((gamma+eps)/2) / (s*sqrt(2))).  25M weights (the 4B-class
    # 9728x2560 shape): sampling error of the fraction is ~1e-4.
    s = 0.02
    w = wls.normal_weights(5000, 9728, 2560, s)
    codes, gamma = oracle.ternary_codes(w)
    assert set(np.unique(codes).tolist()) <= {-1, 0, 1}
    assert gamma[0] == pytest.approx(s * math.sqrt(2 / math.pi), rel=2e-3)
    thr = (float(gamma[0]) + 1e-5) / 2
    p0 = math.erf(thr / (s * math.sqrt(2)))
    frac0 = float((codes == 0).mean())
    assert abs(frac0 - p0) < 1e-3
    assert abs(frac0 - 0.3101) < 3e-3
    # symmetry of +1 / -1 occupancy
    assert abs(float((codes == 1).mean()) - float((codes == -1).mean())) < 2e-3


def test_ternary_codes_are_the_nearest_level():
    # Invariant: every code is the nearest point of {-1,0,1} to w/(gamma+eps)
    # (checked in float64, away from exact ties).
    w = wls.normal_weights(21, 64, 333)
    codes, gamma = oracle.ternary_codes(w)
    r = w.astype(np.float64) / (float(gamma[0]) + 1e-5)
    nearest = np.clip(np.round(r), -1, 1)
    safe = np.abs(np.abs(r) - 0.5) > 1e-5
    assert np.array_equal(codes[safe], nearest[safe].astype(np.int8))


# --------------------------------------------------------------------------
# binary sign codes
# --------------------------------------------------------------------------

def test_binary_signed_zero_and_pack(golden_dir):
    g = _golden(golden_dir, "binary_signed_zero.json")
    w = np.array(g["w"], np.float32)
    codes, s_w = oracle.binary_codes(w)
    assert codes.tolist() == g["codes"]
    assert s_w.tolist() == g["s_w"]
    assert oracle.pack(codes, oracle.BINARY1).tolist() == g["packed"]


def test_binary_scale_is_row_mean_abs():
    w = wls.normal_weights(31, 19, 777)
    codes, s_w = oracle.binary_codes(w)
    for n in range(w.shape[0]):
        assert s_w[n] == _exact_mean_f32(w[n])
    assert np.array_equal(codes, np.where(w >= 0, 1, -1).astype(np.int8))


@pytest.mark.parametrize("K", [1, 7, 8, 9, 192, 1001])
def test_binary_pack_equals_numpy_packbits(K):
    rng = np.random.default_rng(K)
    codes = np.where(rng.random((5, K)) < 0.5, 1, -1).astype(np.int8)
    ref = np.packbits(((1 - codes) // 2).astype(np.uint8), axis=1, bitorder="little")
    assert np.array_equal(oracle.pack(codes, oracle.BINARY1), ref)
    back, st = oracle.unpack(ref, K, oracle.BINARY1)
    assert st == oracle.OK and np.array_equal(back, codes)


# --------------------------------------------------------------------------
# 4-bit tanh-clipped codes
# --------------------------------------------------------------------------

def test_int4_worked_rows(golden_dir):
    g = _golden(golden_dir, "int4_tanh_rows.json")
    codes, s_w = oracle.int4_codes(np.array(g["w"], np.float32))
    assert codes.tolist() == g["codes"]
    assert np.allclose(s_w, g["s_w"], rtol=g["s_w_rel_tol"], atol=0)


def test_tanh_against_libm():
    # Dense sweep of [-20, 20] plus tiny and huge arguments: the oracle's tanh
    # is within 4 units in the last place of libm's.
    zs = np.concatenate([np.linspace(-20, 20, 200001), np.geomspace(1e-300, 1e-3, 2000),
                         -np.geomspace(1e-300, 1e-3, 2000), [0.0, 25.0, 700.0, -700.0]])
    worst = 0.0
    for z in zs:
        ref = math.tanh(z)
        got = oracle.tanh(z)
        if ref == 0.0:
            assert got == 0.0
            continue
        ulp = math.ulp(ref)
        worst = max(worst, abs(got - ref) / ulp)
    assert worst <= 4.0, worst


def test_int4_levels_and_row_extremes():
    # T4NT-0.5B reports 14.8-15.0 of the 15 levels in use on N(0, 0.02)-like
    # weights; the 3584x1280 shape must use all 15, and each row's largest
    # |w| maps to +-7 (the scale is max|w_c|/7).
    w = wls.normal_weights(4000, 3584, 1280)
    codes, s_w = oracle.int4_codes(w)
    assert codes.min() >= -7 and codes.max() <= 7
    assert len(np.unique(codes)) == 15
    idx = np.abs(w).argmax(axis=1)
    assert np.all(np.abs(codes[np.arange(w.shape[0]), idx]) == 7)
    # tanh clipping is mild here: s_w ~ max|w|/7 to first order
    assert np.allclose(s_w, np.abs(w).max(axis=1) / 7, rtol=2e-3)


def test_int4_matches_float64_pipeline_away_from_ties():
    w = wls.normal_weights(41, 64, 256) * 20  # large enough for tanh to bend
    codes, s_w = oracle.int4_codes(w)
    wc = 3.0 * np.tanh(w.astype(np.float64) / 3.0)
    s = np.abs(wc).max(axis=1) / 7
    assert np.allclose(s_w, s, rtol=1e-6)
    r = wc / s[:, None]
    safe = np.abs(np.abs(r - np.floor(r)) - 0.5) > 1e-4
    ref = np.clip(np.round(r), -7, 7).astype(np.int8)
    assert np.array_equal(codes[safe], ref[safe])
    assert safe.mean() > 0.99


# --------------------------------------------------------------------------
# packing invariants
# --------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", [oracle.TERNARY2, oracle.INT4])
def test_codes_are_odd_in_the_weights(fmt):
    # Every step of the ternary and 4-bit quantisers is odd or even in w:
    # mean|W| and max|3 tanh(w/3)| do not see the sign, tanh is odd, and
    # rounding half to even and the clip are symmetric about 0.  So negating
    # the weights negates the codes and keeps the scales, bit for bit.  A
    # floor-style rounding or a one-sided clip breaks this.
    w = wls.normal_weights(120 + fmt, 33, 257)
    w[0, :8] = [0.0, -0.0, 1e-30, -1e-30, 0.02, -0.02, 0.5, -0.5]
    c1, s1 = oracle.quantize(w, fmt)
    c2, s2 = oracle.quantize(-w, fmt)
    assert np.array_equal(c2, -c1)
    assert np.array_equal(np.asarray(s1).view(np.uint32), np.asarray(s2).view(np.uint32))


def test_binary_codes_flip_with_the_weights_except_at_zero():
    # The binary rule is +1 for w >= 0: negation flips every code except at
    # a zero weight (both signed zeros stay +1); the row scales do not change.
    w = wls.normal_weights(125, 17, 129)
    w[0, :4] = [0.0, -0.0, 1e-30, -1e-30]
    c1, s1 = oracle.quantize(w, oracle.BINARY1)
    c2, s2 = oracle.quantize(-w, oracle.BINARY1)
    zero = (w == 0)
    assert np.array_equal(c2[~zero], -c1[~zero])
    assert np.all(c1[zero] == 1) and np.all(c2[zero] == 1)
    assert np.array_equal(s1.view(np.uint32), s2.view(np.uint32))


@pytest.mark.parametrize("fmt,alphabet", [(oracle.TERNARY2, [-1, 0, 1]), (oracle.INT4, list(range(-7, 8))),
                                          (oracle.BINARY1, [-1, 1])])
@pytest.mark.parametrize("K", [1, 3, 4, 5, 31, 32, 33, 255])
def test_pack_roundtrip(fmt, alphabet, K):
    rng = np.random.default_rng(K + 100 * fmt)
    codes = rng.choice(alphabet, size=(6, K)).astype(np.int8)
    for ldp in (None, oracle.row_bytes(fmt, K) + 16):
        packed = oracle.pack(codes, fmt, ldp)
        back, st = oracle.unpack(packed, K, fmt)
        assert st == oracle.OK
        assert np.array_equal(back, codes)
        # bytes past the logical extent are zero
        rb = oracle.row_bytes(fmt, K)
        assert not packed[:, rb:].any()


def test_ternary_four_codes_per_byte():
    # Atomic-1Bit README: ternary weights are packed four per byte.
    for K in (16, 64, 2560):
        assert oracle.row_bytes(oracle.TERNARY2, K) == K // 4
        assert oracle.row_bytes(oracle.INT4, K) == K // 2
        assert oracle.row_bytes(oracle.BINARY1, K) == K // 8


def test_ternary_byte_table_exhaustive():
    # Every value of one byte decodes to four valid codes, or is rejected
    # exactly when one of its 2-bit fields is the reserved pattern 10; a field
    # holds the code as 2-bit two's complement (00 = 0, 01 = +1, 11 = -1).
    for b in range(256):
        fields = [(b >> (2 * j)) & 3 for j in range(4)]
        row = np.zeros((1, 16), np.uint8)
        row[0, 0] = b
        codes, st = oracle.unpack(row, 64, oracle.TERNARY2)
        if 2 in fields:
            assert st == oracle.ERESERVED
            continue
        assert st == oracle.OK
        got = sorted(codes.ravel().tolist())
        want = sorted([{0: 0, 1: 1, 3: -1}[f] for f in fields] + [0] * 60)
        assert got == want
        assert oracle.pack(codes, oracle.TERNARY2, 16)[0, 0] == b


def test_int4_byte_table_exhaustive():
    for b in range(256):
        nib = [b & 15, b >> 4]
        row = np.zeros((1, 16), np.uint8)
        row[0, 0] = b
        codes, st = oracle.unpack(row, 32, oracle.INT4)
        if 8 in nib:
            assert st == oracle.ERESERVED
            continue
        assert st == oracle.OK
        # two's complement: value = nibble - 16 when the top bit is set
        want = sorted([v - 16 if v >= 8 else v for v in nib] + [0] * 30)
        assert sorted(codes.ravel().tolist()) == want
        assert oracle.pack(codes, oracle.INT4, 16)[0, 0] == b


@pytest.mark.parametrize("fmt", [oracle.TERNARY2, oracle.BINARY1, oracle.INT4])
@pytest.mark.parametrize("K", [5, 13, 33])
def test_unowned_bits_rejected(fmt, K):
    # Packing all -1 sets every bit a code owns; any other bit of the row
    # (inside the last partly used word, or in the stride padding) must be
    # rejected as non-canonical.
    codes = -np.ones((2, K), np.int8)
    ldp = oracle.row_bytes(fmt, K) + 16
    packed = oracle.pack(codes, fmt, ldp)
    assert oracle.unpack(packed, K, fmt)[1] == oracle.OK
    free = np.argwhere(np.unpackbits(packed[1], bitorder="little") == 0).ravel()
    assert free.size > 0
    for bit in (free[0], free[-1]):
        bad = packed.copy()
        bad[1, bit // 8] |= np.uint8(1 << (bit % 8))
        assert oracle.unpack(bad, K, fmt)[1] == oracle.ERESERVED

# --------------------------------------------------------------------------
# activation quantiser
# --------------------------------------------------------------------------

def test_act_quant_worked_rows(golden_dir):
    g = _golden(golden_dir, "act_quant_rows.json")
    q, s_x = oracle.act_quant(np.array(g["x"], np.float32), g["eps"])
    assert q.tolist() == g["q"]
    assert s_x.tolist() == g["s_x"]


def test_act_quant_eps_scale_leaves_eps_out(golden_dir):
    # With eps > 0 the codes divide by gamma + eps, but the reconstruction
    # scale stays gamma/127: a slip to (gamma + eps)/127 fails here.
    g = _golden(golden_dir, "act_quant_eps_row.json")
    q, s_x = oracle.act_quant(np.array(g["x"], np.float32), g["eps"])
    assert q.tolist() == g["q"]
    want = (np.array(g["s_x_numerator"], np.float32) / np.float32(127)).astype(np.float32)
    assert np.array_equal(s_x.view(np.uint32), want.view(np.uint32))


def test_act_quant_invariants():
    x = wls.normal_activations(51, 97, 1000)
    q, s_x = oracle.act_quant(x)
    assert q.min() >= -127
    g = np.abs(x).max(axis=1)
    assert np.array_equal(s_x, (g / np.float32(127)).astype(np.float32))
    # the largest |x| of each row maps to +-127
    idx = np.abs(x).argmax(axis=1)
    assert np.all(np.abs(q[np.arange(97), idx]) == 127)
    # reconstruction error at most half a step (plus rounding slack)
    err = np.abs(x.astype(np.float64) - q.astype(np.float64) * s_x[:, None].astype(np.float64))
    assert np.all(err <= s_x[:, None] * (0.5 + 1e-5))
    # codes are monotone in x within a row
    for t in range(5):
        o = np.argsort(x[t], kind="stable")
        assert np.all(np.diff(q[t][o].astype(np.int32)) >= 0)


def test_act_quant_bf16_equals_widened_f32():
    x = wls.normal_activations(52, 33, 515, 0.005, 10.0)
    xb = wls.to_bf16_bits(x)
    widened = (xb.astype(np.uint32) << 16).view(np.float32)
    q1, s1 = oracle.act_quant(xb, bf16_bits=True)
    q2, s2 = oracle.act_quant(widened)
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)


@pytest.mark.parametrize("k", [-80, -40, 40, 80])
def test_act_quant_power_of_two_scale_invariance(k):
    # Multiplying a row by 2^k is exact while every value stays normal, and
    # both the product by 127 and the division by the row max commute with
    # it, so the codes must not change and s_x must scale by 2^k.  Rows far
    # from 1 in magnitude are where a reciprocal of the max over- or
    # underflows.
    x = wls.normal_activations(53, 16, 300, 0.01, 8.0)
    x = x[np.all(np.abs(x) > 1e-6, axis=1)]
    xs = (x.astype(np.float64) * 2.0 ** k).astype(np.float32)
    assert np.all(np.abs(xs) >= np.finfo(np.float32).tiny) and np.all(np.isfinite(xs * np.float32(127)))
    q1, s1 = oracle.act_quant(x)
    q2, s2 = oracle.act_quant(xs)
    assert np.array_equal(q1, q2)
    assert np.array_equal(s2.astype(np.float64), s1.astype(np.float64) * 2.0 ** k)


def _round_f32(r):
    """Nearest binary32 value to the rational r >= 0, ties to even, with
    subnormals (from the IEEE 754 definition, in exact arithmetic)."""
    from fractions import Fraction
    if r == 0:
        return Fraction(0)
    e = r.numerator.bit_length() - r.denominator.bit_length()
    if Fraction(2) ** e > r:
        e -= 1
    quantum = Fraction(2) ** (max(e, -126) - 23)
    n, rem = divmod(r, quantum)
    if rem * 2 > quantum or (rem * 2 == quantum and n % 2 == 1):
        n += 1
    return n * quantum


def test_act_quant_subnormal_rows_exact():
    # Rows whose values are subnormal or near the smallest normal: codes
    # computed in exact rational arithmetic with explicit binary32 rounding
    # of 127x and of the quotient, then rounding half to even.
    from fractions import Fraction
    rng = np.random.default_rng(54)
    rows = [rng.standard_normal(64) * 10.0 ** e for e in (-44, -42, -40, -39, -38, -37)]
    x = np.array(rows).astype(np.float32)
    q, s_x = oracle.act_quant(x)
    for t in range(x.shape[0]):
        vals = [Fraction(float(v)) for v in x[t]]
        g = max(abs(v) for v in vals)
        if g == 0:
            assert not q[t].any() and s_x[t] == 0
            continue
        for kk, v in enumerate(vals):
            sign = -1 if v < 0 else 1
            z = _round_f32(_round_f32(127 * abs(v)) / g)  # |RN(RN(127x)/g)|
            n, rem = divmod(z, 1)
            if rem * 2 > 1 or (rem * 2 == 1 and n % 2 == 1):
                n += 1
            assert q[t, kk] == sign * min(int(n), 127), (t, kk)
        assert Fraction(float(s_x[t])) == _round_f32(g / 127)


def test_act_quant_rejects_nonfinite():
    x = np.ones((2, 8), np.float32)
    x[1, 3] = np.inf
    with pytest.raises(oracle.OracleError) as e:
        oracle.act_quant(x)
    assert e.value.status == oracle.ENONFINITE


# --------------------------------------------------------------------------
# rescale and the whole operator
# --------------------------------------------------------------------------

def test_bf16_rounding_equals_torch():
    import torch
    rng = np.random.default_rng(61)
    y = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 1e3,
                        np.array([0.0, -0.0, np.inf, -np.inf, 3.3895314e38, 1e-40,
                                  1.00390625, 1.01171875, -1.00390625], np.float32)])
    ref = torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f32_to_bf16_bits(y), ref)


@pytest.mark.parametrize("fmt", [oracle.TERNARY2, oracle.BINARY1, oracle.INT4])
def test_linear_equals_float64_product_of_decoded(fmt):
    # Brute force: y must equal (s_x * q) @ (s_w * c)^T evaluated in float64,
    # up to fp32 rounding of the two scale products.
    M, N, K = 9, 21, 160
    w = wls.normal_weights(70 + fmt, N, K)
    x = wls.normal_activations(80 + fmt, M, K)
    codes, s_w = oracle.quantize(w, fmt)
    q, s_x = oracle.act_quant(x)
    packed = oracle.pack(codes, fmt, oracle.row_bytes(fmt, K) + 5)
    y, acc = oracle.linear(q, s_x, packed, s_w, fmt, K)
    sw = np.broadcast_to(s_w.astype(np.float64), (N,))
    ref = (s_x.astype(np.float64)[:, None] * q.astype(np.float64)) @ \
          (sw[:, None] * codes.astype(np.float64)).T
    assert np.allclose(y, ref, rtol=1e-6, atol=0)
    yb, _ = oracle.linear(q, s_x, packed, s_w, fmt, K, out="bf16")
    yb32 = (yb.astype(np.uint32) << 16).view(np.float32)
    assert np.allclose(yb32, ref, rtol=2 ** -8, atol=0)


# Expected relative error of the weight code alone for W ~ N(0, 1), from the
# integrals E[(w - s*c(w))^2]: ternary (thresholds +-g/2, level g = sqrt(2/pi))
# 0.5132; binary (level g) sqrt(1 - 2/pi) = 0.6028; 4-bit: uniform noise of a
# step max|w|/7 with max|w| ~ 3.0 at K = 512, 3.0/7/sqrt(12) = 0.124.
@pytest.mark.parametrize("fmt,expected", [(oracle.TERNARY2, 0.5132), (oracle.BINARY1, 0.6028),
                                          (oracle.INT4, 0.124)])
def test_linear_noise_matches_closed_form(fmt, expected):
    # The quantised layer tracks x @ W^T with the relative Frobenius error the
    # weight code predicts (activation noise adds well under 1%).  A missing or
    # doubled scale, or a wrong threshold, moves this far outside 15%.
    M, N, K = 16, 64, 512
    w = wls.normal_weights(90 + fmt, N, K)
    x = wls.normal_activations(95 + fmt, M, K)
    codes, s_w = oracle.quantize(w, fmt)
    q, s_x = oracle.act_quant(x)
    y, _ = oracle.linear(q, s_x, oracle.pack(codes, fmt), s_w, fmt, K)
    ref = x.astype(np.float64) @ w.astype(np.float64).T
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert abs(rel - expected) < 0.15 * expected, rel
