"""Pins of the oracle's activation prologue (RMSNorm, gain, block Hadamard
rotation, per-token codes) and of the BitNet v1 centred binary quantiser.

As in test_oracle_pins.py, nothing here retypes the oracle's formulas: each
test checks a hand-worked case (tests/golden/, with citations), a library
routine (numpy float64 norms and matrix products, math.fsum, exact integer
arithmetic), an invariant or an error bound.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from binary_weight_transformer_b200 import workloads as wls


def _golden(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def _rn32(value) -> np.float32:
    """fp32 nearest to an exact value given as a Fraction or a float64."""
    return np.float32(float(value))


def _exact(expr: str) -> float:
    # the golden file writes a few closed forms: a/b, a/(c*sqrt(d))
    from decimal import Decimal, getcontext
    getcontext().prec = 60
    expr = expr.replace(" ", "")
    if "sqrt" not in expr:
        return float(Fraction(expr))
    num, den = expr.split("/(")
    c, d = den.rstrip(")").split("*sqrt(")
    return float(Decimal(num) / (Decimal(c) * Decimal(d).sqrt()))


# --------------------------------------------------------------------------
# the activation prologue
# --------------------------------------------------------------------------

def test_prologue_worked_rows(golden_dir):
    g = _golden(golden_dir, "act_prologue_rows.json")
    for case in g["cases"]:
        gain = None if case["g"] is None else np.array(case["g"], np.float32)
        q, s_x = oracle.act_prologue(np.array(case["x"], np.float32), gain, case["norm"], case["eps_norm"],
                                     case["hadamard"])
        assert q.tolist() == case["q"], case["why"]
        assert s_x[0] == _rn32(_exact(case["s_x_exact"])), case["why"]


@pytest.mark.parametrize("bf16", [False, True])
def test_prologue_without_options_is_the_plain_act_quant(bf16):
    # No gain, no norm, no rotation: exactly the (pinned) per-token codes and
    # scale, bit for bit (fp64 then fp32 rounding of gamma/127 equals the fp32
    # quotient for fp32 operands).
    x = wls.normal_activations(1201, 64, 515, 0.01, 8.0)
    if bf16:
        x = wls.to_bf16_bits(x)
    q1, s1 = oracle.act_prologue(x, bf16_bits=bf16)
    q2, s2 = oracle.act_quant(x, 0.0, bf16_bits=bf16)
    assert np.array_equal(q1, q2)
    assert np.array_equal(s1.view(np.uint32), s2.view(np.uint32))


def _midpoint_safe(z):
    """Elements whose float64 code value is not within 1e-4 of a rounding
    midpoint (only those are decided unambiguously by a float64 check)."""
    frac = np.abs(z - np.floor(z) - 0.5)
    return frac > 1e-4


@pytest.mark.parametrize("eps_norm", [0.0, 1e-5, 0.5])
def test_rmsnorm_codes_and_scale_against_float64(eps_norm):
    # Brute force: RMSNorm in float64 with numpy, then the absmax codes in
    # float64.  The codes agree wherever float64 decides them clearly; the
    # scale is max|y|/127 to fp32 accuracy.
    M, K = 48, 1000
    x = wls.normal_activations(1202, M, K, 0.01, 8.0)
    g = (1.0 + 0.1 * np.random.default_rng(1203).standard_normal(K)).astype(np.float32)
    q, s_x = oracle.act_prologue(x, g, True, eps_norm)
    x64 = x.astype(np.float64)
    y = x64 * g.astype(np.float64) / np.sqrt(np.mean(x64 ** 2, axis=1, keepdims=True) + eps_norm)
    gam = np.abs(y).max(axis=1, keepdims=True)
    z = 127.0 * y / gam
    ok = _midpoint_safe(z)
    assert ok.mean() > 0.999
    assert np.array_equal(q[ok], np.rint(z)[ok].astype(np.int8))
    assert np.all(np.abs(s_x.astype(np.float64) * 127.0 / gam[:, 0] - 1.0) <= 2.0 ** -23)


@pytest.mark.parametrize("k", [-60, -20, 20, 60])
def test_rmsnorm_is_invariant_to_powers_of_two(k):
    # With eps = 0, RMSNorm(2^k x) = RMSNorm(x) in real arithmetic, and every
    # step here scales exactly by a power of two, so codes and scale must be
    # bit-identical.
    x = wls.normal_activations(1204, 16, 300, 0.01, 8.0)
    x = x[np.all(np.abs(x) > 1e-6, axis=1)]
    xs = (x.astype(np.float64) * 2.0 ** k).astype(np.float32)
    g = (1.0 + 0.1 * np.random.default_rng(1205).standard_normal(300)).astype(np.float32)
    q1, s1 = oracle.act_prologue(x, g, True, 0.0)
    q2, s2 = oracle.act_prologue(xs, g, True, 0.0)
    assert np.array_equal(q1, q2)
    assert np.array_equal(s1.view(np.uint32), s2.view(np.uint32))


def test_gain_scales_the_scale_not_the_codes():
    # A gain of 2^j on every feature leaves the codes alone and multiplies the
    # scale by exactly 2^j; a negated gain negates the codes.
    x = wls.normal_activations(1206, 20, 256, 0.01, 8.0)
    g = (1.0 + 0.1 * np.random.default_rng(1207).standard_normal(256)).astype(np.float32)
    q1, s1 = oracle.act_prologue(x, g, True, 1e-5)
    q2, s2 = oracle.act_prologue(x, (g * np.float32(8.0)).astype(np.float32), True, 1e-5)
    q3, s3 = oracle.act_prologue(x, -g, True, 1e-5)
    assert np.array_equal(q1, q2) and np.array_equal(s2, (s1 * np.float32(8.0)).astype(np.float32))
    assert np.array_equal(q3, -q1) and np.array_equal(s3, s1)


def test_gain_without_norm_is_act_quant_of_the_product():
    # norm off: the gain alone (the OneBit input value vector) is the plain
    # per-token quantiser applied to the fp32 product x*g.
    x = wls.normal_activations(1208, 30, 192, 0.01, 8.0)
    g = np.exp(0.25 * np.random.default_rng(1209).standard_normal(192)).astype(np.float32)
    q1, s1 = oracle.act_prologue(x, g, False)
    q2, s2 = oracle.act_quant((x * g).astype(np.float32), 0.0)
    assert np.array_equal(q1, q2) and np.array_equal(s1.view(np.uint32), s2.view(np.uint32))


def _hadamard(n):
    i = np.arange(n)
    pc = np.vectorize(lambda v: bin(int(v)).count("1"))(i[:, None] & i[None, :])
    return np.where(pc % 2 == 0, 1, -1).astype(np.int64)


@pytest.mark.parametrize("n", [1, 2, 4, 64, 512])
def test_fwht_equals_the_hadamard_matrix_on_integers(n):
    # Small integers keep every fp32 butterfly exact, so the transform must
    # equal the Sylvester Hadamard matrix (entries (-1)^popcount(i & j)) times
    # the vector in exact integer arithmetic.
    rng = np.random.default_rng(1210 + n)
    v = rng.integers(-100, 101, size=(3, n))
    got = oracle.fwht32(v.astype(np.float32))
    want = v @ _hadamard(n).T
    assert np.array_equal(got.astype(np.int64), want)


def test_fwht_is_an_involution_up_to_n():
    rng = np.random.default_rng(1211)
    v = rng.integers(-1000, 1001, size=(4, 256)).astype(np.float32)
    assert np.array_equal(oracle.fwht32(oracle.fwht32(v)), v * np.float32(256))


def test_fwht_float_error_bound():
    # Each of the log2(n) stages rounds once per element, with partial sums at
    # most 2^s * max|v| at stage s: |fwht32(v) - Hv| <= 2 n max|v| 2^-24.
    n = 512
    v = wls.normal_activations(1212, 8, n, 0.01, 8.0)
    got = oracle.fwht32(v).astype(np.float64)
    want = v.astype(np.float64) @ _hadamard(n).T.astype(np.float64)
    bound = 2.0 * n * np.abs(v).max(axis=1, keepdims=True) * 2.0 ** -24
    assert np.all(np.abs(got - want) <= bound)
    # Parseval: ||Hv||^2 = n ||v||^2
    assert np.allclose((got ** 2).sum(axis=1), n * (v.astype(np.float64) ** 2).sum(axis=1), rtol=1e-5)


@pytest.mark.parametrize("hb", [2, 64, 512])
def test_hadamard_prologue_against_float64_rotation(hb):
    # Brute force: the normalised block rotation H/sqrt(hb) in float64, then
    # float64 absmax codes; the codes agree wherever float64 decides them
    # clearly, and s_x*127 is the largest rotated magnitude.
    M, K = 32, 1024
    x = wls.normal_activations(1213 + hb, M, K, 0.005, 10.0)
    q, s_x = oracle.act_prologue(x, hadamard=hb)
    H = _hadamard(hb).astype(np.float64) / math.sqrt(hb)
    y = (x.astype(np.float64).reshape(M, K // hb, hb) @ H.T).reshape(M, K)
    gam = np.abs(y).max(axis=1, keepdims=True)
    z = 127.0 * y / gam
    ok = _midpoint_safe(z)
    assert ok.mean() > 0.99
    assert np.array_equal(q[ok], np.rint(z)[ok].astype(np.int8))
    assert np.all(np.abs(s_x.astype(np.float64) * 127.0 / gam[:, 0] - 1.0) <= 2.0 ** -20)


def test_hadamard_spreads_an_outlier():
    # A row that is one large value plus noise: without rotation almost every
    # code is 0 or +-1; after a 512-block rotation the energy spreads and the
    # codes use the range (M8.8 0x07C: the transform spreads concentrated
    # channel outliers before quantisation).
    rng = np.random.default_rng(1214)
    x = (0.01 * rng.standard_normal((1, 512))).astype(np.float32)
    x[0, 37] = 100.0
    q0, _ = oracle.act_prologue(x)
    q1, _ = oracle.act_prologue(x, hadamard=512)
    assert np.mean(np.abs(q0) <= 1) > 0.99
    assert np.mean(np.abs(q1) >= 100) > 0.99


def test_prologue_rejects_bad_blocks_and_nonfinite():
    x = np.ones((2, 12), np.float32)
    for hb in (3, 8, 16, -2):  # not a power of two, or not dividing K, or above K
        with pytest.raises(oracle.OracleError) as e:
            oracle.act_prologue(x, hadamard=hb)
        assert e.value.status == oracle.EINVAL
    g = np.ones(12, np.float32)
    g[4] = np.nan
    with pytest.raises(oracle.OracleError) as e:
        oracle.act_prologue(x, g)
    assert e.value.status == oracle.ENONFINITE


# --------------------------------------------------------------------------
# BitNet v1 centred binary codes
# --------------------------------------------------------------------------

def test_centred_codes_worked(golden_dir):
    g = _golden(golden_dir, "binary_centred_rows.json")
    codes, beta, alpha = oracle.binary_centred_codes(np.array(g["w"], np.float32))
    assert codes.tolist() == g["codes"]
    assert alpha[0] == g["alpha"] and beta[0] == g["beta"]


def test_centred_codes_against_fsum():
    # alpha and beta against math.fsum (the exactly rounded sums); codes are
    # the comparison with alpha; a shifted population still splits near half.
    w = (wls.normal_weights(1215, 300, 700) + np.float32(0.013)).astype(np.float32)
    codes, beta, alpha = oracle.binary_centred_codes(w)
    vals = w.astype(np.float64).ravel()
    assert alpha[0] == np.float32(math.fsum(vals) / vals.size)
    assert beta[0] == np.float32(math.fsum(np.abs(vals)) / vals.size)
    assert np.array_equal(codes, np.where(w > alpha[0], 1, -1).astype(np.int8))
    assert abs((codes == 1).mean() - 0.5) < 0.01
    # the uncentred sign rule would put ~74% of these weights at +1
    assert (w >= 0).mean() > 0.7


def test_centred_codes_all_equal_take_minus_one():
    codes, beta, alpha = oracle.binary_centred_codes(np.full((3, 5), 0.25, np.float32))
    assert (codes == -1).all() and alpha[0] == 0.25 and beta[0] == 0.25


# --------------------------------------------------------------------------
# OneBit value vectors folded into the prologue and the epilogue
# --------------------------------------------------------------------------

def test_onebit_fold_tracks_the_rank_one_weight():
    # M8.8 0x06A-0x06B: with W = S * (h g^T) elementwise (signs S, positive
    # value vectors), x W^T = ((x * g) S^T) * h exactly in real arithmetic.
    # Folding g into the activation codes and h into the per-row output scale
    # must therefore track x W^T up to the activation quantisation error only;
    # swapping the two vectors does not.
    M, N, K = 24, 64, 512
    rng = np.random.default_rng(1216)
    S = np.where(rng.standard_normal((N, K)) >= 0, 1, -1).astype(np.int8)
    g = np.exp(0.3 * rng.standard_normal(K)).astype(np.float32)
    h = (0.02 * np.exp(0.3 * rng.standard_normal(N))).astype(np.float32)
    x = wls.normal_activations(1217, M, K, 0.0)
    W = S.astype(np.float64) * np.outer(h, g).astype(np.float64)
    ref = x.astype(np.float64) @ W.T

    codes, _ = oracle.binary_codes((S.astype(np.float32) * np.float32(0.5)))
    assert np.array_equal(codes, S)
    q, s_x = oracle.act_prologue(x, g)
    y = oracle.rescale(oracle.int_dot(q, codes, oracle.BINARY1), h, s_x, "f32")
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert rel < 0.02, rel
    # without the input vector (g dropped): far off
    q2, s2 = oracle.act_prologue(x, None)
    y2 = oracle.rescale(oracle.int_dot(q2, codes, oracle.BINARY1), h, s2, "f32")
    assert np.linalg.norm(y2 - ref) / np.linalg.norm(ref) > 0.1
