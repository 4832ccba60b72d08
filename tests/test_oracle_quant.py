"""Pins of the 8-bit weight oracle (POET-XQ storage of W0') against facts that do not come from
the oracle itself: exact lattices, the uniform-rounding error bound, the tie rule, sign and
power-of-two symmetry, per-column independence, exact rational arithmetic on small inputs, and
the plain layer it must reduce to when W0' is exactly representable.  CPU only."""
from fractions import Fraction

import numpy as np
import pytest

import oracle as O
import oracle.quant as Q


def _lattice(m, n, seed):
    """W[:, j] = k[:, j] * 2^e_j with integer |k| <= 127 and max |k[:, j]| = 127."""
    rng = np.random.default_rng(seed)
    k = rng.integers(-127, 128, size=(m, n))
    k[rng.integers(0, m, size=n), np.arange(n)] = np.where(rng.random(n) < 0.5, -127, 127)
    e = rng.integers(-12, 3, size=n)
    return k, np.ldexp(1.0, e), k * np.ldexp(1.0, e)[None, :]


def test_exact_lattice_round_trips():
    k, s, W = _lattice(40, 24, 1)
    q, scale = Q.quantize_w0_int8(W)
    assert q.dtype == np.int8 and scale.dtype == np.float32
    assert np.array_equal(q.astype(np.int64), k)
    assert np.array_equal(scale.astype(np.float64), s)
    # |k| <= 127 has at most 7 significant bits: bf16 holds k * 2^e exactly
    assert np.array_equal(Q.dequantize_w0_int8(q, scale), W)


def test_zero_column_has_zero_scale_and_codes():
    W = np.random.default_rng(2).standard_normal((16, 8))
    W[:, 3] = 0.0
    q, s = Q.quantize_w0_int8(W)
    assert s[3] == 0 and not np.any(q[:, 3])
    assert np.all(Q.dequantize_w0_int8(q, s)[:, 3] == 0)


def test_ties_round_half_to_even():
    # scale 1 (column max 127); entries at exact halves
    col = np.array([127.0, 2.5, 3.5, -2.5, -3.5, 0.5, -0.5, 126.5])
    q, s = Q.quantize_w0_int8(col[:, None])
    assert s[0] == 1.0
    assert q[:, 0].tolist() == [127, 2, 4, -2, -4, 0, 0, 126]


def test_uniform_rounding_error_bound_and_range():
    rng = np.random.default_rng(3)
    W = rng.standard_normal((300, 50)) * rng.uniform(0.01, 3.0, size=50)[None, :]
    q, s = Q.quantize_w0_int8(W)
    w32 = W.astype(np.float32).astype(np.float64)
    err = np.abs(w32 - q.astype(np.float64) * s.astype(np.float64)[None, :])
    assert np.all(err <= 0.5 * s.astype(np.float64)[None, :] * (1 + 1e-6))
    assert np.all(np.abs(q.astype(np.int64)) <= 127)
    # the column maximum maps to +-127
    j = np.arange(50)
    i = np.argmax(np.abs(w32), axis=0)
    assert np.all(np.abs(q[i, j].astype(np.int64)) == 127)


def test_sign_and_power_of_two_symmetry():
    W = np.random.default_rng(4).standard_normal((64, 32))
    q, s = Q.quantize_w0_int8(W)
    qn, sn = Q.quantize_w0_int8(-W)
    assert np.array_equal(qn, -q) and np.array_equal(sn, s)
    q2, s2 = Q.quantize_w0_int8(W * 4.0)
    assert np.array_equal(q2, q) and np.array_equal(s2, s * 4)


def test_scales_are_per_column():
    rng = np.random.default_rng(5)
    W = rng.standard_normal((48, 20))
    W[7, :] *= 50.0                                    # one large row must not set other scales
    q, s = Q.quantize_w0_int8(W)
    W2 = W.copy()
    W2[:, 4] *= 3.0                                    # changing one column changes only it
    q2, s2 = Q.quantize_w0_int8(W2)
    keep = np.arange(20) != 4
    assert np.array_equal(q2[:, keep], q[:, keep]) and np.array_equal(s2[keep], s[keep])
    assert np.isclose(s2[4], 3 * s[4], rtol=1e-6)
    perm = rng.permutation(20)
    q3, s3 = Q.quantize_w0_int8(W[:, perm])
    assert np.array_equal(q3, q[:, perm]) and np.array_equal(s3, s[perm])


def test_codes_match_exact_rational_rounding():
    """Brute force in exact arithmetic: s = amax / 127 and q = round_half_even(w / s) over the
    rationals, w taken as its fp32 value.  fp32 division could only differ within 2^-24 of a
    half-integer, which these seeded inputs do not come near."""
    rng = np.random.default_rng(6)
    W = (rng.standard_normal((12, 9)) * 0.3).astype(np.float32)
    q, s = Q.quantize_w0_int8(W)
    for j in range(W.shape[1]):
        amax = max(abs(Fraction(float(v))) for v in W[:, j])
        sj = amax / 127
        assert abs(Fraction(float(s[j])) - sj) <= sj * Fraction(1, 1 << 23)
        for i in range(W.shape[0]):
            assert int(q[i, j]) == round(Fraction(float(W[i, j])) / sj)


def test_dequantised_values_are_bf16_of_fp32_product():
    rng = np.random.default_rng(7)
    q = rng.integers(-127, 128, size=(30, 10)).astype(np.int8)
    s = (rng.uniform(0.001, 0.05, size=10)).astype(np.float32)
    d = Q.dequantize_w0_int8(q, s)
    for i in range(30):
        for j in range(10):
            p = float(np.float32(np.float32(int(q[i, j])) * s[j]))
            # bf16 keeps 8 significant bits: the nearest such value, ties to an even last bit
            m, e = np.frexp(p)
            scaled = Fraction(m) * 256
            r = round(scaled)               # round half to even
            assert d[i, j] == float(np.ldexp(float(r) / 256, e)), (i, j)


def test_xq_layer_equals_plain_layer_on_exact_lattice():
    m, n, b, T = 32, 48, 8, 20
    _, _, W = _lattice(m, n, 8)
    rng = np.random.default_rng(9)
    X = rng.standard_normal((T, m))
    pr, pp = rng.permutation(m), rng.permutation(n)
    Gr = O.cnp(rng.standard_normal((m // b, b * (b - 1) // 2)) * 0.05, b)
    Gp = O.cnp(rng.standard_normal((n // b, b * (b - 1) // 2)) * 0.05, b)
    q, s = Q.quantize_w0_int8(W)
    y_xq = O.linear_fwd(X, Q.dequantize_w0_int8(q, s), pr, pp, Gr, Gp)["Y"]
    y = O.linear_fwd(X, W, pr, pp, Gr, Gp)["Y"]
    assert np.array_equal(y_xq, y)


def test_requantized_merge_preserves_the_function_to_quantisation_error():
    """Merge-then-reinitialize of an 8-bit layer: the new 8-bit W0' reproduces the layer up to
    the new rounding (the merge itself is exact, "Reparameterized LLM Training ..." §3)."""
    m, n, b, T = 32, 48, 8, 16
    rng = np.random.default_rng(10)
    W = rng.standard_normal((m, n)) / np.sqrt(n)
    q, s = Q.quantize_w0_int8(W)
    W0m = Q.dequantize_w0_int8(q, s)
    pr, pp = rng.permutation(m), rng.permutation(n)
    q_r = rng.standard_normal((m // b, b * (b - 1) // 2)) * 0.05
    q_p = rng.standard_normal((n // b, b * (b - 1) // 2)) * 0.05
    X = rng.standard_normal((T, m))
    y0 = O.linear_fwd(X, W0m, pr, pp, O.cnp(q_r, b), O.cnp(q_p, b))["Y"]
    out = O.merge_reinit(W0m, pr, pp, q_r, q_p, b, seed=77)
    q2, s2 = Q.requantize_after_merge(out["W0m"])
    I_r = O.cnp(out["q_r"], b)
    I_p = O.cnp(out["q_p"], b)
    y1 = O.linear_fwd(X, Q.dequantize_w0_int8(q2, s2), out["perm_r"], out["perm_p"], I_r, I_p)["Y"]
    y_exact = O.linear_fwd(X, out["W0m"], out["perm_r"], out["perm_p"], I_r, I_p)["Y"]
    assert np.max(np.abs(y_exact - y0)) <= 1e-12 * np.max(np.abs(y0))
    # one code step per weight: |dy| <= sum_i |x_i| (s_j / 2 + bf16 half-ulp)
    bound = np.abs(X[:, out["perm_r"]]).sum(axis=1).max() * (0.5 + 2 ** -8) * s2.max()
    assert np.max(np.abs(y1 - y0)) <= bound
