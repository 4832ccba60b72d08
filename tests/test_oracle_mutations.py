"""Plant plausible mistakes in the oracle (on the CPU only) and check that
its pins catch each one: a dropped term, a wrong sign, a transposed operand,
a wrong index direction."""
import numpy as np
import pytest

import oracle
import oracle.poetx_oracle as OM
import tests.test_oracle as pins

F64 = np.float64


def _patch(monkeypatch, name, fn):
    monkeypatch.setattr(OM, name, fn)
    if hasattr(oracle, name):
        monkeypatch.setattr(oracle, name, fn)


def cnp_drop_q3(q, b):
    Q = OM.unpack_skew(q, b)
    I = np.eye(b)
    Q2 = Q @ Q
    return I + 2.0 * (Q + Q2) + Q2 @ Q2


def cnp_wrong_sign(q, b):
    Q = OM.unpack_skew(q, b)
    I = np.eye(b)
    Q2 = Q @ Q
    return I + 2.0 * (Q - Q2 + Q2 @ Q) + Q2 @ Q2


def blockwise_transposed(A, G, transpose=False):
    nb, b, _ = G.shape
    out = np.empty((A.shape[0], nb * b), dtype=F64)
    for j in range(nb):
        Gj = G[j] if transpose else G[j].T
        out[:, j * b:(j + 1) * b] = A[:, j * b:(j + 1) * b] @ Gj
    return out


def merge_inverse_index(W0, perm_r, perm_p):
    return np.asarray(W0)[np.argsort(perm_r)][:, np.argsort(perm_p)]


def dq_missing_k4(dG, q, b):
    Q = OM.unpack_skew(q, b)
    QT = np.transpose(Q, (0, 2, 1))
    powT = [np.broadcast_to(np.eye(b), Q.shape).copy()]
    for _ in range(3):
        powT.append(powT[-1] @ QT)
    S = np.zeros_like(Q)
    for k, c in {1: 2.0, 2: 2.0, 3: 2.0}.items():
        for i in range(k):
            S += c * (powT[i] @ dG @ powT[k - 1 - i])
    return OM.grad_through_packing(S)


MUTATIONS = {
    "cnp_drop_q3": ("cnp", cnp_drop_q3,
                    [pins.test_golden_b2_closed_form,
                     lambda: pins.test_cnp_reordered_equals_neumann_product(16, 0.05)]),
    "cnp_wrong_sign": ("cnp", cnp_wrong_sign,
                       [pins.test_golden_b2_closed_form,
                        lambda: pins.test_cnp_closed_form_spectrum(8, 0.2)]),
    "blockwise_transposed": ("_blockwise", blockwise_transposed,
                             [lambda: pins.test_input_centric_equals_weight_centric(32, 32, 8),
                              pins.test_backward_matches_torch_autograd]),
    "merge_inverse_index": ("merge_permutations", merge_inverse_index,
                            [pins.test_merged_equals_unmerged,
                             lambda: pins.test_input_centric_equals_weight_centric(24, 40, 8)]),
    "dq_missing_k4": ("dq_from_dG", dq_missing_k4,
                      [pins.test_dq_matches_central_finite_differences,
                       pins.test_backward_matches_torch_autograd]),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(monkeypatch, name):
    target, fn, checks = MUTATIONS[name]
    _patch(monkeypatch, target, fn)
    for check in checks:
        with pytest.raises(AssertionError):
            check()


def test_pins_catch_transposed_packing(monkeypatch):
    orig = OM.unpack_skew

    def unpack_lower(q, b):  # q placed in the lower triangle instead
        return np.transpose(orig(q, b), (0, 2, 1))
    _patch(monkeypatch, "unpack_skew", unpack_lower)
    for check in (pins.test_packed_triu_layout, pins.test_golden_b2_closed_form):
        with pytest.raises(AssertionError):
            check()


def test_pins_catch_flipped_packing_gradient(monkeypatch):
    orig = OM.grad_through_packing
    _patch(monkeypatch, "grad_through_packing", lambda S: -orig(S))
    with pytest.raises(AssertionError):
        pins.test_dq_matches_central_finite_differences()


# ---------------------------------------------------------------- 8-bit weight storage (POET-XQ)
import oracle.quant as QM  # noqa: E402
import tests.test_oracle_quant as qpins  # noqa: E402


def _quant_variant(divisor=127.0, axis=0, rounder=np.rint):
    def quantize(W0m):
        w = np.asarray(W0m, dtype=np.float32)
        amax = np.max(np.abs(w), axis=axis, keepdims=True)
        scale = (amax / np.float32(divisor)).astype(np.float32)
        safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
        q = np.clip(rounder((w / safe).astype(np.float32)), -127, 127)
        q = np.where(scale > 0, q, 0.0).astype(np.int8)
        return q, (scale.reshape(-1) if axis == 0 else scale.reshape(-1)[: w.shape[1]])
    return quantize


QUANT_MUTATIONS = {
    "divide_by_128": _quant_variant(divisor=128.0),
    "per_row_scale": _quant_variant(axis=1),
    "truncate": _quant_variant(rounder=np.trunc),
    "half_away_from_zero": _quant_variant(
        rounder=lambda r: np.sign(r) * np.floor(np.abs(r) + np.float32(0.5))),
}


@pytest.mark.parametrize("name", sorted(QUANT_MUTATIONS))
def test_quant_pins_catch_planted_mistake(monkeypatch, name):
    monkeypatch.setattr(QM, "quantize_w0_int8", QUANT_MUTATIONS[name])
    failed = 0
    for check in (qpins.test_exact_lattice_round_trips, qpins.test_ties_round_half_to_even,
                  qpins.test_uniform_rounding_error_bound_and_range,
                  qpins.test_scales_are_per_column, qpins.test_codes_match_exact_rational_rounding):
        try:
            check()
        except (AssertionError, ValueError, IndexError):
            failed += 1
    assert failed >= 1, name


def test_quant_pins_catch_unrounded_dequantisation(monkeypatch):
    monkeypatch.setattr(QM, "dequantize_w0_int8",
                        lambda q, s: q.astype(np.float64) * np.asarray(s, np.float64)[None, :])
    with pytest.raises(AssertionError):
        qpins.test_dequantised_values_are_bf16_of_fp32_product()
