"""Pins of the float64 oracle against facts fixed by the pages and by
mathematics: identities the pages state, closed forms, special cases that
reduce to a textbook routine, finite differences, an independent autograd
implementation and a published generator's known outputs.  CPU only."""
import os

import numpy as np
import pytest

import oracle as O
import poetx_workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def rand_layer(m, n, b, T, sigma=0.1, seed=0):
    rng = np.random.default_rng(seed)
    return dict(
        X=rng.standard_normal((T, m)), dY=rng.standard_normal((T, n)),
        W0=rng.standard_normal((m, n)),
        q_r=rng.standard_normal((m // b, b * (b - 1) // 2)) * sigma,
        q_p=rng.standard_normal((n // b, b * (b - 1) // 2)) * sigma,
        perm_r=rng.permutation(m), perm_p=rng.permutation(n))


# ---------------------------------------------------------------- packing
def test_packed_triu_layout():
    b = 64
    assert b * (b - 1) // 2 == 2016  # entries per block in the tiny fp32 workload
    q = np.arange(1, 2017, dtype=np.float64)[None]
    Q = O.unpack_skew(q, b)[0]
    assert np.all(Q == -Q.T) and np.all(np.diag(Q) == 0)
    # row-major order over i < j: first row holds 1..63, second row starts at 64
    assert Q[0, 1] == 1 and Q[0, 63] == 63 and Q[1, 2] == 64 and Q[62, 63] == 2016


def test_golden_b2_closed_form():
    rows = np.loadtxt(os.path.join(GOLDEN, "cnp_b2.txt"))
    for r in rows:
        a = r[0]
        G = O.cnp(np.array([[a]]), 2)[0]
        C = O.cayley_exact(np.array([[a]]), 2)[0]
        np.testing.assert_allclose(G.ravel(), r[1:5], rtol=0, atol=1e-14)
        np.testing.assert_allclose(C.ravel(), r[5:9], rtol=0, atol=1e-14)


# ---------------------------------------------------------------- CNP
@pytest.mark.parametrize("b,sigma", [(4, 0.3), (16, 0.05), (64, 0.01)])
def test_cnp_reordered_equals_neumann_product(b, sigma):
    """(I+Q)(I+Q+Q^2+Q^3) == I + 2(Q+Q^2+Q^3) + Q^4: the two forms on the pages."""
    rng = np.random.default_rng(b)
    q = rng.standard_normal((3, b * (b - 1) // 2)) * sigma
    assert rel(O.cnp(q, b), O.cnp_neumann_product(q, b, k=3)) < 1e-13


def test_cnp_q_zero_is_identity():
    G = O.cnp(np.zeros((2, 120)), 16)
    assert np.array_equal(G, np.broadcast_to(np.eye(16), G.shape))


@pytest.mark.parametrize("b,sigma", [(8, 0.2), (32, 0.05), (64, 0.01)])
def test_cnp_closed_form_spectrum(b, sigma):
    """G is a polynomial in the normal matrix Q, so G^T G = (I - Q^4)^2 and
    its singular values are |1 - mu^4| for the eigenvalues +-i mu of Q."""
    rng = np.random.default_rng(7 + b)
    q = rng.standard_normal((2, b * (b - 1) // 2)) * sigma
    G = O.cnp(q, b)
    Q = O.unpack_skew(q, b)
    for j in range(2):
        mu = np.abs(np.linalg.eigvals(Q[j]).imag)
        expect = np.sort(np.abs(1.0 - mu ** 4))
        got = np.sort(np.linalg.svd(G[j], compute_uv=False))
        np.testing.assert_allclose(got, expect, rtol=0, atol=1e-12)
        Q4 = np.linalg.matrix_power(Q[j], 4)
        I = np.eye(b)
        np.testing.assert_allclose(G[j].T @ G[j], (I - Q4) @ (I - Q4), rtol=0, atol=1e-12)


def test_cnp_truncation_error_closed_form():
    """Cayley - CNP = (I+Q) Q^4 (I-Q)^{-1}: the Neumann tail after k = 3."""
    b = 12
    rng = np.random.default_rng(3)
    q = rng.standard_normal((2, b * (b - 1) // 2)) * 0.2
    Q = O.unpack_skew(q, b)
    I = np.eye(b)
    tail = np.stack([(I + Q[j]) @ np.linalg.matrix_power(Q[j], 4) @ np.linalg.inv(I - Q[j])
                     for j in range(2)])
    np.testing.assert_allclose(O.cayley_exact(q, b) - O.cnp(q, b), tail, rtol=0, atol=1e-13)


def test_cayley_exact_is_orthogonal():
    b = 32
    rng = np.random.default_rng(5)
    q = rng.standard_normal((3, b * (b - 1) // 2)) * 0.3
    C = O.cayley_exact(q, b)
    for j in range(3):
        np.testing.assert_allclose(C[j].T @ C[j], np.eye(b), rtol=0, atol=1e-13)


# ---------------------------------------------------------------- forward
def test_forward_q_zero_is_plain_linear():
    """Q = 0 => G = I => Y = X W0 (textbook matmul on the un-merged W0)."""
    d = rand_layer(32, 48, 8, 10)
    W0m = O.merge_permutations(d["W0"], d["perm_r"], d["perm_p"])
    G_r = O.cnp(np.zeros_like(d["q_r"]), 8)
    G_p = O.cnp(np.zeros_like(d["q_p"]), 8)
    Y = O.linear_fwd(d["X"], W0m, d["perm_r"], d["perm_p"], G_r, G_p)["Y"]
    assert rel(Y, np.matmul(d["X"], d["W0"])) < 1e-14


@pytest.mark.parametrize("m,n,b", [(16, 24, 4), (32, 32, 8), (24, 40, 8)])
def test_input_centric_equals_weight_centric(m, n, b):
    d = rand_layer(m, n, b, 7, sigma=0.3, seed=m + n)
    G_r, G_p = O.cnp(d["q_r"], b), O.cnp(d["q_p"], b)
    W0m = O.merge_permutations(d["W0"], d["perm_r"], d["perm_p"])
    Y_ic = O.linear_fwd(d["X"], W0m, d["perm_r"], d["perm_p"], G_r, G_p)["Y"]
    Y_wc = O.linear_fwd_weight_centric(d["X"], d["W0"], d["perm_r"], d["perm_p"], G_r, G_p)
    assert rel(Y_ic, Y_wc) < 1e-13


def test_merged_equals_unmerged():
    m, n, b = 24, 32, 8
    d = rand_layer(m, n, b, 6, sigma=0.3, seed=11)
    G_r, G_p = O.cnp(d["q_r"], b), O.cnp(d["q_p"], b)
    W0m = O.merge_permutations(d["W0"], d["perm_r"], d["perm_p"])
    Y_m = O.linear_fwd(d["X"], W0m, d["perm_r"], d["perm_p"], G_r, G_p)["Y"]
    Y_u = O.linear_fwd_unmerged(d["X"], d["W0"], d["perm_r"], d["perm_p"], G_r, G_p)
    assert rel(Y_m, Y_u) < 1e-13
    # the merged weight is the permutation-matrix product Psi_R W0 Psi_P^T
    Pr, Pp = O.perm_matrix(d["perm_r"]), O.perm_matrix(d["perm_p"])
    assert np.array_equal(W0m, Pr @ d["W0"] @ Pp.T)
    assert np.array_equal(O.unmerge_permutations(W0m, d["perm_r"], d["perm_p"]), d["W0"])


def test_spectrum_preserved_with_exact_cayley():
    m, n, b = 32, 24, 8
    d = rand_layer(m, n, b, 1, sigma=0.4, seed=2)
    R = O.spo_matrix(O.cayley_exact(d["q_r"], b), d["perm_r"])
    P = O.spo_matrix(O.cayley_exact(d["q_p"], b), d["perm_p"])
    s0 = np.linalg.svd(d["W0"], compute_uv=False)
    s1 = np.linalg.svd(R @ d["W0"] @ P, compute_uv=False)
    np.testing.assert_allclose(s1, s0, rtol=1e-12, atol=1e-12)


def test_spectrum_bounds_with_cnp():
    """sigma_min(R) sigma_min(P) s_i <= s_i(R W0 P) <= sigma_max(R) sigma_max(P) s_i."""
    m, n, b = 32, 24, 8
    d = rand_layer(m, n, b, 1, sigma=0.3, seed=4)
    Gr, Gp = O.cnp(d["q_r"], b), O.cnp(d["q_p"], b)
    R, P = O.spo_matrix(Gr, d["perm_r"]), O.spo_matrix(Gp, d["perm_p"])
    sr, sp = np.linalg.svd(R, compute_uv=False), np.linalg.svd(P, compute_uv=False)
    s0 = np.linalg.svd(d["W0"], compute_uv=False)
    s1 = np.linalg.svd(R @ d["W0"] @ P, compute_uv=False)
    assert np.all(s1 <= sr.max() * sp.max() * s0 * (1 + 1e-12))
    assert np.all(s1 >= sr.min() * sp.min() * s0 * (1 - 1e-12))
    assert not np.allclose(s1, s0, rtol=1e-6)  # CNP is not exactly orthogonal


# ---------------------------------------------------------------- backward
def test_dq_matches_central_finite_differences():
    m, n, b, T = 8, 12, 4, 5
    d = rand_layer(m, n, b, T, sigma=0.25, seed=9)
    W0m = O.merge_permutations(d["W0"], d["perm_r"], d["perm_p"])
    G_r, G_p = O.cnp(d["q_r"], b), O.cnp(d["q_p"], b)
    g = O.linear_bwd(d["X"], d["dY"], W0m, d["perm_r"], d["perm_p"], G_r, G_p,
                     d["q_r"], d["q_p"], b)
    h = 1e-6
    for key, other in (("q_r", "q_p"), ("q_p", "q_r")):
        fd = np.zeros_like(d[key])
        for idx in np.ndindex(*d[key].shape):
            qp = d[key].copy(); qp[idx] += h
            qm = d[key].copy(); qm[idx] -= h
            args = {key: qp, other: d[other]}
            Lp = O.layer_loss(d["X"], d["dY"], W0m, d["perm_r"], d["perm_p"],
                              args["q_r"], args["q_p"], b)
            args[key] = qm
            Lm = O.layer_loss(d["X"], d["dY"], W0m, d["perm_r"], d["perm_p"],
                              args["q_r"], args["q_p"], b)
            fd[idx] = (Lp - Lm) / (2 * h)
        assert rel(g["d" + key], fd) < 1e-6, key


def test_dx_matches_dense_transpose():
    m, n, b, T = 24, 16, 8, 9
    d = rand_layer(m, n, b, T, sigma=0.3, seed=12)
    W0m = O.merge_permutations(d["W0"], d["perm_r"], d["perm_p"])
    G_r, G_p = O.cnp(d["q_r"], b), O.cnp(d["q_p"], b)
    g = O.linear_bwd(d["X"], d["dY"], W0m, d["perm_r"], d["perm_p"], G_r, G_p,
                     d["q_r"], d["q_p"], b)
    W_rp = O.spo_matrix(G_r, d["perm_r"]) @ d["W0"] @ O.spo_matrix(G_p, d["perm_p"])
    assert rel(g["dX"], d["dY"] @ W_rp.T) < 1e-13
    assert rel(O.linear_dx_rows(d["dY"][2:5], W0m, d["perm_r"], d["perm_p"], G_r, G_p),
               g["dX"][2:5]) < 1e-14


def test_backward_matches_torch_autograd():
    """An independent implementation: float64 torch autograd through the
    dense weight-centric forward."""
    torch = pytest.importorskip("torch")
    m, n, b, T = 64, 128, 32, 16
    d = rand_layer(m, n, b, T, sigma=0.05, seed=21)
    W0m = O.merge_permutations(d["W0"], d["perm_r"], d["perm_p"])
    G_r, G_p = O.cnp(d["q_r"], b), O.cnp(d["q_p"], b)
    g = O.linear_bwd(d["X"], d["dY"], W0m, d["perm_r"], d["perm_p"], G_r, G_p,
                     d["q_r"], d["q_p"], b)

    def build(qv, size):
        iu = torch.triu_indices(b, b, 1)
        Q = torch.zeros(size // b, b, b, dtype=torch.float64)
        Q[:, iu[0], iu[1]] = qv
        Q = Q - Q.transpose(1, 2)
        I = torch.eye(b, dtype=torch.float64)
        G = (I + Q) @ (I + Q + Q @ Q + Q @ Q @ Q)
        return torch.block_diag(*G)

    qr = torch.tensor(d["q_r"], requires_grad=True)
    qp = torch.tensor(d["q_p"], requires_grad=True)
    X = torch.tensor(d["X"], requires_grad=True)
    Pr = torch.tensor(O.perm_matrix(d["perm_r"]))
    Pp = torch.tensor(O.perm_matrix(d["perm_p"]))
    R = Pr.T @ build(qr, m) @ Pr
    P = Pp.T @ build(qp, n) @ Pp
    Y = X @ (R @ torch.tensor(d["W0"]) @ P)
    (Y * torch.tensor(d["dY"])).sum().backward()
    assert rel(g["Y"], Y.detach().numpy()) < 1e-13
    assert rel(g["dX"], X.grad.numpy()) < 1e-12
    assert rel(g["dq_r"], qr.grad.numpy()) < 1e-12
    assert rel(g["dq_p"], qp.grad.numpy()) < 1e-12


# ---------------------------------------------------------------- merge-reinit
def test_merged_weight_block_form_equals_dense():
    m, n, b = 24, 32, 8
    d = rand_layer(m, n, b, 1, sigma=0.3, seed=13)
    G_r, G_p = O.cnp(d["q_r"], b), O.cnp(d["q_p"], b)
    W0m = O.merge_permutations(d["W0"], d["perm_r"], d["perm_p"])
    W_blk = O.merged_weight_natural(W0m, d["perm_r"], d["perm_p"], G_r, G_p)
    W_dense = O.spo_matrix(G_r, d["perm_r"]) @ d["W0"] @ O.spo_matrix(G_p, d["perm_p"])
    assert rel(W_blk, W_dense) < 1e-14


def test_merge_reinit_preserves_function():
    m, n, b, T = 32, 48, 8, 11
    d = rand_layer(m, n, b, T, sigma=0.2, seed=17)
    W0m = O.merge_permutations(d["W0"], d["perm_r"], d["perm_p"])
    Y0 = O.linear_fwd(d["X"], W0m, d["perm_r"], d["perm_p"],
                      O.cnp(d["q_r"], b), O.cnp(d["q_p"], b))["Y"]
    r = O.merge_reinit(W0m, d["perm_r"], d["perm_p"], d["q_r"], d["q_p"], b, seed=1234)
    assert np.all(r["q_r"] == 0) and np.all(r["q_p"] == 0)
    assert not np.array_equal(r["perm_r"], d["perm_r"])
    Y1 = O.linear_fwd(d["X"], r["W0m"], r["perm_r"], r["perm_p"],
                      O.cnp(r["q_r"], b), O.cnp(r["q_p"], b))["Y"]
    assert rel(Y1, Y0) < 1e-13


# ---------------------------------------------------------------- generator
def test_splitmix64_known_outputs():
    """Published SplitMix64 outputs for initial state 0."""
    assert O.splitmix_stream(0, 3) == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4,
                                       0x06C45D188009454F]
    for s in (0, 1, 0xDEADBEEF, (1 << 64) - 1):
        seq = O.splitmix_stream(s, 5)
        assert [O.splitmix_output(s, i) for i in range(5)] == seq


def test_resampled_permutations_are_uniform_bijections():
    n, trials = 6, 3000
    counts = np.zeros((n, n))
    for s in range(trials):
        p = O.resample_permutation(s, 0, n)
        assert sorted(p.tolist()) == list(range(n))
        counts[np.arange(n), p] += 1
    exp = trials / n
    chi2 = float(((counts - exp) ** 2 / exp).sum())
    assert chi2 < 60.0  # 25 dof: p(chi2 > 60) < 1e-4
    assert not np.array_equal(O.resample_permutation(1, 0, 64), O.resample_permutation(1, 1, 64))


# ---------------------------------------------------------------- workloads
def test_workload_generator_recipe():
    wl = W.WORKLOADS["tiny_fp32"]
    p = W.layer_params(wl)
    assert p["W0"].shape == (512, 512) and p["q_r"].shape == (8, 2016)
    np.testing.assert_allclose(np.linalg.norm(p["W0"].astype(np.float64), axis=1), 1.0, atol=1e-6)
    assert sorted(p["perm_r"].tolist()) == list(range(512))
    a = W.layer_acts(wl)
    assert a["X"].shape == (256, 512) and a["dY"].shape == (256, 512)
    # determinism
    assert np.array_equal(W.layer_params(wl)["q_p"], p["q_p"])
    # bfloat16 keeps 8 significant bits: the spacing above 1.0 is 2^-7
    x = np.array([1.0, 1.0078125, 1.00390625, 1.01171875, 1.005], dtype=np.float32)
    r = W.round_bf16(x)
    assert r[0] == 1.0 and r[1] == 1.0078125          # exact values stay
    assert r[2] == 1.0 and r[3] == 1.015625            # ties go to the even neighbour
    assert r[4] == 1.0078125                           # nearest
