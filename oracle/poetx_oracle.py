"""Float64 CPU oracle of the POET-X linear layer.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
the CPU-baseline / reference legs of the benchmark may import or run this
file.  The CUDA library never calls it and shares no code with it.

Everything here is plain numpy float64: the definitions written out, in the
pages' order and notation, with library matmuls as the only building block.
Inputs stored in bfloat16 or float32 are upcast to float64 once; no
intermediate is rounded.

Sources (web pages on POET / POET-X):
  [POET]  "Reparameterized LLM Training via Orthogonal Equivalence
          Transformation" (paper notes, NeurIPS 2025):
          §整体框架 (W_RP = R W0 P, y = (R W0 P)^T x, spectrum preservation),
          §1 SPO (block-stochastic R = Psi^T Diag(G^1..G^{m/b}) Psi),
          §2 CNP (R = (I+Q)(I-Q)^{-1} ~ (I+Q)(I + sum_{i=1..k} Q^i), k = 3),
          §3 Merge-then-Reinitialize (W <- R W P, reset, resample).
  [P1]    "在单张 H100 上预训练 13B 模型：POET-X 如何把正交变换的内存开销砍到 1/3":
          §第一斧 (input-centric order R^T x, W^T(.), P^T(.)),
          §第二斧 (index-array permutations; 2 of 4 merged into W),
          §第三斧 (each b x b block as one batch element),
          §第四斧 (packed upper triangle; G = 2(Q+Q^2+Q^2 Q) + Q^2 Q^2 + I),
          §第五斧 (forward a = G_R^T x, b = W a, z = G_P^T b).

Conventions (readings of the pages, all listed in the design notes):
  * W0 is m x n (m = in-features); with token-major X [T, m] the layer is
    Y = X R W0 P   (the row form of y = (R W0 P)^T x).
  * A permutation is an int array pi; its matrix Psi has Psi[i, pi[i]] = 1,
    so X Psi^T = X[:, pi] (column gather) and, for C Psi = Y,
    Y[:, pi[i]] = C[:, i] (column scatter).
  * R = Psi_R^T Diag(G_R^1..G_R^{m/b}) Psi_R, P likewise; one SPO factor per
    merge period.
  * The merged weight is W0' = Psi_R W0 Psi_P^T, i.e. W0'[i, j] = W0[pi_R[i], pi_P[j]].
  * q holds the strict upper triangle of each skew block Q in row-major
    (i < j) order: Q[i, j] = q, Q[j, i] = -q, diagonal 0.
"""
from __future__ import annotations

from typing import Dict, Tuple

import numpy as np

from .splitmix import resample_permutation

F64 = np.float64


# --------------------------------------------------------------------------
# packed skew-symmetric parameters  ([P1] §第四斧 item 1: only the upper
# triangle is stored, b(b-1)/2 numbers per block)
# --------------------------------------------------------------------------
def triu_pairs(b: int) -> Tuple[np.ndarray, np.ndarray]:
    """(rows, cols) of the strict upper triangle in row-major order."""
    return np.triu_indices(b, 1)


def unpack_skew(q: np.ndarray, b: int) -> np.ndarray:
    """q [nb, b(b-1)/2] -> Q [nb, b, b] with Q = -Q^T."""
    q = np.asarray(q, dtype=F64)
    nb = q.shape[0]
    iu, ju = triu_pairs(b)
    Q = np.zeros((nb, b, b), dtype=F64)
    Q[:, iu, ju] = q
    Q[:, ju, iu] = -q
    return Q


def grad_through_packing(S: np.ndarray) -> np.ndarray:
    """dL/dq from dL/dQ (Q unconstrained): q enters Q[i,j] with +1 and Q[j,i] with -1."""
    b = S.shape[-1]
    iu, ju = triu_pairs(b)
    return S[:, iu, ju] - S[:, ju, iu]


# --------------------------------------------------------------------------
# Cayley-Neumann parameterisation
# --------------------------------------------------------------------------
def cnp(q: np.ndarray, b: int) -> np.ndarray:
    """G = I + 2(Q + Q^2 + Q^2 Q) + Q^2 Q^2, per block.

    [P1] §第四斧 item 2 (all terms from Q and Q^2); equals [POET] §2 CNP
    with k = 3.
    """
    Q = unpack_skew(q, b)
    I = np.eye(b, dtype=F64)
    Q2 = Q @ Q
    return I + 2.0 * (Q + Q2 + Q2 @ Q) + Q2 @ Q2


def cnp_neumann_product(q: np.ndarray, b: int, k: int = 3) -> np.ndarray:
    """(I + Q)(I + sum_{i=1..k} Q^i): [POET] §2 CNP, the truncated Neumann form."""
    Q = unpack_skew(q, b)
    I = np.eye(b, dtype=F64)
    series = np.broadcast_to(I, Q.shape).copy()
    Qi = np.broadcast_to(I, Q.shape).copy()
    for _ in range(k):
        Qi = Qi @ Q
        series = series + Qi
    return (I + Q) @ series


def cayley_exact(q: np.ndarray, b: int) -> np.ndarray:
    """R = (I + Q)(I - Q)^{-1}: [POET] §2 CNP, the exact Cayley transform."""
    Q = unpack_skew(q, b)
    I = np.eye(b, dtype=F64)
    out = np.empty_like(Q)
    for j in range(Q.shape[0]):
        # X (I - Q) = (I + Q)  <=>  (I - Q)^T X^T = (I + Q)^T
        out[j] = np.linalg.solve((I - Q[j]).T, (I + Q[j]).T).T
    return out


# --------------------------------------------------------------------------
# permutations and block-stochastic orthogonal matrices  ([POET] §1 SPO)
# --------------------------------------------------------------------------
def perm_matrix(pi: np.ndarray) -> np.ndarray:
    n = len(pi)
    Psi = np.zeros((n, n), dtype=F64)
    Psi[np.arange(n), np.asarray(pi)] = 1.0
    return Psi


def block_diag(G: np.ndarray) -> np.ndarray:
    nb, b, _ = G.shape
    D = np.zeros((nb * b, nb * b), dtype=F64)
    for j in range(nb):
        D[j * b:(j + 1) * b, j * b:(j + 1) * b] = G[j]
    return D


def spo_matrix(G: np.ndarray, pi: np.ndarray) -> np.ndarray:
    """Psi^T Diag(G^1..G^{nb}) Psi as a dense matrix (tiny sizes only)."""
    Psi = perm_matrix(pi)
    return Psi.T @ block_diag(np.asarray(G, dtype=F64)) @ Psi


# --------------------------------------------------------------------------
# permutation merging  ([P1] §第二斧: the two permutations next to the fixed
# W are folded into it before the inner loop)
# --------------------------------------------------------------------------
def merge_permutations(W0: np.ndarray, perm_r: np.ndarray, perm_p: np.ndarray) -> np.ndarray:
    """W0' = Psi_R W0 Psi_P^T, i.e. W0'[i, j] = W0[perm_r[i], perm_p[j]]."""
    W0 = np.asarray(W0)
    return W0[np.asarray(perm_r)][:, np.asarray(perm_p)]


def unmerge_permutations(W0m: np.ndarray, perm_r: np.ndarray, perm_p: np.ndarray) -> np.ndarray:
    """Inverse of merge_permutations: W0 = Psi_R^T W0' Psi_P."""
    W0 = np.empty_like(np.asarray(W0m))
    W0[np.ix_(np.asarray(perm_r), np.asarray(perm_p))] = W0m
    return W0


# --------------------------------------------------------------------------
# the layer: input-centric forward and its exact gradient
# --------------------------------------------------------------------------
def _blockwise(A: np.ndarray, G: np.ndarray, transpose: bool = False) -> np.ndarray:
    """Batch-wise block-diagonal product A Diag(G) (or A Diag(G)^T), one b x b
    block per batch element ([P1] §第三斧)."""
    nb, b, _ = G.shape
    out = np.empty((A.shape[0], nb * b), dtype=F64)
    for j in range(nb):
        Gj = G[j].T if transpose else G[j]
        out[:, j * b:(j + 1) * b] = A[:, j * b:(j + 1) * b] @ Gj
    return out


def linear_fwd(X, W0m, perm_r, perm_p, G_r, G_p) -> Dict[str, np.ndarray]:
    """Y = X Psi_R^T Diag(G_R) W0' Diag(G_P) Psi_P, evaluated input-first.

    [P1] §第一斧 (R^T x, then W^T(.), then P^T(.)) and §第五斧
    (a = G_R^T x, b = W a, z = G_P^T b), with the two remaining permutations
    as index gathers/scatters ([P1] §第二斧).  Row-form steps:
      A  = X[:, pi_R]          A'_j = A_j G_R^j
      B  = A' W0'              C_j  = B_j G_P^j
      Y[:, pi_P] = C
    """
    X = np.asarray(X, dtype=F64)
    W0m = np.asarray(W0m, dtype=F64)
    G_r = np.asarray(G_r, dtype=F64)
    G_p = np.asarray(G_p, dtype=F64)
    A = X[:, perm_r]
    A1 = _blockwise(A, G_r)
    B = A1 @ W0m
    C = _blockwise(B, G_p)
    Y = np.empty_like(C)
    Y[:, perm_p] = C
    return {"Y": Y, "A": A, "A1": A1, "B": B, "C": C}


def linear_fwd_weight_centric(X, W0, perm_r, perm_p, G_r, G_p) -> np.ndarray:
    """Y = X (R W0 P) with R, P and their product formed densely (tiny sizes).

    The original weight-centric POET evaluation ([POET] §整体框架,
    W_RP = R W0 P); W0 here is the un-merged weight.
    """
    R = spo_matrix(G_r, perm_r)
    P = spo_matrix(G_p, perm_p)
    W_rp = R @ np.asarray(W0, dtype=F64) @ P
    return np.asarray(X, dtype=F64) @ W_rp


def linear_fwd_unmerged(X, W0, perm_r, perm_p, G_r, G_p) -> np.ndarray:
    """Input-centric evaluation applying all four permutations explicitly."""
    X = np.asarray(X, dtype=F64)
    W0 = np.asarray(W0, dtype=F64)
    Psi_r = perm_matrix(perm_r)
    Psi_p = perm_matrix(perm_p)
    Dr = block_diag(np.asarray(G_r, dtype=F64))
    Dp = block_diag(np.asarray(G_p, dtype=F64))
    t = X @ Psi_r.T
    t = t @ Dr
    t = t @ Psi_r
    t = t @ W0
    t = t @ Psi_p.T
    t = t @ Dp
    return t @ Psi_p


def dq_from_dG(dG: np.ndarray, q: np.ndarray, b: int) -> np.ndarray:
    """Gradient w.r.t. the packed q of L, given dG = dL/dG for G = cnp(q).

    G = I + sum_k c_k Q^k with c = (2, 2, 2, 1) for k = 1..4 ([P1] §第四斧).
    Chain rule for a matrix power: d<dG, Q^k> = sum_{i<k} <(Q^T)^i dG (Q^T)^{k-1-i}, dQ>.
    Then through the packing (+1 on Q[i,j], -1 on Q[j,i]).
    """
    Q = unpack_skew(q, b)
    dG = np.asarray(dG, dtype=F64)
    coeff = {1: 2.0, 2: 2.0, 3: 2.0, 4: 1.0}
    QT = np.transpose(Q, (0, 2, 1))
    powT = [np.broadcast_to(np.eye(b), Q.shape).copy()]
    for _ in range(3):
        powT.append(powT[-1] @ QT)
    S = np.zeros_like(Q)
    for k, c in coeff.items():
        for i in range(k):
            S += c * (powT[i] @ dG @ powT[k - 1 - i])
    return grad_through_packing(S)


def linear_bwd(X, dY, W0m, perm_r, perm_p, G_r, G_p, q_r, q_p, b) -> Dict[str, np.ndarray]:
    """Exact gradient of linear_fwd for L = sum(dY * Y).

      dC = dY[:, pi_P]
      dB_j = dC_j (G_P^j)^T          dG_P^j = B_j^T dC_j
      dA' = dB W0'^T
      dA_j = dA'_j (G_R^j)^T         dG_R^j = A_j^T dA'_j
      dX[:, pi_R] = dA
      dq = dq_from_dG(dG, q)
    """
    f = linear_fwd(X, W0m, perm_r, perm_p, G_r, G_p)
    dY = np.asarray(dY, dtype=F64)
    W0m = np.asarray(W0m, dtype=F64)
    G_r = np.asarray(G_r, dtype=F64)
    G_p = np.asarray(G_p, dtype=F64)
    nbr, nbp = G_r.shape[0], G_p.shape[0]
    dC = dY[:, perm_p]
    dB = _blockwise(dC, G_p, transpose=True)
    dG_p = np.stack([f["B"][:, j * b:(j + 1) * b].T @ dC[:, j * b:(j + 1) * b]
                     for j in range(nbp)])
    dA1 = dB @ W0m.T
    dA = _blockwise(dA1, G_r, transpose=True)
    dG_r = np.stack([f["A"][:, j * b:(j + 1) * b].T @ dA1[:, j * b:(j + 1) * b]
                     for j in range(nbr)])
    dX = np.empty_like(dA)
    dX[:, perm_r] = dA
    return {"dX": dX, "dq_r": dq_from_dG(dG_r, q_r, b), "dq_p": dq_from_dG(dG_p, q_p, b),
            "dG_r": dG_r, "dG_p": dG_p, "dC": dC, "dB": dB, "dA1": dA1,
            "Y": f["Y"], "B": f["B"]}


def layer_loss(X, dY, W0m, perm_r, perm_p, q_r, q_p, b) -> float:
    """L = sum(dY * Y) with G built by CNP from q (for finite differences)."""
    G_r = cnp(q_r, b)
    G_p = cnp(q_p, b)
    Y = linear_fwd(X, W0m, perm_r, perm_p, G_r, G_p)["Y"]
    return float(np.sum(np.asarray(dY, dtype=F64) * Y))


# --------------------------------------------------------------------------
# merge-then-reinitialize  ([POET] §3: W <- R W P, orthogonal factors reset to
# the identity, permutations resampled; [P1] §第二斧 for the merged form)
# --------------------------------------------------------------------------
def merged_weight_natural(W0m, perm_r, perm_p, G_r, G_p) -> np.ndarray:
    """W_new = R W0 P in natural coordinates, by its block form.

    With W0 = Psi_R^T W0' Psi_P:  R W0 P = Psi_R^T Diag(G_R) W0' Diag(G_P) Psi_P.
    M = Diag(G_R) W0' Diag(G_P) is formed block by block, then
    W_new[pi_R[r], pi_P[c]] = M[r, c].
    """
    W0m = np.asarray(W0m, dtype=F64)
    G_r = np.asarray(G_r, dtype=F64)
    G_p = np.asarray(G_p, dtype=F64)
    M = _blockwise(W0m, G_p)                      # W0' Diag(G_P)
    M = _blockwise(M.T, G_r, transpose=True).T     # Diag(G_R) (.)  as ((.)^T Diag(G_R)^T)^T
    return unmerge_permutations(M, perm_r, perm_p)


def merge_reinit(W0m, perm_r, perm_p, q_r, q_p, b, seed) -> Dict[str, np.ndarray]:
    """One merge-then-reinitialize step on a layer.

    W <- R W P (with G from CNP of the current q), new permutations drawn
    from `seed` (lane 0 for R, lane 1 for P), W0'_new = merge of W with the
    new permutations, q <- 0.
    """
    G_r = cnp(q_r, b)
    G_p = cnp(q_p, b)
    W_new = merged_weight_natural(W0m, perm_r, perm_p, G_r, G_p)
    m, n = W_new.shape
    pr_new = resample_permutation(seed, 0, m)
    pp_new = resample_permutation(seed, 1, n)
    return {"W0m": merge_permutations(W_new, pr_new, pp_new), "W": W_new,
            "perm_r": pr_new, "perm_p": pp_new,
            "q_r": np.zeros_like(np.asarray(q_r, dtype=F64)),
            "q_p": np.zeros_like(np.asarray(q_p, dtype=F64))}


# --------------------------------------------------------------------------
# per-row evaluation for sampled checks at full size
# --------------------------------------------------------------------------
def linear_fwd_rows(X_rows, W0m, perm_r, perm_p, G_r, G_p) -> np.ndarray:
    """Y for a few token rows (tokens are independent in the forward pass)."""
    return linear_fwd(X_rows, W0m, perm_r, perm_p, G_r, G_p)["Y"]


def linear_dx_rows(dY_rows, W0m, perm_r, perm_p, G_r, G_p) -> np.ndarray:
    """dX for a few token rows (dX of token t depends only on dY of token t)."""
    dY = np.asarray(dY_rows, dtype=F64)
    W0m = np.asarray(W0m, dtype=F64)
    dC = dY[:, perm_p]
    dB = _blockwise(dC, np.asarray(G_p, dtype=F64), transpose=True)
    dA = _blockwise(dB @ W0m.T, np.asarray(G_r, dtype=F64), transpose=True)
    dX = np.empty_like(dA)
    dX[:, perm_r] = dA
    return dX
