"""fp64 CPU oracle for the LittleBit initialisation: Dual-SVID and Joint-ITQ.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU legs may import or run anything in this directory.  The
CUDA library never calls it, and it imports nothing from the CUDA package.

What it computes, and where each step is defined
------------------------------------------------
* ``svd_factors``: the truncated SVD that both initialisations start from.
  Samsung LittleBit article (aifrontier.co.jp, "samsung-littlebit-sub-1-bit"),
  section 2, the Dual-SVID bullet: the factors come from a truncated SVD of W;
  LittleBit-2 column (physicalainews.jp, "littlebit2-sub-1bit-llm-quantization-2026"),
  chapter 2: W is split by SVD into low-rank factors U, V.
* ``dual_svid``: the same bullet: the signs of the factors become the binary
  U+-, V+-, and their magnitudes are estimated by rank-1 approximations, which
  give the scales h, g and l.
* ``joint_itq``: LittleBit-2 column, chapter 2, "solution 1": an orthogonal R
  is found by iterative rotation (50 iterations by default) on the stacked
  factors [U; V] and applied to both, U <- U R and V <- V R (V here is d_in x s,
  the transpose of the page's s x d_in V), before the signs are taken; the
  product U V^T is unchanged by R.
* ``residual_init``: article section 2, residual-compensation bullet: the
  second path takes what the first path's approximation leaves over.

Readings where the pages are silent or leave a choice open:
* The singular values are split evenly between the factors:
  U' = U_s sqrt(S_s), V' = V_s sqrt(S_s).
* sign(0) = +1, as for the packed factors.
* "rank-1 approximation of the magnitudes": the best rank-1 fit a b^T (least
  squares, i.e. the top singular pair) of |U'| (d_out x s) and of |V'|
  (d_in x s); a and b are taken non-negative (Perron-Frobenius).  The split of
  a b^T between a row scale and the latent scale is a gauge; this oracle
  normalises h = a_U / mean(a_U) and g = a_V / mean(a_V) (mean 1, well inside
  fp16's range) and puts the rest into l = (mean(a_U) b_U) * (mean(a_V) b_V),
  so that h_o l_j g_i = a_U[o] b_U[j] a_V[i] b_V[j].
* The iterative rotation is classic iterative quantisation: from R = I,
  alternate B = sign(X R) and R = the orthogonal Procrustes solution
  argmax_R tr(B^T X R), i.e. the polar factor P Q^T of X^T B = P S Q^T.
* The residual path is initialised by the same Dual-SVID on W - W_hat_1 with
  the same rank s.
"""
from __future__ import annotations

import numpy as np


def _f64(a) -> np.ndarray:
    return np.asarray(a).astype(np.float64)


def sign_pm1(A) -> np.ndarray:
    """+-1 signs with sign(0) = +1 (int8)."""
    return np.where(_f64(A) < 0, -1, 1).astype(np.int8)


# ---------------------------------------------------------------------------
# truncated SVD (library routine as a step)
# ---------------------------------------------------------------------------


def svd_factors(W, s: int):
    """U' (d_out x s), V' (d_in x s) with U' V'^T the best rank-s approximation
    of W, singular values split evenly."""
    U, S, Vt = np.linalg.svd(_f64(W), full_matrices=False)
    r = np.sqrt(S[:s])
    return U[:, :s] * r[None, :], Vt[:s].T * r[None, :]


# ---------------------------------------------------------------------------
# Dual-SVID (article section 2)
# ---------------------------------------------------------------------------


def rank1_nonneg(A):
    """Best rank-1 approximation a b^T of a non-negative matrix A (n x m) in
    the Frobenius norm, with a, b >= 0: the top singular pair, whose vectors a
    non-negative matrix allows to be non-negative.  Returns (a, b)."""
    A = _f64(A)
    U, S, Vt = np.linalg.svd(A, full_matrices=False)
    u, v = U[:, 0], Vt[0]
    if u.sum() < 0:          # the pair is defined up to a joint sign
        u, v = -u, -v
    return np.abs(u) * np.sqrt(S[0]), np.abs(v) * np.sqrt(S[0])


def dual_svid(Uf, Vf):
    """One path from real factors U' (d_out x s), V' (d_in x s): the signs and
    the rank-1 magnitude scales.  Returns a path dict (U, V int8 +-1; h, g, l
    fp64) in the layout of the forward oracle."""
    Uf, Vf = _f64(Uf), _f64(Vf)
    au, bu = rank1_nonneg(np.abs(Uf))
    av, bv = rank1_nonneg(np.abs(Vf))
    mu, mv = au.mean(), av.mean()
    return {"U": sign_pm1(Uf), "V": sign_pm1(Vf), "h": au / mu, "g": av / mv, "l": (bu * mu) * (bv * mv)}


def reconstruct(path) -> np.ndarray:
    """W_hat = diag(h) U diag(l) V^T diag(g) of one path (fp64)."""
    U, V = _f64(path["U"]), _f64(path["V"])
    return (_f64(path["h"])[:, None] * U * _f64(path["l"])[None, :]) @ (V * _f64(path["g"])[:, None]).T


# ---------------------------------------------------------------------------
# Joint-ITQ (LittleBit-2 column, chapter 2, solution 1)
# ---------------------------------------------------------------------------


def procrustes(X, B) -> np.ndarray:
    """argmax over orthogonal R of tr(B^T X R): the polar factor of X^T B."""
    P, _, Qt = np.linalg.svd(_f64(X).T @ _f64(B))
    return P @ Qt


def itq_objective(X, R) -> float:
    """|| sign(X R) - X R ||_F^2, the quantisation loss the rotation lowers."""
    Z = _f64(X) @ _f64(R)
    return float(np.sum((sign_pm1(Z) - Z) ** 2))


def joint_itq(Uf, Vf, iters: int = 50, R0=None, history: list | None = None):
    """Rotation R of the stacked factors X = [U'; V'] ((d_out + d_in) x s) by
    `iters` alternations of B = sign(X R) and R = procrustes(X, B), from R0
    (identity by default).  Returns (R, U' R, V' R).  `history`, if given,
    receives the objective before each iteration and after the last."""
    Uf, Vf = _f64(Uf), _f64(Vf)
    X = np.concatenate([Uf, Vf], axis=0)
    s = X.shape[1]
    R = np.eye(s) if R0 is None else _f64(R0)
    for _ in range(iters):
        if history is not None:
            history.append(itq_objective(X, R))
        B = sign_pm1(X @ R)
        R = procrustes(X, B)
    if history is not None:
        history.append(itq_objective(X, R))
    return R, Uf @ R, Vf @ R


# ---------------------------------------------------------------------------
# the whole initialisation of a layer
# ---------------------------------------------------------------------------


def init_layer(W, s: int, residual: bool = False, itq_iters: int = 0):
    """Paths of a LittleBit layer initialised from a dense W (d_out x d_in):
    truncated SVD, optionally Joint-ITQ, then Dual-SVID; with residual
    compensation a second path from what the first leaves over."""
    W = _f64(W)
    paths = []
    target = W
    for _ in range(2 if residual else 1):
        Uf, Vf = svd_factors(target, s)
        if itq_iters:
            _, Uf, Vf = joint_itq(Uf, Vf, itq_iters)
        p = dual_svid(Uf, Vf)
        paths.append(p)
        target = target - reconstruct(p)
    return paths
