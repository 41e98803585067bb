"""Pins for the initialisation oracle (Dual-SVID and Joint-ITQ): hand-worked
values, exact-recovery cases, brute force on tiny inputs and the invariants
the method relies on."""
import json
import os

import numpy as np
import pytest
from scipy.linalg import hadamard
from scipy.optimize import minimize

from oracle import littlebit_init as ini
from oracle import littlebit_oracle as orc


# ---------------------------------------------------------------- Dual-SVID


def test_dual_svid_hand_worked_2x2(golden_dir):
    with open(os.path.join(golden_dir, "dual_svid_2x2.json")) as f:
        gold = json.load(f)
    W = np.array(gold["W"])
    (p1,) = ini.init_layer(W, 1)
    np.testing.assert_allclose(ini.reconstruct(p1), gold["rank1"]["W_hat"], atol=1e-12)
    np.testing.assert_allclose(p1["h"], gold["rank1"]["h"], atol=1e-12)
    np.testing.assert_allclose(p1["g"], gold["rank1"]["g"], atol=1e-12)
    np.testing.assert_allclose(p1["l"], gold["rank1"]["l"], atol=1e-12)
    (p2,) = ini.init_layer(W, 2)
    np.testing.assert_allclose(ini.reconstruct(p2), gold["rank2"]["W_hat"], atol=1e-12)
    np.testing.assert_allclose(np.sort(p2["l"]), gold["rank2"]["l_sorted"], atol=1e-12)
    np.testing.assert_allclose(p2["h"], gold["rank2"]["h"], atol=1e-12)
    a, b = ini.init_layer(W, 1, residual=True)
    np.testing.assert_allclose(ini.reconstruct(a), gold["rank1_residual"]["W_hat_path1"], atol=1e-12)
    np.testing.assert_allclose(ini.reconstruct(b), gold["rank1_residual"]["W_hat_path2"], atol=1e-12)


@pytest.mark.parametrize("d_out,d_in,seed", [(7, 5, 0), (64, 96, 1), (200, 40, 2)])
def test_dual_svid_recovers_a_rank1_factored_layer(d_out, d_in, seed):
    """s = 1: W = diag(h) u l v^T diag(g) with positive scales is recovered
    exactly, and its signs up to the joint flip of u and v (the latent gauge)."""
    rng = np.random.default_rng(seed)
    u = np.where(rng.random(d_out) < 0.5, -1, 1)
    v = np.where(rng.random(d_in) < 0.5, -1, 1)
    h, g, l = rng.uniform(0.5, 1.5, d_out), rng.uniform(0.5, 1.5, d_in), 0.7
    W = np.outer(h * u * l, g * v)
    (p,) = ini.init_layer(W, 1)
    np.testing.assert_allclose(ini.reconstruct(p), W, rtol=0, atol=1e-12 * np.abs(W).max())
    flip = p["U"][0, 0] * u[0]
    assert np.array_equal(p["U"][:, 0], flip * u) and np.array_equal(p["V"][:, 0], flip * v)
    # the row and column scales are h and g up to the gauge (normalised to mean 1)
    np.testing.assert_allclose(p["h"], h / h.mean(), rtol=1e-12)
    np.testing.assert_allclose(p["g"], g / g.mean(), rtol=1e-12)


@pytest.mark.parametrize("n,cols", [(8, [1, 3, 6]), (16, [0, 2, 5, 9, 14]), (32, [4, 7, 11, 20, 31, 1])])
def test_dual_svid_recovers_orthogonal_sign_factors(n, cols):
    """Sign factors with orthogonal columns (Hadamard columns) and distinct
    latent scales: the truncated SVD is the factorisation itself, so
    Dual-SVID returns W exactly."""
    H = hadamard(n).astype(np.float64)
    l = np.linspace(3.0, 1.0, len(cols))
    W = (H[:, cols] * l[None, :]) @ H[:, cols].T
    (p,) = ini.init_layer(W, len(cols))
    np.testing.assert_allclose(ini.reconstruct(p), W, atol=1e-10)
    assert set(np.unique(p["U"])) <= {-1, 1}


def _rank1_brute(A, starts=20, seed=0):
    """min over a, b of ||A - a b^T||_F by a general-purpose optimiser from
    several random starts (no SVD involved)."""
    n, m = A.shape
    rng = np.random.default_rng(seed)
    f = lambda z: np.sum((A - np.outer(z[:n], z[n:])) ** 2)
    best = np.inf
    for _ in range(starts):
        r = minimize(f, rng.uniform(0.1, 1.0, n + m), method="BFGS", options={"gtol": 1e-12, "maxiter": 10000})
        best = min(best, r.fun)
    return best


@pytest.mark.parametrize("shape,seed", [((3, 2), 0), ((4, 3), 1), ((5, 5), 2), ((2, 6), 3)])
def test_rank1_fit_is_the_least_squares_optimum(shape, seed):
    A = np.abs(np.random.default_rng(seed).standard_normal(shape))
    a, b = ini.rank1_nonneg(A)
    assert np.all(a >= 0) and np.all(b >= 0)
    err = np.sum((A - np.outer(a, b)) ** 2)
    assert err == pytest.approx(_rank1_brute(A), rel=1e-7, abs=1e-10)


def test_rank1_fit_of_an_outer_product_is_exact():
    a0, b0 = np.array([0.5, 2.0, 1.0, 3.0]), np.array([1.5, 0.25, 4.0])
    a, b = ini.rank1_nonneg(np.outer(a0, b0))
    np.testing.assert_allclose(np.outer(a, b), np.outer(a0, b0), rtol=1e-12)


def test_dual_svid_signs_are_the_factor_signs_with_zero_positive():
    Uf = np.array([[1.0, -2.0], [0.0, 3.0], [-0.0, -1.0]])
    Vf = np.array([[-1.0, 2.0], [4.0, 0.0]])
    p = ini.dual_svid(Uf, Vf)
    assert p["U"].tolist() == [[1, -1], [1, 1], [1, -1]]
    assert p["V"].tolist() == [[-1, 1], [1, 1]]


def test_residual_path_takes_the_remainder():
    """The second path is Dual-SVID of W - W_hat_1 (same rank): on a W that is
    two rank-1 sign layers of very different size, the two paths recover it."""
    rng = np.random.default_rng(5)
    d_out, d_in = 48, 40
    parts = []
    for scale in (10.0, 1.0):
        u = np.where(rng.random(d_out) < 0.5, -1, 1) * rng.uniform(0.5, 1.5, d_out)
        v = np.where(rng.random(d_in) < 0.5, -1, 1) * rng.uniform(0.5, 1.5, d_in)
        parts.append(scale * np.outer(u, v))
    W = parts[0] + parts[1]
    a, b = ini.init_layer(W, 1, residual=True)
    err1 = np.linalg.norm(W - ini.reconstruct(a))
    err2 = np.linalg.norm(W - ini.reconstruct(a) - ini.reconstruct(b))
    assert err2 < 0.5 * err1


def test_initialised_layer_runs_through_the_forward_oracle():
    """The paths have the forward oracle's layout: its output equals W_hat x."""
    rng = np.random.default_rng(6)
    W = rng.standard_normal((64, 32))
    paths = ini.init_layer(W, 8, residual=True, itq_iters=5)
    x = rng.standard_normal((3, 32))
    W_hat = sum(ini.reconstruct(p) for p in paths)
    np.testing.assert_allclose(orc.factored_forward(x, paths), x @ W_hat.T, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- Joint-ITQ


def _rot(theta):
    c, s = np.cos(theta), np.sin(theta)
    return np.array([[c, -s], [s, c]])


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_procrustes_step_beats_every_2x2_orthogonal_matrix(seed):
    """s = 2: the Procrustes rotation maximises tr(B^T X R) over all rotations
    and reflections, scanned on a fine grid (no SVD involved)."""
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((30, 2))
    B = ini.sign_pm1(X @ _rot(rng.uniform(0, 6.3)))
    R = ini.procrustes(X, B)
    best = -np.inf
    flip = np.diag([1.0, -1.0])
    for th in np.linspace(0, 2 * np.pi, 20001):
        for Q in (_rot(th), _rot(th) @ flip):
            best = max(best, np.trace(B.T @ X @ Q))
    got = np.trace(B.T @ X @ R)
    assert got >= best - 1e-6 and got <= best + 1e-3 * abs(best)


@pytest.mark.parametrize("n,s,seed", [(60, 4, 0), (300, 16, 1), (500, 40, 2)])
def test_itq_keeps_r_orthogonal_lowers_the_loss_and_keeps_the_product(n, s, seed):
    rng = np.random.default_rng(seed)
    W = rng.standard_normal((n, n // 2)) * (rng.random((n, n // 2)) < 0.1) * 20 + rng.standard_normal((n, n // 2))
    Uf, Vf = ini.svd_factors(W, s)
    hist = []
    R, Ur, Vr = ini.joint_itq(Uf, Vf, 50, history=hist)
    np.testing.assert_allclose(R.T @ R, np.eye(s), atol=1e-10)
    # each alternation minimises over one variable: the loss never rises
    assert all(b <= a * (1 + 1e-12) + 1e-12 for a, b in zip(hist, hist[1:]))
    assert hist[-1] < hist[0]
    assert orc.rotation_residual(Uf, Vf, R) < 1e-12
    np.testing.assert_allclose(Ur @ Vr.T, Uf @ Vf.T, atol=1e-9 * np.abs(Uf @ Vf.T).max())


def test_itq_fixed_point_on_sign_aligned_factors():
    """Factors that already sit on the binary hypercube's directions (X = c B0
    with B0 of full column rank) are a fixed point: R stays the identity."""
    rng = np.random.default_rng(7)
    B0 = np.where(rng.random((40, 6)) < 0.5, -1.0, 1.0)
    X = 0.3 * B0
    R, _, _ = ini.joint_itq(X[:25], X[25:], 10)
    np.testing.assert_allclose(R, np.eye(6), atol=1e-12)


def test_itq_default_is_fifty_iterations():
    import inspect
    assert inspect.signature(ini.joint_itq).parameters["iters"].default == 50


def test_itq_ends_on_a_fixed_point_of_the_alternation():
    """On a small problem the 50 alternations settle: the final R is the
    Procrustes rotation of the signs it gives itself."""
    rng = np.random.default_rng(8)
    W = rng.standard_normal((40, 30))
    Uf, Vf = ini.svd_factors(W, 4)
    R, _, _ = ini.joint_itq(Uf, Vf, 50)
    X = np.concatenate([Uf, Vf])
    np.testing.assert_allclose(ini.procrustes(X, ini.sign_pm1(X @ R)), R, atol=1e-10)


@pytest.mark.parametrize("shape,s,seed", [((4, 3), 1, 0), ((4, 3), 2, 1), ((5, 4), 2, 2)])
def test_svd_factors_are_balanced_and_optimal(shape, s, seed):
    """U' V'^T is the best rank-s approximation of W (checked against a
    general-purpose optimiser over all rank-s products), U' and V' have
    orthogonal columns, and each singular value is split evenly: column j of
    U' and of V' have the same norm."""
    rng = np.random.default_rng(seed)
    W = rng.standard_normal(shape)
    Uf, Vf = ini.svd_factors(W, s)
    G = Uf.T @ Uf
    np.testing.assert_allclose(G, np.diag(np.diag(G)), atol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(Uf, axis=0), np.linalg.norm(Vf, axis=0), rtol=1e-12)
    err = np.sum((W - Uf @ Vf.T) ** 2)
    m, n = shape
    f = lambda z: np.sum((W - z[:m * s].reshape(m, s) @ z[m * s:].reshape(n, s).T) ** 2)
    best = min(minimize(f, np.random.default_rng(k).standard_normal((m + n) * s), method="BFGS",
                        options={"gtol": 1e-12, "maxiter": 20000}).fun for k in range(10))
    assert err == pytest.approx(best, rel=1e-6, abs=1e-9)
