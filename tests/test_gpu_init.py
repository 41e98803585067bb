"""GPU parity of the initialisation (Dual-SVID and Joint-ITQ) against the
fp64 oracle, through the C ABI.  Both sides start from the same fp32 factors
of a truncated SVD, computed on the host."""
import numpy as np
import pytest
import torch

from oracle import littlebit_init as ini
from oracle import littlebit_oracle as orc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lbm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from latent_binary_factorization_b200 import layers, littlebit
    return littlebit, layers


def _weight(d_out, d_in, seed, outliers=True):
    """A synthetic weight with a decaying spectrum and a few large entries
    (the heavy-tailed singular vectors the LittleBit-2 column describes)."""
    rng = np.random.default_rng(seed)
    r = min(d_out, d_in)
    A = rng.standard_normal((d_out, 64)) @ rng.standard_normal((64, d_in)) / 8.0
    W = A + 0.3 * rng.standard_normal((d_out, d_in))
    if outliers:
        W += (rng.random((d_out, d_in)) < 0.002) * rng.standard_normal((d_out, d_in)) * 20
    return W.astype(np.float32)


def _factors(W, s):
    Uf, Vf = ini.svd_factors(W.astype(np.float64), s)
    return np.ascontiguousarray(Uf, dtype=np.float32), np.ascontiguousarray(Vf, dtype=np.float32)


def _fp16_close(got, want, ulps=4):
    """fp16 values equal up to a few units in the last place (the GPU's fp32
    power iteration and the oracle's fp64 SVD round to fp16 separately)."""
    got = got.astype(np.float64)
    want = want.astype(np.float16).astype(np.float64)
    tol = ulps * np.abs(want) * 2.0 ** -10
    return np.all(np.abs(got - want) <= tol + 1e-30)


@pytest.mark.parametrize("d_out,d_in,s", [(256, 256, 16), (512, 768, 40), (1024, 512, 100), (4096, 4096, 188)])
def test_dual_svid_matches_the_oracle(lbm, d_out, d_in, s):
    lb, layers = lbm
    W = _weight(d_out, d_in, seed=s)
    Uf, Vf = _factors(W, s)
    p = lb.init_dual_svid(torch.from_numpy(Uf).cuda(), torch.from_numpy(Vf).cuda())
    torch.cuda.synchronize()
    ref = ini.dual_svid(Uf, Vf)
    # the signs: bit-exact (sign(0) = +1 on both sides)
    assert np.array_equal(p.U_bits.cpu().numpy(), orc.pack_signs(orc.factor_matrix("U", ref["U"]), "U"))
    assert np.array_equal(p.V_bits.cpu().numpy(), orc.pack_signs(orc.factor_matrix("V", ref["V"]), "V"))
    # the scales: the same numbers to a few fp16 ulps
    assert _fp16_close(p.h.cpu().numpy(), ref["h"])
    assert _fp16_close(p.g.cpu().numpy(), ref["g"])
    assert _fp16_close(p.l.cpu().numpy(), ref["l"])
    # and the layer built from them computes the oracle's W_hat x
    layer = lb.Layer(d_in, d_out, s, [p])
    x = torch.randn(3, d_in, device="cuda").half()
    y = lb.forward(layer, x)
    torch.cuda.synchronize()
    ref16 = {"U": ref["U"], "V": ref["V"], "h": ref["h"].astype(np.float16), "g": ref["g"].astype(np.float16),
             "l": ref["l"].astype(np.float16)}
    y_ref = orc.factored_forward(x.cpu().numpy(), [ref16])
    assert orc.rel_l2(y.float().cpu().numpy(), y_ref) <= 2e-3


def test_dual_svid_exact_on_a_rank1_sign_layer(lbm):
    """s = 1 on W = diag(h) u l v^T diag(g): the initialisation recovers W."""
    lb, _ = lbm
    rng = np.random.default_rng(3)
    d_out, d_in = 384, 512
    u, v = np.where(rng.random(d_out) < 0.5, -1, 1), np.where(rng.random(d_in) < 0.5, -1, 1)
    h, g = rng.uniform(0.5, 1.5, d_out), rng.uniform(0.5, 1.5, d_in)
    W = np.outer(h * u, g * v) * 0.3
    Uf, Vf = _factors(W, 1)
    p = lb.init_dual_svid(torch.from_numpy(Uf).cuda(), torch.from_numpy(Vf).cuda())
    torch.cuda.synchronize()
    U = lb.unpack_signs(p.U_bits, "U", d_out, 1).cpu().numpy()[:, 0]
    flip = U[0] * u[0]
    assert np.array_equal(U, flip * u)
    W_hat = ini.reconstruct({"U": U[:, None], "V": lb.unpack_signs(p.V_bits, "V", d_in, 1).cpu().numpy(),
                             "h": p.h.cpu().numpy(), "g": p.g.cpu().numpy(), "l": p.l.cpu().numpy()})
    assert np.linalg.norm(W_hat - W) / np.linalg.norm(W) < 2e-3


@pytest.mark.parametrize("d_out,d_in,s", [(256, 256, 8), (768, 512, 32), (2048, 1024, 64)])
def test_joint_itq_one_step_at_a_time_matches_the_oracle(lbm, d_out, d_in, s):
    """Every alternation of the GPU rotation equals the oracle's alternation
    from the same state: R_{k+1} = procrustes(X, sign(X R_k)), for 50 steps."""
    lb, _ = lbm
    W = _weight(d_out, d_in, seed=d_out + s)
    Uf, Vf = _factors(W, s)
    X0 = np.concatenate([Uf, Vf]).astype(np.float32)
    R = torch.eye(s, device="cuda")
    Xd = torch.from_numpy(X0).cuda()
    X64 = X0.astype(np.float64)
    row_norm = np.linalg.norm(X64, axis=1)
    strict = 0
    for k in range(50):
        R_prev = R.cpu().numpy().astype(np.float64)
        Xk = Xd.clone()
        R = lb.joint_itq(Xk, iters=1, R=R.clone())
        torch.cuda.synchronize()
        got = R.cpu().numpy().astype(np.float64)
        np.testing.assert_allclose(got.T @ got, np.eye(s), atol=1e-4)
        Z = X64 @ R_prev
        B = ini.sign_pm1(Z).astype(np.float64)
        want = ini.procrustes(X64, B)
        # the step maximises tr(B^T X R) over orthogonal R.  Where X R_prev is
        # within fp32 rounding of zero the GPU may take the other sign (both
        # correct); each such entry (i, j) can move the maximum by at most
        # 2 ||x_i||.  So the GPU's R must reach the oracle's maximum up to
        # that slack, and equal the oracle's R where there is no such entry.
        ties = np.argwhere(np.abs(Z) < 4e-6 * row_norm[:, None])
        f_want, f_got = np.trace(B.T @ X64 @ want), np.trace(B.T @ X64 @ got)
        slack = 2.0 * row_norm[ties[:, 0]].sum() + 1e-6 * abs(f_want)
        assert f_got >= f_want - slack, f"step {k}: {f_got} < {f_want} - {slack}"
        if len(ties) == 0:
            strict += 1
            assert np.abs(got - want).max() < 1e-4, f"step {k}: {np.abs(got - want).max():.2e}"
    if X64.size <= 50000:   # small problems see few or no ties: most steps compare R itself
        assert strict >= 10
    # the rotated factors come back in place: X R
    np.testing.assert_allclose(Xk.cpu().numpy(), X0 @ got, atol=1e-4 * np.abs(X0).max())


@pytest.mark.parametrize("d_out,d_in,s", [(1024, 1024, 64), (4096, 4096, 188)])
def test_joint_itq_fifty_iterations(lbm, d_out, d_in, s):
    """50 alternations from the identity in one call: R orthogonal, U'V'^T
    unchanged, and the quantisation loss below the unrotated one and within
    1 % of the oracle's run (the two may take different signs where X R is
    within rounding of zero, and then follow slightly different paths)."""
    lb, _ = lbm
    W = _weight(d_out, d_in, seed=s)
    Uf, Vf = _factors(W, s)
    X0 = np.concatenate([Uf, Vf]).astype(np.float32)
    Xd = torch.from_numpy(X0).cuda()
    R = lb.joint_itq(Xd, iters=50).cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(R.T @ R, np.eye(s), atol=1e-4)
    hist = []
    R_ref, _, _ = ini.joint_itq(Uf, Vf, 50, history=hist)
    loss_gpu = ini.itq_objective(X0, R)
    assert abs(loss_gpu - hist[-1]) <= 1e-2 * hist[-1]
    assert loss_gpu < hist[0]
    Xr = Xd.cpu().numpy().astype(np.float64)
    P = Xr[:d_out] @ Xr[d_out:].T
    np.testing.assert_allclose(P, Uf.astype(np.float64) @ Vf.T, atol=1e-3 * np.abs(Uf @ Vf.T).max())
