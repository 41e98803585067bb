"""Pins for the fp64 oracle: each check fixes the oracle to something other
than itself (hand-worked values, closed forms, brute force, invariants)."""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import littlebit_oracle as orc
from latent_binary_factorization_b200 import synth


def _rows(path):
    with open(path) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


# ---------------------------------------------------------------- eff_bits


def test_eff_bits_hand_worked(golden_dir):
    rows = _rows(os.path.join(golden_dir, "eff_bits.txt"))
    assert len(rows) == 8
    for a, b, s, res, num, den in rows:
        got = orc.eff_bits_exact(int(a), int(b), int(s), bool(int(res)))
        assert got == Fraction(int(num), int(den)), (a, b, s, res)


def test_eff_bits_properties():
    for a, b, s in [(4096, 4096, 86), (4096, 11008, 133), (8192, 28672, 302), (512, 512, 32)]:
        single = orc.eff_bits_exact(a, b, s, False)
        # residual doubles every term of the single-path count
        assert orc.eff_bits_exact(a, b, s, True) == 2 * single
        # a and b enter symmetrically
        assert orc.eff_bits_exact(b, a, s, False) == single
        # one more rank adds (a+b+16) bits per path
        assert orc.eff_bits_exact(a, b, s + 1, False) - single == Fraction(a + b + 16, a * b)
    # 512x512, s=32 is exactly 0.189453125 bits per weight
    assert orc.eff_bits(512, 512, 32, False) == 0.189453125


def test_rank_solver_targets(golden_dir):
    for a, b, bpw, res, s in _rows(os.path.join(golden_dir, "rank_targets.txt")):
        got = orc.solve_rank(int(a), int(b), bpw, bool(int(res)))
        assert got == int(s), (a, b, bpw, res, got)
    # the quoted "about 135" is over the 0.1 budget
    assert orc.eff_bits(4096, 11008, 135, True) > 0.1


# ---------------------------------------------------------------- packing


def test_pack_positions_hand_worked(golden_dir):
    rows = _rows(os.path.join(golden_dir, "pack_positions.txt"))
    assert len(rows) == 8
    for role, R, K, row, k, byte, bit in rows:
        R, K, row, k, byte, bit = map(int, (R, K, row, k, byte, bit))
        F = np.ones((R, K), np.float32)
        F[row, k] = -1.0
        buf = orc.pack_signs(F, role)
        assert buf.size == orc.packed_nbytes(role, R, K)
        nz = np.nonzero(buf)[0]
        assert list(nz) == [byte], (role, row, k, nz)
        assert buf[byte] == (1 << bit), (role, row, k, buf[byte])


@pytest.mark.parametrize("role,R,K", [("V", 16, 256), ("V", 37, 512), ("V", 1, 256),
                                      ("U", 128, 32), ("U", 256, 45), ("U", 384, 1), ("U", 128, 100)])
def test_pack_roundtrip_and_padding(role, R, K):
    F = synth.real_factor(R, K, seed=3, zeros=0.05)
    buf = orc.pack_signs(F, role)
    back = orc.unpack_signs(buf, role, R, K)
    want = np.where(F < 0, -1, 1)            # sign(+0) = sign(-0) = +1
    assert np.array_equal(back, want)
    assert orc.padding_is_zero(buf, role, R, K)
    # one bit per negative entry, nothing else
    popcount = int(np.unpackbits(buf).sum())
    assert popcount == int((F < 0).sum())


def test_pack_of_pm1_is_identity_on_signs():
    rng = np.random.default_rng(5)
    S = (1 - 2 * rng.integers(0, 2, size=(48, 512))).astype(np.int8)
    assert np.array_equal(orc.unpack_signs(orc.pack_signs(S, "V"), "V", 48, 512), S)


def test_pack_layout_is_a_bijection():
    # every in-range element maps to a distinct bit and every bit of a full
    # tile is used exactly once
    for role in ("V", "U"):
        tr, tk = orc.TILE[role]
        row, k = orc._tile_coords(role, 1, 1)
        flat = (row * tk + k).reshape(-1)
        assert np.array_equal(np.sort(flat), np.arange(tr * tk))


# ---------------------------------------------------------------- forward


def test_forward_hand_worked(golden_dir):
    with open(os.path.join(golden_dir, "forward_worked_example.json")) as f:
        ex = json.load(f)
    x = np.array(ex["x"])
    paths = [{k: np.array(v) for k, v in p.items()} for p in ex["paths"]]
    np.testing.assert_array_equal(orc.factored_forward(x, paths[:1]), np.array(ex["y_single_path"]))
    np.testing.assert_array_equal(orc.factored_forward(x, paths), np.array(ex["y_residual"]))


def test_forward_brute_force_loops():
    """W[o,i] = sum_j h_o U_oj l_j V_ij g_i by explicit Python loops, then W x."""
    d_in, d_out, s, B = 5, 3, 2, 2
    paths = synth.layer(d_in, d_out, s, residual=True, seed=11)
    x = synth.activations(B, d_in, seed=11).astype(np.float64)
    y = [[0.0] * d_out for _ in range(B)]
    for p in paths:
        for o in range(d_out):
            for i in range(d_in):
                w = 0.0
                for j in range(s):
                    w += float(p["h"][o]) * float(p["U"][o, j]) * float(p["l"][j]) * float(p["V"][i, j]) * float(p["g"][i])
                for b in range(B):
                    y[b][o] += w * float(x[b, i])
    np.testing.assert_allclose(orc.factored_forward(x, paths), np.array(y), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(orc.dense_forward(x, paths), np.array(y), rtol=1e-13, atol=1e-15)


def test_forward_matches_dense_reconstruction():
    d_in, d_out, s = 96, 40, 7
    paths = synth.layer(d_in, d_out, s, residual=True, seed=2)
    x = synth.activations(3, d_in, seed=2)
    y = orc.factored_forward(x, paths)
    yd = orc.dense_forward(x, paths)
    assert orc.rel_l2(y, yd) < 1e-12


def test_forward_all_plus_closed_form():
    d_in, d_out, s = 64, 24, 9
    p = synth.layer(d_in, d_out, s, residual=False, seed=4)[0]
    p["U"][:] = 1
    p["V"][:] = 1
    x = synth.activations(2, d_in, seed=4).astype(np.float64)
    g, l, h = (p[k].astype(np.float64) for k in "glh")
    want = h[None, :] * l.sum() * (x @ g)[:, None]
    np.testing.assert_allclose(orc.factored_forward(x, [p]), want, rtol=1e-13)


def test_forward_rank_one_closed_form():
    d_in, d_out = 40, 30
    p = synth.layer(d_in, d_out, 1, residual=False, seed=6)[0]
    x = synth.activations(1, d_in, seed=6).astype(np.float64)[0]
    u, v = p["U"][:, 0].astype(np.float64), p["V"][:, 0].astype(np.float64)
    g, l, h = (p[k].astype(np.float64) for k in "glh")
    want = h * u * l[0] * np.dot(v, g * x)
    np.testing.assert_allclose(orc.factored_forward(x[None, :], [p])[0], want, rtol=1e-13)


def test_forward_basis_vector_gives_column():
    d_in, d_out, s = 20, 12, 5
    paths = synth.layer(d_in, d_out, s, residual=True, seed=8)
    W = sum(orc.dense_weight(p) for p in paths)
    for i in (0, 7, 19):
        e = np.zeros((1, d_in))
        e[0, i] = 1.0
        np.testing.assert_allclose(orc.factored_forward(e, paths)[0], W[:, i], rtol=1e-13, atol=1e-16)


def test_forward_linear_in_x():
    d_in, d_out, s = 64, 32, 6
    paths = synth.layer(d_in, d_out, s, residual=True, seed=9)
    x1 = synth.activations(1, d_in, seed=9).astype(np.float64)
    x2 = synth.activations(1, d_in, seed=10).astype(np.float64)
    lhs = orc.factored_forward(2.5 * x1 - x2, paths)
    rhs = 2.5 * orc.factored_forward(x1, paths) - orc.factored_forward(x2, paths)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-14)


def test_residual_is_sum_of_paths():
    d_in, d_out, s = 64, 48, 5
    paths = synth.layer(d_in, d_out, s, residual=True, seed=12)
    x = synth.activations(2, d_in, seed=12)
    both = orc.factored_forward(x, paths)
    np.testing.assert_allclose(both, orc.factored_forward(x, paths[:1]) + orc.factored_forward(x, paths[1:]), rtol=1e-14)


def test_latent_gauge_invariances():
    """Flipping latent column j in both U and V, or permuting latent columns
    together with l, leaves y unchanged; flipping only one factor does not."""
    d_in, d_out, s = 64, 40, 6
    p = synth.layer(d_in, d_out, s, residual=False, seed=13)[0]
    x = synth.activations(2, d_in, seed=13)
    y = orc.factored_forward(x, [p])
    q = {k: v.copy() for k, v in p.items()}
    q["U"][:, 2] *= -1
    q["V"][:, 2] *= -1
    np.testing.assert_allclose(orc.factored_forward(x, [q]), y, rtol=1e-13)
    perm = np.array([3, 0, 5, 1, 4, 2])
    r = {"U": p["U"][:, perm], "V": p["V"][:, perm], "l": p["l"][perm], "h": p["h"], "g": p["g"]}
    np.testing.assert_allclose(orc.factored_forward(x, [r]), y, rtol=1e-13)
    q["V"][:, 2] *= -1
    assert orc.rel_l2(orc.factored_forward(x, [q]), y) > 1e-3


def test_scale_roles_are_not_interchangeable():
    """h scales outputs, g scales inputs: with d_in != d_out a swap is caught."""
    d_in, d_out, s = 32, 16, 4
    p = synth.layer(d_in, d_out, s, residual=False, seed=14)[0]
    x = synth.activations(1, d_in, seed=14).astype(np.float64)
    y = orc.factored_forward(x, [p])
    # doubling h[o] doubles exactly output o
    q = dict(p)
    q["h"] = p["h"].astype(np.float64).copy()
    q["h"][5] *= 2
    y2 = orc.factored_forward(x, [q])
    np.testing.assert_allclose(np.delete(y2, 5, axis=1), np.delete(y, 5, axis=1), rtol=1e-15)
    np.testing.assert_allclose(y2[0, 5], 2 * y[0, 5], rtol=1e-15)
    # zeroing g[i] removes exactly input i's contribution
    q = dict(p)
    q["g"] = p["g"].astype(np.float64).copy()
    q["g"][3] = 0.0
    x0 = x.copy()
    x0[0, 3] = 0.0
    np.testing.assert_allclose(orc.factored_forward(x, [q]), orc.factored_forward(x0, [p]), rtol=1e-13)


def test_sampled_rows_match_full():
    paths = synth.layer(128, 256, 10, residual=True, seed=15)
    x = synth.activations(3, 128, seed=15)
    rows = np.array([0, 17, 255, 128])
    np.testing.assert_array_equal(orc.factored_forward(x, paths, rows=rows), orc.factored_forward(x, paths)[:, rows])


# ---------------------------------------------------------------- rotation gauge


def test_rotation_invariance_and_sign_change():
    rng = np.random.default_rng(21)
    U = rng.standard_normal((64, 8))
    V = rng.standard_normal((48, 8))
    R, _ = np.linalg.qr(rng.standard_normal((8, 8)))
    assert np.allclose(R.T @ R, np.eye(8), atol=1e-13)
    assert orc.rotation_residual(U, V, R) < 1e-12
    # the product is unchanged but the signs that binarisation would keep are not
    assert np.mean(np.sign(U @ R) != np.sign(U)) > 0.2
    # a non-orthogonal R does change the product
    assert orc.rotation_residual(U, V, R + 0.1 * np.eye(8)) > 1e-3


def test_error_measures():
    y = np.array([[3.0, -4.0]])
    assert orc.rel_l2(y, y) == 0.0
    assert orc.rel_l2(np.array([[3.0, -4.0 + 0.5]]), y) == pytest.approx(0.1)
    assert orc.max_abs_ratio(np.array([[3.0, -3.0]]), y) == pytest.approx(0.25)
