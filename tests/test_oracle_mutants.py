"""Mutation check of the oracle's pins.

Each case plants one plausible mistake in the oracle (on the CPU, by
replacing one of its functions for the duration of the case): a dropped
term, a wrong sign, a wrong index or bit position, a transposed or
mis-ordered operand, a swapped scale.  It then runs every pin in
``test_oracle.py`` against the mutated oracle.  At least one pin must fail,
otherwise that mistake could sit in the oracle unnoticed and the GPU parity
tests would inherit it.
"""
import importlib.util
import inspect
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import littlebit_oracle as orc

HERE = os.path.dirname(os.path.abspath(__file__))
_spec = importlib.util.spec_from_file_location("oracle_pins", os.path.join(HERE, "test_oracle.py"))
pins = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(pins)


def _pin_calls(golden_dir):
    """(name, zero-argument callable) for every pin and parameter set."""
    calls = []
    for name, fn in sorted(vars(pins).items()):
        if not (name.startswith("test_") and callable(fn)):
            continue
        params = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if params:
            argnames, argvalues = params[0].args[0], params[0].args[1]
            names = [a.strip() for a in argnames.split(",")]
            for vals in argvalues:
                kw = dict(zip(names, vals if len(names) > 1 else (vals,)))
                calls.append((f"{name}{tuple(kw.values())}", lambda fn=fn, kw=kw: fn(**kw)))
        elif "golden_dir" in inspect.signature(fn).parameters:
            calls.append((name, lambda fn=fn: fn(golden_dir)))
        else:
            calls.append((name, fn))
    return calls


def _failing_pins(golden_dir):
    failed = []
    for name, call in _pin_calls(golden_dir):
        try:
            call()
        except Exception:   # an assertion, or the mutant breaking a shape
            failed.append(name)
    return failed


# ----------------------------------------------------------------- mutants

def _f64(a):
    return np.asarray(a).astype(np.float64)


def _eff(num):
    def eff_bits_exact(a, b, s, residual):
        return Fraction(num(a, b, s, residual), a * b)
    return eff_bits_exact


def _coords(swap_r=False, bit_order_4q=False, u_q_stride=16):
    """Tile coordinates with one planted layout mistake."""
    def _tile_coords(role, n_rb, n_kt):
        rb = np.arange(n_rb).reshape(-1, 1, 1, 1, 1)
        kt = np.arange(n_kt).reshape(1, -1, 1, 1, 1)
        lane = np.arange(32).reshape(1, 1, -1, 1, 1)
        r = np.arange(4).reshape(1, 1, 1, -1, 1)
        n = np.arange(32).reshape(1, 1, 1, 1, -1)
        g, c = lane // 4, lane % 4
        m, q = (n % 4, n // 4) if bit_order_4q else (n // 8, n % 8)
        r_row, r_k = (r // 2, r % 2) if swap_r else (r % 2, r // 2)
        if role == "V":
            row = 16 * rb + g + 8 * r_row
            k = 256 * kt + 32 * q + 16 * r_k + 4 * c + m
        else:
            row = 128 * rb + u_q_stride * q + g + 8 * r_row
            k = 32 * kt + 16 * r_k + 4 * c + m
        shape = (n_rb, n_kt, 32, 4, 32)
        return np.broadcast_to(row, shape), np.broadcast_to(k, shape)
    return _tile_coords


def _pack_zero_negative(F, role):
    """pack_signs with sign(0) read as negative (bit = [v <= 0])."""
    F = np.asarray(F)
    R, K = F.shape
    rp, kp = orc.padded_dims(role, R, K)
    tr, tk = orc.TILE[role]
    row, k = orc._tile_coords(role, rp // tr, kp // tk)
    inside = (row < R) & (k < K)
    vals = F[np.minimum(row, R - 1), np.minimum(k, K - 1)]
    neg = inside & (vals <= 0)
    weights = np.uint64(1) << np.arange(32, dtype=np.uint64)
    words = (neg.astype(np.uint64) * weights).sum(axis=-1).astype(np.uint32)
    return words.astype("<u4").reshape(-1).view(np.uint8).copy()


def _forward(drop_l=False, swap_hg=False, subtract_residual=False, last_path_only=False, negate_v=False,
             roll_l=False, u_wrong_order=False, v_wrong_order=False, h_all_rows=False, drop_g=False):
    """factored_forward with one planted mistake."""
    def factored_forward(x, paths, rows=None):
        x = _f64(x)
        y = None
        for p in paths:
            g, h = (p["h"], p["g"]) if swap_hg else (p["g"], p["h"])
            V = _f64(p["V"])
            if v_wrong_order:   # stored d_in x s read as if it were s x d_in
                V = V.reshape(-1).reshape(V.shape[1], V.shape[0]).T
            if negate_v:
                V = -V
            u = x if drop_g else x * _f64(g)[None, :]
            t = u @ V
            l = _f64(p["l"])
            if roll_l:
                l = np.roll(l, 1)
            tl = t if drop_l else t * l[None, :]
            U = _f64(p["U"])
            if u_wrong_order:
                U = U.reshape(-1).reshape(U.shape[1], U.shape[0]).T
            hh = _f64(h)
            if rows is not None:
                U = U[rows]
                if not h_all_rows:
                    hh = hh[rows]
            yp = (tl @ U.T) * hh[None, :]
            if y is None or last_path_only:
                y = yp
            else:
                y = y - yp if subtract_residual else y + yp
        return y
    return factored_forward


def _dense_without_g(path):
    U, V = _f64(path["U"]), _f64(path["V"])
    h, l = _f64(path["h"]), _f64(path["l"])
    return (h[:, None] * (U * l[None, :])) @ V.T


MUTANTS = {
    # storage cost
    "eff: drop the +16 per rank": {"eff_bits_exact": _eff(
        lambda a, b, s, r: (2 if r else 1) * (s * (a + b) + 16 * (a + b)))},
    "eff: residual keeps 16(a+b)": {"eff_bits_exact": _eff(
        lambda a, b, s, r: (2 * s * (a + b + 16) + 16 * (a + b)) if r else (s * (a + b + 16) + 16 * (a + b)))},
    "eff: drop the 16(a+b) scale term": {"eff_bits_exact": _eff(
        lambda a, b, s, r: (2 if r else 1) * s * (a + b + 16))},
    "eff: 16 per rank counted once per side": {"eff_bits_exact": _eff(
        lambda a, b, s, r: (2 if r else 1) * (s * (a + b + 32) + 16 * (a + b)))},
    # packed layout
    "pack: r%2 and r//2 swapped": {"_tile_coords": _coords(swap_r=True)},
    "pack: bit n = 4q + m": {"_tile_coords": _coords(bit_order_4q=True)},
    "pack: U plane stride 8 rows": {"_tile_coords": _coords(u_q_stride=8)},
    "pack: sign(0) negative": {"pack_signs": _pack_zero_negative},
    # forward
    "fwd: latent scale dropped": {"factored_forward": _forward(drop_l=True)},
    "fwd: h and g swapped": {"factored_forward": _forward(swap_hg=True)},
    "fwd: residual subtracted": {"factored_forward": _forward(subtract_residual=True)},
    "fwd: only the last path kept": {"factored_forward": _forward(last_path_only=True)},
    "fwd: V sign flipped": {"factored_forward": _forward(negate_v=True)},
    "fwd: latent scale off by one": {"factored_forward": _forward(roll_l=True)},
    "fwd: U read in the wrong order": {"factored_forward": _forward(u_wrong_order=True)},
    "fwd: V read in the wrong order": {"factored_forward": _forward(v_wrong_order=True)},
    "fwd: sampled rows keep all of h": {"factored_forward": _forward(h_all_rows=True)},
    "fwd: input scale dropped": {"factored_forward": _forward(drop_g=True)},
    "dense: g dropped": {"dense_weight": _dense_without_g},
    # precision: every oracle function converts through _f64
    "all: fp32 instead of fp64": {"_f64": lambda a: np.asarray(a).astype(np.float32)},
}


def test_pins_pass_on_the_unmutated_oracle(golden_dir):
    assert _failing_pins(golden_dir) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_each_planted_mistake_fails_a_pin(golden_dir, monkeypatch, name):
    for attr, repl in MUTANTS[name].items():
        assert hasattr(orc, attr), attr
        monkeypatch.setattr(orc, attr, repl)
    failed = _failing_pins(golden_dir)
    assert failed, f"no pin catches the planted mistake: {name}"


def test_mutant_helpers_differ_from_the_oracle():
    """Each layout mutant really changes the bit positions (so a pass above
    is not vacuous)."""
    for kw in ({"swap_r": True}, {"bit_order_4q": True}, {"u_q_stride": 8}):
        for role in ("V", "U"):
            a = orc._tile_coords(role, 1, 1)
            b = _coords(**kw)(role, 1, 1)
            if role == "V" and kw.get("u_q_stride"):
                continue   # that mutant only touches role U
            assert any(not np.array_equal(x, y) for x, y in zip(a, b)), (kw, role)
