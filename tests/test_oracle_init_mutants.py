"""Mutation check of the pins of the initialisation oracle (Dual-SVID,
Joint-ITQ) and of the latent-cache half of the forward oracle: each case
plants one plausible mistake (on the CPU, by replacing one function for the
duration of the case) and at least one pin must then fail."""
import importlib.util
import inspect
import os

import numpy as np
import pytest

from oracle import littlebit_init as ini
from oracle import littlebit_oracle as orc

HERE = os.path.dirname(os.path.abspath(__file__))


def _load(name):
    spec = importlib.util.spec_from_file_location(name, os.path.join(HERE, f"{name}.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


PIN_MODULES = [_load("test_oracle_init"), _load("test_oracle_cache")]


def _pin_calls(golden_dir):
    calls = []
    for mod in PIN_MODULES:
        for name, fn in sorted(vars(mod).items()):
            if not (name.startswith("test_") and callable(fn)):
                continue
            params = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
            if params:
                names = [a.strip() for a in params[0].args[0].split(",")]
                for vals in params[0].args[1]:
                    kw = dict(zip(names, vals if len(names) > 1 else (vals,)))
                    calls.append((name, lambda fn=fn, kw=kw: fn(**kw)))
            elif "golden_dir" in inspect.signature(fn).parameters:
                calls.append((name, lambda fn=fn: fn(golden_dir)))
            else:
                calls.append((name, fn))
    return calls


def _failing(golden_dir):
    out = []
    for name, call in _pin_calls(golden_dir):
        try:
            call()
        except Exception:
            out.append(name)
    return out


_orig = {"dual_svid": ini.dual_svid, "procrustes": ini.procrustes, "rank1_nonneg": ini.rank1_nonneg,
         "expand": orc.expand, "latent_cache": orc.latent_cache, "svd_factors": ini.svd_factors}


def _dual_svid_l_without_means(Uf, Vf):
    p = _orig["dual_svid"](Uf, Vf)
    au, bu = ini.rank1_nonneg(np.abs(Uf))
    av, bv = ini.rank1_nonneg(np.abs(Vf))
    p["l"] = bu * bv
    return p


def _dual_svid_h_from_v(Uf, Vf):
    p = _orig["dual_svid"](Uf, Vf)
    av, _ = ini.rank1_nonneg(np.abs(Vf))
    p["h"] = np.resize(av / av.mean(), p["h"].shape)
    return p


def _dual_svid_zero_negative(Uf, Vf):
    p = _orig["dual_svid"](Uf, Vf)
    p["U"] = np.where(np.asarray(Uf) <= 0, -1, 1).astype(np.int8)
    p["V"] = np.where(np.asarray(Vf) <= 0, -1, 1).astype(np.int8)
    return p


def _expand_paths_swapped(t, paths, rows=None):
    return _orig["expand"](t, paths[::-1], rows)


def _expand_without_h(t, paths, rows=None):
    flat = [dict(p, h=np.ones_like(np.asarray(p["h"], dtype=np.float64))) for p in paths]
    return _orig["expand"](t, flat, rows)


def _cache_without_l(x, paths):
    return np.concatenate([orc._f64(x) * orc._f64(p["g"])[None, :] @ orc._f64(p["V"]) for p in paths], axis=1)


def _svd_factors_uneven(W, s):
    U, S, Vt = np.linalg.svd(np.asarray(W, dtype=np.float64), full_matrices=False)
    return U[:, :s] * S[None, :s], Vt[:s].T


MUTANTS = {
    "dual-svid: latent scale without the row/column means": (ini, "dual_svid", _dual_svid_l_without_means),
    "dual-svid: row scale taken from V": (ini, "dual_svid", _dual_svid_h_from_v),
    "dual-svid: sign(0) read as negative": (ini, "dual_svid", _dual_svid_zero_negative),
    "svd: singular values all on U": (ini, "svd_factors", _svd_factors_uneven),
    "rank-1 fit: second singular pair": (ini, "rank1_nonneg", lambda A: tuple(
        np.abs(v) * np.sqrt(S[1]) for v, S in [(np.linalg.svd(A)[0][:, 1], np.linalg.svd(A)[1])]
    ) * 1 + (np.abs(np.linalg.svd(A)[2][1]) * np.sqrt(np.linalg.svd(A)[1][1]),) if min(np.shape(A)) > 1
        else _orig["rank1_nonneg"](2 * np.asarray(A))),
    "itq: Procrustes factor transposed": (ini, "procrustes", lambda X, B: _orig["procrustes"](X, B).T),
    "itq: signs never re-taken": (ini, "procrustes", lambda X, B: _orig["procrustes"](X, np.sign(X) + (X == 0))),
    "cache: paths' columns swapped": (orc, "expand", _expand_paths_swapped),
    "cache: row scale dropped": (orc, "expand", _expand_without_h),
    "cache: latent scale dropped": (orc, "latent_cache", _cache_without_l),
}


def test_pins_pass_on_the_unmutated_oracles(golden_dir):
    assert _failing(golden_dir) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_each_planted_mistake_fails_a_pin(golden_dir, monkeypatch, name):
    mod, attr, repl = MUTANTS[name]
    monkeypatch.setattr(mod, attr, repl)
    assert _failing(golden_dir), f"no pin catches the planted mistake: {name}"
