"""Pins for the latent-cache half of the forward oracle (latent_cache and
expand: the factorised K/V projection cached as its latent, Samsung LittleBit
article, section 4, KV-cache bullet)."""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import littlebit_oracle as orc
from latent_binary_factorization_b200 import synth


def _paths(gold):
    return [{k: np.asarray(v, dtype=np.float64) for k, v in p.items()} for p in gold["paths"]]


def test_latent_cache_hand_worked(golden_dir):
    with open(os.path.join(golden_dir, "latent_cache_worked_example.json")) as f:
        gold = json.load(f)
    paths = _paths(gold)
    x = np.asarray(gold["x"])
    np.testing.assert_allclose(orc.latent_cache(x, paths), gold["cache"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(orc.expand(np.asarray(gold["cache"]), paths), gold["y"], rtol=0, atol=1e-15)


@pytest.mark.parametrize("d_in,d_out,s,residual,batch", [(64, 48, 5, True, 3), (96, 32, 7, False, 2),
                                                         (256, 128, 33, True, 4)])
def test_expand_of_the_cache_is_the_forward(d_in, d_out, s, residual, batch):
    """Rebuilding from the cached latent gives the layer's output, including
    on sampled output rows."""
    paths = synth.layer(d_in, d_out, s, residual, seed=s)
    x = synth.activations(batch, d_in, seed=s)
    t = orc.latent_cache(x, paths)
    assert t.shape == (batch, (2 if residual else 1) * s)
    y = orc.factored_forward(x, paths)
    np.testing.assert_allclose(orc.expand(t, paths), y, rtol=1e-12, atol=1e-12 * np.abs(y).max())
    rows = np.array([0, d_out // 2, d_out - 1])
    np.testing.assert_allclose(orc.expand(t, paths, rows=rows), y[:, rows], rtol=1e-12,
                               atol=1e-12 * np.abs(y).max())


def test_expand_is_linear_in_the_cache():
    paths = synth.layer(64, 32, 6, True, seed=3)
    rng = np.random.default_rng(3)
    a, b = rng.standard_normal((2, 12)), rng.standard_normal((2, 12))
    np.testing.assert_allclose(orc.expand(2 * a - b, paths), 2 * orc.expand(a, paths) - orc.expand(b, paths),
                               rtol=1e-12, atol=1e-12)


def test_kv_cache_ratio_matches_the_article(golden_dir):
    with open(os.path.join(golden_dir, "kv_cache_ratio.txt")) as f:
        rows = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    for d, s, npaths, num, den, one_dec in rows:
        r = orc.kv_cache_ratio(int(d), int(s), int(npaths))
        assert r == Fraction(int(num), int(den))
        assert f"{float(r):.1f}" == one_dec
    # the rank is the one the effective-bit budget gives for that projection
    assert orc.solve_rank(4096, 4096, "0.1", False) == 188
