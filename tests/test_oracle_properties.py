"""Property checks of the oracle over random small shapes (hypothesis): the
packing round trip and its padding for any rows/columns, and the forward's
invariants (dense reconstruction, linearity, residual sum, latent gauge) for
any (d_in, d_out, s, batch).  They complement the fixed-shape pins in
test_oracle.py."""
import numpy as np
from hypothesis import given, settings, strategies as st

from oracle import littlebit_oracle as orc

SETTINGS = settings(max_examples=40, deadline=None)


@SETTINGS
@given(role=st.sampled_from(["V", "U"]), R=st.integers(1, 70), K=st.integers(1, 300),
       seed=st.integers(0, 2 ** 31 - 1))
def test_pack_roundtrip_any_shape(role, R, K, seed):
    rng = np.random.default_rng(seed)
    F = rng.standard_normal((R, K)).astype(np.float32)
    F[rng.random((R, K)) < 0.05] = 0.0
    buf = orc.pack_signs(F, role)
    assert buf.size == orc.packed_nbytes(role, R, K)
    assert np.array_equal(orc.unpack_signs(buf, role, R, K), np.where(F < 0, -1, 1))
    assert orc.padding_is_zero(buf, role, R, K)
    assert int(np.unpackbits(buf).sum()) == int((F < 0).sum())


def _layer(rng, d_in, d_out, s, residual):
    paths = []
    for _ in range(2 if residual else 1):
        paths.append({"U": np.where(rng.random((d_out, s)) < 0.5, -1, 1).astype(np.int8),
                      "V": np.where(rng.random((d_in, s)) < 0.5, -1, 1).astype(np.int8),
                      "h": rng.uniform(0.5, 1.5, d_out).astype(np.float16),
                      "g": rng.uniform(0.5, 1.5, d_in).astype(np.float16),
                      "l": rng.uniform(0.5, 1.5, s).astype(np.float16)})
    return paths


@SETTINGS
@given(d_in=st.integers(1, 40), d_out=st.integers(1, 40), s=st.integers(1, 12), batch=st.integers(1, 4),
       residual=st.booleans(), seed=st.integers(0, 2 ** 31 - 1))
def test_forward_invariants_any_shape(d_in, d_out, s, batch, residual, seed):
    rng = np.random.default_rng(seed)
    paths = _layer(rng, d_in, d_out, s, residual)
    x = rng.standard_normal((batch, d_in)).astype(np.float16)
    y = orc.factored_forward(x, paths)
    assert y.shape == (batch, d_out)
    # equals the dense reconstruction W x
    np.testing.assert_allclose(y, orc.dense_forward(x, paths), rtol=1e-11, atol=1e-11)
    # linear in x
    x2 = rng.standard_normal((batch, d_in))
    np.testing.assert_allclose(orc.factored_forward(x + 3.0 * x2, paths),
                               y + 3.0 * orc.factored_forward(x2, paths), rtol=1e-10, atol=1e-10)
    # the residual output is the sum of the two single-path outputs
    if residual:
        np.testing.assert_allclose(y, orc.factored_forward(x, paths[:1]) + orc.factored_forward(x, paths[1:]),
                                   rtol=1e-12, atol=1e-12)
    # flipping latent column j in both U and V of a path leaves y unchanged
    j = int(rng.integers(0, s))
    flipped = [dict(p) for p in paths]
    flipped[0] = {k: v.copy() for k, v in paths[0].items()}
    flipped[0]["U"][:, j] *= -1
    flipped[0]["V"][:, j] *= -1
    np.testing.assert_allclose(orc.factored_forward(x, flipped), y, rtol=1e-12, atol=1e-12)
