"""GPU parity on seeded random shapes: decode (batch 1..16), prefill (M a
multiple of 128, both GEMM kernels) and mixed-shape stacks, each against the
fp64 oracle.  The shapes are drawn once from a fixed seed, so a failure names
a reproducible case; they cover widths, ranks, column-tile splits and path
boundaries that the fixed-shape tests do not list."""
import numpy as np
import pytest
import torch

from oracle import littlebit_oracle as orc
from latent_binary_factorization_b200 import synth

pytestmark = pytest.mark.gpu

REL_L2 = 2e-3
MAX_ABS = 1e-2


@pytest.fixture(scope="module")
def lbm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from latent_binary_factorization_b200 import layers, littlebit
    return littlebit, layers


def _shapes(seed, n):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        d_in = 256 * int(rng.integers(1, 13))
        d_out = 128 * int(rng.integers(1, 17))
        s = int(rng.choice([int(rng.integers(1, 65)), int(rng.integers(65, 1025))]))
        out.append((d_in, d_out, s, bool(rng.integers(0, 2))))
    return out


DECODE = [(a, b, s, r, 1 + (i * 7) % 16) for i, (a, b, s, r) in enumerate(_shapes(2024, 40))]
PREFILL = [(a, b, s, r, 128 * (1 + i % 5), i % 2 == 0) for i, (a, b, s, r) in enumerate(_shapes(4048, 30))]


def _check(y, y_ref, tag):
    a = y.float().cpu().numpy()
    e, m = orc.rel_l2(a, y_ref), orc.max_abs_ratio(a, y_ref)
    assert e <= REL_L2 and m <= MAX_ABS, f"{tag}: rel_l2={e:.3e} max_abs_ratio={m:.3e}"


@pytest.mark.parametrize("d_in,d_out,s,residual,batch", DECODE)
def test_decode_random_shapes(lbm, d_in, d_out, s, residual, batch):
    lb, layers = lbm
    paths = synth.layer(d_in, d_out, s, residual, seed=d_in + d_out + s)
    layer = layers.upload(paths, d_in, d_out, s)
    xh = synth.activations(batch, d_in, seed=s)
    y = lb.forward(layer, torch.from_numpy(xh).cuda())
    torch.cuda.synchronize()
    _check(y, orc.factored_forward(xh.astype(np.float64), paths), f"{d_in}x{d_out} s={s} r={residual} B={batch}")
    assert lb.device_status() == 0


@pytest.mark.parametrize("d_in,d_out,s,residual,M,bf16", PREFILL)
def test_prefill_random_shapes(lbm, d_in, d_out, s, residual, M, bf16):
    """M = 128 and 384 run the single-SM GEMMs, 256 and 512 pairs of SMs; the
    oracle checks every row (M <= 640)."""
    lb, layers = lbm
    paths = synth.layer(d_in, d_out, s, residual, seed=d_in * 3 + d_out + s)
    layer = layers.upload(paths, d_in, d_out, s)
    if bf16:
        xf = synth.activations(M, d_in, seed=s, dtype="bf16")
        xt, x64 = torch.from_numpy(xf).to(torch.bfloat16), xf.astype(np.float64)
    else:
        xh = synth.activations(M, d_in, seed=s)
        xt, x64 = torch.from_numpy(xh), xh.astype(np.float64)
    y = lb.forward(layer, xt.cuda())
    torch.cuda.synchronize()
    _check(y, orc.factored_forward(x64, paths), f"{d_in}x{d_out} s={s} r={residual} M={M}")
    assert lb.device_status() == 0


@pytest.mark.parametrize("batch", [1, 5, 256])
def test_random_mixed_stack(lbm, batch):
    """Ten random layers in one forward_many call (decode at 1 and 5 rows,
    prefill at 256), every output against the oracle."""
    lb, layers = lbm
    L, X, Y, refs = [], [], [], []
    for i, (a, b, s, r) in enumerate(_shapes(77 + batch, 10)):
        paths = synth.layer(a, b, s, r, seed=900 + i, index=i)
        L.append(layers.upload(paths, a, b, s))
        xh = synth.activations(batch, a, seed=300 + i, index=i)
        X.append(torch.from_numpy(xh).cuda())
        Y.append(torch.full((batch, b), float("nan"), dtype=torch.float16, device="cuda"))
        refs.append(orc.factored_forward(xh.astype(np.float64), paths))
    lb.Stack(L, X, Y)()
    torch.cuda.synchronize()
    for i, (y, ref) in enumerate(zip(Y, refs)):
        _check(y, ref, f"layer {i}")
    assert lb.device_status() == 0


@pytest.mark.parametrize("rows", [1, 3, 256])
def test_random_latent_cache(lbm, rows):
    """Latent rows and their expansion on random shapes: expand(latent(x))
    matches the oracle's forward, and the rows match the oracle's latent."""
    lb, layers = lbm
    for i, (a, b, s, r) in enumerate(_shapes(555 + rows, 4)):
        paths = synth.layer(a, b, s, r, seed=40 + i, index=i)
        layer = layers.upload(paths, a, b, s)
        xh = synth.activations(rows, a, seed=60 + i, index=i)
        (t,) = lb.latent_forward([layer], [torch.from_numpy(xh).cuda()])
        (y,) = lb.latent_expand([layer], [t])
        torch.cuda.synchronize()
        x64 = xh.astype(np.float64)
        t_ref = orc.latent_cache(x64, paths)
        _check(t[:, :t_ref.shape[1]], t_ref, f"latent {a}x{b} s={s} r={r}")
        _check(y, orc.factored_forward(x64, paths), f"expand {a}x{b} s={s} r={r}")
    assert lb.device_status() == 0
