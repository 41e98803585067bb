"""GPU parity of the latent cache (Samsung LittleBit article, section 4, the
KV-cache bullet): the latent-only forward writes a K/V projection's cache
rows t' = [t'_1 | t'_2], and the expand call rebuilds the projection from
them, each against the fp64 oracle, through the C ABI."""
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


def _check(got, ref, tag):
    a = got.float().cpu().numpy()
    e, m = orc.rel_l2(a, ref), orc.max_abs_ratio(a, ref)
    assert e <= REL_L2 and m <= MAX_ABS, f"{tag}: rel_l2={e:.3e} max_abs_ratio={m:.3e}"


def _x(batch, d_in, seed, dtype):
    if dtype == torch.bfloat16:
        xf = synth.activations(batch, d_in, seed=seed, dtype="bf16")
        return torch.from_numpy(xf).to(torch.bfloat16).cuda(), xf.astype(np.float64)
    xh = synth.activations(batch, d_in, seed=seed)
    return torch.from_numpy(xh).cuda(), xh.astype(np.float64)


def test_row_size_matches_the_oracle(lbm):
    lb, layers = lbm
    for s, res in [(1, False), (188, False), (86, True), (620, False), (302, True), (1024, True)]:
        L = lb.Layer(256, 128, s)
        L.paths = [None] * (2 if res else 1)
        assert lb.latent_row_elems(L) == orc.cache_row_elems(s, 2 if res else 1)


@pytest.mark.parametrize("d_in,d_out,s,residual,batch,dtype", [
    (4096, 4096, 188, False, 1, torch.float16),    # 7B K/V projection at 0.1 BPW, one token
    (4096, 4096, 86, True, 3, torch.float16),      # residual variant
    (2048, 1024, 100, True, 16, torch.float16),
    (4096, 4096, 188, False, 256, torch.bfloat16),  # prefill: a prompt's K/V rows
    (1024, 768, 90, True, 128, torch.float16),
    (1024, 768, 90, True, 512, torch.bfloat16),     # pairs of SMs, both paths in one column tile
    (1024, 768, 45, True, 130, torch.float16),      # prefill 128 + decode group of 2
])
def test_latent_forward_and_expand(lbm, d_in, d_out, s, residual, batch, dtype):
    lb, layers = lbm
    paths = synth.layer(d_in, d_out, s, residual, seed=s + batch)
    layer = layers.upload(paths, d_in, d_out, s)
    x, x64 = _x(batch, d_in, s + batch, dtype)
    (t,) = lb.latent_forward([layer], [x])
    torch.cuda.synchronize()
    n = (2 if residual else 1) * s
    t_ref = orc.latent_cache(x64, paths)
    _check(t[:, :n], t_ref, "cache rows")
    # expand the library's own cache rows (exactly the fp16 values it stored)
    (y,) = lb.latent_expand([layer], [t], dtype=dtype)
    torch.cuda.synchronize()
    t_used = t[:, :n].float().cpu().numpy().astype(np.float64)
    _check(y, orc.expand(t_used, paths), "expand of the cache rows")
    _check(y, orc.factored_forward(x64, paths), "expand(latent(x)) = layer(x)")
    assert lb.device_status() == 0


@pytest.mark.parametrize("rows,dtype", [(1, torch.float16), (5, torch.float16), (2048, torch.float16),
                                        (384, torch.bfloat16)])
def test_expand_oracle_cache_rows(lbm, rows, dtype):
    """Cache rows written by the oracle (rounded to fp16), rebuilt on the GPU:
    a decode step re-reading a whole cached prompt (2048 rows) goes through
    the tensor-core GEMM."""
    lb, layers = lbm
    d_in, d_out, s = 4096, 4096, 188
    paths = synth.layer(d_in, d_out, s, False, seed=rows)
    layer = layers.upload(paths, d_in, d_out, s)
    x64 = synth.activations(rows, d_in, seed=rows).astype(np.float64)
    t16 = orc.latent_cache(x64, paths).astype(np.float16)
    ld = lb.latent_row_elems(layer)
    t = torch.zeros((rows, ld), dtype=torch.float16)
    t[:, :s] = torch.from_numpy(t16)
    (y,) = lb.latent_expand([layer], [t.cuda()], dtype=dtype)
    torch.cuda.synchronize()
    _check(y, orc.expand(t16.astype(np.float64), paths), f"rows={rows}")


def test_latent_cache_many_layers(lbm):
    """K and V projections of two blocks in one call each way."""
    lb, layers = lbm
    specs = [(4096, 4096, 188, False), (4096, 4096, 86, True), (2048, 512, 40, True), (1024, 1024, 300, False)]
    L, X, refs, x64s, P = [], [], [], [], []
    for i, (a, b, s, r) in enumerate(specs):
        paths = synth.layer(a, b, s, r, seed=50 + i, index=i)
        x, x64 = _x(2, a, 50 + i, torch.float16)
        L.append(layers.upload(paths, a, b, s))
        X.append(x)
        x64s.append(x64)
        P.append(paths)
    ts = lb.latent_forward(L, X)
    ys = lb.latent_expand(L, ts)
    torch.cuda.synchronize()
    for i, (y, x64, paths) in enumerate(zip(ys, x64s, P)):
        _check(y, orc.factored_forward(x64, paths), f"layer {i}")
