"""The allocation-free forward (littlebit_linear_forward_noalloc) against the
regular forward, through the C ABI.

That entry point exists for callers that cannot let a library allocate
device memory (an application allocator that owns the device, or a hot loop
that cannot take cudaMalloc's synchronisation); its scratch is a fixed array
inside the library.  This file is collected last so that a run stopping at
the first failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

from oracle import littlebit_oracle as orc
from latent_binary_factorization_b200 import synth

pytestmark = pytest.mark.gpu

REL_L2 = 2e-3
MAX_ABS = 1e-2


@pytest.fixture(scope="module")
def env():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from latent_binary_factorization_b200 import layers, littlebit
    lib = littlebit.library()
    f = lib.littlebit_linear_forward_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.POINTER(littlebit.LbLayer), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                  ctypes.c_int, ctypes.c_void_p]
    return littlebit, layers, f


def _noalloc(env, layer, x):
    lb, _, f = env
    y = torch.full((x.shape[0], layer.d_out), float("nan"), dtype=torch.float16, device=x.device)
    L = layer.c_struct()
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    code = f(ctypes.byref(L), ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(y.data_ptr()), x.shape[0], 0, st)
    assert code == 0, lb.STATUS.get(code, code)
    return y


def _compare_oracle(y, x_host, paths):
    a = y.float().cpu().numpy()
    ref = orc.factored_forward(x_host, paths)
    assert orc.rel_l2(a, ref) <= REL_L2 and orc.max_abs_ratio(a, ref) <= MAX_ABS


CASES = [(4096, 4096, 86, True, 1, 31),     # packed output pass (batch 1, two paths)
         (8192, 2048, 300, False, 4, 32),
         (4096, 4096, 86, True, 13, 33)]    # four groups of batch rows, both paths


def test_noalloc_matches_regular_forward_twice_in_a_row(env):
    """The same kernels on the same inputs as the regular forward: the outputs
    are bitwise equal, and within the oracle's tolerance.  Calls follow one
    another on different layers and on the same layer, so a region of the
    shared scratch that kept the previous call's contents would show."""
    lb, layers, _ = env
    built = []
    for d_in, d_out, s, res, batch, seed in CASES:
        paths = synth.layer(d_in, d_out, s, res, seed=seed)
        layer = layers.upload(paths, d_in, d_out, s)
        xh = synth.activations(batch, d_in, seed=seed)
        built.append((layer, torch.from_numpy(xh).cuda(), xh, paths))
    for layer, x, xh, paths in built:
        y_ref = lb.forward(layer, x).clone()
        y = _noalloc(env, layer, x)
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref)
        _compare_oracle(y, xh, paths)
    for layer, x, xh, paths in (built[0], built[2]):
        y1 = _noalloc(env, layer, x).clone()
        y2 = _noalloc(env, layer, x).clone()
        torch.cuda.synchronize()
        y_ref = lb.forward(layer, x)
        torch.cuda.synchronize()
        assert torch.equal(y1, y_ref) and torch.equal(y2, y_ref)
    assert lb.device_status() == 0


def test_noalloc_status_word_is_reported(env):
    """The no-alloc calls keep their device error bits in the array's status
    word, which littlebit_device_status reads and clears: a non-finite input
    raises LB_ERR_RANGE there, and the next clean call raises nothing."""
    lb, layers, _ = env
    d_in, d_out, s, res, batch, seed = CASES[0]
    paths = synth.layer(d_in, d_out, s, res, seed=seed)
    layer = layers.upload(paths, d_in, d_out, s)
    xh = synth.activations(batch, d_in, seed=seed)
    x = torch.from_numpy(xh).cuda()
    assert lb.device_status() == 0
    xb = x.clone()
    xb[0, 17] = float("inf")
    _noalloc(env, layer, xb)
    torch.cuda.synchronize()
    assert lb.device_status() == 1 << 7          # LB_ERR_RANGE
    y = _noalloc(env, layer, x)
    torch.cuda.synchronize()
    assert lb.device_status() == 0
    _compare_oracle(y, xh, paths)


def test_noalloc_rejects_scratch_beyond_its_array(env):
    lb, layers, f = env
    # 32768 inputs (16 slices) x 16 rows x 1024 latent rows x 4 B x 2 paths = 2 MiB of partials alone
    L = lb.LbLayer()
    L.d_in, L.d_out, L.s, L.residual = 32768, 128, 1024, 1
    for p in range(2):
        L.path[p] = lb.LbPath(256, 256, 256, 256, 256)
    x = torch.empty(16, 32768, dtype=torch.float16, device="cuda")
    y = torch.empty(16, 128, dtype=torch.float16, device="cuda")
    code = f(ctypes.byref(L), ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(y.data_ptr()), 16, 0, None)
    assert code == 3   # LB_ERR_SHAPE, before any device work
