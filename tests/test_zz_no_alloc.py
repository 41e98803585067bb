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


def _compare(y, y_ref):
    a, b = y.float().cpu().numpy(), y_ref.float().cpu().numpy()
    assert orc.rel_l2(a, b) <= REL_L2 and orc.max_abs_ratio(a, b) <= MAX_ABS


def test_noalloc_matches_regular_forward_twice_in_a_row(env):
    lb, layers, _ = env
    cases = [(4096, 4096, 86, True, 1, 31), (8192, 2048, 300, False, 4, 32)]
    built = []
    for d_in, d_out, s, res, batch, seed in cases:
        paths = synth.layer(d_in, d_out, s, res, seed=seed)
        layer = layers.upload(paths, d_in, d_out, s)
        x = torch.from_numpy(synth.activations(batch, d_in, seed=seed)).cuda()
        built.append((layer, x))
    # two calls in a row, different layers: the second must not see the
    # first call's leftovers in the shared scratch
    for layer, x in built:
        y_ref = lb.forward(layer, x).clone()
        y = _noalloc(env, layer, x)
        torch.cuda.synchronize()
        _compare(y, y_ref)
    # and the same layer twice in a row
    layer, x = built[0]
    y1 = _noalloc(env, layer, x).clone()
    y2 = _noalloc(env, layer, x).clone()
    torch.cuda.synchronize()
    y_ref = lb.forward(layer, x)
    torch.cuda.synchronize()
    _compare(y1, y_ref)
    _compare(y2, y_ref)


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
