"""GPU parity of the prefill forward (batch >= 128, tcgen05 tensor cores)
against the fp64 oracle, through the C ABI."""
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


def _x(M, d_in, seed, dtype):
    if dtype == torch.bfloat16:
        xf = synth.activations(M, d_in, seed=seed, dtype="bf16")         # float32, bf16-exact
        return torch.from_numpy(xf).to(torch.bfloat16), xf.astype(np.float64)
    xh = synth.activations(M, d_in, seed=seed)
    return torch.from_numpy(xh), xh.astype(np.float64)


def _check(y, y_ref, tag):
    a = y.float().cpu().numpy()
    e, m = orc.rel_l2(a, y_ref), orc.max_abs_ratio(a, y_ref)
    assert e <= REL_L2 and m <= MAX_ABS, f"{tag}: rel_l2={e:.3e} max_abs_ratio={m:.3e}"
    return e


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("d_in,d_out,s,residual,M", [
    (512, 512, 32, False, 128),      # tiny config, one tile
    (512, 512, 32, True, 256),
    (1024, 384, 100, True, 256),     # ragged N tile of GEMM2 (384 = 256 + 128), ragged rank
    (768, 640, 1, False, 128),       # rank 1
    (256, 128, 45, True, 384),       # smallest shapes
    (1024, 512, 1024, True, 128),    # maximum rank, both paths: GEMM1 N = GEMM2 K = 2048
])
def test_prefill_small_full_output(lbm, dtype, d_in, d_out, s, residual, M):
    lb, layers = lbm
    paths = synth.layer(d_in, d_out, s, residual, seed=s + M)
    layer = layers.upload(paths, d_in, d_out, s)
    xt, x64 = _x(M, d_in, seed=s, dtype=dtype)
    y = lb.forward(layer, xt.cuda())
    torch.cuda.synchronize()
    assert y.dtype == dtype
    _check(y, orc.factored_forward(x64, paths), f"{d_in}x{d_out} s={s} M={M}")
    assert lb.device_status() == 0


@pytest.mark.parametrize("d_in,d_out,s", [(4096, 4096, 290), (4096, 11008, 431), (11008, 4096, 431)])
def test_prefill_7b_0p3bpw_full_size_sampled_tokens(lbm, d_in, d_out, s):
    """Llama-2-7B linear layers at 0.3 BPW with residual, M = 2048 bf16 tokens;
    the oracle checks 64 sampled token rows over all outputs."""
    lb, layers = lbm
    paths = synth.layer(d_in, d_out, s, True, seed=d_out)
    layer = layers.upload(paths, d_in, d_out, s)
    xt, x64 = _x(2048, d_in, seed=7, dtype=torch.bfloat16)
    y = lb.forward(layer, xt.cuda())
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(1).choice(2048, 64, replace=False))
    _check(y[rows], orc.factored_forward(x64[rows], paths), f"7B {d_in}x{d_out}")


def test_prefill_matches_decode_on_same_rows(lbm):
    """The tensor-core prefill and the decode kernels agree row by row."""
    lb, layers = lbm
    paths = synth.layer(2048, 1024, 133, True, seed=3)
    layer = layers.upload(paths, 2048, 1024, 133)
    xt, _ = _x(128, 2048, seed=3, dtype=torch.float16)
    y_pre = lb.forward(layer, xt.cuda())
    y_dec = torch.cat([lb.forward(layer, xt[i:i + 16].cuda()) for i in range(0, 128, 16)])
    torch.cuda.synchronize()
    a, b = y_pre.float().cpu().numpy(), y_dec.float().cpu().numpy()
    assert orc.rel_l2(a, b) <= 2 * REL_L2


@pytest.mark.parametrize("d_in,d_out,s,residual", [(1024, 640, 290, True), (2048, 768, 133, True),
                                                   (1024, 384, 188, False)])
def test_pair_and_single_sm_gemms_agree(lbm, d_in, d_out, s, residual):
    """The same 384 rows through the pair-of-SMs GEMMs (M = 256: rows 0..255)
    and the single-SM GEMMs (M = 384 and M = 128): every row matches the
    oracle, and the two kernels agree row by row within fp16 rounding of t'
    and y.  The shapes give unequal column tiles (640 = 224 + 224 + 192 and a
    path boundary inside a tile)."""
    lb, layers = lbm
    paths = synth.layer(d_in, d_out, s, residual, seed=s + 5)
    layer = layers.upload(paths, d_in, d_out, s)
    xt, x64 = _x(384, d_in, seed=s, dtype=torch.bfloat16)
    xd = xt.cuda()
    y_all = lb.forward(layer, xd)                 # M = 384: single-SM tiles
    y_pair = lb.forward(layer, xd[:256].contiguous())   # M = 256: pairs of SMs
    y_tail = lb.forward(layer, xd[256:].contiguous())   # M = 128: single-SM
    torch.cuda.synchronize()
    ref = orc.factored_forward(x64, paths)
    _check(y_pair, ref[:256], "pair GEMM")
    _check(y_all, ref, "single-SM GEMM")
    assert torch.equal(y_tail, y_all[256:])
    a, b = y_pair.float().cpu().numpy(), y_all[:256].float().cpu().numpy()
    assert orc.rel_l2(a, b) <= REL_L2
    assert lb.device_status() == 0


def test_prefill_forward_many(lbm):
    lb, layers = lbm
    specs = [(1024, 1024, 64, True), (1024, 2048, 100, False), (2048, 512, 77, True)]
    L, X, Y, refs = [], [], [], []
    for i, (a, b, s, r) in enumerate(specs):
        paths = synth.layer(a, b, s, r, seed=50 + i, index=i)
        xt, x64 = _x(256, a, seed=50 + i, dtype=torch.bfloat16)
        L.append(layers.upload(paths, a, b, s))
        X.append(xt.cuda())
        Y.append(torch.empty(256, b, dtype=torch.bfloat16, device="cuda"))
        refs.append(orc.factored_forward(x64, paths))
    lb.Stack(L, X, Y)()
    torch.cuda.synchronize()
    for i, (y, ref) in enumerate(zip(Y, refs)):
        _check(y, ref, f"layer {i}")


@pytest.mark.parametrize("M", [256, 384])
def test_prefill_forward_many_shared_inputs(lbm, M):
    """Layers of one prefill call that read the same x (q, k and v; gate and
    up) share one converted operand: every output matches the oracle and is
    bit-identical to its one-layer call.  M = 256 runs the GEMMs on pairs of
    SMs, M = 384 on single SMs."""
    lb, layers = lbm
    groups = [[(1024, 1024, 64, True)] * 3, [(1024, 2048, 100, False)] * 2, [(2048, 512, 77, True)],
              [(1024, 768, 45, True)]]
    L, X, Y, refs = [], [], [], []
    k = 0
    for g, members in enumerate(groups):
        xt, x64 = _x(M, members[0][0], seed=60 + g, dtype=torch.bfloat16)
        x = xt.cuda()
        for (a, b, s, r) in members:
            paths = synth.layer(a, b, s, r, seed=70 + k, index=k)
            L.append(layers.upload(paths, a, b, s))
            X.append(x)
            Y.append(torch.full((M, b), float("nan"), dtype=torch.bfloat16, device="cuda"))
            refs.append(orc.factored_forward(x64, paths))
            k += 1
    lb.Stack(L, X, Y)()
    torch.cuda.synchronize()
    for i, (y, ref) in enumerate(zip(Y, refs)):
        _check(y, ref, f"layer {i}")
        assert torch.equal(y, lb.forward(L[i], X[i])), f"layer {i} differs from its one-layer call"
    assert lb.device_status() == 0


@pytest.mark.parametrize("shared", [False, True])
def test_prefill_chunked_stack_matches_single_layer_calls(lbm, shared):
    """A stack whose operand buffers span several chunks (preparation of one
    chunk overlapped with the GEMMs of the previous one, two workspace halves
    reused in turn) gives, layer by layer, exactly what one-layer calls give;
    a second call in a row, after the halves hold the last call's operands,
    gives it again.  With `shared`, layers read their inputs in groups of three
    (as q, k and v do), and some groups straddle a chunk boundary."""
    lb, layers = lbm
    gen = torch.Generator(device="cuda").manual_seed(11)
    M, n = 2048, 40   # ~29 MB of operands per layer: three chunks
    L, X, Y = [], [], []
    for i in range(n):
        L.append(layers.random_layer(4096, 4096, 290, True, gen)[0])
        if shared and i % 3:
            X.append(X[-1])
        else:
            X.append(torch.randn(M, 4096, generator=gen, device="cuda").to(torch.bfloat16))
        Y.append(torch.full((M, 4096), float("nan"), dtype=torch.bfloat16, device="cuda"))
    st = lb.Stack(L, X, Y)
    st()
    for rep in range(2):
        torch.cuda.synchronize()
        for i in range(n):
            y1 = lb.forward(L[i], X[i])
            assert torch.equal(Y[i], y1), f"layer {i} differs from its single-layer call (pass {rep})"
        for y in Y:
            y.fill_(float("nan"))
        st()
    assert lb.device_status() == 0


def test_prefill_stack_in_cuda_graph(lbm):
    """A two-chunk prefill stack (side-stream preparation forked from and
    joined to the caller's stream) captured into a CUDA graph on the stream of
    an earlier eager call and replayed gives exactly the eager result."""
    lb, layers = lbm
    gen = torch.Generator(device="cuda").manual_seed(12)
    M, n = 2048, 20   # ~29 MB of operands per layer: two chunks
    L, X, Y = [], [], []
    for i in range(n):
        L.append(layers.random_layer(4096, 4096, 290, True, gen)[0])
        X.append(torch.randn(M, 4096, generator=gen, device="cuda").to(torch.bfloat16))
        Y.append(torch.empty(M, 4096, dtype=torch.bfloat16, device="cuda"))
    st = lb.Stack(L, X, Y)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        st()
    torch.cuda.synchronize()
    ref = [y.clone() for y in Y]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        st()
    for y in Y:
        y.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    for i, (y, r) in enumerate(zip(Y, ref)):
        assert torch.equal(y, r), f"layer {i}"
    del g


RANGE_BIT = 1 << 7   # LB_ERR_RANGE


def test_prefill_range_errors_are_reported(lbm):
    """Prefill holds x and t' in fp16.  A bf16 input beyond fp16's finite
    range, and a latent value t' = l * t beyond it, cannot be held there: the
    call raises LB_ERR_RANGE in the device status instead of returning inf
    silently.  In-range inputs raise nothing."""
    lb, layers = lbm
    d_in, d_out, s, M = 512, 256, 40, 128
    paths = synth.layer(d_in, d_out, s, True, seed=21)
    layer = layers.upload(paths, d_in, d_out, s)
    xt, _ = _x(M, d_in, seed=21, dtype=torch.bfloat16)
    x = xt.cuda()
    lb.forward(layer, x)
    assert lb.device_status() == 0
    # |x| = 1e5 is a finite bf16 value and an fp16 overflow
    xb = x.clone()
    xb[7, 100] = 1.0e5
    lb.forward(layer, xb)
    assert lb.device_status() & RANGE_BIT
    assert lb.device_status() == 0            # read and cleared
    # t' overflow: large latent scales make l * t exceed 65504
    big = [dict(p) for p in paths]
    for p in big:
        p["l"] = np.full(s, 30000.0, np.float16)
    big_layer = layers.upload(big, d_in, d_out, s)
    lb.forward(big_layer, x)
    assert lb.device_status() & RANGE_BIT
    # the stream keeps working and in-range calls are exact again
    y = lb.forward(layer, x)
    assert lb.device_status() == 0
    _check(y, orc.factored_forward(xt.float().numpy().astype(np.float64), paths), "after range errors")


def test_prefill_nonfinite_fp16_input_is_reported(lbm):
    lb, layers = lbm
    d_in, d_out, s, M = 256, 128, 16, 128
    paths = synth.layer(d_in, d_out, s, False, seed=22)
    layer = layers.upload(paths, d_in, d_out, s)
    xt, _ = _x(M, d_in, seed=22, dtype=torch.float16)
    x = xt.cuda()
    x[3, 5] = float("inf")
    lb.forward(layer, x)
    assert lb.device_status() & RANGE_BIT
