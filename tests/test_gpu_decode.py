"""GPU parity: sign packing (bit-exact) and the decode forward (batch 1..16)
against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

from oracle import littlebit_oracle as orc
from latent_binary_factorization_b200 import synth

pytestmark = pytest.mark.gpu

REL_L2 = 2e-3      # relative L2 error over the whole output tensor
MAX_ABS = 1e-2     # max |err| / max |y_ref|


@pytest.fixture(scope="module")
def lbm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from latent_binary_factorization_b200 import layers, littlebit
    return littlebit, layers


def _check(y_gpu, y_ref, tag=""):
    y = y_gpu.float().cpu().numpy()
    e, m = orc.rel_l2(y, y_ref), orc.max_abs_ratio(y, y_ref)
    assert e <= REL_L2 and m <= MAX_ABS, f"{tag} rel_l2={e:.3e} max_abs_ratio={m:.3e}"
    return e, m


# ----------------------------------------------------------------- packing

@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16, torch.int8])
@pytest.mark.parametrize("role,n_long,s", [("V", 256, 1), ("V", 512, 33), ("V", 4096, 86), ("V", 768, 16),
                                           ("U", 128, 1), ("U", 384, 45), ("U", 4096, 188), ("U", 256, 32)])
def test_pack_bit_exact(lbm, dtype, role, n_long, s):
    lb, _ = lbm
    F = synth.real_factor(n_long, s, seed=7, zeros=0.05)      # natural orientation (n_long x s)
    if dtype == torch.int8:
        F = np.where(F < 0, -1, 1).astype(np.int8)
    t = torch.from_numpy(F).to(dtype=dtype, device="cuda") if dtype != torch.int8 else torch.from_numpy(F).cuda()
    host = t.float().cpu().numpy()        # the values the kernel sees (after dtype rounding)
    got = lb.pack_signs(t, role).cpu().numpy()
    want = orc.pack_signs(orc.factor_matrix(role, host), role)
    assert np.array_equal(got, want)


def test_pack_strided_and_signed_zero(lbm):
    lb, _ = lbm
    base = torch.randn(300, 512, device="cuda")
    base[::7, ::3] = 0.0
    base[1::7, ::5] = -0.0
    base[2, 2] = float("nan")
    view = base.t()[:, :300]              # (512 x 300) with strides (1, 512)
    got = lb.pack_signs(view, "U").cpu().numpy()
    want = orc.pack_signs(view.cpu().numpy(), "U")
    assert np.array_equal(got, want)


def test_pack_full_size_70b_factor(lbm):
    """Largest factor of the 70B MLP workload (28672 x 620), role V and U."""
    lb, _ = lbm
    gen = torch.Generator(device="cuda").manual_seed(3)
    S = (1 - 2 * torch.randint(0, 2, (28672, 620), generator=gen, device="cuda", dtype=torch.int8)).to(torch.int8)
    Sh = S.cpu().numpy()
    for role in ("V", "U"):
        got = lb.pack_signs(S, role).cpu().numpy()
        assert np.array_equal(got, orc.pack_signs(orc.factor_matrix(role, Sh), role)), role


@pytest.mark.parametrize("role,n_long,s", [("V", 256, 1), ("V", 4096 + 256, 86), ("V", 512, 1024),
                                           ("U", 128, 1), ("U", 4096, 188), ("U", 384, 45)])
def test_unpack_inverts_pack(lbm, role, n_long, s):
    """unpack(pack(F)) = sign(F) as +-1, and it equals the oracle's unpacking
    of the same bytes."""
    lb, _ = lbm
    F = synth.real_factor(n_long, s, seed=n_long + s, zeros=0.05)
    t = torch.from_numpy(F).cuda()
    packed = lb.pack_signs(t, role)
    got = lb.unpack_signs(packed, role, n_long, s).cpu().numpy()
    assert np.array_equal(got, np.where(F < 0, -1, 1).astype(np.int8))
    R, K = (s, n_long) if role == "V" else (n_long, s)
    want = orc.unpack_signs(packed.cpu().numpy(), role, R, K)
    assert np.array_equal(got, orc.factor_matrix(role, want) if role == "V" else want)


# ----------------------------------------------------------------- forward

def _run(lbm, d_in, d_out, s, residual, batch, seed=0):
    lb, layers = lbm
    paths = synth.layer(d_in, d_out, s, residual, seed=seed)
    x = synth.activations(batch, d_in, seed=seed)
    layer = layers.upload(paths, d_in, d_out, s)
    y = lb.forward(layer, torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    return y, x, paths


def test_tiny_config_against_dense_reconstruction(lbm):
    """512 -> 512, s = 32, single path, batch 1: also equals dense W x."""
    y, x, paths = _run(lbm, 512, 512, 32, False, 1, seed=1)
    _check(y, orc.factored_forward(x, paths), "factored")
    _check(y, orc.dense_forward(x, paths), "dense")


@pytest.mark.parametrize("batch", [1, 2, 3, 4, 5, 8, 13, 16])
@pytest.mark.parametrize("residual,s", [(False, 188), (True, 86)])
def test_7b_attention_projection(lbm, batch, residual, s):
    y, x, paths = _run(lbm, 4096, 4096, s, residual, batch, seed=batch)
    _check(y, orc.factored_forward(x, paths), f"B={batch}")


@pytest.mark.parametrize("d_in,d_out,s,residual,batch", [
    (256, 128, 1, False, 1),            # smallest shapes, rank 1
    (256, 128, 1, True, 3),
    (768, 384, 33, True, 2),            # s just over one 32-block
    (4096 + 256, 640, 100, False, 1),   # ragged last input slice
    (8192 + 512, 256, 17, True, 4),     # three slices, last one ragged
    (4096, 11008, 133, True, 1),        # 7B MLP gate/up at 0.1 BPW
    (11008, 4096, 135, True, 2),        # 7B MLP down, the quoted rank
    (1024, 1024, 1024, False, 1),       # maximum rank
    (1024, 512, 1024, True, 16),        # maximum rank, both paths, full batch
    (512, 256, 511, True, 16),          # ragged rank, full batch
    (768, 384, 40, True, 16),           # one partial slice (3 of 8 K-tiles) at batch 16
    (1280, 256, 70, False, 8),          # one partial slice (5 of 8 K-tiles) at batch 8
    (4096, 4096, 86, True, 12),         # three groups of batch rows
])
def test_shapes_and_ragged_edges(lbm, d_in, d_out, s, residual, batch):
    y, x, paths = _run(lbm, d_in, d_out, s, residual, batch, seed=s)
    _check(y, orc.factored_forward(x, paths), f"{d_in}x{d_out} s={s}")


def test_all_plus_signs_and_zero_input(lbm):
    lb, layers = lbm
    d_in, d_out, s = 512, 256, 40
    paths = synth.layer(d_in, d_out, s, False, seed=5)
    paths[0]["U"][:] = 1
    paths[0]["V"][:] = 1
    layer = layers.upload(paths, d_in, d_out, s)
    x = synth.activations(2, d_in, seed=5)
    x[1] = 0
    y = lb.forward(layer, torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    y_ref = orc.factored_forward(x, paths)
    _check(y[:1], y_ref[:1], "all +1")
    assert torch.count_nonzero(y[1]).item() == 0


def test_basis_vector_input_gives_weight_column(lbm):
    lb, layers = lbm
    d_in, d_out, s = 1024, 512, 64
    paths = synth.layer(d_in, d_out, s, True, seed=6)
    layer = layers.upload(paths, d_in, d_out, s)
    W = sum(orc.dense_weight(p) for p in paths)
    x = np.zeros((3, d_in), np.float16)
    cols = [0, 517, 1023]
    for r, i in enumerate(cols):
        x[r, i] = 1.0
    y = lb.forward(layer, torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    _check(y, W[:, cols].T, "basis")


@pytest.mark.parametrize("B", [1, 2])
def test_forward_many_mixed_stack(lbm, B):
    """One forward_many call over layers of different shapes, ranks and path
    counts.  At batch 1 with residual layers the output pass takes both paths
    as one K range (single-path layers, and chunks that span the two paths'
    K-tiles, included)."""
    lb, layers = lbm
    specs = [(4096, 4096, 86, True), (4096, 11008, 133, True), (11008, 4096, 133, True),
             (512, 512, 32, False), (8192, 1024, 620, False)]
    L, X, Y, refs = [], [], [], []
    for i, (a, b, s, r) in enumerate(specs):
        paths = synth.layer(a, b, s, r, seed=100 + i, index=i)
        x = synth.activations(B, a, seed=100 + i, index=i)
        L.append(layers.upload(paths, a, b, s))
        X.append(torch.from_numpy(x).cuda())
        Y.append(torch.empty(B, b, dtype=torch.float16, device="cuda"))
        refs.append(orc.factored_forward(x, paths))
    stack = lb.Stack(L, X, Y)
    for _ in range(3):            # repeated calls reuse the workspace and counters
        for y in Y:
            y.fill_(float("nan"))
        stack()
        torch.cuda.synchronize()
        for i, (y, ref) in enumerate(zip(Y, refs)):
            _check(y, ref, f"layer {i}")


def test_device_status_clean_after_forward(lbm):
    lb, layers = lbm
    paths = synth.layer(2048, 1024, 200, True, seed=4)
    layer = layers.upload(paths, 2048, 1024, 200)
    x = torch.from_numpy(synth.activations(3, 2048, seed=4)).cuda()
    lb.forward(layer, x)
    assert lb.device_status() == 0


def test_bounded_wait_timeout_is_reported_and_recoverable(lbm):
    """The error path of a bounded device wait, run for real: a wait on a
    barrier that nothing completes gives up after 1000 polls (about 1 ms) and
    raises LB_ERR_TIMEOUT; the status read returns the bit and clears it, a
    workspace growth carries an unread bit over, and the stream keeps working."""
    lb, layers = lbm
    timeout_bit = 1 << 5                                         # LB_ERR_TIMEOUT
    st = torch.cuda.Stream()
    lb.check_wait_timeout(st, polls=1000)                        # no workspace yet on this stream
    assert lb.device_status(st) == timeout_bit
    assert lb.device_status(st) == 0

    paths = synth.layer(2048, 1024, 200, True, seed=6)
    layer = layers.upload(paths, 2048, 1024, 200)
    xh = synth.activations(2, 2048, seed=6)
    x = torch.from_numpy(xh).cuda()
    ref = orc.factored_forward(xh, paths)
    st.wait_stream(torch.cuda.current_stream())                  # packed factors and x are ready
    with torch.cuda.stream(st):
        y = lb.forward(layer, x, stream=st)
    assert lb.device_status(st) == 0
    _check(y, ref, "after the self-check")

    lb.check_wait_timeout(st, polls=1000)
    # 16384 inputs at batch 16: about 1.4 MB of scratch, more than the 1 MB
    # workspace the first forward allocated, so this call regrows it
    big = synth.layer(16384, 1024, 300, True, seed=7)
    big_layer = layers.upload(big, 16384, 1024, 300)
    xbh = synth.activations(16, 16384, seed=7)
    xb = torch.from_numpy(xbh).cuda()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        yb = lb.forward(big_layer, xb, stream=st)
    assert lb.device_status(st) == timeout_bit
    _check(yb, orc.factored_forward(xbh, big), "after a workspace growth")
    with torch.cuda.stream(st):
        y2 = lb.forward(layer, x, stream=st)
    assert lb.device_status(st) == 0
    _check(y2, ref, "second forward")


def test_repeatable_and_deterministic(lbm):
    lb, layers = lbm
    paths = synth.layer(4096, 4096, 86, True, seed=9)
    layer = layers.upload(paths, 4096, 4096, 86)
    x = torch.from_numpy(synth.activations(1, 4096, seed=9)).cuda()
    y1 = lb.forward(layer, x).clone()
    y2 = lb.forward(layer, x).clone()
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_full_size_70b_mlp_sampled_rows(lbm):
    """Full-size 70B MLP up projection (8192 -> 28672, single path s = 620,
    batch 1) in the launch configuration of the stack benchmark; the oracle
    checks a sample of output rows one by one."""
    lb, layers = lbm
    gen = torch.Generator(device="cuda").manual_seed(11)
    layer, host = layers.random_layer(8192, 28672, 620, False, gen, keep_signs=True)
    x = torch.randn(1, 8192, generator=gen, device="cuda").half()
    y = lb.forward(layer, x)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(0).choice(28672, 512, replace=False))
    y_ref = orc.factored_forward(x.cpu().numpy(), host, rows=rows)
    _check(y[:, rows], y_ref, "70B sampled")


@pytest.mark.parametrize("B", [1, 3])
def test_forward_many_in_cuda_graph(lbm, B):
    """The decode stack captured into a CUDA graph (on the stream of an earlier
    eager call, whose workspace and tables it reuses) and replayed gives
    exactly what the eager call gave, twice in a row."""
    lb, layers = lbm
    specs = [(4096, 4096, 86, True), (8192, 2048, 620, False), (1024, 4096, 45, True)]
    L, X, Y = [], [], []
    for i, (a, b, s, r) in enumerate(specs):
        paths = synth.layer(a, b, s, r, seed=300 + i, index=i)
        L.append(layers.upload(paths, a, b, s))
        X.append(torch.from_numpy(synth.activations(B, a, seed=300 + i, index=i)).cuda())
        Y.append(torch.empty(B, b, dtype=torch.float16, device="cuda"))
    stack = lb.Stack(L, X, Y)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        stack()
    torch.cuda.synchronize()
    ref = [y.clone() for y in Y]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        stack()
    for _ in range(2):
        for y in Y:
            y.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        for i, (y, r) in enumerate(zip(Y, ref)):
            assert torch.equal(y, r), f"layer {i}"
    del g


@pytest.mark.parametrize("batch", [17, 40, 130])
def test_batches_between_decode_and_prefill(lbm, batch):
    """Batches above 16 that are not a multiple of 128: the leading multiple
    of 128 rows take the prefill path, the rest the decode path in groups of
    at most 16 rows."""
    lb, layers = lbm
    d_in, d_out, s = 1024, 768, 90
    paths = synth.layer(d_in, d_out, s, True, seed=batch)
    x = synth.activations(batch, d_in, seed=batch)
    layer = layers.upload(paths, d_in, d_out, s)
    y = lb.forward(layer, torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    _check(y, orc.factored_forward(x, paths), f"B={batch}")


@pytest.mark.parametrize("d_in,d_out,s,residual,batch", [
    (28672, 8192, 620, False, 1),     # 70B MLP down projection, single path
    (28672, 8192, 620, False, 4),
    (28672, 8192, 302, True, 1),      # 70B MLP down projection, residual
    (28672, 8192, 302, True, 4),
    (8192, 28672, 302, True, 1),      # 70B MLP gate/up, residual
    (8192, 28672, 302, True, 4),
])
def test_full_size_70b_mlp_matrices_sampled_rows(lbm, d_in, d_out, s, residual, batch):
    """Every full-size matrix shape of the 70B MLP stack (14 input slices on
    the down projection; the residual rank s = 302 with both paths), at batch
    1 and 4, in the launch configuration of the stack benchmark: the oracle
    computes 512 sampled output rows of every batch row."""
    lb, layers = lbm
    gen = torch.Generator(device="cuda").manual_seed(d_in + s + batch)
    layer, host = layers.random_layer(d_in, d_out, s, residual, gen, keep_signs=True)
    x = torch.randn(batch, d_in, generator=gen, device="cuda").half()
    y = lb.forward(layer, x)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(d_in).choice(d_out, 512, replace=False))
    y_ref = orc.factored_forward(x.cpu().numpy(), host, rows=rows)
    _check(y[:, rows], y_ref, f"{d_in}->{d_out} s={s} res={residual} B={batch}")
    assert lb.device_status() == 0


def _outlier_activations(batch, d_in, seed, frac=0.01):
    """x ~ N(0,1) with a fraction `frac` of the entries scaled by 10^2..10^3
    (log-uniform): the heavy-tailed activations of real LLM layers."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((batch, d_in))
    mask = rng.random((batch, d_in)) < frac
    x[mask] *= 10.0 ** rng.uniform(2.0, 3.0, size=int(mask.sum()))
    return x.astype(np.float16)


@pytest.mark.parametrize("d_in,d_out,s,residual", [(4096, 4096, 86, True), (11008, 4096, 133, True),
                                                   (4096, 4096, 188, False)])
@pytest.mark.parametrize("batch", [1, 16])
def test_outlier_activations(lbm, d_in, d_out, s, residual, batch):
    """Outlier activations (1 % of the entries 100-1000x the rest): the 16-bit
    fixed point of g*x per input slice and batch row keeps the result within
    the forward's tolerances."""
    lb, layers = lbm
    paths = synth.layer(d_in, d_out, s, residual, seed=s + batch)
    x = _outlier_activations(batch, d_in, seed=s + batch)
    layer = layers.upload(paths, d_in, d_out, s)
    y = lb.forward(layer, torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    _check(y, orc.factored_forward(x, paths), f"outliers B={batch}")


@pytest.mark.parametrize("batch", [1, 4])
def test_single_outlier_per_slice_and_small_rows(lbm, batch):
    """The worst case for a per-slice step: one entry per 2048-input slice at
    4000x the rest, and batch rows of very different magnitude (each row has
    its own step)."""
    lb, layers = lbm
    d_in, d_out, s = 8192, 2048, 150
    paths = synth.layer(d_in, d_out, s, True, seed=77)
    rng = np.random.default_rng(77)
    x = rng.standard_normal((batch, d_in))
    for sl in range(d_in // 2048):
        x[:, sl * 2048 + rng.integers(0, 2048)] = 4000.0
    x *= (10.0 ** -np.arange(batch))[:, None]          # rows 1, 0.1, 0.01, ...
    x = x.astype(np.float16)
    layer = layers.upload(paths, d_in, d_out, s)
    y = lb.forward(layer, torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    y_ref = orc.factored_forward(x, paths)
    for b in range(batch):   # each row on its own scale
        _check(y[b:b + 1], y_ref[b:b + 1], f"row {b}")


def test_nonfinite_decode_input_is_reported(lbm):
    """An inf or NaN in x cannot be quantised: the decode forward raises
    LB_ERR_RANGE in the device status, and the next clean call raises nothing."""
    lb, layers = lbm
    range_bit = 1 << 7
    d_in, d_out, s = 2048, 512, 64
    paths = synth.layer(d_in, d_out, s, True, seed=23)
    layer = layers.upload(paths, d_in, d_out, s)
    xh = synth.activations(3, d_in, seed=23)
    for bad in (float("inf"), float("nan")):
        x = torch.from_numpy(xh).cuda()
        x[1, 1000] = bad
        lb.forward(layer, x)
        assert lb.device_status() & range_bit
    y = lb.forward(layer, torch.from_numpy(xh).cuda())
    assert lb.device_status() == 0
    _check(y, orc.factored_forward(xh, paths), "after a non-finite input")


@pytest.mark.parametrize("B", [1, 3, 16])
def test_forward_many_shared_inputs(lbm, B):
    """Layers of one call that read the same x (a block's q, k and v
    projections; gate and up) are quantised from one read of x: every
    layer's output still matches the oracle, and a layer listed twice with
    the same input gives identical outputs."""
    lb, layers = lbm
    groups = [[(4096, 4096, 86, True)] * 3, [(4096, 4096, 86, True)], [(4096, 11008, 133, True)] * 2,
              [(11008, 4096, 133, True)], [(1024, 512, 40, False), (1024, 768, 300, True)]]
    L, X, Y, refs = [], [], [], []
    k = 0
    for g, members in enumerate(groups):
        xh = synth.activations(B, members[0][0], seed=200 + g, index=g)
        x = torch.from_numpy(xh).cuda()
        for (a, b, s, r) in members:
            paths = synth.layer(a, b, s, r, seed=400 + k, index=k)
            L.append(layers.upload(paths, a, b, s))
            X.append(x)
            Y.append(torch.full((B, b), float("nan"), dtype=torch.float16, device="cuda"))
            refs.append(orc.factored_forward(xh, paths))
            k += 1
    # the same layer twice on the same input
    L.append(L[0])
    X.append(X[0])
    Y.append(torch.empty_like(Y[0]))
    refs.append(refs[0])
    lb.Stack(L, X, Y)()
    torch.cuda.synchronize()
    for i, (y, ref) in enumerate(zip(Y, refs)):
        _check(y, ref, f"layer {i}")
    assert torch.equal(Y[0], Y[-1])
    assert lb.device_status() == 0
