"""Thin ctypes binding of liblittlebit.so (include/littlebit.h).

Argument marshalling only: every step of the layer runs in the CUDA library.
Tensors are torch CUDA tensors (torch supplies device memory and streams).
If the library has not been built, importing this module raises ImportError;
there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblittlebit.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -c 'import __graft_entry__ as g; g.build()'` "
        "(the LittleBit layer has no CPU implementation)"
    )

_lib = ctypes.CDLL(LIB_PATH)

LB_F16, LB_BF16, LB_F32, LB_I8 = 0, 1, 2, 3
LB_ROLE_V, LB_ROLE_U = 0, 1
ROLE = {"V": LB_ROLE_V, "U": LB_ROLE_U}
STATUS = {0: "LB_OK", 1: "LB_ERR_ARG", 2: "LB_ERR_ALIGN", 3: "LB_ERR_SHAPE", 4: "LB_ERR_CUDA",
          5: "LB_ERR_TIMEOUT", 6: "LB_ERR_UNSUPPORTED", 7: "LB_ERR_RANGE"}
_DTYPE = {torch.float16: LB_F16, torch.bfloat16: LB_BF16, torch.float32: LB_F32, torch.int8: LB_I8}


class LbPath(ctypes.Structure):
    _fields_ = [("V_bits", ctypes.c_void_p), ("U_bits", ctypes.c_void_p), ("h", ctypes.c_void_p),
                ("g", ctypes.c_void_p), ("l", ctypes.c_void_p)]


class LbLayer(ctypes.Structure):
    _fields_ = [("d_in", ctypes.c_int), ("d_out", ctypes.c_int), ("s", ctypes.c_int),
                ("residual", ctypes.c_int), ("path", LbPath * 2)]


_lib.littlebit_packed_bytes.restype = ctypes.c_size_t
_lib.littlebit_packed_bytes.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
_lib.littlebit_eff_bits.restype = ctypes.c_double
_lib.littlebit_eff_bits.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
_lib.littlebit_pack_signs.restype = ctypes.c_int
_lib.littlebit_pack_signs.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p,
                                      ctypes.c_void_p]
_lib.littlebit_unpack_signs.restype = ctypes.c_int
_lib.littlebit_unpack_signs.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                        ctypes.c_void_p]
_lib.littlebit_linear_forward.restype = ctypes.c_int
_lib.littlebit_linear_forward.argtypes = [ctypes.POINTER(LbLayer), ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
_lib.littlebit_linear_forward_many.restype = ctypes.c_int
_lib.littlebit_linear_forward_many.argtypes = [ctypes.POINTER(LbLayer), ctypes.c_int,
                                               ctypes.POINTER(ctypes.c_void_p),
                                               ctypes.POINTER(ctypes.c_void_p), ctypes.c_int, ctypes.c_int,
                                               ctypes.c_void_p]
_lib.littlebit_linear_forward_many_timed.restype = ctypes.c_int
_lib.littlebit_linear_forward_many_timed.argtypes = [ctypes.POINTER(LbLayer), ctypes.c_int,
                                                     ctypes.POINTER(ctypes.c_void_p),
                                                     ctypes.POINTER(ctypes.c_void_p), ctypes.c_int, ctypes.c_int,
                                                     ctypes.c_void_p, ctypes.POINTER(ctypes.c_void_p), ctypes.c_int]
_lib.littlebit_linear_forward_many_host.restype = ctypes.c_int
_lib.littlebit_linear_forward_many_host.argtypes = [ctypes.POINTER(LbLayer), ctypes.c_int, ctypes.c_void_p,
                                                    ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                    ctypes.c_void_p]
_lib.littlebit_latent_row_elems.restype = ctypes.c_int
_lib.littlebit_latent_row_elems.argtypes = [ctypes.c_int, ctypes.c_int]
for _name in ("littlebit_latent_forward", "littlebit_latent_expand"):
    getattr(_lib, _name).restype = ctypes.c_int
    getattr(_lib, _name).argtypes = [ctypes.POINTER(LbLayer), ctypes.c_int, ctypes.POINTER(ctypes.c_void_p),
                                     ctypes.POINTER(ctypes.c_void_p), ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
_lib.littlebit_init_dual_svid.restype = ctypes.c_int
_lib.littlebit_init_dual_svid.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
_lib.littlebit_joint_itq.restype = ctypes.c_int
_lib.littlebit_joint_itq.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                     ctypes.c_int, ctypes.c_void_p]
_lib.littlebit_device_status.restype = ctypes.c_int
_lib.littlebit_device_status.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_uint)]
_lib.littlebit_check_wait_timeout.restype = ctypes.c_int
_lib.littlebit_check_wait_timeout.argtypes = [ctypes.c_void_p, ctypes.c_int]
_lib.littlebit_release.restype = None
_lib.littlebit_release.argtypes = []
_lib.littlebit_status_string.restype = ctypes.c_char_p
_lib.littlebit_status_string.argtypes = [ctypes.c_int]
_lib.littlebit_last_cuda_error.restype = ctypes.c_char_p
_lib.littlebit_last_cuda_error.argtypes = []


class LittleBitError(RuntimeError):
    def __init__(self, code: int, where: str):
        msg = _lib.littlebit_status_string(code).decode()
        if code == 4:
            msg += f" ({_lib.littlebit_last_cuda_error().decode()})"
        super().__init__(f"{where}: {msg}")
        self.code = code
        self.status = STATUS.get(code, str(code))


def _check(code: int, where: str) -> None:
    if code != 0:
        raise LittleBitError(code, where)


def _stream(stream=None) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _activation(t: torch.Tensor, rows: int | None, cols: int, name: str) -> None:
    """A row-major (rows x cols) CUDA activation buffer: the library reads and
    writes it through a raw pointer, so a CPU tensor or a strided view would
    be misread."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dim() != 2 or t.shape[1] != cols or (rows is not None and t.shape[0] != rows):
        raise ValueError(f"{name} must have shape ({rows if rows is not None else 'batch'}, {cols}), "
                         f"got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def library():
    """The loaded ctypes CDLL (for tests that call the C ABI directly)."""
    return _lib


def packed_bytes(role: str, rows: int, cols: int) -> int:
    return int(_lib.littlebit_packed_bytes(ROLE[role], rows, cols))


def eff_bits(d_in: int, d_out: int, s: int, residual: bool) -> float:
    return float(_lib.littlebit_eff_bits(d_in, d_out, s, int(bool(residual))))


def pack_signs(factor: torch.Tensor, role: str, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Pack the signs of a CUDA factor tensor (V: d_in x s, U: d_out x s)."""
    if factor.dim() != 2 or not factor.is_cuda:
        raise ValueError("factor must be a 2-D CUDA tensor")
    n_long, s = factor.shape
    rows, cols = (s, n_long) if role == "V" else (n_long, s)
    nbytes = packed_bytes(role, rows, cols)
    if out is None:
        out = torch.empty(nbytes, dtype=torch.uint8, device=factor.device)
    if out.numel() < nbytes:
        raise ValueError("output buffer too small")
    _check(_lib.littlebit_pack_signs(ctypes.c_void_p(factor.data_ptr()), _DTYPE[factor.dtype], n_long, s,
                                     factor.stride(0), factor.stride(1), ROLE[role],
                                     ctypes.c_void_p(out.data_ptr()), _stream(stream)),
           "littlebit_pack_signs")
    return out


def unpack_signs(packed: torch.Tensor, role: str, n_long: int, s: int, stream=None) -> torch.Tensor:
    """Packed factor bytes (CUDA) back to its +-1 values, n_long x s int8."""
    out = torch.empty((n_long, s), dtype=torch.int8, device=packed.device)
    _check(_lib.littlebit_unpack_signs(ctypes.c_void_p(packed.data_ptr()), ROLE[role], n_long, s,
                                       ctypes.c_void_p(out.data_ptr()), _stream(stream)),
           "littlebit_unpack_signs")
    return out


@dataclass
class Path:
    """One path of a layer, all CUDA tensors: packed V/U bytes, fp16 h, g, l."""
    V_bits: torch.Tensor
    U_bits: torch.Tensor
    h: torch.Tensor
    g: torch.Tensor
    l: torch.Tensor


@dataclass
class Layer:
    d_in: int
    d_out: int
    s: int
    paths: list = field(default_factory=list)

    @property
    def residual(self) -> bool:
        return len(self.paths) == 2

    def c_struct(self) -> LbLayer:
        if len(self.paths) not in (1, 2):
            raise ValueError("a layer has one path, or two with residual compensation")
        for p in self.paths:
            for name in ("V_bits", "U_bits", "h", "g", "l"):
                if not getattr(p, name).is_cuda:
                    raise ValueError(f"path tensor {name} must be a CUDA tensor")
        L = LbLayer()
        L.d_in, L.d_out, L.s, L.residual = self.d_in, self.d_out, self.s, int(self.residual)
        for i, p in enumerate(self.paths):
            L.path[i] = LbPath(p.V_bits.data_ptr(), p.U_bits.data_ptr(), p.h.data_ptr(), p.g.data_ptr(),
                               p.l.data_ptr())
        return L


def forward(layer: Layer, x: torch.Tensor, y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y = layer(x); x is (batch, d_in) fp16 (decode) on the layer's device."""
    _activation(x, None, layer.d_in, "x")
    batch = x.shape[0]
    if y is None:
        y = torch.empty((batch, layer.d_out), dtype=x.dtype, device=x.device)
    _activation(y, batch, layer.d_out, "y")
    if y.dtype != x.dtype:
        raise ValueError("y must have x's dtype")
    L = layer.c_struct()
    _check(_lib.littlebit_linear_forward(ctypes.byref(L), ctypes.c_void_p(x.data_ptr()),
                                         ctypes.c_void_p(y.data_ptr()), batch, _DTYPE[x.dtype], _stream(stream)),
           "littlebit_linear_forward")
    return y


class Stack:
    """A list of independent layers run by one forward_many call per step.

    Holds the marshalled C structs and pointer arrays so that repeated calls
    do no Python-side allocation."""

    def __init__(self, layers: list, xs: list, ys: list):
        if not layers or not len(layers) == len(xs) == len(ys):
            raise ValueError("layers, xs and ys must be non-empty lists of the same length")
        self.layers, self.xs, self.ys = layers, xs, ys
        self.batch = xs[0].shape[0]
        for i, (L, x, y) in enumerate(zip(layers, xs, ys)):
            _activation(x, self.batch, L.d_in, f"xs[{i}]")
            _activation(y, self.batch, L.d_out, f"ys[{i}]")
            if x.dtype != xs[0].dtype or y.dtype != x.dtype:
                raise ValueError(f"xs[{i}] and ys[{i}] must share xs[0]'s dtype")
        self.dtype = _DTYPE[xs[0].dtype]
        n = len(layers)
        self._n = n
        self._arr = (LbLayer * n)(*[L.c_struct() for L in layers])
        self._xp = (ctypes.c_void_p * n)(*[x.data_ptr() for x in xs])
        self._yp = (ctypes.c_void_p * n)(*[y.data_ptr() for y in ys])

    def __call__(self, stream=None, events: list | None = None) -> None:
        """One forward of every layer.  ``events`` (decode only): up to three
        torch.cuda.Event recorded after the quantise, latent and finalize
        launches (the output pass follows the last)."""
        if not events:
            _check(_lib.littlebit_linear_forward_many(self._arr, self._n, self._xp, self._yp, self.batch,
                                                      self.dtype, _stream(stream)),
                   "littlebit_linear_forward_many")
        else:
            evs = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
            _check(_lib.littlebit_linear_forward_many_timed(self._arr, self._n, self._xp, self._yp, self.batch,
                                                            self.dtype, _stream(stream), evs, len(events)),
                   "littlebit_linear_forward_many_timed")


class HostStack:
    """A list of independent layers whose activations live in host memory.

    One call copies every layer's input in, runs the stack forward and copies
    every output back, in ``n_chunks`` groups of layers whose copies overlap
    the neighbouring groups' kernels.  ``x_host`` holds the layers' inputs
    back to back (layer i: batch x d_in[i], row-major), ``y_host`` the outputs
    the same way; both CPU tensors, page-locked (``pin_memory=True``) for the
    overlap.  y_host is complete once the stream has been synchronised."""

    def __init__(self, layers: list, batch: int, dtype=torch.float16):
        assert layers and batch >= 1
        self.layers, self.batch, self.dtype = layers, batch, dtype
        self._n = len(layers)
        self._arr = (LbLayer * self._n)(*[L.c_struct() for L in layers])
        self.x_numel = batch * sum(L.d_in for L in layers)
        self.y_numel = batch * sum(L.d_out for L in layers)

    def __call__(self, x_host: torch.Tensor, y_host: torch.Tensor, n_chunks: int = 8, stream=None) -> None:
        for t, numel in ((x_host, self.x_numel), (y_host, self.y_numel)):
            if t.device.type != "cpu" or not t.is_contiguous() or t.numel() != numel or t.dtype != self.dtype:
                raise ValueError(f"host buffer must be a contiguous CPU {self.dtype} tensor of {numel} elements")
        _check(_lib.littlebit_linear_forward_many_host(self._arr, self._n, ctypes.c_void_p(x_host.data_ptr()),
                                                       ctypes.c_void_p(y_host.data_ptr()), self.batch,
                                                       _DTYPE[self.dtype], int(n_chunks), _stream(stream)),
               "littlebit_linear_forward_many_host")


def latent_row_elems(layer: Layer) -> int:
    """fp16 elements between a layer's latent cache rows (npaths*s rounded up
    to a multiple of 8)."""
    return int(_lib.littlebit_latent_row_elems(layer.s, int(layer.residual)))


def _ptrs(ts):
    return (ctypes.c_void_p * len(ts))(*[t.data_ptr() for t in ts])


def latent_forward(layers: list, xs: list, ts: list | None = None, stream=None) -> list:
    """Latent cache rows of each layer's input: ts[i] = [t'_1 | t'_2] of xs[i]
    (fp16, batch x latent_row_elems), the K/V projection kept as its latent."""
    batch = xs[0].shape[0]
    for i, (L, x) in enumerate(zip(layers, xs)):
        _activation(x, batch, L.d_in, f"xs[{i}]")
    if ts is None:
        ts = [torch.empty((batch, latent_row_elems(L)), dtype=torch.float16, device=x.device)
              for L, x in zip(layers, xs)]
    for i, (L, t) in enumerate(zip(layers, ts)):
        _activation(t, batch, latent_row_elems(L), f"ts[{i}]")
        if t.dtype != torch.float16:
            raise ValueError("cache rows are fp16")
    arr = (LbLayer * len(layers))(*[L.c_struct() for L in layers])
    _check(_lib.littlebit_latent_forward(arr, len(layers), _ptrs(xs), _ptrs(ts), batch, _DTYPE[xs[0].dtype],
                                         _stream(stream)), "littlebit_latent_forward")
    return ts


def latent_expand(layers: list, ts: list, ys: list | None = None, dtype=torch.float16, stream=None) -> list:
    """Projections rebuilt from cache rows: ys[i] = sum_p h_p (.) U_p t'_p."""
    rows = ts[0].shape[0]
    for i, (L, t) in enumerate(zip(layers, ts)):
        _activation(t, rows, latent_row_elems(L), f"ts[{i}]")
        if t.dtype != torch.float16:
            raise ValueError("cache rows are fp16")
    if ys is None:
        ys = [torch.empty((rows, L.d_out), dtype=dtype, device=t.device) for L, t in zip(layers, ts)]
    for i, (L, y) in enumerate(zip(layers, ys)):
        _activation(y, rows, L.d_out, f"ys[{i}]")
    arr = (LbLayer * len(layers))(*[L.c_struct() for L in layers])
    _check(_lib.littlebit_latent_expand(arr, len(layers), _ptrs(ts), _ptrs(ys), rows, _DTYPE[ys[0].dtype],
                                        _stream(stream)), "littlebit_latent_expand")
    return ys


def _f32_rows(t: torch.Tensor, rows: int, cols: int, name: str) -> None:
    if not (isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == torch.float32 and t.is_contiguous()
            and tuple(t.shape) == (rows, cols)):
        raise ValueError(f"{name} must be a contiguous CUDA float32 tensor of shape ({rows}, {cols})")


def init_dual_svid(Uf: torch.Tensor, Vf: torch.Tensor, iters: int = 32, stream=None) -> Path:
    """One path from real factors U' (d_out x s) and V' (d_in x s), fp32 CUDA:
    packed signs and the rank-1 magnitude scales h, g, l (fp16)."""
    d_out, s = Uf.shape
    d_in = Vf.shape[0]
    _f32_rows(Uf, d_out, s, "Uf")
    _f32_rows(Vf, d_in, s, "Vf")
    dev = Uf.device
    p = Path(V_bits=torch.empty(packed_bytes("V", s, d_in), dtype=torch.uint8, device=dev),
             U_bits=torch.empty(packed_bytes("U", d_out, s), dtype=torch.uint8, device=dev),
             h=torch.empty(d_out, dtype=torch.float16, device=dev), g=torch.empty(d_in, dtype=torch.float16, device=dev),
             l=torch.empty(s, dtype=torch.float16, device=dev))
    _check(_lib.littlebit_init_dual_svid(ctypes.c_void_p(Uf.data_ptr()), ctypes.c_void_p(Vf.data_ptr()), d_out, d_in,
                                         s, int(iters), ctypes.c_void_p(p.U_bits.data_ptr()),
                                         ctypes.c_void_p(p.V_bits.data_ptr()), ctypes.c_void_p(p.h.data_ptr()),
                                         ctypes.c_void_p(p.g.data_ptr()), ctypes.c_void_p(p.l.data_ptr()),
                                         _stream(stream)), "littlebit_init_dual_svid")
    return p


def joint_itq(X: torch.Tensor, iters: int = 50, R: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Rotate the stacked factors X = [U'; V'] ((d_out + d_in) x s, fp32 CUDA)
    in place by the Joint-ITQ rotation; returns R (s x s).  With R given, the
    alternations start from it (and it is overwritten)."""
    n_rows, s = X.shape
    _f32_rows(X, n_rows, s, "X")
    given = R is not None
    if R is None:
        R = torch.empty((s, s), dtype=torch.float32, device=X.device)
    _f32_rows(R, s, s, "R")
    _check(_lib.littlebit_joint_itq(ctypes.c_void_p(X.data_ptr()), n_rows, s, int(iters), ctypes.c_void_p(R.data_ptr()),
                                    int(given), _stream(stream)), "littlebit_joint_itq")
    return R


def forward_many(layers: list, xs: list, ys: list, stream=None) -> None:
    Stack(layers, xs, ys)(stream)


def device_status(stream=None) -> int:
    """Wait for the stream and return (and clear) the device error bits its
    forward kernels raised; 0 means none."""
    out = ctypes.c_uint(0)
    _check(_lib.littlebit_device_status(_stream(stream), ctypes.byref(out)), "littlebit_device_status")
    return int(out.value)


def check_wait_timeout(stream=None, polls: int = 1000) -> None:
    """Enqueue the self-check of the bounded-wait error path: a wait on a
    barrier that nothing completes gives up after `polls` polls and raises
    the LB_ERR_TIMEOUT bit, which the next device_status() returns."""
    _check(_lib.littlebit_check_wait_timeout(_stream(stream), int(polls)), "littlebit_check_wait_timeout")


def release() -> None:
    _lib.littlebit_release()
