"""CPU-side checks of the C-ABI library: it loads, exports every entry point
the header declares, and its host-only functions agree with the oracle."""
import ctypes
import os
import re

import pytest

from oracle import littlebit_oracle as orc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "latent_binary_factorization_b200", "liblittlebit.so")


def _header_functions():
    funcs = set()
    for name in os.listdir(os.path.join(ROOT, "include")):
        if name.endswith(".h"):
            with open(os.path.join(ROOT, "include", name)) as f:
                text = f.read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            funcs |= set(re.findall(r"\b(littlebit_\w+)\s*\(", text))
    return sorted(funcs)


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        from latent_binary_factorization_b200 import build_ext
        build_ext.build()
    return ctypes.CDLL(LIB)


def test_header_declares_entry_points():
    funcs = _header_functions()
    for f in ("littlebit_pack_signs", "littlebit_linear_forward", "littlebit_linear_forward_many",
              "littlebit_packed_bytes", "littlebit_eff_bits"):
        assert f in funcs


def test_library_exports_every_declared_symbol(lib):
    for f in _header_functions():
        assert hasattr(lib, f), f"{f} declared in include/ but not exported"


def test_host_functions_match_oracle(lib):
    lib.littlebit_eff_bits.restype = ctypes.c_double
    lib.littlebit_eff_bits.argtypes = [ctypes.c_int] * 4
    lib.littlebit_packed_bytes.restype = ctypes.c_size_t
    lib.littlebit_packed_bytes.argtypes = [ctypes.c_int] * 3
    for a, b, s, r in [(4096, 4096, 86, 1), (8192, 28672, 620, 0), (512, 512, 32, 0), (4096, 11008, 133, 1)]:
        assert lib.littlebit_eff_bits(a, b, s, r) == pytest.approx(orc.eff_bits(a, b, s, bool(r)), rel=1e-15)
    for role, code in (("V", 0), ("U", 1)):
        for R, K in [(86, 4096), (1, 256), (620, 28672), (4096, 86), (128, 1), (11008, 133)]:
            assert lib.littlebit_packed_bytes(code, R, K) == orc.packed_nbytes(role, R, K)


def test_status_strings(lib):
    lib.littlebit_status_string.restype = ctypes.c_char_p
    lib.littlebit_status_string.argtypes = [ctypes.c_int]
    for code in range(7):
        assert lib.littlebit_status_string(code).startswith(b"LB_")


def test_forward_rejects_bad_arguments_without_device_work(lib):
    """Argument checks happen on the host before any CUDA call."""
    from latent_binary_factorization_b200 import littlebit as lb
    L = lb.LbLayer()
    L.d_in, L.d_out, L.s, L.residual = 100, 128, 4, 0       # d_in not a multiple of 256
    f = lb.library().littlebit_linear_forward
    x = ctypes.c_void_p(16)
    assert f(ctypes.byref(L), x, x, 1, 0, None) == 3           # LB_ERR_SHAPE
    L.d_in, L.s = 256, 0
    assert f(ctypes.byref(L), x, x, 1, 0, None) == 3           # s < 1
    L.s = 4
    assert f(ctypes.byref(L), x, x, 1, 0, None) == 1           # null factor pointers
    for p in range(2):
        L.path[p] = lb.LbPath(16, 32, 64, 48, 6)
    L.residual = 2
    assert f(ctypes.byref(L), x, x, 1, 0, None) == 1           # residual must be 0/1
    L.residual = 0
    L.path[0] = lb.LbPath(8, 32, 64, 48, 6)                      # V not 16-byte aligned
    assert f(ctypes.byref(L), x, x, 1, 0, None) == 2
    L.path[0] = lb.LbPath(16, 32, 64, 40, 6)                     # g not 16-byte aligned
    assert f(ctypes.byref(L), x, x, 1, 0, None) == 2
    L.path[0] = lb.LbPath(16, 32, 66, 48, 6)                     # h not 16-byte aligned
    assert f(ctypes.byref(L), x, x, 1, 0, None) == 2
    L.path[0] = lb.LbPath(16, 32, 64, 48, 6)
    assert f(ctypes.byref(L), ctypes.c_void_p(24), x, 1, 0, None) == 2   # x misaligned
    assert f(ctypes.byref(L), x, x, 0, 0, None) == 3           # batch 0
    assert f(ctypes.byref(L), x, x, 100, 1, None) == 6         # bf16 off a multiple of 128 rows
    assert f(ctypes.byref(L), x, x, 100, 2, None) == 6         # f32 activations
    assert f(ctypes.byref(L), x, x, 1, 1, None) == 6           # decode wants fp16
    pack = lb.library().littlebit_pack_signs
    assert pack(None, 0, 4, 4, 4, 1, 0, ctypes.c_void_p(16), None) == 1
    assert pack(ctypes.c_void_p(16), 9, 4, 4, 4, 1, 0, ctypes.c_void_p(16), None) == 1
    assert pack(ctypes.c_void_p(16), 0, 0, 4, 4, 1, 0, ctypes.c_void_p(16), None) == 3
    assert pack(ctypes.c_void_p(16), 0, 4, 4, 4, 1, 0, ctypes.c_void_p(8), None) == 2
    host = lb.library().littlebit_linear_forward_many_host
    hx = ctypes.c_void_p(4096)                                   # never dereferenced: rejected first
    assert host(ctypes.byref(L), 1, None, hx, 1, 0, 4, None) == 1            # null x_host
    assert host(ctypes.byref(L), 1, hx, hx, 1, 0, 0, None) == 1              # n_chunks < 1
    assert host(ctypes.byref(L), 0, hx, hx, 1, 0, 4, None) == 1              # no layers
    assert host(ctypes.byref(L), 1, hx, hx, 1, 2, 4, None) == 6              # f32 activations
    L.d_in = 100
    assert host(ctypes.byref(L), 1, hx, hx, 1, 0, 4, None) == 3              # bad layer shape
    L.d_in = 256
    chk = lb.library().littlebit_check_wait_timeout
    assert chk(None, 0) == 1                                     # polls < 1
    assert chk(None, (1 << 22) + 1) == 1                         # polls above the kernels' own limit


def test_header_compiles_as_c_and_links(tmp_path):
    """A C program (tests/c_abi_host_check.c) compiles against the header with
    a C compiler, links with the library and runs its host entry points."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    exe = tmp_path / "c_abi_host_check"
    libdir = os.path.dirname(LIB)
    subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_host_check.c"), "-o", str(exe),
                    "-L", libdir, "-llittlebit", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    from oracle import littlebit_oracle as orc
    assert abs(float(out[0].split()[1]) - float(orc.eff_bits_exact(4096, 4096, 86, True))) < 1e-8
    assert int(out[1].split()[1]) == orc.packed_nbytes("V", 86, 4096)
    assert out[2] == "forward 3"
    assert out[3].startswith("status LB_ERR_SHAPE")
    assert out[4] == "host 1"


def test_binding_rejects_buffers_the_library_would_misread():
    """CPU tensors, strided views and wrong shapes are refused in Python,
    before a pointer reaches the library (a host pointer would fault a kernel)."""
    import torch
    from latent_binary_factorization_b200 import littlebit as lb
    z = torch.zeros(16, dtype=torch.uint8)
    s16 = torch.zeros(256, dtype=torch.float16)
    layer = lb.Layer(256, 128, 4, [lb.Path(z, z, s16[:128], s16, s16[:4])])
    with pytest.raises(ValueError):
        layer.c_struct()                                       # path tensors on the CPU
    with pytest.raises(ValueError):
        lb.forward(layer, torch.zeros(1, 256, dtype=torch.float16))   # x on the CPU
    with pytest.raises(ValueError):
        lb.Stack([layer], [], [])                              # lengths differ
    with pytest.raises(ValueError):
        lb.Stack([layer], [torch.zeros(1, 256, dtype=torch.float16)], [torch.zeros(1, 128, dtype=torch.float16)])
    with pytest.raises(ValueError):
        lb.Layer(256, 128, 4, []).c_struct()                   # no path
    with pytest.raises(ValueError):
        lb.HostStack([layer], 1)                               # path tensors on the CPU


PER_DEVICE_CHECK = r"""
#include <cstdio>
#include "per_device.h"
int main() {
  lb::PerDevice cache;
  int runs = 0, v = 0;
  auto init = [&](int dev) { return [&, dev](int& out) { ++runs; out = 100 + dev; return 0; }; };
  // first use on device 0 runs the set-up; device 1 has its own slot
  if (cache.get(0, v, init(0)) || v != 100 || runs != 1) return 1;
  if (cache.get(1, v, init(1)) || v != 101 || runs != 2) return 2;
  // later uses return each device's own value without running it again
  if (cache.get(0, v, init(0)) || v != 100 || runs != 2) return 3;
  if (cache.get(1, v, init(1)) || v != 101 || runs != 2) return 4;
  // a failed set-up is reported and leaves nothing cached
  int fails = 0;
  if (cache.get(2, v, [&](int& out) { ++fails; out = 7; return 9; }) != 9) return 5;
  if (cache.get(2, v, [&](int& out) { ++fails; out = 7; return 0; }) || v != 7 || fails != 2) return 6;
  // an ordinal outside the table runs the set-up every time
  if (cache.get(lb::kMaxDevices, v, init(0)) || cache.get(lb::kMaxDevices, v, init(0)) || runs != 4) return 7;
  std::puts("ok");
  return 0;
}
"""


def test_kernel_attribute_caches_are_per_device(tmp_path):
    """The launch set-up caches (shared-memory attribute, occupancy) are kept
    per device ordinal: a process driving two GPUs sets each one up."""
    import shutil
    import subprocess
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("no g++")
    src = tmp_path / "per_device_check.cc"
    src.write_text(PER_DEVICE_CHECK)
    exe = tmp_path / "per_device_check"
    csrc = os.path.join(ROOT, "latent_binary_factorization_b200", "csrc")
    subprocess.run([gxx, "-std=c++17", "-O1", "-I", csrc, str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.returncode
