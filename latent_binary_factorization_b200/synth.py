"""Seeded synthetic inputs for the LittleBit layer.

This module only draws random numbers; it holds none of the layer's
arithmetic, so both the CUDA path and the CPU oracle can be fed from it.

Recipe (the shapes and distributions of the Llama-2-shaped workloads):
  x        ~ N(0, 1), rounded to fp16 (decode) or bf16 (prefill)
  U, V     i.i.d. fair +-1 signs
  h, g, l  ~ Uniform[0.5, 1.5] / sqrt(s), rounded to fp16
Each tensor gets its own stream, spawned from one ``numpy.random.SeedSequence``
per (seed, layer) so that a layer's tensors do not depend on the others.
"""
from __future__ import annotations

import numpy as np

_TENSORS = ("x", "V0", "U0", "h0", "g0", "l0", "V1", "U1", "h1", "g1", "l1", "F")


def _rng(seed: int, layer: int, name: str) -> np.random.Generator:
    ss = np.random.SeedSequence([seed, layer, _TENSORS.index(name)])
    return np.random.default_rng(ss)


def signs(rng: np.random.Generator, shape) -> np.ndarray:
    """Fair +-1 signs as int8."""
    return (1 - 2 * rng.integers(0, 2, size=shape, dtype=np.int8)).astype(np.int8)


def scales(rng: np.random.Generator, n: int, s: int) -> np.ndarray:
    return (rng.uniform(0.5, 1.5, size=n) / np.sqrt(s)).astype(np.float16)


def layer(d_in: int, d_out: int, s: int, residual: bool, seed: int = 0, index: int = 0) -> list[dict]:
    """One LittleBit layer: a list of 1 or 2 paths, each a dict of numpy arrays.

    U (d_out, s) int8 +-1, V (d_in, s) int8 +-1, h (d_out,), g (d_in,), l (s,) fp16.
    """
    paths = []
    for p in range(2 if residual else 1):
        paths.append(
            {
                "U": signs(_rng(seed, index, f"U{p}"), (d_out, s)),
                "V": signs(_rng(seed, index, f"V{p}"), (d_in, s)),
                "h": scales(_rng(seed, index, f"h{p}"), d_out, s),
                "g": scales(_rng(seed, index, f"g{p}"), d_in, s),
                "l": scales(_rng(seed, index, f"l{p}"), s, s),
            }
        )
    return paths


def activations(batch: int, d_in: int, seed: int = 0, index: int = 0, dtype: str = "f16") -> np.ndarray:
    """x ~ N(0,1) as fp16 (numpy) or, for dtype="bf16", as float32 values that
    are exactly representable in bf16 (round-to-nearest-even of the fp32 draw)."""
    x = _rng(seed, index, "x").standard_normal((batch, d_in)).astype(np.float32)
    if dtype == "f16":
        return x.astype(np.float16)
    if dtype == "bf16":
        return round_to_bf16(x)
    raise ValueError(dtype)


def real_factor(rows: int, cols: int, seed: int = 0, index: int = 0, zeros: float = 0.0) -> np.ndarray:
    """Real-valued float32 matrix ~ N(0,1) for the pack tests; a fraction
    ``zeros`` of the entries is set to +0.0 or -0.0."""
    rng = _rng(seed, index, "F")
    F = rng.standard_normal((rows, cols)).astype(np.float32)
    if zeros > 0:
        mask = rng.random((rows, cols)) < zeros
        neg = rng.random((rows, cols)) < 0.5
        F[mask & ~neg] = 0.0
        F[mask & neg] = -0.0
    return F


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returned as float32."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    r = ((b + 0x7FFF + lsb) >> 16) << 16
    return r.astype(np.uint32).view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """uint16 bf16 encodings of float32 values that are already bf16-exact."""
    return (np.ascontiguousarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)
