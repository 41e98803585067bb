"""Building packed LittleBit layers on the GPU (factors packed by the CUDA kernel)."""
from __future__ import annotations

import math

import numpy as np
import torch

from . import littlebit as lb


def upload(paths: list, d_in: int, d_out: int, s: int, device="cuda") -> lb.Layer:
    """Layer from host factors: per path U (d_out x s), V (d_in x s) signs or
    real values, and fp16 h, g, l (numpy or torch).  Signs are packed on the GPU."""
    out = lb.Layer(d_in, d_out, s)
    for p in paths:
        U = torch.as_tensor(np.ascontiguousarray(p["U"])).to(device)
        V = torch.as_tensor(np.ascontiguousarray(p["V"])).to(device)
        out.paths.append(
            lb.Path(
                V_bits=lb.pack_signs(V, "V"),
                U_bits=lb.pack_signs(U, "U"),
                h=torch.as_tensor(np.asarray(p["h"], dtype=np.float16)).to(device),
                g=torch.as_tensor(np.asarray(p["g"], dtype=np.float16)).to(device),
                l=torch.as_tensor(np.asarray(p["l"], dtype=np.float16)).to(device),
            )
        )
    return out


def random_layer(d_in: int, d_out: int, s: int, residual: bool, gen: torch.Generator, device="cuda",
                 keep_signs: bool = False):
    """A layer with fair random signs and scales ~ Uniform[0.5, 1.5]/sqrt(s),
    drawn on the device from ``gen``.  Returns (layer, host copies of the
    factors as numpy dicts, or None)."""
    layer = lb.Layer(d_in, d_out, s)
    host = [] if keep_signs else None
    for _ in range(2 if residual else 1):
        V = (1 - 2 * torch.randint(0, 2, (d_in, s), generator=gen, device=device, dtype=torch.int8)).to(torch.int8)
        U = (1 - 2 * torch.randint(0, 2, (d_out, s), generator=gen, device=device, dtype=torch.int8)).to(torch.int8)

        def sc(n):
            return ((torch.rand(n, generator=gen, device=device) + 0.5) / math.sqrt(s)).to(torch.float16)

        h, g, l = sc(d_out), sc(d_in), sc(s)
        layer.paths.append(lb.Path(V_bits=lb.pack_signs(V, "V"), U_bits=lb.pack_signs(U, "U"), h=h, g=g, l=l))
        if keep_signs:
            host.append({"V": V.cpu().numpy(), "U": U.cpu().numpy(), "h": h.cpu().numpy(),
                         "g": g.cpu().numpy(), "l": l.cpu().numpy()})
        del U, V
    return layer, host


def packed_bytes(layer: lb.Layer) -> int:
    """Bytes the forward streams for the factors and scales of ``layer``."""
    total = 0
    for p in layer.paths:
        total += p.V_bits.numel() + p.U_bits.numel() + 2 * (p.h.numel() + p.g.numel() + p.l.numel())
    return total
