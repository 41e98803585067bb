"""fp64 CPU oracle for the LittleBit latent-factorized binary linear layer.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
or run anything in this directory.  The CUDA library never calls it, and this
module imports nothing from the CUDA package: the two share no code.

What it computes, and where each piece is defined
-------------------------------------------------
* ``eff_bits_exact`` / ``solve_rank``: storage cost of one layer, from the
  LittleBit-2 column (physicalainews.jp, "littlebit2-sub-1bit-llm-quantization-2026"),
  chapter 1, the two bullets that define the effective bit width for the
  single path (``s(a+b+16) + 16(a+b)`` bits) and for the residual path
  (``2s(a+b+16) + 32(a+b)`` bits), both divided by ``a*b``; a = input width,
  b = output width, s = latent rank (``split_dim``).
* ``factored_forward``: the layer output.  The Samsung LittleBit article
  (aifrontier.co.jp, "samsung-littlebit-sub-1-bit"), section 2: W is
  approximated by the product of two rank-s factors U, V binarised to +-1,
  with fp16 row scale h, column scale g and latent scale l; the compute is
  two small binary matrix products plus elementwise scaling; with residual
  compensation a second path of the same form is run and the two outputs are
  added.  Written out per path p:
      y = sum_p  h_p * ( U_p @ ( l_p * ( V_p^T @ ( g_p * x ) ) ) )
  i.e. W_p = diag(h_p) U_p diag(l_p) V_p^T diag(g_p).
* ``pack_signs`` / ``unpack_signs``: the 1-bit storage of U and V.  The pages
  only say the factors are binarised with sign() and stored at one bit each
  (the ``s(a+b)`` term of the cost formula); the bit layout is this library's
  own choice, restated here from its specification (tile shapes below).
* ``latent_cache`` / ``expand``: the two halves of the forward, split where
  the article (section 4, "KV cache" bullet) says a factorised K/V
  projection can be cached: the r-wide latent t' instead of the d-wide row.
* ``rotation_residual``: the gauge freedom the LittleBit-2 column (chapter 2,
  "solution 1", Joint-ITQ) relies on: (U R)(R^T V^T) = U V^T for orthogonal R.

Readings where the pages are silent:
* sign(0) is taken as +1 (bit = [v < 0]); the pages only say "binarise to +-1".
* the residual path uses the same rank s as the main path (the cost formula's
  factor 2 multiplies every term).
* inputs are taken at the exact values stored in fp16/bf16 and converted to
  fp64 exactly; no GPU rounding is mirrored.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

# ---------------------------------------------------------------------------
# storage cost (LittleBit-2 column, chapter 1, effective-bit bullets)
# ---------------------------------------------------------------------------


def eff_bits_exact(a: int, b: int, s: int, residual: bool) -> Fraction:
    """Effective bits per weight as an exact rational number.

    single path:   num_bits = s*(a+b+16) + 16*(a+b)
    residual path: num_bits = 2*s*(a+b+16) + 32*(a+b)
    eff_bit = num_bits / (a*b)
    """
    if residual:
        num = 2 * s * (a + b + 16) + 32 * (a + b)
    else:
        num = s * (a + b + 16) + 16 * (a + b)
    return Fraction(num, a * b)


def eff_bits(a: int, b: int, s: int, residual: bool) -> float:
    return float(eff_bits_exact(a, b, s, residual))


def solve_rank(a: int, b: int, bpw, residual: bool) -> int:
    """Largest rank s >= 1 whose effective bit width does not exceed ``bpw``.

    ``bpw`` may be a string such as "0.1" (read as an exact decimal) or a
    Fraction.  The pages give no rounding rule; "largest s within budget" is
    the plain reading.  Returns 0 if even s = 1 is over budget.
    """
    target = Fraction(bpw) if not isinstance(bpw, float) else Fraction(str(bpw))
    s = 0
    while eff_bits_exact(a, b, s + 1, residual) <= target:
        s += 1
    return s


# ---------------------------------------------------------------------------
# bit layout of the packed factors (this library's format, restated)
# ---------------------------------------------------------------------------
#
# A factor is viewed as a +-1 matrix F with R rows and K columns, where the
# rows are the outputs of the pass that reads it and K is the contraction:
#   role "V": F[j, i] = V[i, j]   (R = s latent rows,  K = d_in)
#   role "U": F[o, j] = U[o, j]   (R = d_out rows,     K = s)
# F is cut into tiles of TR x TK elements, 4096 bits = 512 bytes each:
#   role "V": TR = 16,  TK = 256     role "U": TR = 128, TK = 32
# Rows and columns are zero-padded (bit 0) up to whole tiles.  Tile (rb, kt)
# starts at byte 512 * (rb * n_kt + kt).  Inside a tile, "lane" L = 0..31 owns
# bytes 16L .. 16L+15, read as four little-endian uint32 words w_0..w_3.
# With g = L // 4 and c = L % 4, bit n = 8m + q of word w_r (m = 0..3,
# q = 0..7) holds the sign of element (row, k):
#   role "V": row = 16 rb + g + 8 (r % 2)
#             k   = 256 kt + 32 q + 16 (r // 2) + 4 c + m
#   role "U": row = 128 rb + 16 q + g + 8 (r % 2)
#             k   = 32 kt + 16 (r // 2) + 4 c + m
# and the bit is 1 exactly when F[row, k] < 0.

TILE = {"V": (16, 256), "U": (128, 32)}


def padded_dims(role: str, rows: int, cols: int) -> tuple[int, int]:
    tr, tk = TILE[role]
    return (-(-rows // tr)) * tr, (-(-cols // tk)) * tk


def packed_nbytes(role: str, rows: int, cols: int) -> int:
    rp, kp = padded_dims(role, rows, cols)
    return rp * kp // 8


def _tile_coords(role: str, n_rb: int, n_kt: int):
    """(row, k) of every bit, indexed [rb, kt, lane, word, bit]."""
    rb = np.arange(n_rb).reshape(-1, 1, 1, 1, 1)
    kt = np.arange(n_kt).reshape(1, -1, 1, 1, 1)
    lane = np.arange(32).reshape(1, 1, -1, 1, 1)
    r = np.arange(4).reshape(1, 1, 1, -1, 1)
    n = np.arange(32).reshape(1, 1, 1, 1, -1)
    g, c = lane // 4, lane % 4
    m, q = n // 8, n % 8
    if role == "V":
        row = 16 * rb + g + 8 * (r % 2)
        k = 256 * kt + 32 * q + 16 * (r // 2) + 4 * c + m
    elif role == "U":
        row = 128 * rb + 16 * q + g + 8 * (r % 2)
        k = 32 * kt + 16 * (r // 2) + 4 * c + m
    else:
        raise ValueError(role)
    shape = (n_rb, n_kt, 32, 4, 32)
    return np.broadcast_to(row, shape), np.broadcast_to(k, shape)


def pack_signs(F: np.ndarray, role: str) -> np.ndarray:
    """Pack the signs of F (rows x cols, any real dtype) into uint8 bytes."""
    F = np.asarray(F)
    R, K = F.shape
    rp, kp = padded_dims(role, R, K)
    tr, tk = TILE[role]
    row, k = _tile_coords(role, rp // tr, kp // tk)
    inside = (row < R) & (k < K)
    vals = F[np.minimum(row, R - 1), np.minimum(k, K - 1)]
    neg = inside & (vals < 0)
    weights = np.uint64(1) << np.arange(32, dtype=np.uint64)
    words = (neg.astype(np.uint64) * weights).sum(axis=-1).astype(np.uint32)
    return words.astype("<u4").reshape(-1).view(np.uint8).copy()


def unpack_signs(buf: np.ndarray, role: str, R: int, K: int) -> np.ndarray:
    """Inverse of ``pack_signs``: int8 +-1 matrix of shape (R, K)."""
    rp, kp = padded_dims(role, R, K)
    tr, tk = TILE[role]
    words = np.asarray(buf, dtype=np.uint8).view("<u4").reshape(rp // tr, kp // tk, 32, 4)
    bits = (words[..., None] >> np.arange(32, dtype=np.uint32)) & 1
    row, k = _tile_coords(role, rp // tr, kp // tk)
    out = np.zeros((rp, kp), dtype=np.int8)
    out[row, k] = 1 - 2 * bits.astype(np.int8)
    return out[:R, :K].copy()


def padding_is_zero(buf: np.ndarray, role: str, R: int, K: int) -> bool:
    """True when every bit outside the R x K matrix is 0."""
    rp, kp = padded_dims(role, R, K)
    tr, tk = TILE[role]
    words = np.asarray(buf, dtype=np.uint8).view("<u4").reshape(rp // tr, kp // tk, 32, 4)
    bits = (words[..., None] >> np.arange(32, dtype=np.uint32)) & 1
    row, k = _tile_coords(role, rp // tr, kp // tk)
    outside = (row >= R) | (k >= K)
    return not bool(np.any(bits.astype(bool) & outside))


def factor_matrix(role: str, M: np.ndarray) -> np.ndarray:
    """The R x K view of a factor: V (d_in x s) -> V^T; U (d_out x s) -> U."""
    return np.asarray(M).T if role == "V" else np.asarray(M)


# ---------------------------------------------------------------------------
# the forward (Samsung LittleBit article, section 2)
# ---------------------------------------------------------------------------


def _f64(a) -> np.ndarray:
    return np.asarray(a).astype(np.float64)


def factored_forward(x, paths, rows=None) -> np.ndarray:
    """y (batch x d_out, fp64) of the factored layer, optionally only ``rows``.

    x: (batch, d_in).  paths: one dict per path with
      U (d_out, s) +-1,  V (d_in, s) +-1,  h (d_out,),  g (d_in,),  l (s,).
    Order of operations is the one the article states: column scale g on the
    input, binary V^T product, latent scale l, binary U product, row scale h;
    a residual path's output is added.
    """
    x = _f64(x)
    y = None
    for p in paths:
        u = x * _f64(p["g"])[None, :]            # g (.) x
        t = u @ _f64(p["V"])                      # V^T (g (.) x)    (batch, s)
        tl = t * _f64(p["l"])[None, :]            # l (.) t
        U = _f64(p["U"]) if rows is None else _f64(p["U"])[rows]
        h = _f64(p["h"]) if rows is None else _f64(p["h"])[rows]
        z = tl @ U.T                              # U (l (.) t)      (batch, d_out)
        yp = z * h[None, :]                       # h (.) z
        y = yp if y is None else y + yp
    return y


def latent(x, path) -> np.ndarray:
    """t' = l (.) (V^T (g (.) x)) for one path, fp64 (batch x s)."""
    x = _f64(x)
    return ((x * _f64(path["g"])[None, :]) @ _f64(path["V"])) * _f64(path["l"])[None, :]


# ---------------------------------------------------------------------------
# the latent cache (Samsung LittleBit article, section 4, the KV-cache bullet)
# ---------------------------------------------------------------------------
#
# Because a K or V projection is factorised, its output can be kept as the
# latent t' (r numbers per token) instead of the d-wide projection; the
# projection is rebuilt from the latent with the U pass when it is used.
# A token's cache row holds the paths' latents side by side: path p's s values
# at columns p*s .. p*s + s - 1 (the second half of the forward, written out).


def latent_cache(x, paths) -> np.ndarray:
    """Cache rows of x: [t'_1 | t'_2], t'_p = l_p (.) (V_p^T (g_p (.) x)), fp64
    (batch x npaths*s)."""
    return np.concatenate([latent(x, p) for p in paths], axis=1)


def expand(t_cache, paths, rows=None) -> np.ndarray:
    """The projection rebuilt from cache rows: y = sum_p h_p (.) (U_p t'_p),
    fp64 (n x d_out); t_cache is n x npaths*s as written by latent_cache."""
    t = _f64(t_cache)
    s = np.asarray(paths[0]["l"]).shape[0]
    y = None
    for i, p in enumerate(paths):
        tp = t[:, i * s:(i + 1) * s]
        U = _f64(p["U"]) if rows is None else _f64(p["U"])[rows]
        h = _f64(p["h"]) if rows is None else _f64(p["h"])[rows]
        yp = (tp @ U.T) * h[None, :]
        y = yp if y is None else y + yp
    return y


def cache_row_elems(s: int, npaths: int, align: int = 8) -> int:
    """Elements of one cache row when rows are padded to whole 16-byte units
    (8 fp16 values): npaths*s rounded up to a multiple of `align`."""
    n = npaths * s
    return -(-n // align) * align


def kv_cache_ratio(d: int, s: int, npaths: int, align: int = 8) -> Fraction:
    """Bytes of a d-wide fp16 K (or V) row over the bytes of its cache row."""
    return Fraction(d, cache_row_elems(s, npaths, align))


def dense_weight(path) -> np.ndarray:
    """W = diag(h) U diag(l) V^T diag(g), fp64 (d_out x d_in)."""
    U, V = _f64(path["U"]), _f64(path["V"])
    h, g, l = _f64(path["h"]), _f64(path["g"]), _f64(path["l"])
    return (h[:, None] * (U * l[None, :])) @ (V.T * g[None, :])


def dense_forward(x, paths) -> np.ndarray:
    W = sum(dense_weight(p) for p in paths)
    return _f64(x) @ W.T


# ---------------------------------------------------------------------------
# rotation gauge (LittleBit-2 column, chapter 2, Joint-ITQ)
# ---------------------------------------------------------------------------


def rotation_residual(U: np.ndarray, V: np.ndarray, R: np.ndarray) -> float:
    """|| (U R)(R^T V^T) - U V^T ||_F / || U V^T ||_F for real factors."""
    U, V, R = _f64(U), _f64(V), _f64(R)
    ref = U @ V.T
    rot = (U @ R) @ (R.T @ V.T)
    return float(np.linalg.norm(rot - ref) / np.linalg.norm(ref))


# ---------------------------------------------------------------------------
# error measures used by the parity tests
# ---------------------------------------------------------------------------


def rel_l2(y, y_ref) -> float:
    y, y_ref = _f64(y), _f64(y_ref)
    den = np.linalg.norm(y_ref)
    return float(np.linalg.norm(y - y_ref) / den) if den > 0 else float(np.linalg.norm(y))


def max_abs_ratio(y, y_ref) -> float:
    """max|y - y_ref| / max|y_ref|."""
    y, y_ref = _f64(y), _f64(y_ref)
    den = np.max(np.abs(y_ref))
    return float(np.max(np.abs(y - y_ref)) / den) if den > 0 else float(np.max(np.abs(y)))
