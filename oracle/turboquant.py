"""fp64 reference of the TurboQuant KV compression -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` may import this
module; it shares no code with the product package.

Definition followed: the C attention library's README, "TurboQuant KV Cache
Compression" -- each cached K or V row of head size d is rotated by a
randomized Hadamard transform (random +-1 signs applied BEFORE the Hadamard
transform), normalised by its L2 norm, each coordinate quantised to 2-4 bits
by Lloyd-Max scalar quantisation against a precomputed codebook of the
Beta(d/2, d/2) distribution, and the codes bit-packed; K4/V2 by default,
which the page puts at 9.14 times less memory than an fp32 cache.

Readings (the page fixes no more than the above):
  * rotation: y = H (s * x) / sqrt(d), H the Sylvester-ordered Hadamard
    matrix (H_1 = [1], H_2n = [[H, H], [H, -H]]), s the signs; orthonormal,
    so ||y|| = ||x|| and x = s * (H y) / sqrt(d);
  * normalisation: u = y / ||x||, coordinates in [-1, 1]; the Beta(d/2, d/2)
    law is that of t = (u + 1) / 2, i.e. the density of u is proportional to
    (1 - u^2)^(d/2 - 1);
  * codebook: the 2^b-level Lloyd-Max quantiser of that law (levels the
    conditional means of their cells, cell edges the midpoints between
    levels), in u-space, ascending;
  * code of u: the number of cell edges below u (the nearest level, a tie
    going to the lower one); a zero row has u = 0;
  * packing: channel i's b-bit code at bits [i b, i b + b) of the row's
    little-endian bit stream (least significant bit first), d b / 8 bytes;
  * one fp32 norm per row beside the codes (K4/V2 at d = 64: 512 bytes of
    fp32 K and V against 32 + 4 + 16 + 4 = 56, the page's 9.14x);
  * dequantisation: x_hat = s * (H (||x|| level[code])) / sqrt(d).
"""
from __future__ import annotations

import functools

import numpy as np


def fwht(x) -> np.ndarray:
    """Unnormalised Walsh-Hadamard transform along the last axis (Sylvester
    order): returns H x.  The butterfly (a + b, a - b) at strides 1, 2, 4, ..."""
    y = np.array(x, dtype=np.float64, copy=True)
    n = y.shape[-1]
    if n & (n - 1):
        raise ValueError("length must be a power of two")
    lead = y.shape[:-1]
    h = 1
    while h < n:
        y = y.reshape(lead + (n // (2 * h), 2, h))
        a, b = y[..., 0, :].copy(), y[..., 1, :].copy()
        y[..., 0, :] = a + b
        y[..., 1, :] = a - b
        y = y.reshape(lead + (n,))
        h *= 2
    return y


def rotate(x, signs) -> np.ndarray:
    """y = H (s * x) / sqrt(d)."""
    x = np.asarray(x, dtype=np.float64)
    s = np.asarray(signs, dtype=np.float64)
    return fwht(x * s) / np.sqrt(x.shape[-1])


def unrotate(y, signs) -> np.ndarray:
    """The inverse rotation: x = s * (H y) / sqrt(d)."""
    y = np.asarray(y, dtype=np.float64)
    s = np.asarray(signs, dtype=np.float64)
    return s * fwht(y) / np.sqrt(y.shape[-1])


def codebook(d: int, bits: int) -> np.ndarray:
    """The 2^bits Lloyd-Max levels of the Beta(d/2, d/2) law in u-space
    (computed once per (d, bits); see _codebook)."""
    return np.array(_codebook_cached(int(d), int(bits)))


@functools.lru_cache(maxsize=None)
def _codebook_cached(d: int, bits: int):
    return tuple(_codebook(d, bits))


def _codebook(d: int, bits: int, iters: int = 100000, tol: float = 1e-15) -> np.ndarray:
    """The 2^bits Lloyd-Max levels (u-space, ascending) of u = 2t - 1 with
    t ~ Beta(d/2, d/2).  Cell mass and first moment come from the regularised
    incomplete beta function: for t in [a, b],
      P = I_b(a', a') - I_a(a', a'),  E[t; cell] = (1/2) (I_b(a'+1, a') - I_a(a'+1, a'))
    with a' = d/2 (the mean of Beta(a', a') is 1/2)."""
    from scipy.special import betainc, betaincinv
    a = d / 2.0
    n = 1 << bits
    # start from the quantiles at the cell centres
    t = betaincinv(a, a, (np.arange(n) + 0.5) / n)
    for _ in range(iters):
        edges = np.concatenate(([0.0], (t[:-1] + t[1:]) / 2, [1.0]))
        mass = np.diff(betainc(a, a, edges))
        first = 0.5 * np.diff(betainc(a + 1.0, a, edges))
        t_new = first / mass
        done = np.max(np.abs(t_new - t)) < tol
        t = t_new
        if done:
            break
    return 2.0 * t - 1.0


def edges_of(levels) -> np.ndarray:
    """Cell edges: the midpoints between consecutive levels."""
    lv = np.asarray(levels, dtype=np.float64)
    return (lv[:-1] + lv[1:]) / 2


def quantize(x, signs, levels):
    """(codes, norms) of rows x [..., d]: codes uint8 [..., d] unpacked,
    norms float64 [...]."""
    x = np.asarray(x, dtype=np.float64)
    y = rotate(x, signs)
    norms = np.sqrt(np.sum(x * x, axis=-1))
    safe = np.where(norms > 0, norms, 1.0)
    u = np.where(norms[..., None] > 0, y / safe[..., None], 0.0)
    codes = np.searchsorted(edges_of(levels), u, side="left").astype(np.uint8)
    return codes, norms


def unit_coords(x, signs) -> np.ndarray:
    """u = rotate(x) / ||x|| (0 for a zero row): the values the codes decide on."""
    x = np.asarray(x, dtype=np.float64)
    norms = np.sqrt(np.sum(x * x, axis=-1))
    safe = np.where(norms > 0, norms, 1.0)
    return np.where(norms[..., None] > 0, rotate(x, signs) / safe[..., None], 0.0)


def pack(codes, bits: int) -> np.ndarray:
    """Codes [..., d] -> bytes [..., d * bits / 8], LSB-first bit stream."""
    c = np.asarray(codes, dtype=np.uint8)
    d = c.shape[-1]
    if (d * bits) % 8:
        raise ValueError("d * bits must be a multiple of 8")
    bit_planes = ((c[..., :, None] >> np.arange(bits, dtype=np.uint8)) & 1).astype(np.uint8)
    stream = bit_planes.reshape(c.shape[:-1] + (d * bits,))
    return np.packbits(stream, axis=-1, bitorder="little")


def unpack(packed, bits: int, d: int) -> np.ndarray:
    """Bytes [..., d * bits / 8] -> codes uint8 [..., d]."""
    p = np.asarray(packed, dtype=np.uint8)
    stream = np.unpackbits(p, axis=-1, bitorder="little")[..., : d * bits]
    planes = stream.reshape(p.shape[:-1] + (d, bits)).astype(np.uint8)
    return np.sum(planes << np.arange(bits, dtype=np.uint8), axis=-1, dtype=np.uint8)


def compress(x, signs, bits: int, levels):
    """(packed codes uint8 [..., d*bits/8], norms float32 [...]) of rows x."""
    codes, norms = quantize(x, signs, levels)
    return pack(codes, bits), norms.astype(np.float32)


def dequantize(packed, norms, signs, bits: int, levels, d: int) -> np.ndarray:
    """x_hat = s * (H (norm * level[code])) / sqrt(d), fp64 [..., d]."""
    codes = unpack(packed, bits, d)
    lv = np.asarray(levels, dtype=np.float64)
    y = np.asarray(norms, dtype=np.float64)[..., None] * lv[codes]
    return unrotate(y, signs)


def bytes_per_row(d: int, bits: int) -> int:
    """Packed codes plus the fp32 norm."""
    return d * bits // 8 + 4
