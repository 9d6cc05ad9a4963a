"""Encode / pack / unpack / dequantize — oracle (test only).

Steps, in the pages' order:
  [TQAI §The Paper]        keep ||x|| separately in FP16; quantize the unit vector
  [ADAPTQ §How it works 1] y = (1/sqrt d) · H · D · (x / ||x||)
  [TQAI §The Paper], [ADAPTQ §How it works 2]
                           each y_i -> index of its Lloyd-Max cell for N(0,1/d)
  [TQAI §What's Next], [ADAPTQ §Key Features]
                           pack the b-bit indices (2/3/4 bits)
  [TQAI §Compression numbers]  K4/V2, K3/V2, K4/V3 at d = 128

Readings where the pages are silent (the library freezes the same ones):
  - The unit vector uses the unrounded norm; the stored norm is
    fp16(||x||) with round-to-nearest-even, saturated at 65504.
  - Thresholds in N(0,1/d) units are t_j/sqrt(d); equivalently the index is
    #{ j : zeta_i >= t_j } with zeta = sqrt(d)·y and the N(0,1) thresholds
    t_j (a value on a threshold goes to the upper cell).
  - A zero vector has norm 0 and zeta = 0, so every index is N/2.
  - Packing is LSB-first contiguous: row bit (i·b + k) is bit k of idx_i;
    row byte j holds row bits 8j..8j+7.
"""
from __future__ import annotations

import numpy as np

from . import codebook as _cb
from . import rotation as _rot

FP16_MAX = 65504.0
_CB_CACHE: dict = {}


def codebook(bits: int):
    """(centroids, thresholds) in N(0,1) units, cached per bit width."""
    if bits not in _CB_CACHE:
        c, t = _cb.lloyd_max_normal(bits)
        _CB_CACHE[bits] = (c, t)
    return _CB_CACHE[bits]


# ------------------------------------------------------------ input dtypes
def promote(bits16: np.ndarray, dtype: str) -> np.ndarray:
    """fp16 / bf16 bit patterns -> float64, exactly."""
    bits16 = np.asarray(bits16, dtype=np.uint16)
    if dtype == "f16":
        return bits16.view(np.float16).astype(np.float64)
    if dtype == "bf16":
        return (bits16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    raise ValueError(dtype)


def fp16_norm_bits(n: np.ndarray) -> np.ndarray:
    """Stored norm: fp16 round-to-nearest-even of min(n, 65504), as bits."""
    return np.minimum(n, FP16_MAX).astype(np.float16).view(np.uint16)


# ------------------------------------------------------------ quantization
def quantize_index(zeta: np.ndarray, thresholds: np.ndarray) -> np.ndarray:
    """idx = #{ j : zeta >= t_j } (binary search over the sorted thresholds)."""
    return np.searchsorted(thresholds, zeta, side="right").astype(np.int64)


def encode(x: np.ndarray, bits: int, seed: int):
    """Encode float64 rows x[n, d].

    Returns (idx[n, d] int64, norm[n] float64 unrounded, norm_bits[n] uint16,
             zeta[n, d] float64, margin[n, d] float64) where margin is the
    distance of zeta_i to the nearest threshold (in N(0,1) units).
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    _, t = codebook(bits)
    norm = np.sqrt(np.sum(x * x, axis=-1))
    z = (x * _rot.sign_vector(seed, d)) @ _rot.hadamard(d).T   # H·(D⊙x)
    safe = np.where(norm > 0.0, norm, 1.0)
    zeta = z / safe[:, None]        # = sqrt(d)·y with y = (1/sqrt d)·H·D·x/||x||
    zeta[norm == 0.0] = 0.0
    idx = quantize_index(zeta, t)
    tp = np.concatenate(([-np.inf], t, [np.inf]))
    margin = np.minimum(zeta - tp[idx], tp[idx + 1] - zeta)
    return idx, norm, fp16_norm_bits(norm), zeta, margin


def pack(idx: np.ndarray, bits: int) -> np.ndarray:
    """LSB-first contiguous packing of idx[n, d] into uint8[n, d*bits/8]."""
    idx = np.asarray(idx, dtype=np.int64)
    n, d = idx.shape
    planes = (idx[:, :, None] >> np.arange(bits)) & 1        # [n, d, bits]
    rowbits = planes.reshape(n, d * bits).astype(np.uint8)   # bit i*b+k
    return np.packbits(rowbits, axis=1, bitorder="little")


def unpack(rows: np.ndarray, bits: int, d: int) -> np.ndarray:
    """Inverse of pack: uint8[n, d*bits/8] -> idx[n, d] int64."""
    rows = np.asarray(rows, dtype=np.uint8)
    n = rows.shape[0]
    rowbits = np.unpackbits(rows, axis=1, bitorder="little")[:, :d * bits]
    planes = rowbits.reshape(n, d, bits).astype(np.int64)
    return np.sum(planes << np.arange(bits), axis=-1)


# ------------------------------------------------------------ dequantization
def dequant_rotated(idx: np.ndarray, bits: int) -> np.ndarray:
    """Rotated-domain unit-vector estimate: c[idx] / sqrt(d) (N(0,1/d) codebook)."""
    c, _ = codebook(bits)
    d = idx.shape[-1]
    return c[idx] / np.sqrt(d)


def dequant(idx: np.ndarray, norm_bits: np.ndarray, bits: int, seed: int) -> np.ndarray:
    """Original-space reconstruction x_hat = fp16norm · R^T · (c[idx]/sqrt d)."""
    n16 = np.asarray(norm_bits, dtype=np.uint16).view(np.float16).astype(np.float64)
    return n16[:, None] * _rot.unrotate(dequant_rotated(idx, bits), seed)


def encode_rows(x: np.ndarray, bits: int, seed: int):
    """Convenience: (packed rows uint8[n, d*bits/8], norm bits uint16[n])."""
    idx, _, nb, _, _ = encode(x, bits, seed)
    return pack(idx, bits), nb
