"""Stage-2 residual sketch (QJL) and the unbiased inner-product estimate —
oracle (test only).

"We Built a Python Library That Cuts LLM Memory Usage by 80%", section "Why
not both stages?": the method has a second stage that adds a one-bit
correction of the stage-1 residual so that inner products become unbiased;
that page leaves it out of softmax attention, where its variance hurts. The
pages give no further detail, so the definition below is the plain reading
of a one-bit Johnson-Lindenstrauss sketch of the residual; every choice
marked "reading" is the library's and the CUDA path implements the same.

For a key x with stage-1 code (idx, fp16 norm nK) and R = H·diag(D)/sqrt(d):
  r~    = R·x - nK · c[idx]/sqrt(d)     residual in rotated coordinates,
                                          = R·(x - x_hat)          (reading)
  S     : [m, d], i.i.d. N(0, 1), m = d (one bit per coordinate); drawn by
          the caller and passed in                                  (reading)
  bit_i = 1 iff (S·r~)_i >= 0, packed LSB-first, m/8 bytes per row  (reading)
  gamma = ||r~|| (= ||x - x_hat||), stored fp16 round-to-nearest-even,
          saturated at 65504                                        (reading)
For a query q with q~ = R·q, the estimate of <q, x> is
  <q~, nK·c[idx]/sqrt(d)> + gamma · sqrt(pi/2)/m · <S·q~, 2·bit - 1>
and the attention-style score is that estimate / sqrt(d). Since S·R has
i.i.d. N(0, 1) entries too, sketching in rotated coordinates is the same
sketch of x - x_hat in the original ones. For s ~ N(0, I),
E[sign(s·r)·(s·q)] = sqrt(2/pi)·<q, r>/||r||, which makes the correction
unbiased for <q, r>.
"""
from __future__ import annotations

import numpy as np

from . import codec as _codec
from . import rotation as _rot

FP16_MAX = 65504.0


def residual_rotated(x: np.ndarray, bits: int, seed: int):
    """Stage-1 code of the rows x[n, d] and their rotated residuals.
    Returns (idx[n, d], norm_bits[n] uint16, r_rot[n, d] float64)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    idx, _, nb, _, _ = _codec.encode(x, bits, seed)
    n16 = nb.view(np.float16).astype(np.float64)
    r_rot = _rot.rotate(x, seed) - n16[:, None] * _codec.dequant_rotated(idx, bits)
    return idx, nb, r_rot


def sketch(r_rot: np.ndarray, S: np.ndarray):
    """Sign bits of S·r~ packed LSB-first (uint8[n, m/8]), the projections
    S·r~ [n, m] (for comparison windows), and fp16 bits of ||r~||."""
    u = np.asarray(r_rot, dtype=np.float64) @ np.asarray(S, dtype=np.float64).T
    bits = (u >= 0.0).astype(np.uint8)
    rows = np.packbits(bits, axis=1, bitorder="little")
    gamma = np.sqrt(np.sum(np.asarray(r_rot, dtype=np.float64) ** 2, axis=1))
    gamma_bits = np.minimum(gamma, FP16_MAX).astype(np.float16).view(np.uint16)
    return rows, u, gamma_bits


def encode(x: np.ndarray, bits: int, seed: int, S: np.ndarray):
    """Stage 1 and the residual sketch of the rows x[n, d].
    Returns (packed stage-1 rows, norm bits, sketch rows, gamma bits, S·r~)."""
    idx, nb, r_rot = residual_rotated(x, bits, seed)
    rows, u, gb = sketch(r_rot, S)
    return _codec.pack(idx, bits), nb, rows, gb, u


def correction(q_rot: np.ndarray, sketch_rows: np.ndarray, gamma_bits: np.ndarray,
               S: np.ndarray) -> np.ndarray:
    """gamma · sqrt(pi/2)/m · <S·q~, 2·bit - 1> for each query row [nq, d]
    and key row [n]: returns [nq, n]."""
    S = np.asarray(S, dtype=np.float64)
    m = S.shape[0]
    pm = 2.0 * np.unpackbits(np.asarray(sketch_rows, np.uint8), axis=1,
                             bitorder="little")[:, :m].astype(np.float64) - 1.0
    g = np.asarray(gamma_bits, dtype=np.uint16).view(np.float16).astype(np.float64)
    sq = np.asarray(q_rot, dtype=np.float64) @ S.T               # [nq, m]
    return (sq @ pm.T) * g[None, :] * np.sqrt(np.pi / 2.0) / m


def inner_products(q: np.ndarray, packed_k: np.ndarray, norms_k: np.ndarray,
                   sketch_rows: np.ndarray, gamma_bits: np.ndarray, bits: int,
                   seed: int, S: np.ndarray, with_sketch: bool = True) -> np.ndarray:
    """Estimates of <q_a, x_t> for query rows q[nq, d] and the key rows of
    one kv head (packed_k[n], norms_k[n], sketch rows, gamma bits)."""
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[-1]
    q_rot = _rot.rotate(q, seed)
    idx = _codec.unpack(packed_k, bits, d)
    nk = np.asarray(norms_k, dtype=np.uint16).view(np.float16).astype(np.float64)
    est = (q_rot @ _codec.dequant_rotated(idx, bits).T) * nk[None, :]
    if with_sketch:
        est = est + correction(q_rot, sketch_rows, gamma_bits, S)
    return est


def scores(q: np.ndarray, packed_k: np.ndarray, norms_k: np.ndarray,
           sketch_rows: np.ndarray, gamma_bits: np.ndarray, ctx_lens: np.ndarray,
           gqa: int, bits: int, seed: int, S: np.ndarray,
           with_sketch: bool = True) -> np.ndarray:
    """Scores estimate/sqrt(d) for q[B, Hq, d] over a cache
    [B, Hkv, cap, ...]; positions t >= min(ctx, cap) are 0."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    Hkv, cap = packed_k.shape[1], packed_k.shape[2]
    out = np.zeros((B, Hq, cap))
    for b in range(B):
        L = max(0, min(int(ctx_lens[b]), cap))
        if L == 0:
            continue
        for g in range(Hkv):
            hs = slice(g * gqa, (g + 1) * gqa)
            out[b, hs, :L] = inner_products(q[b, hs], packed_k[b, g, :L], norms_k[b, g, :L],
                                            sketch_rows[b, g, :L], gamma_bits[b, g, :L],
                                            bits, seed, S, with_sketch) / np.sqrt(d)
    return out
