"""Decode attention over the packed cache — oracle (test only).

[ADAPTQ §How it works, item 3]: the query is rotated once and the scores are
taken against the packed indices through the codebook, without rebuilding
the cache. [TQAI §Test Suite]: the quantity approximated is
softmax(Q·K^T / sqrt d)·V. [TQPLUS §2 Sparse V]: positions whose attention
weight is negligible skip the V dequantization.

With R = H·diag(D)/sqrt(d) orthonormal, k_hat_t = nK_t · R^T · cK[idx_t]/sqrt(d)
and v_hat_t likewise, so for one query head:
  q~   = R·q
  s_t  = (q · k_hat_t)/sqrt(d) = (1/sqrt d) · nK_t · sum_i q~_i · cK[idx_t,i]/sqrt(d)
  w_t  = exp(s_t - max s),   l = sum over all t < L of w_t
  acc  = sum over ungated t of w_t · nV_t · cV[idx'_t]/sqrt(d)   (rotated domain)
  out  = R^T · (acc / l)                                         (rotated back once)

Readings where the pages are silent or open (the library uses the same):
  - GQA: query head h reads kv head h // gqa (consecutive heads share).
  - L = min(ctx_len, cap); L <= 0 gives out = 0.
  - Sparse-V gate: the weight a position would get cannot be known exactly in
    a single pass, so the gate uses a block-local bound: position t is gated
    for head h iff exp(s_t - M_blk(t)) < tau, M_blk(t) the head's maximum
    score over the aligned 64-position block holding t. Since
    exp(s_t - M_blk) >= exp(s_t - max s) >= w_t / l, a gated position has
    softmax weight below tau. Gated positions stay in l. tau <= 0: no gate.

Context parallelism (the pages describe one device; splitting the context
is the library's extension): each device attends over a contiguous slice of
the positions and reports a log-sum-exp record per query head,
  m2  = log2(e) · max_t s_t
  l   = sum_t exp(s_t - max s)
  acc = sum over ungated t of exp(s_t - max s) · nV_t · cV[idx'_t]
with cV the N(0,1) codebook, i.e. acc lives in the unnormalized Hadamard
domain z = H·(D⊙v) of the encoder. An empty slice reports acc = 0,
m2 = -inf, l = 0. Records of disjoint slices merge exactly:
  M = max_p m2_p,  l = sum_p 2^(m2_p - M) · l_p,  acc likewise,
  out = D⊙(H·(acc / l)) / d.
Slices start at multiples of 64 positions so that the gate's blocks are the
same as in one pass over the whole context.
"""
from __future__ import annotations

import numpy as np

from . import codec as _codec
from . import rotation as _rot

GATE_BLOCK = 64


def attend_head_group(qs: np.ndarray, idx_k: np.ndarray, nk_bits: np.ndarray,
                      idx_v: np.ndarray, nv_bits: np.ndarray, bits_k: int,
                      bits_v: int, seed: int, tau: float):
    """Attention of the query heads qs[g, d] against one kv head's L rows.

    idx_k, idx_v: [L, d] indices; nk_bits, nv_bits: [L] fp16 norm bits.
    Returns (out[g, d] float64, gated[g, L] bool).
    """
    qs = np.asarray(qs, dtype=np.float64)
    g, d = qs.shape
    L = idx_k.shape[0]
    if L <= 0:
        return np.zeros((g, d)), np.zeros((g, 0), dtype=bool)
    nk = np.asarray(nk_bits, dtype=np.uint16).view(np.float16).astype(np.float64)
    nv = np.asarray(nv_bits, dtype=np.uint16).view(np.float16).astype(np.float64)
    q_rot = _rot.rotate(qs, seed)                              # [g, d]
    k_rot = _codec.dequant_rotated(idx_k, bits_k)              # [L, d]
    v_rot = _codec.dequant_rotated(idx_v, bits_v)              # [L, d]
    s = (q_rot @ k_rot.T) * nk[None, :] / np.sqrt(d)           # [g, L]
    m = s.max(axis=1, keepdims=True)
    w = np.exp(s - m)
    l = w.sum(axis=1, keepdims=True)
    if tau > 0.0:
        nblk = (L + GATE_BLOCK - 1) // GATE_BLOCK
        pad = np.full((g, nblk * GATE_BLOCK), -np.inf)
        pad[:, :L] = s
        mblk = pad.reshape(g, nblk, GATE_BLOCK).max(axis=2)    # [g, nblk]
        m_of_t = np.repeat(mblk, GATE_BLOCK, axis=1)[:, :L]
        gated = np.exp(s - m_of_t) < tau
    else:
        gated = np.zeros((g, L), dtype=bool)
    wv = np.where(gated, 0.0, w) * nv[None, :]
    acc = wv @ v_rot                                           # [g, d]
    return _rot.unrotate(acc / l, seed), gated


def attend(q: np.ndarray, packed_k: np.ndarray, norms_k: np.ndarray,
           packed_v: np.ndarray, norms_v: np.ndarray, ctx_lens: np.ndarray,
           gqa: int, bits_k: int, bits_v: int, seed: int, tau: float = 0.0,
           heads=None):
    """Batched decode attention.

    q: float64 [B, Hq, d]; packed_k: uint8 [B, Hkv, cap, d*bits_k/8];
    norms_k: uint16 [B, Hkv, cap] (likewise for V); ctx_lens: [B].
    heads: optional iterable of (b, kv_head) pairs to compute (others stay 0).
    Returns (out [B, Hq, d] float64, n_gated int, gate_margin list) where
    gate_margin holds |ln(exp(s - M_blk)/tau)| of every position, for the
    comparison window of the gate decision.
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    Hkv, cap = packed_k.shape[1], packed_k.shape[2]
    out = np.zeros((B, Hq, d))
    n_gated = 0
    pairs = heads if heads is not None else [(b, g) for b in range(B) for g in range(Hkv)]
    for b, g in pairs:
        L = int(min(int(ctx_lens[b]), cap))
        if L <= 0:
            continue
        ik = _codec.unpack(packed_k[b, g, :L], bits_k, d)
        iv = _codec.unpack(packed_v[b, g, :L], bits_v, d)
        hs = slice(g * gqa, (g + 1) * gqa)
        o, gated = attend_head_group(q[b, hs], ik, norms_k[b, g, :L], iv,
                                     norms_v[b, g, :L], bits_k, bits_v, seed, tau)
        out[b, hs] = o
        n_gated += int(gated.sum())
    return out, n_gated


def partial_head_group(qs: np.ndarray, idx_k: np.ndarray, nk_bits: np.ndarray,
                       idx_v: np.ndarray, nv_bits: np.ndarray, bits_k: int,
                       bits_v: int, seed: int, tau: float):
    """Log-sum-exp record of the query heads qs[g, d] over the L rows of one
    kv head in one context slice. Returns (rec[g, d + 2], gated[g, L]) with
    rec[:, :d] = acc, rec[:, d] = m2, rec[:, d + 1] = l (module docstring)."""
    qs = np.asarray(qs, dtype=np.float64)
    g, d = qs.shape
    L = idx_k.shape[0]
    rec = np.zeros((g, d + 2))
    if L <= 0:
        rec[:, d] = -np.inf
        return rec, np.zeros((g, 0), dtype=bool)
    nk = np.asarray(nk_bits, dtype=np.uint16).view(np.float16).astype(np.float64)
    nv = np.asarray(nv_bits, dtype=np.uint16).view(np.float16).astype(np.float64)
    q_rot = _rot.rotate(qs, seed)
    s = (q_rot @ _codec.dequant_rotated(idx_k, bits_k).T) * nk[None, :] / np.sqrt(d)
    m = s.max(axis=1, keepdims=True)
    w = np.exp(s - m)
    if tau > 0.0:
        nblk = (L + GATE_BLOCK - 1) // GATE_BLOCK
        pad = np.full((g, nblk * GATE_BLOCK), -np.inf)
        pad[:, :L] = s
        mblk = pad.reshape(g, nblk, GATE_BLOCK).max(axis=2)
        gated = np.exp(s - np.repeat(mblk, GATE_BLOCK, axis=1)[:, :L]) < tau
    else:
        gated = np.zeros((g, L), dtype=bool)
    # codebook values in N(0,1) units: sqrt(d) times the rotated unit coordinates
    cv = _codec.dequant_rotated(idx_v, bits_v) * np.sqrt(d)
    rec[:, :d] = (np.where(gated, 0.0, w) * nv[None, :]) @ cv
    rec[:, d] = m[:, 0] / np.log(2.0)
    rec[:, d + 1] = w.sum(axis=1)
    return rec, gated


def attend_partial(q: np.ndarray, packed_k: np.ndarray, norms_k: np.ndarray,
                   packed_v: np.ndarray, norms_v: np.ndarray, ctx_lens: np.ndarray,
                   gqa: int, bits_k: int, bits_v: int, seed: int, tau: float = 0.0):
    """Records [B, Hq, d + 2] of one context slice (the cache arrays and
    ctx_lens describe the slice: its rows start at local position 0)."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    Hkv, cap = packed_k.shape[1], packed_k.shape[2]
    rec = np.zeros((B, Hq, d + 2))
    n_gated = 0
    for b in range(B):
        L = max(int(min(int(ctx_lens[b]), cap)), 0)
        for g in range(Hkv):
            ik = _codec.unpack(packed_k[b, g, :L], bits_k, d)
            iv = _codec.unpack(packed_v[b, g, :L], bits_v, d)
            hs = slice(g * gqa, (g + 1) * gqa)
            rec[b, hs], gated = partial_head_group(q[b, hs], ik, norms_k[b, g, :L], iv,
                                                   norms_v[b, g, :L], bits_k, bits_v, seed, tau)
            n_gated += int(gated.sum())
    return rec, n_gated


def combine(recs: np.ndarray, seed: int) -> np.ndarray:
    """Merge the records [P, B, Hq, d + 2] of P disjoint slices into the
    attention output [B, Hq, d]; heads whose every slice is empty give 0."""
    recs = np.asarray(recs, dtype=np.float64)
    d = recs.shape[-1] - 2
    m2 = recs[..., d]
    M = m2.max(axis=0)                                          # [B, Hq]
    live = np.isfinite(M)
    f = np.where(np.isfinite(m2), np.exp2(m2 - np.where(live, M, 0.0)[None]), 0.0)
    l = (f * recs[..., d + 1]).sum(axis=0)
    acc = (f[..., None] * recs[..., :d]).sum(axis=0)
    y = acc / np.where(live, l, 1.0)[..., None]
    # D ⊙ (H · y) / d = R^T · y / sqrt(d)
    out = _rot.unrotate(y, seed) / np.sqrt(d)
    return np.where(live[..., None], out, 0.0)


def gate_values(qs, idx_k, nk_bits, bits_k, seed):
    """exp(s_t - M_blk(t)) for each head and position (for test windows)."""
    qs = np.asarray(qs, dtype=np.float64)
    g, d = qs.shape
    L = idx_k.shape[0]
    nk = np.asarray(nk_bits, dtype=np.uint16).view(np.float16).astype(np.float64)
    s = (_rot.rotate(qs, seed) @ _codec.dequant_rotated(idx_k, bits_k).T) * nk / np.sqrt(d)
    nblk = (L + GATE_BLOCK - 1) // GATE_BLOCK
    pad = np.full((g, nblk * GATE_BLOCK), -np.inf)
    pad[:, :L] = s
    mblk = pad.reshape(g, nblk, GATE_BLOCK).max(axis=2)
    return np.exp(s - np.repeat(mblk, GATE_BLOCK, axis=1)[:, :L])
