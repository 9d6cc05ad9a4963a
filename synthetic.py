"""Seeded synthetic workloads shared by the tests, the benchmark and the oracle.

This module only draws random numbers and lays them out; it holds none of the
compression or attention arithmetic. Every array is reproducible from
(DATA_SEED, workload name, purpose, index) through numpy's PCG64.

Workloads (d = 128 everywhere; K and V head vectors ~ N(0, 1)):

  single_head_1k      1 q head / 1 kv head, 1024 cached tokens, K4/V2, fp16.
                      4 outlier K channels (drawn once), scaled x20.
  llama3_8b_decode    batch 1, 32 q heads, 8 kv heads (GQA 4), ctx 32768,
                      K4/V2, fp16, 4 outlier K channels x20 per kv head.
  qwen14b_decode      batch 1, 40 q heads, 8 kv heads (GQA 5), ctx 131072,
                      K3/V2, bf16; on 3 K channels per kv head (2% of 128,
                      rounded) the N(0,1) values are replaced by Laplace(0,1).
  batched_serving     batch 64, 32 q heads, 8 kv heads, ctx_b ~ U{1024..16384}
                      (inclusive), capacity 16384, K4/V3, fp16, sparse-V gate
                      at 1e-6.
  bulk_prefill_encode 32 layers x 8 kv heads x 32768 tokens, K4/V2, fp16,
                      4 outlier K channels x20 per (layer, kv head).

Queries are ~ N(0, 1) in the workload's dtype. The sign-vector seed is 0.
The kv buffers use the encoder's input layout [2][n_tok][n_kv_heads][d]
(K block then V block) as raw 16-bit patterns (fp16 or bf16).
"""
from __future__ import annotations

import dataclasses
import zlib
from typing import Optional

import numpy as np

DATA_SEED = 1234
SIGN_SEED = 0
HEAD_DIM = 128


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    d: int
    ctx: Optional[int]          # fixed context length (None: ragged)
    ctx_range: Optional[tuple]  # inclusive (lo, hi) for ragged batches
    cap_tok: int
    bits_k: int
    bits_v: int
    dtype: str                  # "f16" or "bf16"
    outlier: str                # "x20" | "laplace" | "none"
    n_outlier: int
    tau: float = 0.0
    layers: int = 1

    @property
    def gqa(self) -> int:
        return self.n_q_heads // self.n_kv_heads


WORKLOADS = {
    "single_head_1k": Workload("single_head_1k", 1, 1, 1, HEAD_DIM, 1024, None,
                               1024, 4, 2, "f16", "x20", 4),
    "llama3_8b_decode": Workload("llama3_8b_decode", 1, 32, 8, HEAD_DIM, 32768,
                                 None, 32768, 4, 2, "f16", "x20", 4),
    "qwen14b_decode": Workload("qwen14b_decode", 1, 40, 8, HEAD_DIM, 131072,
                               None, 131072, 3, 2, "bf16", "laplace", 3),
    "batched_serving": Workload("batched_serving", 64, 32, 8, HEAD_DIM, None,
                                (1024, 16384), 16384, 4, 3, "f16", "none", 0,
                                tau=1e-6),
    "bulk_prefill_encode": Workload("bulk_prefill_encode", 1, 8, 8, HEAD_DIM,
                                    32768, None, 32768, 4, 2, "f16", "x20", 4,
                                    layers=32),
}


def rng_for(workload: str, purpose: str, *index: int) -> np.random.Generator:
    """Independent PCG64 stream per (workload, purpose, index...)."""
    key = [DATA_SEED, zlib.crc32(workload.encode()), zlib.crc32(purpose.encode())]
    key += [int(i) for i in index]
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(key)))


# ---------------------------------------------------------------- dtype bits
def f16_bits(a: np.ndarray) -> np.ndarray:
    """float -> IEEE fp16 bit patterns (numpy's round-to-nearest-even)."""
    return np.asarray(a, dtype=np.float32).astype(np.float16).view(np.uint16)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round-to-nearest-even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def to_bits(a: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f16":
        return f16_bits(a)
    if dtype == "bf16":
        return bf16_bits(a)
    raise ValueError(dtype)


# ---------------------------------------------------------------- generators
def outlier_channels(w: Workload, layer: int = 0) -> np.ndarray:
    """[n_kv_heads][n_outlier] distinct channel indices, drawn once."""
    rng = rng_for(w.name, "outlier-channels", layer)
    return np.stack([rng.choice(w.d, size=w.n_outlier, replace=False)
                     for _ in range(w.n_kv_heads)]) if w.n_outlier else \
        np.zeros((w.n_kv_heads, 0), dtype=np.int64)


def kv_f32(w: Workload, seq: int, n_tok: int, layer: int = 0,
           tok_start: int = 0) -> np.ndarray:
    """float32 [2][n_tok][n_kv_heads][d] for tokens tok_start.. of a sequence.

    Tokens are drawn in fixed chunks of 1024 so any token range is
    reproducible independently of how the caller slices it.
    """
    chunk = 1024
    out = np.empty((2, n_tok, w.n_kv_heads, w.d), dtype=np.float32)
    chans = outlier_channels(w, layer)
    c0, c1 = tok_start // chunk, (tok_start + n_tok + chunk - 1) // chunk
    for c in range(c0, c1):
        rng = rng_for(w.name, "kv", layer, seq, c)
        blk = rng.standard_normal((2, chunk, w.n_kv_heads, w.d), dtype=np.float32)
        if w.outlier == "x20":
            for h in range(w.n_kv_heads):
                blk[0, :, h, chans[h]] *= 20.0
        elif w.outlier == "laplace":
            lap = rng.laplace(0.0, 1.0, size=(chunk, w.n_kv_heads, w.n_outlier))
            for h in range(w.n_kv_heads):
                for j, ch in enumerate(chans[h]):
                    blk[0, :, h, ch] = lap[:, h, j]
        lo = max(tok_start, c * chunk)
        hi = min(tok_start + n_tok, (c + 1) * chunk)
        out[:, lo - tok_start:hi - tok_start] = blk[:, lo - c * chunk:hi - c * chunk]
    return out


def kv_bits(w: Workload, seq: int, n_tok: int, layer: int = 0,
            tok_start: int = 0) -> np.ndarray:
    """uint16 [2][n_tok][n_kv_heads][d] fp16/bf16 patterns (encoder input)."""
    return to_bits(kv_f32(w, seq, n_tok, layer, tok_start), w.dtype)


def query_bits(w: Workload, scale: float = 1.0, step: int = 0) -> np.ndarray:
    """uint16 [batch][n_q_heads][d] query patterns, ~ N(0, scale^2)."""
    rng = rng_for(w.name, "query", step)
    q = rng.standard_normal((w.batch, w.n_q_heads, w.d), dtype=np.float32) * scale
    return to_bits(q, w.dtype)


def ctx_lens(w: Workload) -> np.ndarray:
    """int32 [batch] context lengths."""
    if w.ctx is not None:
        return np.full(w.batch, w.ctx, dtype=np.int32)
    lo, hi = w.ctx_range
    rng = rng_for(w.name, "ctx-lens")
    return rng.integers(lo, hi + 1, size=w.batch).astype(np.int32)



def projection_matrix(d: int, index: int = 0) -> np.ndarray:
    """[d][d] float32 with i.i.d. N(0, 1) entries: the random projection of
    the residual sketch, drawn by the caller and passed to both sides."""
    return rng_for("residual-sketch", "projection", d, index).standard_normal((d, d)) \
        .astype(np.float32)
