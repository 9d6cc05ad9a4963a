"""Helpers for the GPU parity tests: oracle-built inputs and device buffers.

Every expected value comes from the oracle on seeded synthetic inputs; the
packed caches fed to the GPU attention are built by the oracle's encoder, so
no oracle input ever comes from the CUDA path. The oracle work runs in a
process pool started with 'spawn' (before any CUDA call in the workers).
"""
from __future__ import annotations

import functools
import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor

import numpy as np

import synthetic as S

_POOL = None


def pool() -> ProcessPoolExecutor:
    global _POOL
    if _POOL is None:
        n = max(1, min(32, (os.cpu_count() or 2) - 1))
        _POOL = ProcessPoolExecutor(max_workers=n, mp_context=mp.get_context("spawn"),
                                    initializer=_worker_init)
    return _POOL


def _worker_init():
    os.environ["OPENBLAS_NUM_THREADS"] = "1"
    os.environ["OMP_NUM_THREADS"] = "1"
    try:
        import threadpoolctl
        threadpoolctl.threadpool_limits(1)
    except Exception:
        pass


# ------------------------------------------------------------ oracle side
def oracle_encode_heads(kv_bits: np.ndarray, dtype: str, which: int, bits: int,
                        seed: int, chunk: int = 32768):
    """Oracle encode of kv_bits[which] ([n][H][d] 16-bit patterns).

    Returns idx uint8 [H][n][d], norm bits uint16 [H][n], margin float32
    [H][n][d] (distance of zeta to the nearest threshold, N(0,1) units).
    """
    from oracle import codec
    n, H, d = kv_bits.shape[1:]
    idx = np.empty((H, n, d), np.uint8)
    nb = np.empty((H, n), np.uint16)
    mg = np.empty((H, n, d), np.float32)
    for h in range(H):
        for s in range(0, n, chunk):
            x = codec.promote(kv_bits[which, s:s + chunk, h], dtype)
            i, _, b, _, m = codec.encode(x, bits, seed)
            idx[h, s:s + chunk] = i
            nb[h, s:s + chunk] = b
            mg[h, s:s + chunk] = m
    return idx, nb, mg


def _seq_cache(name: str, seq: int, n_tok: int, seed: int):
    """Worker: oracle-encoded packed rows of one sequence (all kv heads)."""
    from oracle import codec
    w = S.WORKLOADS[name]
    kv = S.kv_bits(w, seq, n_tok)
    out = []
    for which, bits in ((0, w.bits_k), (1, w.bits_v)):
        idx, nb, _ = oracle_encode_heads(kv, w.dtype, which, bits, seed)
        rows = np.stack([codec.pack(idx[h].astype(np.int64), bits) for h in range(w.n_kv_heads)])
        out += [rows, nb]
    return out


@functools.lru_cache(maxsize=4)
def oracle_cache(name: str, seed: int = S.SIGN_SEED):
    """(packed_k, norms_k, packed_v, norms_v, ctx) for a workload, built by
    the oracle from the workload's synthetic K/V ([B][H][cap][row] layout;
    rows past each sequence's context are zero)."""
    w = S.WORKLOADS[name]
    ctx = S.ctx_lens(w)
    B, H, cap, d = w.batch, w.n_kv_heads, w.cap_tok, w.d
    pk = np.zeros((B, H, cap, d * w.bits_k // 8), np.uint8)
    pv = np.zeros((B, H, cap, d * w.bits_v // 8), np.uint8)
    nk = np.zeros((B, H, cap), np.uint16)
    nv = np.zeros((B, H, cap), np.uint16)
    futs = [pool().submit(_seq_cache, name, b, int(ctx[b]), seed) for b in range(B)]
    for b, f in enumerate(futs):
        rk, bk, rv, bv = f.result()
        L = int(ctx[b])
        pk[b, :, :L], nk[b, :, :L], pv[b, :, :L], nv[b, :, :L] = rk, bk, rv, bv
    return pk, nk, pv, nv, ctx


def _oracle_attend_part(q, pk, nk, pv, nv, ctx, gqa, bk, bv, seed, tau):
    from oracle import attention
    return attention.attend(q, pk, nk, pv, nv, ctx, gqa, bk, bv, seed, tau)


def oracle_attend(q64, pk, nk, pv, nv, ctx, gqa, bk, bv, seed, tau=0.0):
    """Oracle attention; each (batch, kv head) pair is one pool task that
    receives only its own slice of the cache."""
    B, H = pk.shape[:2]
    out = np.zeros(q64.shape)
    futs = []
    for b in range(B):
        L = int(min(max(int(ctx[b]), 0), pk.shape[2]))
        for g in range(H):
            hs = slice(g * gqa, (g + 1) * gqa)
            futs.append((b, hs, pool().submit(
                _oracle_attend_part, q64[b:b + 1, hs], pk[b:b + 1, g:g + 1, :L],
                nk[b:b + 1, g:g + 1, :L], pv[b:b + 1, g:g + 1, :L], nv[b:b + 1, g:g + 1, :L],
                np.array([L]), gqa, bk, bv, seed, tau)))
    n_gated = 0
    for b, hs, f in futs:
        o, ng = f.result()
        out[b, hs] = o[0]
        n_gated += ng
    return out, n_gated


# ------------------------------------------------------------ device side
def dev(a: np.ndarray):
    """numpy -> CUDA tensor (16-bit patterns travel as int16)."""
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).cuda()


def host(t) -> np.ndarray:
    a = t.cpu().numpy()
    return a.view(np.uint16) if a.dtype == np.int16 else a


def gpu_encode(kv_bits, dtype, bits_k, bits_v, seed, cap=None, tok_offset=0,
               fill=0, status=None):
    """Run tq_encode on kv_bits [2][n][H][d]; returns host copies of the cache."""
    import torch
    import compressed_decode_attention_b200 as tq
    _, n, H, d = kv_bits.shape
    cap = cap or n + tok_offset
    pk = torch.full((H, cap, d * bits_k // 8), fill, dtype=torch.uint8, device="cuda")
    pv = torch.full((H, cap, d * bits_v // 8), fill, dtype=torch.uint8, device="cuda")
    nk = torch.full((H, cap), fill, dtype=torch.int16, device="cuda")
    nv = torch.full((H, cap), fill, dtype=torch.int16, device="cuda")
    st = status if status is not None else torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.tq_encode(dev(kv_bits), tq.TQ_F16 if dtype == "f16" else tq.TQ_BF16, n, H, d,
                 bits_k, bits_v, seed, pk, pv, nk, nv, cap, tok_offset, st)
    torch.cuda.synchronize()
    return host(pk), host(nk), host(pv), host(nv), int(st.item())


# Error bound of the kernel's fp32 scores against the oracle's float64 ones,
# used to find the positions where the two may take the sparse-V gate
# decision differently. A score s_t = (nK_t/sqrt d)·sum_i q~_i·c_i/sqrt(d) is
# formed on tensor cores from fp16 high+low parts of q~ and of the codebook
# values (the missing low x low term and the rounding of the low parts leave
# < 3·2^-22 of each product), accumulated in fp32 over 128 products, eight
# k-steps and three partial products (about ten roundings of at most 2^-23
# of the running magnitude), then scaled twice by exact factors with one
# rounding each: < 2^-19 of the sum S_t of the products' magnitudes in all.
# So |ds_t| <= SCORE_EPS_ABS·S_t + SCORE_EPS_REL·|s_t|, with a factor of 8
# to spare in the first term.
SCORE_EPS_ABS = 2.0 ** -16
SCORE_EPS_REL = 2.0 ** -22


def _gate_table(q, pk, nk, L, gqa, bk, seed, tau):
    """Worker: (gated count, ambiguous count) per query head of one kv head.
    A position is ambiguous when its float64 gate value exp(s - M_blk) lies
    within the score error bound (relative, in the log domain) of tau."""
    from oracle import attention, codec, rotation
    d = q.shape[-1]
    idx = codec.unpack(pk, bk, d)
    gv = attention.gate_values(q, idx, nk, bk, seed)             # [g, L]
    nkf = nk.view(np.float16).astype(np.float64)
    q_rot = rotation.rotate(q, seed)
    k_rot = codec.dequant_rotated(idx, bk)
    s = (q_rot @ k_rot.T) * nkf / np.sqrt(d)
    mag = (np.abs(q_rot) @ np.abs(k_rot).T) * nkf / np.sqrt(d)
    bound = SCORE_EPS_ABS * mag + SCORE_EPS_REL * np.abs(s)
    nblk = (L + attention.GATE_BLOCK - 1) // attention.GATE_BLOCK
    pad = np.zeros((q.shape[0], nblk * attention.GATE_BLOCK))
    pad[:, :L] = bound
    bmax = np.repeat(pad.reshape(q.shape[0], nblk, -1).max(axis=2), attention.GATE_BLOCK, axis=1)[:, :L]
    with np.errstate(divide="ignore"):
        amb = np.abs(np.log(gv) - np.log(tau)) <= bound + bmax
    return (gv < tau).sum(axis=1), amb.sum(axis=1)


def oracle_gate_table(q64, pk, nk, ctx, gqa, bk, seed, tau):
    """Per (sequence, query head): the oracle's gated-position count and the
    number of positions whose decision the score error bound leaves open."""
    B, H = pk.shape[:2]
    Hq = q64.shape[1]
    cnt = np.zeros((B, Hq), np.int64)
    amb = np.zeros((B, Hq), np.int64)
    futs = []
    for b in range(B):
        L = int(min(max(int(ctx[b]), 0), pk.shape[2]))
        for g in range(H):
            if L > 0:
                hs = slice(g * gqa, (g + 1) * gqa)
                futs.append((b, hs, pool().submit(_gate_table, q64[b, hs], pk[b, g, :L],
                                                  nk[b, g, :L], L, gqa, bk, seed, tau)))
    for b, hs, f in futs:
        cnt[b, hs], amb[b, hs] = f.result()
    return cnt, amb


def gpu_attend(q_bits, q_dtype, pk, nk, pv, nv, ctx, gqa, bk, bv, seed, tau=0.0,
               n_ctas=0, out_dtype=None, workspace=None, head_counts=False):
    """tq_attend on host arrays; returns (out float32/bits, status, skipped),
    plus the per (sequence, query head) gate counts of tq_attend_gate_counts
    when head_counts is set."""
    import torch
    import compressed_decode_attention_b200 as tq
    B, H, cap = pk.shape[:3]
    Hq = q_bits.shape[1]
    d = q_bits.shape[2]
    out_dtype = tq.TQ_F32 if out_dtype is None else out_dtype
    ws_bytes = tq.tq_attend_workspace_size(B, Hq, cap, d)
    ws = workspace if workspace is not None else \
        torch.zeros(ws_bytes // 4, dtype=torch.float32, device="cuda")
    if out_dtype == tq.TQ_F32:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device="cuda")
    else:
        out = torch.empty((B, Hq, d), dtype=torch.int16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sk = torch.zeros(1, dtype=torch.int64, device="cuda")
    qt = dev(q_bits)
    q_enum = {"f16": tq.TQ_F16, "bf16": tq.TQ_BF16, "f32": tq.TQ_F32}[q_dtype]
    args = (qt, q_enum, dev(pk), dev(nk), dev(pv), dev(nv), dev(np.asarray(ctx, np.int32)),
            B, Hq, gqa, d, bk, bv, seed, cap, tau, n_ctas, ws, ws_bytes)
    if head_counts:
        hk = torch.zeros((B, Hq), dtype=torch.int32, device="cuda")
        tq.tq_attend_gate_counts(*args, hk, out, out_dtype, dev_status=st, sparse_v_skipped=sk)
    else:
        tq.tq_attend(*args, out, out_dtype, dev_status=st, sparse_v_skipped=sk)
    torch.cuda.synchronize()
    if head_counts:
        return host(out), int(st.item()), int(sk.item()), hk.cpu().numpy().astype(np.int64)
    return host(out), int(st.item()), int(sk.item())


def _encode_slice(kv_slice, dtype, bits, seed):
    """Worker: oracle encode of [n][d] 16-bit patterns."""
    kv = kv_slice[None, :, None, :]
    idx, nb, mg = oracle_encode_heads(np.stack([kv[0], kv[0]]), dtype, 0, bits, seed)
    return idx[0], nb[0], mg[0]


def oracle_encode_parallel(kv_bits, dtype, which, bits, seed, chunk=65536):
    """oracle_encode_heads spread over the pool by (head, token chunk)."""
    n, H, d = kv_bits.shape[1:]
    idx = np.empty((H, n, d), np.uint8)
    nb = np.empty((H, n), np.uint16)
    mg = np.empty((H, n, d), np.float32)
    futs = []
    for h in range(H):
        for s in range(0, n, chunk):
            sl = np.ascontiguousarray(kv_bits[which, s:s + chunk, h])
            futs.append((h, s, pool().submit(_encode_slice, sl, dtype, bits, seed)))
    for h, s, f in futs:
        i, b, m = f.result()
        idx[h, s:s + len(b)], nb[h, s:s + len(b)], mg[h, s:s + len(b)] = i, b, m
    return idx, nb, mg


# Comparison rule for encoded indices: bit-exact except at coordinates whose
# rotated value lies within this distance (N(0,1) units, i.e. 1e-5/sqrt(d) in
# the N(0,1/d) units of the codebook) of a threshold; those must be at most
# NEAR_FRACTION of all coordinates.
NEAR_WINDOW = 1e-5
NEAR_FRACTION = 1e-4


def check_indices(idx_gpu, idx_oracle, margin):
    """Bit-exact outside the boundary window. Returns (mismatches, near, total)
    so the caller can bound the exempted count over a whole encode call."""
    near = margin < NEAR_WINDOW
    bad = (idx_gpu != idx_oracle) & ~near
    assert not bad.any(), f"{int(bad.sum())} index mismatches outside the boundary window"
    return int((idx_gpu != idx_oracle).sum()), int(near.sum()), int(near.size)


def check_near_fraction(stats):
    """The exempted (near-threshold) coordinates of one encode call, K and V
    together, are at most NEAR_FRACTION of all its coordinates."""
    near = sum(s[1] for s in stats)
    total = sum(s[2] for s in stats)
    assert near <= NEAR_FRACTION * total, (near, total)


def check_norms(nb_gpu, nb_oracle):
    """Stored fp16 norms within one ulp (non-negative fp16 bit patterns are
    ordered like the values they encode)."""
    diff = np.abs(nb_gpu.astype(np.int64) - nb_oracle.astype(np.int64))
    assert diff.max(initial=0) <= 1, int(diff.max())
