"""GPU parity of tq_prefill_attend (causal attention of a chunk of new query
tokens over the compressed cache) against the float64 oracle, B200.

Token i of sequence b sits at position p = ctx_b - n_tok + i; its output must
equal, within 2e-3, the oracle decode attention of that query over cache
positions 0..p (the cache under test, built by the oracle's encoder).
"""
import numpy as np
import pytest

import synthetic as S
from gpu_support import dev, host, pool
from oracle import codec

pytestmark = pytest.mark.gpu
ATOL = 2e-3
D = 128


def _cache(bk, bv, B, Hkv, cap, ctx, seed, rng):
    pk = np.zeros((B, Hkv, cap, D * bk // 8), np.uint8)
    pv = np.zeros((B, Hkv, cap, D * bv // 8), np.uint8)
    nk = np.zeros((B, Hkv, cap), np.uint16)
    nv = np.zeros((B, Hkv, cap), np.uint16)
    for b in range(B):
        L = int(min(max(ctx[b], 0), cap))
        for g in range(Hkv):
            k = rng.standard_normal((L, D)) * 2
            k[:, :4] *= 10.0                     # outlier channels
            v = rng.standard_normal((L, D))
            pk[b, g, :L], nk[b, g, :L] = codec.encode_rows(codec.promote(S.f16_bits(k), "f16"),
                                                           bk, seed)
            pv[b, g, :L], nv[b, g, :L] = codec.encode_rows(codec.promote(S.f16_bits(v), "f16"),
                                                           bv, seed)
    return pk, nk, pv, nv


def _oracle_token(q, pk, nk, pv, nv, p, gqa, bk, bv, seed):
    from oracle import attention
    if p < 0:
        return np.zeros(q.shape)
    out, _ = attention.attend(q[None], pk[None, :, :p + 1], nk[None, :, :p + 1],
                              pv[None, :, :p + 1], nv[None, :, :p + 1], np.array([p + 1]),
                              gqa, bk, bv, seed, 0.0)
    return out[0]


def _run(bk, bv, ctx, cap, Hkv, gqa, T, seed, rng_seed, q_dtype="f16", out_dtype="f32",
         qscale=1.0, n_splits=1):
    import torch
    import compressed_decode_attention_b200 as tq
    rng = np.random.default_rng(rng_seed)
    ctx = np.asarray(ctx, np.int32)
    B, Hq = len(ctx), Hkv * gqa
    pk, nk, pv, nv = _cache(bk, bv, B, Hkv, cap, ctx, seed, rng)
    qx = rng.standard_normal((B, T, Hq, D)) * qscale
    qb = S.to_bits(qx, q_dtype) if q_dtype != "f32" else qx.astype(np.float32)
    q64 = codec.promote(qb, q_dtype) if q_dtype != "f32" else qb.astype(np.float64)
    enum = {"f16": tq.TQ_F16, "bf16": tq.TQ_BF16, "f32": tq.TQ_F32}
    if out_dtype == "f32":
        out = torch.empty((B, T, Hq, D), dtype=torch.float32, device="cuda")
    else:
        out = torch.empty((B, T, Hq, D), dtype=torch.int16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    if n_splits == 1:
        tq.tq_prefill_attend(dev(qb), enum[q_dtype], dev(pk), dev(nk), dev(pv), dev(nv),
                             dev(ctx), B, T, Hq, gqa, D, bk, bv, seed, cap, out, enum[out_dtype],
                             dev_status=st)
    else:
        wsb = tq.tq_prefill_workspace_size(B, T, Hq, D, n_splits)
        ws = torch.full((wsb // 4,), float("nan"), dtype=torch.float32, device="cuda")
        tq.tq_prefill_attend_split(dev(qb), enum[q_dtype], dev(pk), dev(nk), dev(pv), dev(nv),
                                   dev(ctx), B, T, Hq, gqa, D, bk, bv, seed, cap, n_splits, ws,
                                   wsb, out, enum[out_dtype], dev_status=st)
    torch.cuda.synchronize()
    got = host(out)
    if out_dtype == "f16":
        got = got.view(np.float16).astype(np.float64)
    elif out_dtype == "bf16":
        got = (got.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    futs = {}
    for b in range(B):
        L = int(min(max(ctx[b], 0), cap))
        for t in range(T):
            p = L - T + t
            futs[b, t] = pool().submit(_oracle_token, q64[b, t], pk[b], nk[b], pv[b], nv[b], p,
                                       gqa, bk, bv, seed)
    want = np.zeros((B, T, Hq, D))
    for (b, t), f in futs.items():
        want[b, t] = f.result()
    # an fp16 / bf16 output adds its own rounding: unit roundoff 2^-11 / 2^-8
    # relative to |out|
    u = {"f32": 0.0, "f16": 2.0 ** -11, "bf16": 2.0 ** -8}[out_dtype]
    err = np.max(np.abs(got - want) - u * np.abs(want))
    print(f"K{bk}/V{bv} g={gqa} T={T}: max|err| = {err:.3e}")
    return err, int(st.item())


@pytest.mark.parametrize("bk,bv,gqa,T,q_dtype", [
    (4, 2, 4, 40, "f16"),     # 32 tokens per tile: a full and a partial tile
    (3, 2, 5, 30, "bf16"),    # 25 tokens per tile (125 of 128 rows)
    (4, 3, 8, 20, "f32"),     # 16 tokens per tile
    (2, 4, 1, 130, "f16"),    # 128 tokens per tile
    (3, 3, 2, 64, "f16"),
])
def test_prefill_matches_oracle(bk, bv, gqa, T, q_dtype):
    err, st = _run(bk, bv, [300, 180], 320, 2, gqa, T, 0, bk * 10 + bv + gqa, q_dtype)
    assert err <= ATOL
    assert st == 0


@pytest.mark.parametrize("bk,bv", [(bk, bv) for bk in (2, 3, 4) for bv in (2, 3, 4)])
def test_prefill_every_bit_pair(bk, bv):
    """Every (b_K, b_V) instantiation of the kernel (each has its own
    shared-memory layout and table copies), on a chunk of two partial tiles."""
    err, st = _run(bk, bv, [150], 160, 1, 4, 40, 0, 300 + 10 * bk + bv)
    assert err <= ATOL
    assert st == 0


@pytest.mark.parametrize("out_dtype", ["f16", "bf16"])
def test_prefill_output_dtypes(out_dtype):
    err, _ = _run(4, 2, [200], 256, 1, 4, 24, 3, 7, out_dtype=out_dtype)
    assert err <= ATOL                  # beyond the output type's own rounding


def test_prefill_context_shorter_than_chunk():
    """ctx = 5 < 12 tokens: the first 7 tokens have no positions (out = 0,
    TQ_DEV_CTX_EMPTY), the others attend causally."""
    err, st = _run(4, 2, [5, 70], 128, 2, 4, 12, 0, 9)
    assert err <= ATOL
    assert st == 4


def test_prefill_long_context_sharp_queries():
    """1500 cached positions (24 chunks), queries x4 (sharper softmax)."""
    err, st = _run(4, 2, [1500], 1536, 2, 4, 33, 0, 11, qscale=4.0)
    assert err <= ATOL


def test_prefill_full_workload_sampled():
    """The bench's prefill line: a 1024-token chunk at the end of an
    8192-position context, 32 query / 8 kv heads, K4/V2, fp16 output;
    tokens sampled across the tiles (first, tile edges, last) against the
    oracle."""
    import torch
    import compressed_decode_attention_b200 as tq
    rng = np.random.default_rng(41)
    B, Hkv, gqa, T, L, bk, bv, seed = 1, 8, 4, 1024, 8192, 4, 2, 0
    Hq = Hkv * gqa
    pk, nk, pv, nv = _cache(bk, bv, B, Hkv, L, np.array([L]), seed, rng)
    qb = S.f16_bits(rng.standard_normal((B, T, Hq, D)))
    q64 = codec.promote(qb, "f16")
    out = torch.empty((B, T, Hq, D), dtype=torch.int16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.tq_prefill_attend(dev(qb), tq.TQ_F16, dev(pk), dev(nk), dev(pv), dev(nv),
                         dev(np.array([L], np.int32)), B, T, Hq, gqa, D, bk, bv, seed, L, out,
                         tq.TQ_F16, dev_status=st)
    torch.cuda.synchronize()
    got = host(out).view(np.float16).astype(np.float64)
    sample = [0, 1, 31, 32, 511, 512, 1000, 1023]
    futs = {t: pool().submit(_oracle_token, q64[0, t], pk[0], nk[0], pv[0], nv[0], L - T + t,
                             gqa, bk, bv, seed) for t in sample}
    for t, f in futs.items():
        want = f.result()
        err = np.max(np.abs(got[0, t] - want) - 2.0 ** -11 * np.abs(want))
        assert err <= ATOL, (t, err)
    assert int(st.item()) == 0


@pytest.mark.parametrize("n_splits,bk,bv,gqa,T", [
    (2, 4, 2, 4, 40),
    (3, 3, 2, 5, 30),
    (4, 4, 3, 8, 20),
    (8, 2, 4, 1, 130),
])
def test_prefill_split_context_matches_oracle(n_splits, bk, bv, gqa, T):
    """The context of every tile split n ways (records merged by the combine
    kernel), including splits with no chunk: the oracle bar as unsplit."""
    err, st = _run(bk, bv, [300, 180], 320, 2, gqa, T, 0, 100 + bk * 10 + n_splits,
                   n_splits=n_splits)
    assert err <= ATOL
    assert st == 0


def test_prefill_split_short_context_and_dtypes():
    """ctx = 5 < 12 tokens with 4 splits: tokens without positions give 0 and
    TQ_DEV_CTX_EMPTY through the merge; bf16 output."""
    err, st = _run(4, 2, [5, 70], 128, 2, 4, 12, 0, 9, n_splits=4)
    assert err <= ATOL
    assert st == 4
    err, _ = _run(4, 2, [200], 256, 1, 4, 24, 3, 7, out_dtype="bf16", n_splits=3)
    assert err <= ATOL


@pytest.mark.parametrize("forced", [0, 4])
def test_prefill_split_full_workload_sampled(forced):
    """The bench's prefill chunk with the split count the library picks for
    this device (forced = 0) and with 4 context splits."""
    import torch
    import compressed_decode_attention_b200 as tq
    rng = np.random.default_rng(43)
    B, Hkv, gqa, T, L, bk, bv, seed = 1, 8, 4, 1024, 8192, 4, 2, 0
    Hq = Hkv * gqa
    pk, nk, pv, nv = _cache(bk, bv, B, Hkv, L, np.array([L]), seed, rng)
    qb = S.f16_bits(rng.standard_normal((B, T, Hq, D)))
    q64 = codec.promote(qb, "f16")
    n_splits = forced or tq.tq_prefill_splits(B, T, Hq, gqa, L)
    assert n_splits >= 1
    wsb = tq.tq_prefill_workspace_size(B, T, Hq, D, n_splits)
    ws = torch.empty(max(wsb, 16) // 4, dtype=torch.float32, device="cuda")
    out = torch.empty((B, T, Hq, D), dtype=torch.int16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.tq_prefill_attend_split(dev(qb), tq.TQ_F16, dev(pk), dev(nk), dev(pv), dev(nv),
                               dev(np.array([L], np.int32)), B, T, Hq, gqa, D, bk, bv, seed, L,
                               n_splits, ws, wsb, out, tq.TQ_F16, dev_status=st)
    torch.cuda.synchronize()
    got = host(out).view(np.float16).astype(np.float64)
    sample = [0, 31, 32, 500, 1023]
    futs = {t: pool().submit(_oracle_token, q64[0, t], pk[0], nk[0], pv[0], nv[0], L - T + t,
                             gqa, bk, bv, seed) for t in sample}
    for t, f in futs.items():
        want = f.result()
        err = np.max(np.abs(got[0, t] - want) - 2.0 ** -11 * np.abs(want))
        assert err <= ATOL, (t, err)
    assert int(st.item()) == 0
