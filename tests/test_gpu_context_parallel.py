"""GPU parity of context-parallel attention (tq_attend_partial per slice,
then tq_attend_combine), B200.

The ranks of a context-parallel group are emulated on one GPU: each slice of
the cache lives in device buffers of its own, as on its own rank, and its
records go to row p of the gathered buffer that the all-gather would fill.
- The merged output is within 2e-3 of the float64 oracle attention over the
  whole context, and within 2e-4 of tq_attend on the whole cache.
- Each slice's records match the oracle's records of that slice: the base-2
  maximum within 1e-3, the normalized value sum acc / l within 2e-3 (it maps
  to the output through an orthonormal matrix, scaled by 1/sqrt(d)).
- The gate skips the same positions as one pass (slices are whole blocks).
"""
import numpy as np
import pytest

import synthetic as S
from gpu_support import dev, gpu_attend, host, oracle_attend, pool
from oracle import codec

pytestmark = pytest.mark.gpu
ATOL = 2e-3


def _cache(bk, bv, B, Hkv, cap, ctx, seed, rng, d):
    pk = np.zeros((B, Hkv, cap, d * bk // 8), np.uint8)
    pv = np.zeros((B, Hkv, cap, d * bv // 8), np.uint8)
    nk = np.zeros((B, Hkv, cap), np.uint16)
    nv = np.zeros((B, Hkv, cap), np.uint16)
    for b in range(B):
        L = int(min(max(ctx[b], 0), cap))
        for g in range(Hkv):
            k = rng.standard_normal((L, d)) * 2
            k[:, :4] *= 10.0                               # outlier channels
            v = rng.standard_normal((L, d))
            pk[b, g, :L], nk[b, g, :L] = codec.encode_rows(codec.promote(S.f16_bits(k), "f16"),
                                                           bk, seed)
            pv[b, g, :L], nv[b, g, :L] = codec.encode_rows(codec.promote(S.f16_bits(v), "f16"),
                                                           bv, seed)
    return pk, nk, pv, nv


def _oracle_records(q64, part, loc, gqa, bk, bv, seed, tau):
    from oracle import attention
    return attention.attend_partial(q64, *part, loc, gqa, bk, bv, seed, tau)[0]


def _run(bk, bv, ctx, cap, Hkv, gqa, d, n_parts, seed=0, tau=0.0, qscale=1.0, n_ctas=0,
         out_dtype="f32", rng_seed=0, check_records=True):
    import torch
    import compressed_decode_attention_b200 as tq
    from compressed_decode_attention_b200.context_parallel import local_ctx_lens, slice_bounds
    rng = np.random.default_rng(rng_seed)
    ctx = np.asarray(ctx, np.int32)
    B, Hq = len(ctx), Hkv * gqa
    arrs = _cache(bk, bv, B, Hkv, cap, ctx, seed, rng, d)
    qb = S.f16_bits(rng.standard_normal((B, Hq, d)) * qscale)
    q64 = codec.promote(qb, "f16")
    qd = dev(qb)
    gathered = torch.full((n_parts, B, Hq, d + 2), float("nan"), dtype=torch.float32,
                          device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sk = torch.zeros(1, dtype=torch.int64, device="cuda")
    ws_bytes = tq.tq_attend_workspace_size(B, Hq, cap, d)
    ws = torch.zeros(ws_bytes // 4, dtype=torch.float32, device="cuda")
    futs = []
    for p in range(n_parts):
        a, b = slice_bounds(cap, n_parts, p)
        loc = local_ctx_lens(np.minimum(ctx, cap), a, b).astype(np.int32)
        part = [np.ascontiguousarray(x[:, :, a:b]) for x in arrs]
        if b == a:                                  # a rank with no positions
            part = [np.zeros(x.shape[:2] + (8,) + x.shape[3:], x.dtype) for x in arrs]
        lc = part[0].shape[2]
        c = [dev(x) for x in part]
        tq.tq_attend_partial(qd, tq.TQ_F16, c[0], c[1], c[2], c[3], dev(loc), B, Hq, gqa, d, bk,
                             bv, seed, lc, tau, n_ctas, ws, ws_bytes, gathered[p],
                             dev_status=st, sparse_v_skipped=sk)
        if check_records:
            futs.append(pool().submit(_oracle_records, q64, part, loc, gqa, bk, bv, seed, tau))
    enum = {"f16": tq.TQ_F16, "bf16": tq.TQ_BF16, "f32": tq.TQ_F32}[out_dtype]
    out = torch.empty((B, Hq, d), dtype=torch.float32 if out_dtype == "f32" else torch.int16,
                      device="cuda")
    cst = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.tq_attend_combine(gathered, n_parts, B, Hq, d, seed, out, enum, dev_status=cst)
    torch.cuda.synchronize()
    got = host(out)
    if out_dtype == "f16":
        got = got.view(np.float16).astype(np.float64)
    elif out_dtype == "bf16":
        got = (got.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    recs = host(gathered).astype(np.float64)

    # records of every slice against the oracle's
    for p, f in enumerate(futs):
        want = f.result()
        live = np.isfinite(want[..., d])
        assert np.array_equal(np.isfinite(recs[p][..., d]), live)
        assert np.all(recs[p][~live][..., d] == -np.inf)
        assert np.all(recs[p][~live][..., :d] == 0) and np.all(recs[p][~live][..., d + 1] == 0)
        if live.any():
            assert np.abs(recs[p][live][:, d] - want[live][:, d]).max() <= 1e-3
            y_got = recs[p][live][:, :d] / recs[p][live][:, d + 1:] / np.sqrt(d)
            y_want = want[live][:, :d] / want[live][:, d + 1:] / np.sqrt(d)
            assert np.abs(y_got - y_want).max() <= ATOL

    # merged output: oracle over the whole context, and one pass on the GPU
    want, n_gated = oracle_attend(q64, *arrs, ctx, gqa, bk, bv, seed, tau)
    u = {"f32": 0.0, "f16": 2.0 ** -11, "bf16": 2.0 ** -8}[out_dtype]
    err = np.max(np.abs(got - want) - u * np.abs(want))
    assert err <= ATOL, err
    one, st1, sk1 = gpu_attend(qb, "f16", *arrs, ctx, gqa, bk, bv, seed, tau, n_ctas,
                               out_dtype=enum)
    if out_dtype == "f32":
        assert np.abs(got - one).max() <= 2e-4
    assert int(sk.item()) == sk1
    return int(st.item()), int(cst.item()), int(sk.item()), n_gated


@pytest.mark.parametrize("d,bk,bv,gqa,n_parts", [
    (128, 4, 2, 4, 2),
    (128, 3, 2, 5, 3),
    (128, 4, 3, 4, 4),
    (64, 4, 2, 4, 3),
    (256, 3, 2, 5, 2),
])
def test_slices_merge_to_one_pass(d, bk, bv, gqa, n_parts):
    """Ragged contexts: one sequence ends inside the first slice (later
    slices are empty for it), one is empty everywhere."""
    st, cst, _, _ = _run(bk, bv, [640, 100, 0, 513], 640, 2, gqa, d, n_parts,
                         rng_seed=d + bk * 10 + n_parts)
    assert st & 4 and cst == 4                       # the empty sequence


def test_gate_with_slices():
    """Sharp queries and tau = 1e-3: the slices skip exactly the positions one
    pass skips, and the merged output keeps the one-pass parity."""
    _, _, sk, ng = _run(4, 2, [1024, 700], 1024, 2, 4, 128, 4, tau=1e-3, qscale=8.0,
                        rng_seed=5)
    assert sk > 0


def test_many_slices_and_forced_ctas():
    """40 slices of 64 positions (more parts than a warp has lanes) and
    slices spread over several CTAs each (the cross-CTA merge)."""
    _run(4, 2, [2560, 1900], 2560, 1, 4, 128, 40, rng_seed=6, check_records=False)
    _run(4, 2, [2560, 1900], 2560, 2, 4, 128, 2, n_ctas=37, rng_seed=7)


@pytest.mark.parametrize("out_dtype", ["f16", "bf16"])
def test_combine_output_dtypes(out_dtype):
    _run(4, 2, [300, 64], 320, 2, 4, 128, 2, out_dtype=out_dtype, rng_seed=8,
         check_records=False)


def test_all_slices_empty():
    import torch
    import compressed_decode_attention_b200 as tq
    n, B, Hq, d = 3, 2, 4, 128
    rec = np.zeros((n, B, Hq, d + 2), np.float32)
    rec[..., d] = -np.inf
    out = torch.full((B, Hq, d), 7.0, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.tq_attend_combine(dev(rec), n, B, Hq, d, 0, out, tq.TQ_F32, dev_status=st)
    torch.cuda.synchronize()
    assert np.all(host(out) == 0.0)
    assert int(st.item()) == 4


def test_odd_record_count_alignment():
    """batch x heads odd (3 x 5): row p of the gathered buffer is only 8-byte
    aligned, which the records allow."""
    _run(4, 2, [300, 200, 129], 320, 1, 5, 128, 3, rng_seed=9)


def test_full_workload_four_slices_as_timed():
    """The bench's context-parallel line: the Llama-3-8B-shaped layer (8 kv
    heads x 32768 positions) split into 4 slices that are views of one
    cache (row offset, cap_tok kept as the head stride), merged by
    tq_attend_combine; against the oracle over the whole context."""
    import torch
    import compressed_decode_attention_b200 as tq
    from compressed_decode_attention_b200.context_parallel import slice_bounds
    from gpu_support import oracle_cache
    w = S.WORKLOADS["llama3_8b_decode"]
    pk, nk, pv, nv, ctx = oracle_cache("llama3_8b_decode")
    B, H, cap, d = pk.shape[0], pk.shape[1], pk.shape[2], w.d
    qb = S.query_bits(w, step=5)
    c = [dev(x) for x in (pk, nk, pv, nv)]
    rk, rv = d * w.bits_k // 8, d * w.bits_v // 8
    P = 4
    rec = torch.empty((P, B, w.n_q_heads, d + 2), dtype=torch.float32, device="cuda")
    ws_bytes = tq.tq_attend_workspace_size(B, w.n_q_heads, cap, d)
    ws = torch.zeros(ws_bytes // 4, dtype=torch.float32, device="cuda")
    qd = dev(qb)
    for r in range(P):
        a, b = slice_bounds(int(ctx[0]), P, r)
        lens = dev(np.array([b - a], np.int32))
        tq.tq_attend_partial(qd, tq.TQ_F16, c[0].data_ptr() + a * rk, c[1].data_ptr() + 2 * a,
                             c[2].data_ptr() + a * rv, c[3].data_ptr() + 2 * a, lens, B,
                             w.n_q_heads, w.gqa, d, w.bits_k, w.bits_v, 0, cap, 0.0, 0, ws,
                             ws_bytes, rec[r])
    out = torch.empty((B, w.n_q_heads, d), dtype=torch.int16, device="cuda")
    tq.tq_attend_combine(rec, P, B, w.n_q_heads, d, 0, out, tq.TQ_F16)
    torch.cuda.synchronize()
    want, _ = oracle_attend(codec.promote(qb, "f16"), pk, nk, pv, nv, ctx, w.gqa, w.bits_k,
                            w.bits_v, 0)
    got = host(out).view(np.float16).astype(np.float64)
    assert np.max(np.abs(got - want) - 2.0 ** -11 * np.abs(want)) <= ATOL
