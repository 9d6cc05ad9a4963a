"""GPU parity of the stage-2 residual sketch (tq_qjl_encode) and the score
estimate (tq_qjl_scores) against the float64 oracle, B200.

- Sketch bits equal the oracle's except where the projection (S·r~)_i lies
  within 1e-4·|S_i|·|r~| of zero (the GPU forms r~ and S·r~ in fp32); such
  bits are at most 1e-3 of all. Residual norms within one fp16 ulp.
- Scores within 2e-3 of the oracle's, computed from the same cache (built by
  the oracle), with and without the sketch term.
"""
import numpy as np
import pytest

import synthetic as S
from gpu_support import dev, host
from oracle import codec, qjl

pytestmark = pytest.mark.gpu
ATOL = 2e-3


def _keys(rng, n, H, d, dtype="f16"):
    k = rng.standard_normal((n, H, d)) * 2.0
    k[:, :, :4] *= 10.0                               # outlier channels
    bits = S.to_bits(k, dtype)
    return bits, codec.promote(bits, dtype)


@pytest.mark.parametrize("d,bits,dtype", [(128, 4, "f16"), (128, 2, "bf16"), (128, 3, "f16"),
                                          (64, 4, "f16"), (256, 3, "f16")])
def test_sketch_matches_oracle(d, bits, dtype):
    import torch
    import compressed_decode_attention_b200 as tq
    rng = np.random.default_rng(d + bits)
    n, H, cap, off, seed = 300, 2, 320, 7, 4
    kb, kx = _keys(rng, n, H, d, dtype)
    Sm = S.projection_matrix(d)
    pk = np.zeros((H, cap, d * bits // 8), np.uint8)
    nk = np.zeros((H, cap), np.uint16)
    want_rows = np.zeros((H, n, d // 8), np.uint8)
    want_g = np.zeros((H, n), np.uint16)
    want_u = np.zeros((H, n, d))
    rr = np.zeros((H, n))
    for h in range(H):
        p, nb, rows, gb, u = qjl.encode(kx[:, h], bits, seed, Sm.astype(np.float64))
        pk[h, off:off + n], nk[h, off:off + n] = p, nb
        want_rows[h], want_g[h], want_u[h] = rows, gb, u
        rr[h] = np.sqrt(np.sum(qjl.residual_rotated(kx[:, h], bits, seed)[2] ** 2, axis=1))
    sketch = torch.full((H, cap, d // 8), 0x5A, dtype=torch.uint8, device="cuda")
    gamma = torch.full((H, cap), 0x7E00, dtype=torch.int16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.tq_qjl_encode(dev(kb), tq.TQ_F16 if dtype == "f16" else tq.TQ_BF16, n, H, d, bits, seed,
                     dev(Sm), dev(pk), dev(nk), sketch, gamma, cap, off, st)
    torch.cuda.synchronize()
    got = host(sketch)
    gg = host(gamma)
    assert int(st.item()) == 0
    # rows outside [off, off + n) untouched
    assert np.all(got[:, :off] == 0x5A) and np.all(got[:, off + n:] == 0x5A)
    assert np.all(gg[:, :off] == 0x7E00) and np.all(gg[:, off + n:] == 0x7E00)
    gb_bits = np.unpackbits(got[:, off:off + n], axis=-1, bitorder="little")
    wb_bits = np.unpackbits(want_rows, axis=-1, bitorder="little")
    snorm = np.linalg.norm(Sm.astype(np.float64), axis=1)
    margin = np.abs(want_u) / (snorm[None, None, :] * np.maximum(rr[:, :, None], 1e-30))
    bad = (gb_bits != wb_bits) & (margin >= 1e-4)
    assert not bad.any(), int(bad.sum())
    assert (gb_bits != wb_bits).mean() <= 1e-3
    ulp = np.abs(gg[:, off:off + n].astype(np.int64) - want_g.astype(np.int64))
    assert ulp.max() <= 1


def _cache(rng, B, H, cap, ctx, d, bits, seed, Sm):
    pk = np.zeros((B, H, cap, d * bits // 8), np.uint8)
    nk = np.zeros((B, H, cap), np.uint16)
    sk = np.zeros((B, H, cap, d // 8), np.uint8)
    gk = np.zeros((B, H, cap), np.uint16)
    for b in range(B):
        L = int(min(max(ctx[b], 0), cap))
        for h in range(H):
            _, kx = _keys(rng, L, 1, d)
            pk[b, h, :L], nk[b, h, :L], sk[b, h, :L], gk[b, h, :L], _ = qjl.encode(
                kx[:, 0], bits, seed, Sm.astype(np.float64))
    return pk, nk, sk, gk


@pytest.mark.parametrize("d,bits,gqa,q_dtype,sketch", [
    (128, 4, 4, "f16", True),
    (128, 4, 4, "f16", False),
    (128, 2, 5, "bf16", True),
    (128, 3, 8, "f32", True),
    (64, 4, 1, "f16", True),
    (256, 3, 4, "f16", True),
])
def test_scores_match_oracle(d, bits, gqa, q_dtype, sketch):
    import torch
    import compressed_decode_attention_b200 as tq
    rng = np.random.default_rng(10 * d + bits + gqa)
    B, H, cap, seed = 3, 2, 1280, 2
    ctx = np.array([1280, 700, 0], np.int32)
    Sm = S.projection_matrix(d, 3)
    pk, nk, sk, gk = _cache(rng, B, H, cap, ctx, d, bits, seed, Sm)
    qx = rng.standard_normal((B, H * gqa, d))
    qb = S.to_bits(qx, q_dtype) if q_dtype != "f32" else qx.astype(np.float32)
    q64 = codec.promote(qb, q_dtype) if q_dtype != "f32" else qb.astype(np.float64)
    out = torch.full((B, H * gqa, cap), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    enum = {"f16": tq.TQ_F16, "bf16": tq.TQ_BF16, "f32": tq.TQ_F32}[q_dtype]
    tq.tq_qjl_scores(dev(qb), enum, dev(pk), dev(nk), dev(sk), dev(gk), dev(Sm), dev(ctx), B,
                     H * gqa, gqa, d, bits, seed, cap, sketch, out, dev_status=st)
    torch.cuda.synchronize()
    got = host(out)
    want = qjl.scores(q64, pk, nk, sk, gk, ctx, gqa, bits, seed, Sm.astype(np.float64), sketch)
    for b in range(B):
        L = int(min(max(ctx[b], 0), cap))
        assert np.all(np.isnan(got[b, :, L:]))          # not written
        if L:
            err = np.abs(got[b, :, :L] - want[b, :, :L]).max()
            assert err <= ATOL, err
    assert int(st.item()) == 4                          # the empty sequence


def test_gpu_sketch_rows_feed_the_scores():
    """tq_encode -> tq_qjl_encode -> tq_qjl_scores on the GPU against the
    oracle scores on the GPU's own rows (bits that differ from the oracle's
    encode sit at near-zero projections and cancel to first order)."""
    import torch
    import compressed_decode_attention_b200 as tq
    rng = np.random.default_rng(77)
    n, H, d, bits, seed, gqa = 2048, 2, 128, 4, 0, 4
    kb, _ = _keys(rng, n, H, d)
    vb = S.f16_bits(rng.standard_normal((n, H, d)))
    Sm = S.projection_matrix(d, 9)
    kv = np.stack([kb, vb])
    pk = torch.zeros((H, n, d * bits // 8), dtype=torch.uint8, device="cuda")
    pv = torch.zeros((H, n, d * 2 // 8), dtype=torch.uint8, device="cuda")
    nk = torch.zeros((H, n), dtype=torch.int16, device="cuda")
    nv = torch.zeros((H, n), dtype=torch.int16, device="cuda")
    sk = torch.zeros((H, n, d // 8), dtype=torch.uint8, device="cuda")
    gk = torch.zeros((H, n), dtype=torch.int16, device="cuda")
    tq.tq_encode(dev(kv), tq.TQ_F16, n, H, d, bits, 2, seed, pk, pv, nk, nv, n, 0)
    tq.tq_qjl_encode(dev(kb), tq.TQ_F16, n, H, d, bits, seed, dev(Sm), pk, nk, sk, gk, n, 0)
    qb = S.f16_bits(rng.standard_normal((1, H * gqa, d)))
    out = torch.empty((1, H * gqa, n), dtype=torch.float32, device="cuda")
    ctx = dev(np.array([n], np.int32))
    tq.tq_qjl_scores(dev(qb), tq.TQ_F16, pk, nk, sk, gk, dev(Sm), ctx, 1, H * gqa, gqa, d, bits,
                     seed, n, 1, out)
    torch.cuda.synchronize()
    want = qjl.scores(codec.promote(qb, "f16"), host(pk)[None], host(nk)[None], host(sk)[None],
                      host(gk)[None], np.array([n]), gqa, bits, seed, Sm.astype(np.float64))
    assert np.abs(host(out) - want).max() <= ATOL


def _oracle_head_sketch(kx, pk_h, nk_h, bits, seed, Sm):
    """Worker: oracle sketch rows / gamma / projections of one kv head."""
    from oracle import qjl as oq
    r_rot = oq.residual_rotated(kx, bits, seed)[2]
    rows, u, gb = oq.sketch(r_rot, Sm)
    return rows, gb, u, np.sqrt(np.sum(r_rot ** 2, axis=1))


def test_full_workload_sketch_and_scores():
    """The bench's QJL line at full size: the Llama-3-8B-shaped layer's keys
    (8 kv heads x 32768) sketched on the GPU against the oracle, then the
    scores of its 32 query heads from the GPU's own rows."""
    import torch
    import compressed_decode_attention_b200 as tq
    from gpu_support import oracle_cache, pool
    w = S.WORKLOADS["llama3_8b_decode"]
    pk, nk, pv, nv, ctx = oracle_cache("llama3_8b_decode")
    H, cap, d, bits, n = w.n_kv_heads, w.cap_tok, w.d, w.bits_k, int(ctx[0])
    kv = S.kv_bits(w, 0, n)                               # [2][n][H][d], the cached keys
    Sm = S.projection_matrix(d)
    sk = torch.zeros((1, H, cap, d // 8), dtype=torch.uint8, device="cuda")
    gk = torch.zeros((1, H, cap), dtype=torch.int16, device="cuda")
    tq.tq_qjl_encode(dev(np.ascontiguousarray(kv[0])), tq.TQ_F16, n, H, d, bits, 0, dev(Sm),
                     dev(pk[0]), dev(nk[0]), sk, gk, cap, 0)
    torch.cuda.synchronize()
    got_rows, got_g = host(sk)[0], host(gk)[0]
    futs = [pool().submit(_oracle_head_sketch, codec.promote(kv[0, :, h], "f16"), pk[0, h],
                          nk[0, h], bits, 0, Sm.astype(np.float64)) for h in (0, 5)]
    snorm = np.linalg.norm(Sm.astype(np.float64), axis=1)
    for h, f in zip((0, 5), futs):
        rows, gb, u, rr = f.result()
        gbits = np.unpackbits(got_rows[h, :n], axis=-1, bitorder="little")
        wbits = np.unpackbits(rows, axis=-1, bitorder="little")
        margin = np.abs(u) / (snorm[None, :] * np.maximum(rr[:, None], 1e-30))
        assert not ((gbits != wbits) & (margin >= 1e-4)).any()
        assert (gbits != wbits).mean() <= 1e-3
        assert np.abs(got_g[h, :n].astype(np.int64) - gb.astype(np.int64)).max() <= 1
    qb = S.query_bits(w, step=7)
    out = torch.empty((1, w.n_q_heads, cap), dtype=torch.float32, device="cuda")
    tq.tq_qjl_scores(dev(qb), tq.TQ_F16, dev(pk), dev(nk), sk, gk, dev(Sm), dev(ctx), 1,
                     w.n_q_heads, w.gqa, d, bits, 0, cap, 1, out)
    torch.cuda.synchronize()
    want = qjl.scores(codec.promote(qb, "f16"), pk, nk, got_rows[None], got_g[None], ctx, w.gqa,
                      bits, 0, Sm.astype(np.float64))
    assert np.abs(host(out) - want).max() <= ATOL
