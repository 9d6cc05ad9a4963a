"""GPU parity of tq_attend_append: one decode step (encode the new token of
every sequence into cache row ctx - 1, then attend over ctx positions) in one
launch, B200.

- The row it writes holds the oracle's encode of the new token under the
  encode bar (indices bit-exact outside the boundary window, norms within one
  fp16 ulp), and equals what tq_encode writes for the same token bit for bit;
  every other row is left as it was.
- The output is within 2e-3 of the float64 oracle attention run on the cache
  the call leaves behind (attend parity on the cache under test).
- The output equals tq_encode followed by tq_attend (same CTA split) bit for
  bit.
"""
import numpy as np
import pytest

import synthetic as S
from gpu_support import check_indices, check_norms, dev, host, oracle_attend
from oracle import codec

pytestmark = pytest.mark.gpu
ATOL = 2e-3


def _cache(bk, bv, B, Hkv, cap, ctx, seed, rng, D=128):
    """Oracle-encoded random cache with rows 0 .. L_b - 2 filled; row L_b - 1
    holds unrelated bytes that the append must replace."""
    pk = rng.integers(0, 256, (B, Hkv, cap, D * bk // 8), dtype=np.uint8)
    pv = rng.integers(0, 256, (B, Hkv, cap, D * bv // 8), dtype=np.uint8)
    nk = rng.integers(0, 0x3C00, (B, Hkv, cap), dtype=np.uint16)
    nv = rng.integers(0, 0x3C00, (B, Hkv, cap), dtype=np.uint16)
    for b in range(B):
        L = int(min(max(ctx[b], 0), cap))
        for g in range(Hkv):
            if L <= 1:
                continue
            k = rng.standard_normal((L - 1, D)) * 2
            v = rng.standard_normal((L - 1, D))
            pk[b, g, :L - 1], nk[b, g, :L - 1] = codec.encode_rows(
                codec.promote(S.f16_bits(k), "f16"), bk, seed)
            pv[b, g, :L - 1], nv[b, g, :L - 1] = codec.encode_rows(
                codec.promote(S.f16_bits(v), "f16"), bv, seed)
    return pk, nk, pv, nv


def _run(bk, bv, ctx, cap, Hkv, gqa, kv_dtype, seed, tau=0.0, n_ctas=0, qscale=1.0,
         rng_seed=0, D=128):
    import torch
    import compressed_decode_attention_b200 as tq
    rng = np.random.default_rng(rng_seed)
    ctx = np.asarray(ctx, np.int32)
    B, Hq = len(ctx), Hkv * gqa
    pk, nk, pv, nv = _cache(bk, bv, B, Hkv, cap, ctx, seed, rng, D)
    new = rng.standard_normal((2, B, Hkv, D))
    new[0, :, :, :4] *= 20.0                       # outlier K channels
    new_bits = S.to_bits(new, kv_dtype)
    qb = S.f16_bits(rng.standard_normal((B, Hq, D)) * qscale)
    kv_enum = tq.TQ_F16 if kv_dtype == "f16" else tq.TQ_BF16

    def call(fused):
        c = [dev(x) for x in (pk, nk, pv, nv)]
        ws_bytes = tq.tq_attend_workspace_size(B, Hq, cap, D)
        ws = torch.zeros(ws_bytes // 4, dtype=torch.float32, device="cuda")
        out = torch.empty((B, Hq, D), dtype=torch.float32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        sk = torch.zeros(1, dtype=torch.int64, device="cuda")
        ctx_d = dev(ctx)
        if fused:
            tq.tq_attend_append(dev(qb), tq.TQ_F16, dev(new_bits), kv_enum, c[0], c[1], c[2],
                                c[3], ctx_d, B, Hq, gqa, D, bk, bv, seed, cap, tau, n_ctas, ws,
                                ws_bytes, out, tq.TQ_F32, dev_status=st, sparse_v_skipped=sk)
        else:
            for b in range(B):
                L = int(min(ctx[b], cap))
                if L < 1:
                    continue
                one = dev(np.ascontiguousarray(new_bits[:, b:b + 1]))
                tq.tq_encode(one, kv_enum, 1, Hkv, D, bk, bv, seed, c[0][b], c[2][b], c[1][b],
                             c[3][b], cap, L - 1, st)
            tq.tq_attend(dev(qb), tq.TQ_F16, c[0], c[1], c[2], c[3], ctx_d, B, Hq, gqa, D, bk,
                         bv, seed, cap, tau, n_ctas, ws, ws_bytes, out, tq.TQ_F32,
                         dev_status=st, sparse_v_skipped=sk)
        torch.cuda.synchronize()
        return [host(x) for x in c], host(out), int(st.item()), int(sk.item())

    (gk, gnk, gv, gnv), out, st, sk = call(True)
    (ek, enk, ev, env), out_e, st_e, sk_e = call(False)

    # the appended rows: oracle encode bar, and identical to tq_encode's rows
    for b in range(B):
        L = int(min(max(ctx[b], 0), cap))
        keep = np.ones(cap, bool)
        if L >= 1:
            keep[L - 1] = False
            for which, bits, rows, norms in ((0, bk, gk, gnk), (1, bv, gv, gnv)):
                x = codec.promote(new_bits[which, b], kv_dtype)
                idx, _, nbits, _, margin = codec.encode(x, bits, seed)
                check_indices(codec.unpack(rows[b, :, L - 1], bits, D), idx, margin)
                check_norms(norms[b, :, L - 1], nbits)
        for ref, got in ((pk, gk), (nk, gnk), (pv, gv), (nv, gnv)):
            np.testing.assert_array_equal(got[b][:, keep], ref[b][:, keep])
    for got, exp in ((gk, ek), (gnk, enk), (gv, ev), (gnv, env)):
        np.testing.assert_array_equal(got, exp)
    np.testing.assert_array_equal(out, out_e)
    assert (st, sk) == (st_e, sk_e)

    # attention parity on the cache the call left behind
    q64 = codec.promote(qb, "f16")
    want, ng = oracle_attend(q64, gk, gnk, gv, gnv, ctx, gqa, bk, bv, seed, tau)
    err = np.abs(out - want).max()
    assert err <= ATOL, err
    return st, sk, ng


def test_append_k4v2_ragged_empty_and_clamped():
    st, _, _ = _run(4, 2, [700, 64, 1, 0, 1000], 768, 2, 4, "f16", 0, rng_seed=1)
    assert st == 1 | 4          # one clamped, one empty sequence


@pytest.mark.parametrize("n_ctas", [0, 7, 37])
def test_append_k3v2_bf16_group5(n_ctas):
    _run(3, 2, [513, 129, 64, 2], 640, 2, 5, "bf16", 0, n_ctas=n_ctas, rng_seed=2)


def test_append_k4v3_gate():
    st, sk, ng = _run(4, 3, [1500, 333, 960], 1536, 2, 4, "f16", 5, tau=1e-6, qscale=8.0,
                      rng_seed=3)
    assert ng > 0 and st == 0


def test_append_single_sequence_eight_heads():
    _run(4, 2, [4096], 4096, 8, 4, "f16", 0, rng_seed=4)


@pytest.mark.parametrize("d,bk,bv,gqa", [(64, 4, 2, 4), (64, 3, 2, 5), (256, 4, 3, 4),
                                         (256, 3, 2, 5)])
def test_append_head_dims(d, bk, bv, gqa):
    """d = 64 and 256: the new token's rows (d/32 lanes per vector) and the
    attention over the updated cache."""
    _run(bk, bv, [700, 64, 1, 1000], 768, 2, gqa, "f16", 0, rng_seed=10 + d + bk, D=d)


def test_per_layer_bit_choice_in_one_step():
    """A decode step over layers with different bit widths (K4/V2, K3/V2,
    K4/V3, K2/V4), sharing one workspace, each layer one tq_attend_append
    call: every layer's output and appended rows match the oracle (a model
    may choose the bits per layer)."""
    import torch
    import compressed_decode_attention_b200 as tq
    rng = np.random.default_rng(77)
    B, Hkv, gqa, cap, seed = 2, 2, 4, 512, 3
    Hq = Hkv * gqa
    ctx = np.array([300, 97], np.int32)
    ws_bytes = tq.tq_attend_workspace_size(B, Hq, cap, 128)
    ws = torch.zeros(ws_bytes // 4, dtype=torch.float32, device="cuda")
    layers = [(4, 2), (3, 2), (4, 3), (2, 4)]
    caches, news, qs, outs = [], [], [], []
    for bk, bv in layers:
        pk, nk, pv, nv = _cache(bk, bv, B, Hkv, cap, ctx, seed, rng)
        caches.append([dev(x) for x in (pk, nk, pv, nv)])
        news.append(S.f16_bits(rng.standard_normal((2, B, Hkv, 128))))
        qs.append(S.f16_bits(rng.standard_normal((B, Hq, 128))))
        outs.append(torch.empty((B, Hq, 128), dtype=torch.float32, device="cuda"))
    ctx_d = dev(ctx)
    for l, (bk, bv) in enumerate(layers):
        c = caches[l]
        tq.tq_attend_append(dev(qs[l]), tq.TQ_F16, dev(news[l]), tq.TQ_F16, c[0], c[1], c[2],
                            c[3], ctx_d, B, Hq, gqa, 128, bk, bv, seed, cap, 0.0, 0, ws, ws_bytes,
                            outs[l], tq.TQ_F32)
    torch.cuda.synchronize()
    for l, (bk, bv) in enumerate(layers):
        gk, gnk, gv, gnv = [host(x) for x in caches[l]]
        for b in range(B):
            for which, bits, rows in ((0, bk, gk), (1, bv, gv)):
                x = codec.promote(news[l][which, b], "f16")
                idx, _, _, _, margin = codec.encode(x, bits, seed)
                check_indices(codec.unpack(rows[b, :, ctx[b] - 1], bits, 128), idx, margin)
        want, _ = oracle_attend(codec.promote(qs[l], "f16"), gk, gnk, gv, gnv, ctx, gqa, bk, bv,
                                seed)
        assert np.abs(host(outs[l]) - want).max() <= ATOL, (bk, bv)


def test_append_full_workload_bench_configuration():
    """The bench's decode step at full size: the Llama-3-8B-shaped layer
    (8 kv heads, 32768 positions, K4/V2, GQA 4, one CTA per SM) with its
    last row replaced by the new token, fp16 output as timed."""
    import torch
    import compressed_decode_attention_b200 as tq
    from gpu_support import oracle_cache
    w = S.WORKLOADS["llama3_8b_decode"]
    pk, nk, pv, nv, ctx = oracle_cache("llama3_8b_decode")
    B, H, cap, d = pk.shape[0], pk.shape[1], pk.shape[2], w.d
    rng = np.random.default_rng(31)
    new = rng.standard_normal((2, B, H, d))
    new_bits = S.f16_bits(new)
    qb = S.query_bits(w, step=3)
    c = [dev(x) for x in (pk, nk, pv, nv)]
    ws_bytes = tq.tq_attend_workspace_size(B, w.n_q_heads, cap, d)
    ws = torch.zeros(ws_bytes // 4, dtype=torch.float32, device="cuda")
    out = torch.empty((B, w.n_q_heads, d), dtype=torch.int16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.tq_attend_append(dev(qb), tq.TQ_F16, dev(new_bits), tq.TQ_F16, c[0], c[1], c[2], c[3],
                        dev(ctx), B, w.n_q_heads, w.gqa, d, w.bits_k, w.bits_v, 0, cap, 0.0, 0,
                        ws, ws_bytes, out, tq.TQ_F16, dev_status=st)
    torch.cuda.synchronize()
    gk, gnk, gv, gnv = [host(x) for x in c]
    L = int(ctx[0])
    for which, bits, rows, norms in ((0, w.bits_k, gk, gnk), (1, w.bits_v, gv, gnv)):
        x = codec.promote(new_bits[which, 0], "f16")
        idx, _, nbits, _, margin = codec.encode(x, bits, 0)
        check_indices(codec.unpack(rows[0, :, L - 1], bits, d), idx, margin)
        check_norms(norms[0, :, L - 1], nbits)
    keep = np.ones(cap, bool)
    keep[L - 1] = False
    np.testing.assert_array_equal(gk[0][:, keep], pk[0][:, keep])
    np.testing.assert_array_equal(gv[0][:, keep], pv[0][:, keep])
    want, _ = oracle_attend(codec.promote(qb, "f16"), gk, gnk, gv, gnv, ctx, w.gqa, w.bits_k,
                            w.bits_v, 0)
    got = host(out).view(np.float16).astype(np.float64)
    # fp16 output: its own rounding (2^-11 relative) on top of the bound
    assert np.max(np.abs(got - want) - 2.0 ** -11 * np.abs(want)) <= ATOL
    assert int(st.item()) == 0
