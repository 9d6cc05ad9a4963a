"""GPU parity at head dimensions 64 and 256 (B200): encode, dequant and
attention against the oracle, with the bars of the d = 128 tests.

"We Built a Python Library That Cuts LLM Memory Usage by 80%" (§The Paper)
computes the codebook for a given head dimension; the randomized Hadamard
rotation takes any power of two, and d = 64 and 256 are the head sizes the
pages name besides 128. The library runs d/32 lanes per vector in the encode
and d/32 values per lane, d/16 MMA k-steps and d/16 PV tiles in attention.
"""
import numpy as np
import pytest

import synthetic as S
from gpu_support import (check_indices, check_norms, dev, gpu_attend, gpu_encode, host,
                         oracle_attend, oracle_encode_heads, oracle_gate_table)
from oracle import codec

pytestmark = pytest.mark.gpu
SEED = S.SIGN_SEED
ATOL = 2e-3
DIMS = [64, 256]


def _kv_bits(d, n, H, dtype, rng):
    """K/V ~N(0,1) with 4 outlier K channels x20 (per head), as 16-bit patterns."""
    x = rng.standard_normal((2, n, H, d))
    for h in range(H):
        x[0, :, h, rng.choice(d, 4, replace=False)] *= 20.0
    return S.to_bits(x, dtype)


@pytest.mark.parametrize("d", DIMS)
@pytest.mark.parametrize("bk,bv,dtype", [(4, 2, "f16"), (3, 2, "bf16"), (4, 3, "f16"),
                                         (2, 4, "bf16")])
def test_encode_head_dims(d, bk, bv, dtype):
    rng = np.random.default_rng(d * 10 + bk)
    kv = _kv_bits(d, 1500, 3, dtype, rng)
    pk, nk, pv, nv, st = gpu_encode(kv, dtype, bk, bv, SEED, cap=1504, tok_offset=3)
    assert st == 0
    for which, bits, rows, nb in ((0, bk, pk, nk), (1, bv, pv, nv)):
        idx_o, nb_o, mg = oracle_encode_heads(kv, dtype, which, bits, SEED)
        H, n = idx_o.shape[:2]
        idx_g = codec.unpack(rows[:, 3:3 + n].reshape(H * n, -1), bits, d).reshape(H, n, d)
        check_indices(idx_g, idx_o, mg)
        check_norms(nb[:, 3:3 + n], nb_o)


@pytest.mark.parametrize("d", DIMS)
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_dequant_head_dims(d, bits):
    import torch
    import compressed_decode_attention_b200 as tq
    rng = np.random.default_rng(d + bits)
    kv = _kv_bits(d, 300, 2, "f16", rng)
    idx, nb, _ = oracle_encode_heads(kv, "f16", 0, bits, SEED)
    H, n, _ = idx.shape
    cap = 320
    rows_c = np.zeros((H, cap, d * bits // 8), np.uint8)
    nb_c = np.zeros((H, cap), np.uint16)
    for h in range(H):
        rows_c[h, :n] = codec.pack(idx[h].astype(np.int64), bits)
        nb_c[h, :n] = nb[h]
    for domain in (0, 1):
        out = torch.empty((H, n, d), dtype=torch.float32, device="cuda")
        tq.tq_dequant(dev(rows_c), dev(nb_c), n, H, d, bits, SEED, cap, domain, out)
        torch.cuda.synchronize()
        got = host(out)
        for h in range(H):
            if domain == 1:
                want = codec.dequant_rotated(idx[h].astype(np.int64), bits)
                np.testing.assert_allclose(got[h], want, rtol=1e-6, atol=0)
            else:
                want = codec.dequant(idx[h].astype(np.int64), nb[h], bits, SEED)
                scale = np.linalg.norm(want, axis=1, keepdims=True) + 1e-30
                assert np.max(np.abs(got[h] - want) / scale) < 2e-6


def _cache(bk, bv, B, Hkv, cap, ctx, seed, rng, d):
    pk = np.zeros((B, Hkv, cap, d * bk // 8), np.uint8)
    pv = np.zeros((B, Hkv, cap, d * bv // 8), np.uint8)
    nk = np.zeros((B, Hkv, cap), np.uint16)
    nv = np.zeros((B, Hkv, cap), np.uint16)
    for b in range(B):
        L = int(min(max(ctx[b], 0), cap))
        for g in range(Hkv):
            k = rng.standard_normal((L, d)) * 2
            k[:, :4] *= 10.0
            v = rng.standard_normal((L, d))
            pk[b, g, :L], nk[b, g, :L] = codec.encode_rows(codec.promote(S.f16_bits(k), "f16"),
                                                           bk, seed)
            pv[b, g, :L], nv[b, g, :L] = codec.encode_rows(codec.promote(S.f16_bits(v), "f16"),
                                                           bv, seed)
    return pk, nk, pv, nv


@pytest.mark.parametrize("d", DIMS)
@pytest.mark.parametrize("bk,bv,gqa,tau,qscale,n_ctas", [
    (4, 2, 4, 0.0, 1.0, 0),
    (3, 2, 5, 0.0, 1.0, 7),
    (4, 3, 4, 1e-6, 8.0, 37),
    (2, 4, 8, 0.0, 1.0, 0),
    (3, 3, 1, 0.0, 1.0, 300),
])
def test_attend_head_dims(d, bk, bv, gqa, tau, qscale, n_ctas):
    rng = np.random.default_rng(d + 100 * bk + 10 * bv + gqa)
    ctx = np.array([700, 64, 1, 129, 0])
    Hkv = 2
    pk, nk, pv, nv = _cache(bk, bv, len(ctx), Hkv, 768, ctx, SEED, rng, d)
    qb = S.f16_bits(rng.standard_normal((len(ctx), Hkv * gqa, d)) * qscale)
    q64 = codec.promote(qb, "f16")
    want, ng_o = oracle_attend(q64, pk, nk, pv, nv, ctx, gqa, bk, bv, SEED, tau)
    got, st, ng_g, heads_g = gpu_attend(qb, "f16", pk, nk, pv, nv, ctx, gqa, bk, bv, SEED,
                                        tau=tau, n_ctas=n_ctas, head_counts=True)
    err = np.abs(got - want).max()
    print(f"d={d} K{bk}/V{bv} g={gqa}: max|err| = {err:.3e}, gated {ng_o}/{ng_g}")
    assert err <= ATOL
    assert st == 4                      # the empty sequence
    if tau > 0:
        # per (sequence, query head): equal outside the score error band
        assert ng_o > 0
        cnt_o, amb = oracle_gate_table(q64, pk, nk, ctx, gqa, bk, SEED, tau)
        assert cnt_o.sum() == ng_o and heads_g.sum() == ng_g
        assert np.all(np.abs(heads_g - cnt_o) <= amb)
    else:
        assert ng_g == 0 and not heads_g.any()
