"""Pins for the oracle's compressed-domain decode attention (CPU).

The brute force below rebuilds K and V in the original space with its own
unpacking (numpy.unpackbits) and scipy's Hadamard matrix, then runs plain
softmax(q·K^T/sqrt d)·V — the quantity named in "We Built a Python Library
That Cuts LLM Memory Usage by 80%", section "Test Suite". The oracle instead
rotates the query once and accumulates V in the rotated domain ("AdapTQ" PyPI
page, "How it works", item 3); the two must agree to rounding.
"""
import numpy as np
import pytest
import scipy.linalg

from oracle import attention, codec, rotation
from oracle import codebook as cb


def _rows_to_idx(rows, bits, d):
    b = np.unpackbits(rows, axis=-1, bitorder="little")[..., :d * bits]
    b = b.reshape(rows.shape[:-1] + (d, bits)).astype(np.int64)
    return (b * (1 << np.arange(bits))).sum(-1)


def _brute(q, pk, nk, pv, nv, ctx, gqa, bk, bv, seed, tau=0.0):
    """Dequantize to the original space, then dense masked softmax attention."""
    B, Hq, d = q.shape
    h = scipy.linalg.hadamard(d).astype(np.float64)
    sv = rotation.sign_vector(seed, d)
    ck, _ = cb.lloyd_max_normal(bk)
    cv, _ = cb.lloyd_max_normal(bv)
    out = np.zeros((B, Hq, d))
    for b in range(B):
        L = min(int(ctx[b]), pk.shape[2])
        if L <= 0:
            continue
        for hq in range(Hq):
            g = hq // gqa
            nK = nk[b, g, :L].view(np.float16).astype(np.float64)
            nV = nv[b, g, :L].view(np.float16).astype(np.float64)
            # x_hat = n · D ⊙ (H · c[idx]) / d
            K = nK[:, None] * sv * (ck[_rows_to_idx(pk[b, g, :L], bk, d)] @ h) / d
            V = nV[:, None] * sv * (cv[_rows_to_idx(pv[b, g, :L], bv, d)] @ h) / d
            s = K @ q[b, hq] / np.sqrt(d)
            p = np.exp(s - s.max())
            if tau > 0:
                keep = np.ones(L, dtype=bool)
                for blk in range(0, L, 64):
                    e = slice(blk, min(L, blk + 64))
                    keep[e] = np.exp(s[e] - s[e].max()) >= tau
                out[b, hq] = (p * keep) @ V / p.sum()
            else:
                out[b, hq] = p @ V / p.sum()
    return out


def _cache(B, Hkv, cap, d, bk, bv, seed, rng, same_key=False):
    pk = np.zeros((B, Hkv, cap, d * bk // 8), np.uint8)
    pv = np.zeros((B, Hkv, cap, d * bv // 8), np.uint8)
    nk = np.zeros((B, Hkv, cap), np.uint16)
    nv = np.zeros((B, Hkv, cap), np.uint16)
    for b in range(B):
        for g in range(Hkv):
            k = rng.standard_normal((cap, d)) * rng.uniform(0.5, 2.0)
            if same_key:
                k[:] = k[0]
            v = rng.standard_normal((cap, d))
            pk[b, g], nk[b, g] = codec.encode_rows(k, bk, seed)
            pv[b, g], nv[b, g] = codec.encode_rows(v, bv, seed)
    return pk, nk, pv, nv


@pytest.mark.parametrize("bk,bv,gqa", [(4, 2, 1), (3, 2, 5), (4, 3, 4)])
def test_matches_dense_brute_force(bk, bv, gqa):
    rng = np.random.default_rng(bk * 10 + bv)
    B, Hkv, cap, d, seed = 2, 2, 150, 128, 9
    pk, nk, pv, nv = _cache(B, Hkv, cap, d, bk, bv, seed, rng)
    q = rng.standard_normal((B, Hkv * gqa, d)) * 2
    ctx = np.array([150, 97])
    got, _ = attention.attend(q, pk, nk, pv, nv, ctx, gqa, bk, bv, seed)
    want = _brute(q, pk, nk, pv, nv, ctx, gqa, bk, bv, seed)
    np.testing.assert_allclose(got, want, atol=1e-12)


@pytest.mark.parametrize("tau", [1e-3, 0.05, 0.5])
def test_gate_matches_brute_force(tau):
    rng = np.random.default_rng(4)
    B, Hkv, cap, d, seed, gqa = 1, 2, 200, 128, 1, 2
    pk, nk, pv, nv = _cache(B, Hkv, cap, d, 4, 3, seed, rng)
    q = rng.standard_normal((B, Hkv * gqa, d)) * 4
    ctx = np.array([200])
    got, ng = attention.attend(q, pk, nk, pv, nv, ctx, gqa, 4, 3, seed, tau)
    want = _brute(q, pk, nk, pv, nv, ctx, gqa, 4, 3, seed, tau)
    np.testing.assert_allclose(got, want, atol=1e-12)
    assert ng > 0


def test_context_of_one_returns_that_value():
    rng = np.random.default_rng(1)
    pk, nk, pv, nv = _cache(1, 1, 4, 128, 4, 2, 0, rng)
    q = rng.standard_normal((1, 3, 128))
    got, _ = attention.attend(q, pk, nk, pv, nv, np.array([1]), 3, 4, 2, 0)
    v0 = codec.dequant(codec.unpack(pv[0, 0, :1], 2, 128), nv[0, 0, :1], 2, 0)[0]
    for h in range(3):
        np.testing.assert_allclose(got[0, h], v0, atol=1e-13)


def test_identical_keys_average_values():
    rng = np.random.default_rng(2)
    pk, nk, pv, nv = _cache(1, 1, 64, 128, 4, 2, 0, rng, same_key=True)
    q = rng.standard_normal((1, 1, 128))
    got, _ = attention.attend(q, pk, nk, pv, nv, np.array([64]), 1, 4, 2, 0)
    vh = codec.dequant(codec.unpack(pv[0, 0], 2, 128), nv[0, 0], 2, 0)
    np.testing.assert_allclose(got[0, 0], vh.mean(0), atol=1e-13)


def test_duplicated_heads_and_gqa_mapping():
    rng = np.random.default_rng(3)
    pk, nk, pv, nv = _cache(1, 2, 80, 128, 4, 2, 0, rng)
    q1 = rng.standard_normal(128)
    q = np.stack([q1, q1, q1, q1])[None]
    got, _ = attention.attend(q, pk, nk, pv, nv, np.array([80]), 2, 4, 2, 0)
    np.testing.assert_array_equal(got[0, 0], got[0, 1])
    np.testing.assert_array_equal(got[0, 2], got[0, 3])
    assert np.abs(got[0, 0] - got[0, 2]).max() > 1e-3   # different kv heads


def test_gate_special_cases():
    rng = np.random.default_rng(5)
    pk, nk, pv, nv = _cache(1, 1, 130, 128, 4, 2, 0, rng)
    q = rng.standard_normal((1, 2, 128)) * 3
    ctx = np.array([130])
    base, n0 = attention.attend(q, pk, nk, pv, nv, ctx, 2, 4, 2, 0, 0.0)
    neg, nn = attention.attend(q, pk, nk, pv, nv, ctx, 2, 4, 2, 0, -1.0)
    assert n0 == 0 and nn == 0
    np.testing.assert_array_equal(base, neg)
    # tau > 1 gates everything (e^0 = 1 < tau): out = 0
    allg, na = attention.attend(q, pk, nk, pv, nv, ctx, 2, 4, 2, 0, 1.5)
    assert na == 2 * 130
    np.testing.assert_array_equal(allg, 0.0)
    # tau = 1: only each block's maximum survives (e^0 = 1 is not < 1)
    one, n1 = attention.attend(q, pk, nk, pv, nv, ctx, 2, 4, 2, 0, 1.0)
    assert n1 == 2 * (130 - 3)     # 3 blocks: 64, 64, 2 positions


def test_gate_error_bound_against_exact_weights():
    """Gated positions have softmax weight < tau; dropping them moves the
    output by at most sum(p_t · max|v_hat_t|) over the gated set."""
    rng = np.random.default_rng(6)
    pk, nk, pv, nv = _cache(1, 1, 256, 128, 4, 2, 0, rng)
    q = rng.standard_normal((1, 1, 128)) * 6
    ctx = np.array([256])
    tau = 1e-2
    base, _ = attention.attend(q, pk, nk, pv, nv, ctx, 1, 4, 2, 0)
    gated_out, ng = attention.attend(q, pk, nk, pv, nv, ctx, 1, 4, 2, 0, tau)
    idx_k = codec.unpack(pk[0, 0], 4, 128)
    gv = attention.gate_values(q[0], idx_k, nk[0, 0], 4, 0)[0]
    kh = codec.dequant(idx_k, nk[0, 0], 4, 0)
    s = kh @ q[0, 0] / np.sqrt(128)
    p = np.exp(s - s.max())
    p /= p.sum()
    gated = gv < tau
    assert gated.sum() == ng > 0
    assert np.all(p[gated] < tau)
    vh = codec.dequant(codec.unpack(pv[0, 0], 2, 128), nv[0, 0], 2, 0)
    bound = np.sum(p[gated] * np.abs(vh[gated]).max(1))
    assert np.abs(base - gated_out).max() <= bound + 1e-15


def test_context_clamp_and_empty():
    rng = np.random.default_rng(7)
    pk, nk, pv, nv = _cache(3, 1, 70, 128, 4, 2, 0, rng)
    q = rng.standard_normal((3, 1, 128))
    a, _ = attention.attend(q, pk, nk, pv, nv, np.array([500, 0, -3]), 1, 4, 2, 0)
    b, _ = attention.attend(q, pk, nk, pv, nv, np.array([70, 0, 0]), 1, 4, 2, 0)
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(a[1:], 0.0)


# ---- context parallelism: per-slice log-sum-exp records and their merge

def _slice(arrs, ctx, a, b):
    """The cache rows [a, b) of every sequence as a cache of its own, and the
    number of valid rows each sequence has in it."""
    pk, nk, pv, nv = arrs
    loc = np.clip(np.minimum(ctx, pk.shape[2]) - a, 0, b - a)
    return (pk[:, :, a:b], nk[:, :, a:b], pv[:, :, a:b], nv[:, :, a:b]), loc


@pytest.mark.parametrize("tau", [0.0, 0.05])
def test_context_slices_combine_to_whole(tau):
    """Records of 64-aligned slices (one of them empty for every sequence)
    merge to the dense brute-force attention over the whole context."""
    rng = np.random.default_rng(11)
    B, Hkv, cap, d, seed, gqa, bk, bv = 3, 2, 300, 128, 4, 2, 4, 2
    arrs = _cache(B, Hkv, cap, d, bk, bv, seed, rng)
    q = rng.standard_normal((B, Hkv * gqa, d)) * 3
    ctx = np.array([300, 130, 0])
    recs = []
    for a, b in [(0, 64), (64, 192), (192, 300), (300, 300)]:
        part, loc = _slice(arrs, ctx, a, b)
        rec, _ = attention.attend_partial(q, *part, loc, gqa, bk, bv, seed, tau)
        recs.append(rec)
    got = attention.combine(np.stack(recs), seed)
    want = _brute(q, *arrs, ctx, gqa, bk, bv, seed, tau)
    np.testing.assert_allclose(got, want, atol=1e-12)
    np.testing.assert_array_equal(got[2], 0.0)
    # slice order does not matter
    np.testing.assert_allclose(attention.combine(np.stack(recs[::-1]), seed), got, atol=1e-14)


def test_partial_record_closed_form():
    """One slice's record against the original-space quantities: 2^m2 · l is
    sum_t exp(s_t), and D⊙(H·acc)/d is sum_t exp(s_t - max s) · v_hat_t."""
    rng = np.random.default_rng(12)
    d, L, seed = 128, 90, 6
    pk, nk, pv, nv = _cache(1, 1, L, d, 3, 3, seed, rng)
    q = rng.standard_normal((1, 1, d)) * 2
    rec, _ = attention.attend_partial(q, pk, nk, pv, nv, np.array([L]), 1, 3, 3, seed)
    kh = codec.dequant(codec.unpack(pk[0, 0], 3, d), nk[0, 0], 3, seed)
    vh = codec.dequant(codec.unpack(pv[0, 0], 3, d), nv[0, 0], 3, seed)
    s = kh @ q[0, 0] / np.sqrt(d)
    w = np.exp(s - s.max())
    assert rec[0, 0, d] == pytest.approx(s.max() * np.log2(np.e), abs=1e-12)
    assert np.exp2(rec[0, 0, d]) * rec[0, 0, d + 1] == pytest.approx(np.exp(s).sum(), rel=1e-12)
    h = scipy.linalg.hadamard(d).astype(np.float64)
    sv = rotation.sign_vector(seed, d)
    np.testing.assert_allclose(sv * (h @ rec[0, 0, :d]) / d, w @ vh, atol=1e-11)


def test_empty_slice_record_and_all_empty_combine():
    rng = np.random.default_rng(13)
    pk, nk, pv, nv = _cache(2, 1, 64, 128, 4, 2, 0, rng)
    q = rng.standard_normal((2, 2, 128))
    rec, _ = attention.attend_partial(q, pk, nk, pv, nv, np.array([0, -5]), 2, 4, 2, 0)
    np.testing.assert_array_equal(rec[..., :128], 0.0)
    assert np.all(rec[..., 128] == -np.inf) and np.all(rec[..., 129] == 0.0)
    np.testing.assert_array_equal(attention.combine(np.stack([rec, rec]), 0), 0.0)
