"""GPU parity of tq_encode and tq_dequant against the oracle (B200).

Indices must be bit-exact except at coordinates within 1e-5 (N(0,1) units)
of a decision threshold, which may flip with the kernel's float32 rounding
and must number at most 1e-4 of all coordinates; stored fp16 norms must be
within one ulp of the oracle's.
"""
import numpy as np
import pytest

import synthetic as S
from gpu_support import (check_indices, check_near_fraction, check_norms, dev,
                         gpu_encode, host, oracle_encode_heads, oracle_encode_parallel)
from oracle import codec

pytestmark = pytest.mark.gpu
SEED = S.SIGN_SEED


def _compare(kv, dtype, bk, bv, seed, pk, nk, pv, nv, lo=0, parallel=False,
             count_rule=False):
    """count_rule: also bound the exempted fraction (workload-scale calls;
    on a few hundred vectors the expected count is below one)."""
    n, H, d = kv.shape[1:]
    enc = oracle_encode_parallel if parallel else oracle_encode_heads
    stats = []
    for which, bits, rows, nb in ((0, bk, pk, nk), (1, bv, pv, nv)):
        idx_o, nb_o, mg = enc(kv, dtype, which, bits, seed)
        r = rows[:, lo:lo + n].reshape(H * n, -1)
        idx_g = codec.unpack(r, bits, d).reshape(H, n, d)
        stats.append(check_indices(idx_g, idx_o, mg))
        check_norms(nb[:, lo:lo + n], nb_o)
    if count_rule:
        check_near_fraction(stats)
    print(f"mismatches/near/total per K,V: {stats}")
    return stats


@pytest.mark.parametrize("name", ["single_head_1k", "llama3_8b_decode", "qwen14b_decode"])
def test_encode_full_workload(name):
    w = S.WORKLOADS[name]
    kv = S.kv_bits(w, 0, w.ctx)
    pk, nk, pv, nv, st = gpu_encode(kv, w.dtype, w.bits_k, w.bits_v, SEED)
    assert st == 0
    _compare(kv, w.dtype, w.bits_k, w.bits_v, SEED, pk, nk, pv, nv, parallel=True,
             count_rule=True)


def test_encode_k4v3_batched_serving_sequence():
    w = S.WORKLOADS["batched_serving"]
    n = int(S.ctx_lens(w)[0])
    kv = S.kv_bits(w, 0, n)
    pk, nk, pv, nv, st = gpu_encode(kv, w.dtype, w.bits_k, w.bits_v, SEED, cap=w.cap_tok)
    assert st == 0
    _compare(kv, w.dtype, w.bits_k, w.bits_v, SEED, pk, nk, pv, nv, parallel=True,
             count_rule=True)


@pytest.mark.parametrize("layer", [0, 1, 30, 31])
def test_encode_bulk_prefill_whole_layer(layer):
    """Four whole layers of the bulk-encode workload (32768 tokens x 8 kv
    heads each, the bench's launch), every vector checked against the
    oracle; the exempted near-threshold count is bounded per layer."""
    w = S.WORKLOADS["bulk_prefill_encode"]
    kv = S.kv_bits(w, 0, w.ctx, layer=layer)
    pk, nk, pv, nv, st = gpu_encode(kv, w.dtype, w.bits_k, w.bits_v, SEED)
    assert st == 0
    _compare(kv, w.dtype, w.bits_k, w.bits_v, SEED, pk, nk, pv, nv, parallel=True,
             count_rule=True)


def test_round_trip_bulk_layer_quality():
    """Encode -> dequant on the GPU over one whole bulk layer: the mean
    rotated-domain squared error ||y - y^||^2 (y = R x/||x||, per-coordinate
    MSE in N(0,1) units) equals the oracle's on the same vectors, and for V
    (plain N(0,1) input) it lies within [0.95, 1.01] of the codebook MSE D_2
    (the finite-d marginal has lighter tails than N(0,1))."""
    import torch
    import compressed_decode_attention_b200 as tq
    from oracle import codebook as ocb, rotation
    w = S.WORKLOADS["bulk_prefill_encode"]
    kv = S.kv_bits(w, 0, w.ctx, layer=2)
    pk, nk, pv, nv, st = gpu_encode(kv, w.dtype, w.bits_k, w.bits_v, SEED)
    H, n, d = w.n_kv_heads, w.ctx, w.d
    for which, bits, rows, nb in ((0, w.bits_k, pk, nk), (1, w.bits_v, pv, nv)):
        out = torch.empty((H, n, d), dtype=torch.float32, device="cuda")
        tq.tq_dequant(dev(rows), dev(nb), n, H, d, bits, SEED, n, 1, out)
        torch.cuda.synchronize()
        yhat_g = host(out).astype(np.float64)
        idx_o, _, _ = oracle_encode_parallel(kv, w.dtype, which, bits, SEED)
        mse_g, mse_o = 0.0, 0.0
        for h in range(H):
            x = codec.promote(kv[which, :, h], w.dtype)
            y = rotation.rotate(x / np.linalg.norm(x, axis=1, keepdims=True), SEED)
            mse_g += np.sum((y - yhat_g[h]) ** 2)
            mse_o += np.sum((y - codec.dequant_rotated(idx_o[h].astype(np.int64), bits)) ** 2)
        mse_g /= H * n
        mse_o /= H * n
        print(f"bits {bits}: rotated MSE gpu {mse_g:.6f} oracle {mse_o:.6f}")
        assert abs(mse_g - mse_o) <= 1e-6 * mse_o
        if which == 1:
            c, t = ocb.lloyd_max_normal(bits)
            assert 0.95 <= mse_g / ocb.quantizer_mse(c, t) <= 1.01


@pytest.mark.parametrize("bk,bv", [(2, 2), (3, 3), (4, 4), (2, 4), (3, 2)])
def test_encode_bit_widths(bk, bv):
    w = S.WORKLOADS["llama3_8b_decode"]
    kv = S.kv_bits(w, 3, 700)
    pk, nk, pv, nv, _ = gpu_encode(kv, "f16", bk, bv, 12345)
    _compare(kv, "f16", bk, bv, 12345, pk, nk, pv, nv)


def test_ragged_range_with_offset_leaves_other_rows():
    w = S.WORKLOADS["llama3_8b_decode"]
    kv = S.kv_bits(w, 5, 1000)
    pk, nk, pv, nv, _ = gpu_encode(kv, "f16", 4, 2, SEED, cap=1100, tok_offset=37, fill=0x5A)
    _compare(kv, "f16", 4, 2, SEED, pk, nk, pv, nv, lo=37)
    for rows in (pk, pv):
        assert np.all(rows[:, :37] == 0x5A) and np.all(rows[:, 1037:] == 0x5A)
    for nb in (nk, nv):
        assert np.all(nb[:, :37] == 0x5A) and np.all(nb[:, 1037:] == 0x5A)


def test_single_token_append():
    w = S.WORKLOADS["llama3_8b_decode"]
    kv = S.kv_bits(w, 9, 1)
    pk, nk, pv, nv, _ = gpu_encode(kv, "f16", 4, 2, SEED, cap=64, tok_offset=63, fill=0x11)
    _compare(kv, "f16", 4, 2, SEED, pk, nk, pv, nv, lo=63)
    assert np.all(pk[:, :63] == 0x11)


def test_zero_vectors():
    kv = np.zeros((2, 70, 2, 128), np.uint16)
    pk, nk, pv, nv, st = gpu_encode(kv, "f16", 3, 2, SEED)
    assert st == 0
    np.testing.assert_array_equal(codec.unpack(pk.reshape(-1, 48), 3, 128), 4)
    np.testing.assert_array_equal(codec.unpack(pv.reshape(-1, 32), 2, 128), 2)
    assert np.all(nk == 0) and np.all(nv == 0)


def test_norm_saturation_flag():
    rng = np.random.default_rng(1)
    big = rng.uniform(30000, 60000, size=(2, 64, 1, 128)) * rng.choice([-1, 1], size=(2, 64, 1, 128))
    kv = S.f16_bits(big)
    pk, nk, pv, nv, st = gpu_encode(kv, "f16", 4, 2, SEED)
    assert st & 2
    assert np.all(nk == 0x7BFF) and np.all(nv == 0x7BFF)
    _compare(kv, "f16", 4, 2, SEED, pk, nk, pv, nv)


def test_bf16_wide_range():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((2, 300, 3, 128)) * 10.0 ** rng.integers(-6, 6, size=(2, 300, 3, 1))
    kv = S.bf16_bits(x.astype(np.float32))
    pk, nk, pv, nv, st = gpu_encode(kv, "bf16", 4, 3, 77)
    _compare(kv, "bf16", 4, 3, 77, pk, nk, pv, nv)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_dequant_matches_oracle(bits):
    import torch
    import compressed_decode_attention_b200 as tq
    w = S.WORKLOADS["llama3_8b_decode"]
    kv = S.kv_bits(w, 11, 300)
    idx, nb, _ = oracle_encode_heads(kv, "f16", 0, bits, SEED)
    H, n, d = idx.shape
    rows = np.stack([codec.pack(idx[h].astype(np.int64), bits) for h in range(H)])
    cap = 320
    rows_c = np.zeros((H, cap, rows.shape[-1]), np.uint8)
    rows_c[:, :n] = rows
    nb_c = np.zeros((H, cap), np.uint16)
    nb_c[:, :n] = nb
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
