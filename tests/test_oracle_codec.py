"""Pins for the oracle's encode / pack / dequant (CPU).

Checks against: closed-form inputs whose rotated coordinates are chosen in
advance, the zero vector, hand-derived packed bytes, the byte accounting and
the codec statistics printed in "We Built a Python Library That Cuts LLM
Memory Usage by 80%" (sections "Compression numbers" and "The CLI"), and
fp16 rounding/saturation of the stored norm.
"""
import numpy as np
import pytest
import scipy.linalg

from conftest import golden_rows
from oracle import codebook as cb
from oracle import codec, rotation


def _x_from_zeta(zeta, seed):
    """x with H·(D⊙x)/||x|| = zeta, for ||zeta|| = sqrt(d): x = D⊙(H·zeta)/sqrt(d)."""
    d = zeta.shape[-1]
    h = scipy.linalg.hadamard(d).astype(np.float64)
    return rotation.sign_vector(seed, d) * (zeta @ h) / np.sqrt(d)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_closed_form_indices(bits):
    """Rotated coordinates placed on chosen centroids decode to those indices."""
    d, seed = 128, 11
    c, _ = cb.lloyd_max_normal(bits)
    rng = np.random.default_rng(bits)
    # every level once, the rest on the two innermost levels (keeps the
    # squared norm of the first d-2 coordinates below d), in random order
    n = len(c)
    inner = rng.integers(n // 2 - 1, n // 2 + 1, size=d - 2 - n)
    want = np.concatenate((np.arange(n), inner, [0, 0]))
    want[:-2] = rng.permutation(want[:-2])
    zeta = c[want].astype(np.float64)
    # fix the norm to sqrt(d) with two coordinates set to +-r
    rest = d - np.sum(zeta[:-2] ** 2)
    assert rest > 0
    r = np.sqrt(rest / 2)
    zeta[-2], zeta[-1] = r, -r
    x = _x_from_zeta(zeta, seed)
    idx, norm, _, z, margin = codec.encode(x[None], bits, seed)
    assert norm[0] == pytest.approx(np.sqrt(d), rel=1e-14)
    np.testing.assert_allclose(z[0], zeta, atol=1e-12)
    np.testing.assert_array_equal(idx[0, :-2], want[:-2])
    assert np.all(margin[0, :-2] > 1e-3)


def test_basis_vector_through_rotation():
    """x = D⊙H[:,k] rotates to sqrt(d)·e_k: top index at k, N/2 elsewhere."""
    d, seed, bits = 128, 0, 4
    h = scipy.linalg.hadamard(d).astype(np.float64)
    for k in (0, 5, 127):
        x = rotation.sign_vector(seed, d) * h[:, k]
        idx, norm, nb, _, _ = codec.encode(x[None], bits, seed)
        assert norm[0] == pytest.approx(np.sqrt(d))
        want = np.full(d, 8)
        want[k] = 15
        np.testing.assert_array_equal(idx[0], want)


def test_zero_vector():
    idx, norm, nb, z, _ = codec.encode(np.zeros((1, 128)), 3, 0)
    assert norm[0] == 0 and nb[0] == 0
    np.testing.assert_array_equal(idx[0], np.full(128, 4))
    np.testing.assert_array_equal(codec.dequant(idx, nb, 3, 0), np.zeros((1, 128)))


def test_ties_go_to_upper_cell():
    _, t = cb.lloyd_max_normal(3)
    got = codec.quantize_index(np.array([t[0], t[3], t[6], -10.0, 10.0]), t)
    np.testing.assert_array_equal(got, [1, 4, 7, 0, 7])


def test_packing_golden_bytes():
    for row in golden_rows("packing_lsb_first.txt"):
        fields = " ".join(row).split("|")
        bits = int(fields[0])
        ids = [int(v) for v in fields[1].split()]
        want = bytes(int(v, 16) for v in fields[2].split())
        idx = np.zeros((1, 128), dtype=np.int64)
        idx[0, :len(ids)] = ids
        got = codec.pack(idx, bits)[0].tobytes()
        assert got[:len(want)] == want, bits
        assert got[len(want):] == bytes(len(got) - len(want))


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 8])
def test_pack_roundtrip(bits):
    rng = np.random.default_rng(bits)
    idx = rng.integers(0, 1 << bits, size=(50, 128))
    rows = codec.pack(idx, bits)
    assert rows.shape == (50, 128 * bits // 8)
    np.testing.assert_array_equal(codec.unpack(rows, bits, 128), idx)


def test_byte_accounting():
    for name, bk, bv, avg, fp16_bytes, total in golden_rows("byte_accounting.txt"):
        bk, bv, d = int(bk), int(bv), 128
        rk = codec.pack(np.zeros((1, d), dtype=np.int64), bk).shape[1]
        rv = codec.pack(np.zeros((1, d), dtype=np.int64), bv).shape[1]
        assert (rk + rv) * 8 / (2 * d) == float(avg), name
        assert 2 * d * 2 == int(fp16_bytes)
        assert rk + rv + 2 + 2 == int(total), name


def test_norm_rounding_and_saturation():
    n = np.array([1.0, 1.0 + 2 ** -11, 1.0 + 3 * 2 ** -11, 65504.0, 65519.0, 70000.0])
    got = codec.fp16_norm_bits(n)
    # ties to even: 1+2^-11 -> 1.0 ; 1+3*2^-11 -> 1+2^-9... (next even) ; saturate
    np.testing.assert_array_equal(got, [0x3C00, 0x3C00, 0x3C02, 0x7BFF, 0x7BFF, 0x7BFF])


def test_bf16_and_f16_promotion():
    np.testing.assert_array_equal(codec.promote(np.array([0x3F80, 0xC000, 0x0000], np.uint16), "bf16"),
                                  [1.0, -2.0, 0.0])
    np.testing.assert_array_equal(codec.promote(np.array([0x3C00, 0xC000, 0x7BFF], np.uint16), "f16"),
                                  [1.0, -2.0, 65504.0])


@pytest.mark.parametrize("bits", [2, 4])
def test_codec_statistics_match_printed_benchmark(bits):
    rows = {int(r[0]): [float(v) for v in r[1:]] for r in golden_rows("tqai_benchmark.txt")}
    nmse_p, snr_p, cos_p = rows[bits]
    rng = np.random.default_rng(2024)
    x = rng.standard_normal((20000, 128))
    idx, _, nb, _, _ = codec.encode(x, bits, 0)
    xh = codec.dequant(idx, nb, bits, 0)
    nmse = np.mean(np.sum((x - xh) ** 2, 1) / np.sum(x * x, 1))
    cos = np.mean(np.sum(x * xh, 1) / np.linalg.norm(x, axis=1) / np.linalg.norm(xh, axis=1))
    assert nmse == pytest.approx(nmse_p, rel=0.02)
    assert -10 * np.log10(nmse) == pytest.approx(snr_p, abs=0.1)
    assert cos == pytest.approx(cos_p, abs=1.5e-3)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_rotated_domain_mse_near_codebook_mse(bits):
    """Unit vectors: MSE of the rotated coordinates within [0.95, 1.01] of D_b.

    The exact marginal of a rotated unit vector is a scaled Beta with lighter
    tails than N(0, 1/d), so the observed error sits slightly below D_b.
    """
    c, t = cb.lloyd_max_normal(bits)
    db = cb.quantizer_mse(c, t)
    rng = np.random.default_rng(77)
    x = rng.standard_normal((20000, 128))
    idx, norm, _, _, _ = codec.encode(x, bits, 5)
    y = rotation.rotate(x / norm[:, None], 5)
    err = np.mean(np.sum((y - codec.dequant_rotated(idx, bits)) ** 2, 1))
    assert 0.95 * db <= err <= 1.01 * db


def test_outlier_channels_are_spread():
    """Large channels no longer dominate after rotation: error stays at D_b scale."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((5000, 128))
    x[:, [3, 40, 77, 100]] *= 20.0
    idx, _, nb, _, _ = codec.encode(x, 4, 0)
    xh = codec.dequant(idx, nb, 4, 0)
    nmse = np.mean(np.sum((x - xh) ** 2, 1) / np.sum(x * x, 1))
    assert nmse < 0.0105
