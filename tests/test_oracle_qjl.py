"""Pins for the oracle's residual sketch (QJL) and its inner-product estimate
(CPU).

The sketch is defined only by what it must achieve ("We Built a Python
Library That Cuts LLM Memory Usage by 80%", section "Why not both stages?":
a one-bit residual correction that makes inner products unbiased), so the
pins are statistical and structural:
- over independent Gaussian projections, the mean correction equals
  <q, x - x_hat> (unbiasedness) and its variance equals the closed form
  ((pi/2)·|q|^2·|r|^2 - <q, r>^2)/m, derived below;
- the residual is x - x_hat of the original space (dense brute force);
- sketching in rotated coordinates equals sketching the original-space
  residual with S·R;
- the stage-1 part is the dense inner product with x_hat;
- bit order and packing by hand on a small case.

Variance: with r_hat = r/|r|, q = a·r_hat + q_perp and s ~ N(0, I), the term
X = sign(s·r)(s·q) = a|s·r_hat| + sign(s·r_hat)(s·q_perp) has E[X] =
a·sqrt(2/pi) and E[X^2] = a^2 + |q_perp|^2 = |q|^2, so the estimate
|r|·sqrt(pi/2)/m·sum_i X_i has variance (|r|^2·(pi/2)/m)·(|q|^2 - 2a^2/pi).
"""
import numpy as np
import pytest
import scipy.linalg

import synthetic as S
from oracle import codec, qjl, rotation


def _key_and_query(rng, d=128):
    x = rng.standard_normal((1, d)) * 2.0
    x[0, :4] *= 10.0
    q = rng.standard_normal((1, d))
    return x, q


def _corrections(x, q, bits, seed, n_draws, rng):
    """Correction term of one key and query over n_draws independent S."""
    d = x.shape[1]
    idx, nb, r_rot = qjl.residual_rotated(x, bits, seed)
    q_rot = rotation.rotate(q, seed)
    out = np.empty(n_draws)
    for i in range(n_draws):
        Sm = rng.standard_normal((d, d))
        rows, _, gb = qjl.sketch(r_rot, Sm)
        out[i] = qjl.correction(q_rot, rows, gb, Sm)[0, 0]
    return out, r_rot, nb


@pytest.mark.parametrize("bits", [2, 4])
def test_correction_is_unbiased_with_the_closed_form_variance(bits):
    rng = np.random.default_rng(100 + bits)
    x, q = _key_and_query(rng)
    d = x.shape[1]
    c, r_rot, nb = _corrections(x, q, bits, 3, 3000, rng)
    # the residual of the original space, by brute force
    idx = codec.encode(x, bits, 3)[0]
    r = x - codec.dequant(idx, nb, bits, 3)
    gamma = np.linalg.norm(r)
    g16 = float(np.float16(gamma))
    # the stored fp16 gamma scales the expectation by g16/gamma
    want_mean = float(q[0] @ r[0]) * g16 / gamma
    want_var = ((np.pi / 2) * float(q[0] @ q[0]) * gamma ** 2 - float(q[0] @ r[0]) ** 2) / d
    want_var *= (g16 / gamma) ** 2
    se = np.sqrt(want_var / len(c))
    assert abs(c.mean() - want_mean) < 4 * se
    assert c.var(ddof=1) == pytest.approx(want_var, rel=0.1)


def test_residual_is_the_original_space_difference():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((5, 128))
    idx, nb, r_rot = qjl.residual_rotated(x, 3, 9)
    r = x - codec.dequant(idx, nb, 3, 9)
    h = scipy.linalg.hadamard(128).astype(np.float64)
    dense_r = (r * rotation.sign_vector(9, 128)) @ h.T / np.sqrt(128)
    np.testing.assert_allclose(r_rot, dense_r, atol=1e-12)


def test_rotated_sketch_equals_original_space_sketch_with_S_R():
    rng = np.random.default_rng(8)
    d, seed = 64, 5
    x, q = _key_and_query(rng, d)
    Sm = rng.standard_normal((d, d))
    idx, nb, r_rot = qjl.residual_rotated(x, 4, seed)
    rows, u, gb = qjl.sketch(r_rot, Sm)
    r = x - codec.dequant(idx, nb, 4, seed)
    R = scipy.linalg.hadamard(d) * rotation.sign_vector(seed, d)[None, :] / np.sqrt(d)
    SR = Sm @ R
    u_orig = r @ SR.T
    assert np.min(np.abs(u_orig)) > 1e-9                        # no sign on a knife edge
    np.testing.assert_array_equal(np.packbits((u_orig >= 0).astype(np.uint8), axis=1,
                                              bitorder="little"), rows)
    got = qjl.correction(rotation.rotate(q, seed), rows, gb, Sm)[0, 0]
    pm = np.where(u_orig[0] >= 0, 1.0, -1.0)
    g16 = float(np.asarray(gb).view(np.float16)[0])
    want = g16 * np.sqrt(np.pi / 2) / d * float((q[0] @ SR.T) @ pm)
    assert got == pytest.approx(want, rel=1e-12)


def test_stage_one_part_is_the_dense_inner_product_with_x_hat():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((20, 128))
    q = rng.standard_normal((3, 128))
    Sm = S.projection_matrix(128)
    pk, nb, rows, gb, _ = qjl.encode(x, 4, 2, Sm)
    got = qjl.inner_products(q, pk, nb, rows, gb, 4, 2, Sm, with_sketch=False)
    xh = codec.dequant(codec.unpack(pk, 4, 128), nb, 4, 2)
    np.testing.assert_allclose(got, q @ xh.T, atol=1e-11)


def test_sketch_bits_by_hand():
    """d = 16: bit i of the row is [(S r~)_i >= 0], LSB first."""
    rng = np.random.default_rng(10)
    r_rot = rng.standard_normal((2, 16))
    Sm = rng.standard_normal((16, 16))
    rows, u, gb = qjl.sketch(r_rot, Sm)
    for n in range(2):
        for i in range(16):
            ui = sum(Sm[i, j] * r_rot[n, j] for j in range(16))
            assert ((rows[n, i // 8] >> (i % 8)) & 1) == (1 if ui >= 0 else 0)
        assert np.float16(gb[n:n + 1].view(np.float16)[0]) == np.float16(np.linalg.norm(r_rot[n]))


def test_zero_residual_gives_no_correction():
    """gamma = 0: the estimate is the stage-1 inner product exactly."""
    rng = np.random.default_rng(11)
    q = rng.standard_normal((2, 128))
    Sm = rng.standard_normal((128, 128))
    rows = np.full((3, 16), 0xA5, np.uint8)
    got = qjl.correction(rotation.rotate(q, 0), rows, np.zeros(3, np.uint16), Sm)
    np.testing.assert_array_equal(got, 0.0)


def test_scores_layout_and_empty_sequences():
    rng = np.random.default_rng(13)
    B, Hkv, cap, d, gqa = 2, 2, 24, 128, 2
    Sm = S.projection_matrix(d)
    pk = np.zeros((B, Hkv, cap, 64), np.uint8)
    nk = np.zeros((B, Hkv, cap), np.uint16)
    sr = np.zeros((B, Hkv, cap, 16), np.uint8)
    gk = np.zeros((B, Hkv, cap), np.uint16)
    for b in range(B):
        for g in range(Hkv):
            pk[b, g], nk[b, g], sr[b, g], gk[b, g], _ = qjl.encode(
                rng.standard_normal((cap, d)), 4, 1, Sm)
    q = rng.standard_normal((B, Hkv * gqa, d))
    out = qjl.scores(q, pk, nk, sr, gk, np.array([20, 0]), gqa, 4, 1, Sm)
    np.testing.assert_array_equal(out[1], 0.0)
    np.testing.assert_array_equal(out[0, :, 20:], 0.0)
    want = qjl.inner_products(q[0, 2:4], pk[0, 1, :20], nk[0, 1, :20], sr[0, 1, :20],
                              gk[0, 1, :20], 4, 1, Sm) / np.sqrt(d)
    np.testing.assert_allclose(out[0, 2:4, :20], want, atol=1e-13)
