"""The pins catch plausible oracle mistakes (CPU).

Each case plants one mistake in the oracle (monkeypatched for the duration of
the case only) and checks that at least one pin test then fails.
"""
import numpy as np
import pytest

import test_oracle_attention as ta
import test_oracle_codebook as tcb
import test_oracle_codec as tc
import test_oracle_rotation as tr
from oracle import attention, codebook, codec, rotation


def _fails(fn, *args):
    with pytest.raises(AssertionError):
        fn(*args)


def test_sign_bit_choice_is_pinned(monkeypatch):
    real = rotation.splitmix64
    monkeypatch.setattr(rotation, "sign_vector", lambda seed, d: np.array(
        [-1.0 if (v >> 62) & 1 else 1.0 for v in real(seed, d)]))
    _fails(tr.test_sign_vector_definition)


def test_missing_sign_flip_in_encode(monkeypatch):
    # the encoder loses D; the closed-form input is still built with the real D
    real_signs = rotation.sign_vector
    real_helper = tc._x_from_zeta
    def helper(z, s):
        monkeypatch.setattr(rotation, "sign_vector", real_signs)
        try:
            return real_helper(z, s)
        finally:
            monkeypatch.setattr(rotation, "sign_vector", lambda seed, d: np.ones(d))
    monkeypatch.setattr(tc, "_x_from_zeta", helper)
    monkeypatch.setattr(rotation, "sign_vector", lambda seed, d: np.ones(d))
    _fails(tc.test_closed_form_indices, 4)


def test_query_rotation_without_signs(monkeypatch):
    real_rotate = rotation.rotate
    monkeypatch.setattr(rotation, "rotate",
                        lambda x, seed: x @ rotation.hadamard(x.shape[-1]).T / np.sqrt(x.shape[-1]))
    _fails(ta.test_matches_dense_brute_force, 4, 2, 1)
    monkeypatch.setattr(rotation, "rotate", real_rotate)


def test_dropped_score_scale(monkeypatch):
    real = codec.dequant_rotated
    monkeypatch.setattr(codec, "dequant_rotated", lambda idx, bits: real(idx, bits) * np.sqrt(idx.shape[-1]))
    _fails(ta.test_matches_dense_brute_force, 4, 2, 1)


def test_ties_to_lower_cell(monkeypatch):
    monkeypatch.setattr(codec, "quantize_index",
                        lambda z, t: np.searchsorted(t, z, side="left").astype(np.int64))
    _fails(tc.test_ties_go_to_upper_cell)


def test_msb_first_packing(monkeypatch):
    def pack_msb(idx, bits):
        n, d = idx.shape
        planes = (idx[:, :, None] >> np.arange(bits)[::-1]) & 1
        return np.packbits(planes.reshape(n, d * bits).astype(np.uint8), axis=1)
    monkeypatch.setattr(codec, "pack", pack_msb)
    _fails(tc.test_packing_golden_bytes)


def test_wrong_threshold_rule(monkeypatch):
    real = codebook.lloyd_max_normal
    def bad(bits, **kw):
        c, t = real(bits)
        return c, t * 1.01
    monkeypatch.setattr(codebook, "lloyd_max_normal", bad)
    _fails(tcb.test_fixed_point_with_independent_normal, 3)


def test_gate_with_global_max(monkeypatch):
    monkeypatch.setattr(attention, "GATE_BLOCK", 1 << 20)
    _fails(ta.test_gate_matches_brute_force, 0.05)


def test_wrong_gqa_mapping(monkeypatch):
    real = attention.attend_head_group
    def swapped(qs, *a, **k):
        return real(qs[::-1].copy(), *a, **k)
    monkeypatch.setattr(attention, "attend_head_group", swapped)
    _fails(ta.test_matches_dense_brute_force, 4, 3, 4)


def test_norm_not_saturated(monkeypatch):
    def unsaturated(n):
        with np.errstate(over="ignore"):
            return np.asarray(n).astype(np.float16).view(np.uint16)
    monkeypatch.setattr(codec, "fp16_norm_bits", unsaturated)
    _fails(tc.test_norm_rounding_and_saturation)


def test_combine_without_rescaling(monkeypatch):
    real_exp2 = np.exp2
    monkeypatch.setattr(attention.np, "exp2", lambda x: np.where(np.isfinite(x), 1.0, 0.0))
    try:
        _fails(ta.test_context_slices_combine_to_whole, 0.0)
    finally:
        monkeypatch.setattr(attention.np, "exp2", real_exp2)


def test_record_max_in_natural_units(monkeypatch):
    real = attention.partial_head_group
    def natural(*args):
        rec, gated = real(*args)
        d = rec.shape[-1] - 2
        rec = rec.copy()
        rec[:, d] *= np.log(2.0)
        return rec, gated
    monkeypatch.setattr(attention, "partial_head_group", natural)
    _fails(ta.test_partial_record_closed_form)
    _fails(ta.test_context_slices_combine_to_whole, 0.0)


def test_sketch_without_the_sqrt_pi_over_2_factor(monkeypatch):
    from oracle import qjl
    real = qjl.correction
    monkeypatch.setattr(qjl, "correction",
                        lambda *a: real(*a) / np.sqrt(np.pi / 2.0))
    import test_oracle_qjl as tq
    _fails(tq.test_correction_is_unbiased_with_the_closed_form_variance, 4)


def test_sketch_bit_convention_flipped(monkeypatch):
    from oracle import qjl
    real = qjl.sketch
    def flipped(r_rot, Sm):
        rows, u, gb = real(r_rot, Sm)
        return np.invert(rows), u, gb
    monkeypatch.setattr(qjl, "sketch", flipped)
    import test_oracle_qjl as tq
    _fails(tq.test_correction_is_unbiased_with_the_closed_form_variance, 2)
    _fails(tq.test_sketch_bits_by_hand)


def test_sketch_of_the_unrotated_residual(monkeypatch):
    from oracle import qjl
    real = qjl.residual_rotated
    def unrotated(x, bits, seed):
        idx, nb, r_rot = real(x, bits, seed)
        return idx, nb, rotation.unrotate(r_rot, seed)
    monkeypatch.setattr(qjl, "residual_rotated", unrotated)
    import test_oracle_qjl as tq
    _fails(tq.test_residual_is_the_original_space_difference)
    _fails(tq.test_rotated_sketch_equals_original_space_sketch_with_S_R)


def test_centroid_at_cell_midpoint(monkeypatch):
    # the centroid step takes the middle of the cell instead of E[X | cell]
    def midpoint(a, b):
        return a + 1.0 if b == float("inf") else 0.5 * (a + b)
    monkeypatch.setattr(codebook, "cell_centroid", midpoint)
    monkeypatch.setattr(codec, "_CB_CACHE", {})
    _fails(tcb.test_matches_max_1960_table, 3)


def test_dequant_without_the_norm(monkeypatch):
    # the original-space reconstruction forgets to scale the unit vector
    monkeypatch.setattr(codec, "dequant", lambda idx, nb, bits, seed:
                        rotation.unrotate(codec.dequant_rotated(idx, bits), seed))
    _fails(tc.test_codec_statistics_match_printed_benchmark, 4)


def test_gated_positions_dropped_from_the_sum(monkeypatch):
    # the softmax sum runs over the positions that pass the gate only
    def dropped(qs, idx_k, nk_bits, idx_v, nv_bits, bits_k, bits_v, seed, tau):
        qs = np.asarray(qs, dtype=np.float64)
        g, d = qs.shape
        L = idx_k.shape[0]
        nk = np.asarray(nk_bits, dtype=np.uint16).view(np.float16).astype(np.float64)
        nv = np.asarray(nv_bits, dtype=np.uint16).view(np.float16).astype(np.float64)
        s = (rotation.rotate(qs, seed) @ codec.dequant_rotated(idx_k, bits_k).T) * nk / np.sqrt(d)
        w = np.exp(s - s.max(axis=1, keepdims=True))
        nblk = (L + attention.GATE_BLOCK - 1) // attention.GATE_BLOCK
        pad = np.full((g, nblk * attention.GATE_BLOCK), -np.inf)
        pad[:, :L] = s
        mblk = pad.reshape(g, nblk, attention.GATE_BLOCK).max(axis=2)
        gated = np.exp(s - np.repeat(mblk, attention.GATE_BLOCK, axis=1)[:, :L]) < tau
        kept = np.where(gated, 0.0, w)
        acc = (kept * nv) @ codec.dequant_rotated(idx_v, bits_v)
        return rotation.unrotate(acc / kept.sum(axis=1, keepdims=True), seed), gated
    monkeypatch.setattr(attention, "attend_head_group", dropped)
    _fails(ta.test_gate_matches_brute_force, 0.05)
