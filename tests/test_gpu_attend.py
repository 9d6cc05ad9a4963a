"""GPU parity of tq_attend against the float64 oracle on the same packed
cache (built by the oracle's encoder), B200.

Bar: max |out_gpu - out_oracle| <= 2e-3 on float32 output; fp16/bf16 output
equals the round-to-nearest-even of the float32 output within one ulp. The
sparse-V gate is compared head by head: for every (sequence, query head) the
number of gated positions (tq_attend_gate_counts) equals the oracle's except
for positions whose float64 gate value exp(s - M_blk) lies within the
kernel's score error bound of tau (gpu_support.SCORE_EPS_*: derived from the
fp16 high/low operands and fp32 accumulation of the scores); the total count
(tq_attend's counter) obeys the same rule.
"""
import numpy as np
import pytest

import synthetic as S
from gpu_support import gpu_attend, oracle_attend, oracle_cache, oracle_gate_table, pool
from oracle import attention, codec

pytestmark = pytest.mark.gpu
SEED = S.SIGN_SEED
ATOL = 2e-3


def _check_gate(q64, cache, gqa, bk, tau, ng_o, ng_g, heads_g):
    """Per (sequence, query head) and total gate counts within the derived
    ambiguity of the oracle's; returns the total ambiguous count."""
    pk, nk, _, _, ctx = cache
    cnt_o, amb = oracle_gate_table(q64, pk, nk, ctx, gqa, bk, SEED, tau)
    assert cnt_o.sum() == ng_o
    diff = np.abs(heads_g - cnt_o)
    assert np.all(diff <= amb), (int((diff > amb).sum()), int(diff.max()))
    assert heads_g.sum() == ng_g
    assert abs(ng_g - ng_o) <= amb.sum()
    return int(amb.sum())


def _run(name, scale=1.0, tau=None, n_ctas=0):
    w = S.WORKLOADS[name]
    pk, nk, pv, nv, ctx = oracle_cache(name)
    qb = S.query_bits(w, scale=scale)
    q64 = codec.promote(qb, w.dtype)
    tau = w.tau if tau is None else tau
    want, ng_o = oracle_attend(q64, pk, nk, pv, nv, ctx, w.gqa, w.bits_k, w.bits_v, SEED, tau)
    got, st, ng_g, heads_g = gpu_attend(qb, w.dtype, pk, nk, pv, nv, ctx, w.gqa, w.bits_k,
                                        w.bits_v, SEED, tau=tau, n_ctas=n_ctas, head_counts=True)
    if tau <= 0:
        assert ng_g == 0 and not heads_g.any()
    return w, q64, (pk, nk, pv, nv, ctx), want, got, st, ng_o, ng_g, tau, heads_g


@pytest.mark.parametrize("name", ["single_head_1k", "llama3_8b_decode", "qwen14b_decode",
                                  "batched_serving"])
def test_attend_full_workload(name):
    w, q64, cache, want, got, st, ng_o, ng_g, tau, heads_g = _run(name)
    err = np.abs(got - want).max()
    print(f"{name}: max|err| = {err:.3e}, gated oracle {ng_o} gpu {ng_g}")
    assert err <= ATOL
    assert st == 0
    if tau > 0:
        _check_gate(q64, cache, w.gqa, w.bits_k, tau, ng_o, ng_g, heads_g)


def test_forced_gate_batched_serving():
    """Queries scaled x8 sharpen the softmax so the 1e-6 gate fires often;
    the gate is checked head by head on all 64 x 32 (sequence, head) pairs."""
    w, q64, cache, want, got, st, ng_o, ng_g, tau, heads_g = _run("batched_serving", scale=8.0)
    assert ng_o > 1000
    amb = _check_gate(q64, cache, w.gqa, w.bits_k, tau, ng_o, ng_g, heads_g)
    print(f"forced gate: oracle {ng_o}, gpu {ng_g}, ambiguous {amb}")
    assert (heads_g > 0).sum() > 1000      # most (sequence, head) pairs gate something
    assert np.abs(got - want).max() <= ATOL


@pytest.mark.parametrize("tau", [1e-2, 0.5, 1.0, 2.0])
def test_gate_thresholds_single_head(tau):
    w, q64, cache, want, got, st, ng_o, ng_g, tau, heads_g = _run("single_head_1k", scale=3.0,
                                                                  tau=tau)
    _check_gate(q64, cache, w.gqa, w.bits_k, tau, ng_o, ng_g, heads_g)
    assert np.abs(got - want).max() <= ATOL
    if tau > 1:
        assert ng_g == 1024 and np.all(got == 0)
    if tau <= 1:                           # each block's maximum is never gated
        assert ng_g <= 1024 - 16


@pytest.mark.parametrize("n_ctas", [1, 3, 7, 16, 1024])
def test_cta_counts_single_head(n_ctas):
    """1024 positions = 16 blocks: ranges that split the sequence unevenly,
    one block per CTA, and more CTAs than blocks."""
    _, _, _, want, got, _, _, _, _, _ = _run("single_head_1k", n_ctas=n_ctas)
    assert np.abs(got - want).max() <= ATOL


@pytest.mark.parametrize("n_ctas", [5, 37, 300])
def test_cta_counts_ragged_batch(n_ctas):
    """CTA ranges that cross sequence and kv-head boundaries, ragged lengths."""
    rng = np.random.default_rng(n_ctas)
    ctx = np.array([1, 700, 64, 0, 129, 1000, 63, 512])
    pk, nk, pv, nv = _small_cache(4, 2, len(ctx), 2, 1024, ctx, 21, rng)
    qb = S.f16_bits(rng.standard_normal((len(ctx), 8, 128)))
    q64 = codec.promote(qb, "f16")
    want, _ = oracle_attend(q64, pk, nk, pv, nv, ctx, 4, 4, 2, 21)
    got, st, _ = gpu_attend(qb, "f16", pk, nk, pv, nv, ctx, 4, 4, 2, 21, n_ctas=n_ctas)
    assert np.abs(got - want).max() <= ATOL
    assert st == 4


@pytest.mark.parametrize("n_ctas", [5, 12, 37, 300, 0])
def test_cta_counts_equal_block_counts(n_ctas):
    """Every (sequence, kv head) segment has 11 blocks (lengths 641..704):
    the partition then aligns CTA ranges with segments when the grid allows
    (5 CTAs for 12 segments does not, 37 gives three CTAs per segment over
    11 blocks, 300 one block per CTA)."""
    rng = np.random.default_rng(100 + n_ctas)
    ctx = np.array([704, 641, 700, 650, 683, 704])
    pk, nk, pv, nv = _small_cache(4, 2, len(ctx), 2, 768, ctx, 22, rng)
    qb = S.f16_bits(rng.standard_normal((len(ctx), 8, 128)))
    q64 = codec.promote(qb, "f16")
    want, _ = oracle_attend(q64, pk, nk, pv, nv, ctx, 4, 4, 2, 22)
    got, st, _ = gpu_attend(qb, "f16", pk, nk, pv, nv, ctx, 4, 4, 2, 22, n_ctas=n_ctas)
    assert np.abs(got - want).max() <= ATOL
    assert st == 0


def test_workspace_counters_return_to_zero_and_calls_repeat():
    import torch
    import compressed_decode_attention_b200 as tq
    rng = np.random.default_rng(31)
    ctx = np.array([900, 2000, 5])
    pk, nk, pv, nv = _small_cache(3, 2, 1, 3, 2048, ctx, 2, rng)
    qb = S.f16_bits(rng.standard_normal((3, 6, 128)))
    ws_bytes = tq.tq_attend_workspace_size(3, 6, 2048, 128)
    ws = torch.zeros(ws_bytes // 4, dtype=torch.float32, device="cuda")
    outs = []
    for n_ctas in (0, 9, 9, 0):
        o, _, _ = gpu_attend(qb, "f16", pk, nk, pv, nv, ctx, 2, 3, 2, 2, n_ctas=n_ctas,
                             workspace=ws)
        counters = ws[: (3 * 6 * 4 + 255) // 256 * 64].view(torch.int32)
        assert int(counters.abs().sum().item()) == 0
        outs.append(o)
    np.testing.assert_array_equal(outs[0], outs[3])
    np.testing.assert_array_equal(outs[1], outs[2])
    # Different CTA counts split the positions differently; the softmax
    # weights x V norms enter the P.V product rounded to fp16 (relative step
    # 2^-11) against each chunk's own maximum, so the two splits agree to
    # about 1e-4, ten times inside the oracle bar.
    assert np.abs(outs[0] - outs[1]).max() <= 2e-4


def _small_cache(bk, bv, B, Hkv, cap, ctx, seed, rng, dtype="f16"):
    pk = np.zeros((B, Hkv, cap, 128 * bk // 8), np.uint8)
    pv = np.zeros((B, Hkv, cap, 128 * bv // 8), np.uint8)
    nk = np.zeros((B, Hkv, cap), np.uint16)
    nv = np.zeros((B, Hkv, cap), np.uint16)
    for b in range(B):
        for g in range(Hkv):
            L = int(min(max(ctx[b], 0), cap))
            k = rng.standard_normal((L, 128)) * 2
            v = rng.standard_normal((L, 128))
            kx = codec.promote(S.to_bits(k, dtype), dtype)
            vx = codec.promote(S.to_bits(v, dtype), dtype)
            pk[b, g, :L], nk[b, g, :L] = codec.encode_rows(kx, bk, seed)
            pv[b, g, :L], nv[b, g, :L] = codec.encode_rows(vx, bv, seed)
    return pk, nk, pv, nv


@pytest.mark.parametrize("bk,bv,gqa", [(2, 2, 1), (3, 3, 8), (4, 4, 2), (2, 4, 3),
                                       (3, 4, 6), (2, 3, 7), (4, 2, 5), (3, 2, 4), (4, 3, 1)])
def test_bit_widths_and_group_sizes(bk, bv, gqa):
    rng = np.random.default_rng(bk * 100 + bv * 10 + gqa)
    ctx = np.array([300, 77])
    pk, nk, pv, nv = _small_cache(bk, bv, 2, 2, 320, ctx, 99, rng)
    qb = S.f16_bits(rng.standard_normal((2, 2 * gqa, 128)))
    q64 = codec.promote(qb, "f16")
    want, _ = oracle_attend(q64, pk, nk, pv, nv, ctx, gqa, bk, bv, 99)
    got, st, _ = gpu_attend(qb, "f16", pk, nk, pv, nv, ctx, gqa, bk, bv, 99)
    assert np.abs(got - want).max() <= ATOL


def test_context_edge_cases_and_status():
    rng = np.random.default_rng(8)
    cap = 256
    ctx = np.array([1, 0, 65, 5000, -4, 256, 64, 129])
    pk, nk, pv, nv = _small_cache(4, 2, len(ctx), 1, cap, ctx, 3, rng)
    qb = S.f16_bits(rng.standard_normal((len(ctx), 2, 128)))
    q64 = codec.promote(qb, "f16")
    want, _ = oracle_attend(q64, pk, nk, pv, nv, ctx, 2, 4, 2, 3)
    got, st, _ = gpu_attend(qb, "f16", pk, nk, pv, nv, ctx, 2, 4, 2, 3)
    assert np.abs(got - want).max() <= ATOL
    assert np.all(got[1] == 0) and np.all(got[4] == 0)
    assert st == (1 | 4)   # clamped and empty
    # context of one position returns that position's value
    v0 = codec.dequant(codec.unpack(pv[0, 0, :1], 2, 128), nv[0, 0, :1], 2, 3)[0]
    np.testing.assert_allclose(got[0, 0], v0, atol=ATOL)


@pytest.mark.parametrize("q_dtype", ["f16", "bf16", "f32"])
def test_query_dtypes(q_dtype):
    rng = np.random.default_rng(12)
    ctx = np.array([200])
    pk, nk, pv, nv = _small_cache(4, 2, 1, 2, 200, ctx, 5, rng)
    qf = rng.standard_normal((1, 8, 128)).astype(np.float32)
    if q_dtype == "f32":
        qb, q64 = qf, qf.astype(np.float64)
    else:
        qb = S.to_bits(qf, q_dtype)
        q64 = codec.promote(qb, q_dtype)
    want, _ = oracle_attend(q64, pk, nk, pv, nv, ctx, 4, 4, 2, 5)
    got, _, _ = gpu_attend(qb, q_dtype, pk, nk, pv, nv, ctx, 4, 4, 2, 5)
    assert np.abs(got - want).max() <= ATOL


@pytest.mark.parametrize("out_dtype", [0, 1])
def test_output_dtypes_round_float32_result(out_dtype):
    import torch
    w = S.WORKLOADS["single_head_1k"]
    pk, nk, pv, nv, ctx = oracle_cache("single_head_1k")
    qb = S.query_bits(w)
    f32, _, _ = gpu_attend(qb, "f16", pk, nk, pv, nv, ctx, 1, 4, 2, SEED)
    lo, _, _ = gpu_attend(qb, "f16", pk, nk, pv, nv, ctx, 1, 4, 2, SEED, out_dtype=out_dtype)
    ref = S.f16_bits(f32) if out_dtype == 0 else S.bf16_bits(f32)
    assert np.abs(lo.astype(np.int64) - ref.astype(np.int64)).max() <= 1
