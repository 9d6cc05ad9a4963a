"""The bounds-checked build (TQ_DEBUG) runs the kernels' GPU cases clean.

libtq_debug.so is the library compiled with TQ_DEBUG: every bulk copy of
cached rows (attention, prefill) and every row store of the encoders checks
that its rows lie inside the sequence's capacity; a failed check sets
TQ_DEV_DEBUG_CHECK and skips the access instead of trapping, so the context
stays usable (compute-sanitizer's stand-in on this pool). Each case runs a
workload on the checked build, requires the status to stay free of that bit
(and of any other), and compares the result with the oracle.
"""
import os

import numpy as np
import pytest

import synthetic as S
from gpu_support import dev, host, oracle_attend
from oracle import codec

pytestmark = pytest.mark.gpu
TQ_DEV_DEBUG_CHECK = 16
ATOL = 2e-3
D = 128


@pytest.fixture(scope="module")
def debug_lib():
    import compressed_decode_attention_b200 as tq
    from compressed_decode_attention_b200 import build
    path = os.path.join(os.path.dirname(tq.LIB_PATH), "libtq_debug.so")
    if not os.path.exists(path):
        build.build(variant="debug")
    return tq.load_library(path)


def _with(lib, fn):
    """Run fn with the package bound to lib, then restore the production one."""
    import compressed_decode_attention_b200 as tq
    saved = tq._lib
    tq._lib = lib
    try:
        return fn()
    finally:
        tq._lib = saved


def _cache(rng, B, Hkv, cap, ctx, bk, bv, seed):
    pk = np.zeros((B, Hkv, cap, D * bk // 8), np.uint8)
    pv = np.zeros((B, Hkv, cap, D * bv // 8), np.uint8)
    nk = np.zeros((B, Hkv, cap), np.uint16)
    nv = np.zeros((B, Hkv, cap), np.uint16)
    for b in range(B):
        for g in range(Hkv):
            k = codec.promote(S.f16_bits(rng.standard_normal((ctx[b], D))), "f16")
            v = codec.promote(S.f16_bits(rng.standard_normal((ctx[b], D))), "f16")
            pk[b, g, :ctx[b]], nk[b, g, :ctx[b]] = codec.encode_rows(k, bk, seed)
            pv[b, g, :ctx[b]], nv[b, g, :ctx[b]] = codec.encode_rows(v, bv, seed)
    return pk, nk, pv, nv


def test_attention_ragged_batch(debug_lib):
    import torch
    import compressed_decode_attention_b200 as tq
    rng = np.random.default_rng(71)
    B, Hkv, gqa, cap, seed = 3, 2, 4, 1024, 5
    ctx = np.array([1000, 7, 513], np.int32)
    pk, nk, pv, nv = _cache(rng, B, Hkv, cap, ctx, 4, 2, seed)
    qb = S.f16_bits(rng.standard_normal((B, Hkv * gqa, D)))
    out = torch.empty((B, Hkv * gqa, D), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    wsb = tq.tq_attend_workspace_size(B, Hkv * gqa, cap, D)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")

    def run():
        tq.tq_attend(dev(qb), tq.TQ_F16, dev(pk), dev(nk), dev(pv), dev(nv), dev(ctx), B,
                     Hkv * gqa, gqa, D, 4, 2, seed, cap, 0.0, 0, ws, wsb, out, tq.TQ_F32,
                     dev_status=st)
        torch.cuda.synchronize()
    _with(debug_lib, run)
    assert int(st.item()) == 0
    want, _ = oracle_attend(codec.promote(qb, "f16"), pk, nk, pv, nv, ctx, gqa, 4, 2, seed)
    assert np.max(np.abs(host(out) - want)) <= ATOL


def test_prefill_with_splits(debug_lib):
    import torch
    import compressed_decode_attention_b200 as tq
    from oracle import attention
    rng = np.random.default_rng(72)
    B, Hkv, gqa, cap, T, seed, n_splits = 2, 2, 4, 640, 40, 3, 3
    ctx = np.array([600, 200], np.int32)
    pk, nk, pv, nv = _cache(rng, B, Hkv, cap, ctx, 4, 2, seed)
    Hq = Hkv * gqa
    qb = S.f16_bits(rng.standard_normal((B, T, Hq, D)))
    out = torch.empty((B, T, Hq, D), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    wsb = tq.tq_prefill_workspace_size(B, T, Hq, D, n_splits)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device="cuda")

    def run():
        tq.tq_prefill_attend_split(dev(qb), tq.TQ_F16, dev(pk), dev(nk), dev(pv), dev(nv),
                                   dev(ctx), B, T, Hq, gqa, D, 4, 2, seed, cap, n_splits, ws,
                                   wsb, out, tq.TQ_F32, dev_status=st)
        torch.cuda.synchronize()
    _with(debug_lib, run)
    assert int(st.item()) == 0
    got = host(out)
    q64 = codec.promote(qb, "f16")
    for b in range(B):
        for t in (0, T // 2, T - 1):
            p = int(ctx[b]) - T + t
            want, _ = attention.attend(q64[b, t][None], pk[b][None, :, :p + 1],
                                       nk[b][None, :, :p + 1], pv[b][None, :, :p + 1],
                                       nv[b][None, :, :p + 1], np.array([p + 1]), gqa, 4, 2,
                                       seed, 0.0)
            assert np.max(np.abs(got[b, t] - want[0])) <= ATOL, (b, t)


@pytest.mark.parametrize("n_tok", [700, 100])       # the tensor-core and the FWHT encoders
def test_encode_with_offset(debug_lib, n_tok):
    import torch
    import compressed_decode_attention_b200 as tq
    rng = np.random.default_rng(73)
    H, off, cap, seed = 2, 37, 1024, 9
    kv = S.f16_bits(rng.standard_normal((2, n_tok, H, D)))
    pk = torch.zeros((H, cap, 64), dtype=torch.uint8, device="cuda")
    pv = torch.zeros((H, cap, 32), dtype=torch.uint8, device="cuda")
    nk = torch.zeros((H, cap), dtype=torch.int16, device="cuda")
    nv = torch.zeros((H, cap), dtype=torch.int16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")

    def run():
        tq.tq_encode(dev(kv), tq.TQ_F16, n_tok, H, D, 4, 2, seed, pk, pv, nk, nv, cap, off, st)
        torch.cuda.synchronize()
    _with(debug_lib, run)
    assert int(st.item()) == 0
    for which, bits, rows in ((0, 4, pk), (1, 2, pv)):
        for h in range(H):
            idx_o, _, _, _, mg = codec.encode(codec.promote(kv[which, :, h], "f16"), bits, seed)
            idx_g = codec.unpack(host(rows)[h, off:off + n_tok], bits, D)
            assert np.all((idx_g == idx_o) | (mg < 1e-5))
        assert np.all(host(rows)[:, :off] == 0) and np.all(host(rows)[:, off + n_tok:] == 0)
