"""The kernels' bounded waits give up cleanly (failure detection without a
GPU fault).

Every wait in the attention kernel is bounded: a wait for staged cache data
(an mbarrier completed by bulk copies) and the decode step's wait for the
helper warp's flag. When one runs out, the kernel sets TQ_DEV_WAIT_TIMEOUT,
waits (bounded again) for its own copies still in flight, stops issuing and
ends normally, so the context stays usable.

The test uses libtq_waittest.so, a test-only build of the same sources with
TQ_TEST_INJECT_WAIT_FAULTS: waits give up after ~1e5 cycles, and two waits
cannot complete, without any invalid access:
  - tq_attend: every warp arms the mbarrier of its first ring slot for 16
    bytes more than its bulk copies deliver (every byte still lands);
  - tq_attend_append: the helper warp never raises the flag its owner warp
    waits for.
Each case checks that the launch returns without a CUDA error and reports
the timeout, and that the production library then gives the oracle's
result on the same inputs in the same process.
"""
import os

import numpy as np
import pytest

import synthetic as S
from gpu_support import dev, host, oracle_attend
from oracle import codec

pytestmark = pytest.mark.gpu
TQ_DEV_WAIT_TIMEOUT = 8
ATOL = 2e-3


@pytest.fixture(scope="module")
def waittest_lib():
    import compressed_decode_attention_b200 as tq
    from compressed_decode_attention_b200 import build
    path = os.path.join(os.path.dirname(tq.LIB_PATH), "libtq_waittest.so")
    if not os.path.exists(path):
        build.build(variant="waittest")
    return tq.load_library(path)


def _case(rng, B=2, Hkv=2, gqa=4, cap=1024, ctx=(1000, 513), seed=3):
    d = 128
    pk = np.zeros((B, Hkv, cap, 64), np.uint8)
    pv = np.zeros((B, Hkv, cap, 32), np.uint8)
    nk = np.zeros((B, Hkv, cap), np.uint16)
    nv = np.zeros((B, Hkv, cap), np.uint16)
    for b in range(B):
        for g in range(Hkv):
            k = codec.promote(S.f16_bits(rng.standard_normal((ctx[b], d))), "f16")
            v = codec.promote(S.f16_bits(rng.standard_normal((ctx[b], d))), "f16")
            pk[b, g, :ctx[b]], nk[b, g, :ctx[b]] = codec.encode_rows(k, 4, seed)
            pv[b, g, :ctx[b]], nv[b, g, :ctx[b]] = codec.encode_rows(v, 2, seed)
    qb = S.f16_bits(rng.standard_normal((B, Hkv * gqa, d)))
    return qb, pk, nk, pv, nv, np.asarray(ctx, np.int32), gqa, seed


def _attend(L, tq, qb, pk, nk, pv, nv, ctx, gqa, seed, new_kv=None):
    """One attention (or decode-step) call through library handle L; returns
    (output, device status). Raises if the launch or the stream failed."""
    import torch
    B, Hkv, cap = pk.shape[:3]
    Hq, d = qb.shape[1], qb.shape[2]
    ws_bytes = tq.tq_attend_workspace_size(B, Hq, cap, d)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    out = torch.empty((B, Hq, d), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    bufs = [dev(x) for x in (qb, pk, nk, pv, nv, ctx)]
    P = tq._ptr
    if new_kv is None:
        rc = L.tq_attend(P(bufs[0]), tq.TQ_F16, P(bufs[1]), P(bufs[2]), P(bufs[3]), P(bufs[4]),
                         P(bufs[5]), B, Hq, gqa, d, 4, 2, seed, cap, 0.0, 0, P(ws), ws_bytes,
                         P(st), None, P(out), tq.TQ_F32, None)
    else:
        kvt = dev(new_kv)
        rc = L.tq_attend_append(P(bufs[0]), tq.TQ_F16, P(kvt), tq.TQ_F16, P(bufs[1]), P(bufs[2]),
                                P(bufs[3]), P(bufs[4]), P(bufs[5]), B, Hq, gqa, d, 4, 2, seed,
                                cap, 0.0, 0, P(ws), ws_bytes, P(st), None, P(out), tq.TQ_F32,
                                None)
    assert rc == tq.TQ_OK, rc
    torch.cuda.synchronize()              # raises if the kernel faulted
    return host(out), int(st.item())


def test_ring_slot_wait_gives_up(waittest_lib):
    import compressed_decode_attention_b200 as tq
    rng = np.random.default_rng(7)
    qb, pk, nk, pv, nv, ctx, gqa, seed = _case(rng)
    _, st = _attend(waittest_lib, tq, qb, pk, nk, pv, nv, ctx, gqa, seed)
    assert st & TQ_DEV_WAIT_TIMEOUT
    # the context is still usable: the production build is exact next
    got, st2 = _attend(tq.lib(), tq, qb, pk, nk, pv, nv, ctx, gqa, seed)
    assert st2 == 0
    want, _ = oracle_attend(codec.promote(qb, "f16"), pk, nk, pv, nv, ctx, gqa, 4, 2, seed)
    assert np.abs(got - want).max() <= ATOL


def test_decode_step_flag_wait_gives_up(waittest_lib):
    import compressed_decode_attention_b200 as tq
    rng = np.random.default_rng(8)
    qb, pk, nk, pv, nv, ctx, gqa, seed = _case(rng)
    new_kv = S.f16_bits(rng.standard_normal((2, len(ctx), pk.shape[1], 128)))
    _, st = _attend(waittest_lib, tq, qb, pk, nk, pv, nv, ctx, gqa, seed, new_kv=new_kv)
    assert st & TQ_DEV_WAIT_TIMEOUT
    _, st2 = _attend(tq.lib(), tq, qb, pk, nk, pv, nv, ctx, gqa, seed, new_kv=new_kv)
    assert st2 == 0
