"""The allocation-free attention entry point (tq_attend_noalloc) gives the
same output as tq_attend with a caller workspace, bit for bit, on two calls
in a row: both run the same kernel with the same grid on the same inputs,
and the partial results merge in a fixed order, so any difference would be
a stale counter or a misplaced slot in the shared scratch.

tq_attend_noalloc serves callers that cannot allocate device memory while
they run attention; it takes its scratch from a fixed array inside the
library. This file sorts last so that a run stopping at the first failure
has already run every other test; it also passes on its own.
"""
import numpy as np
import pytest

import synthetic as S
from oracle import codec

pytestmark = pytest.mark.gpu


def _cache(rng, B, Hkv, cap, ctx, bk, bv, seed):
    pk = np.zeros((B, Hkv, cap, 16 * bk), np.uint8)
    pv = np.zeros((B, Hkv, cap, 16 * bv), np.uint8)
    nk = np.zeros((B, Hkv, cap), np.uint16)
    nv = np.zeros((B, Hkv, cap), np.uint16)
    for b in range(B):
        L = int(ctx[b])
        for g in range(Hkv):
            k = codec.promote(S.f16_bits(rng.standard_normal((L, 128))), "f16")
            v = codec.promote(S.f16_bits(rng.standard_normal((L, 128))), "f16")
            pk[b, g, :L], nk[b, g, :L] = codec.encode_rows(k, bk, seed)
            pv[b, g, :L], nv[b, g, :L] = codec.encode_rows(v, bv, seed)
    return pk, nk, pv, nv


def test_noalloc_matches_workspace_entry_point_twice():
    import torch
    import compressed_decode_attention_b200 as tq

    def dev(a):
        a = np.ascontiguousarray(a)
        return torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).cuda()

    rng = np.random.default_rng(2025)
    B, Hq, gqa, cap, seed = 3, 8, 4, 1024, 5
    ctx = np.array([1000, 257, 64], np.int32)
    pk, nk, pv, nv = _cache(rng, B, Hq // gqa, cap, ctx, 4, 2, seed)
    args = [dev(pk), dev(nk), dev(pv), dev(nv), dev(ctx)]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def run(q, use_workspace):
        out = torch.empty((B, Hq, 128), dtype=torch.float32, device="cuda")
        common = (q, tq.TQ_F16, *args, B, Hq, gqa, 128, 4, 2, seed, cap, 1e-3, 0)
        if use_workspace:
            ws_bytes = tq.tq_attend_workspace_size(B, Hq, cap, 128)
            ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
            tq.tq_attend(*common, ws, ws_bytes, out, tq.TQ_F32, dev_status=status)
        else:
            tq.tq_attend_noalloc(*common, out, tq.TQ_F32, dev_status=status)
        torch.cuda.synchronize()
        return out.cpu().numpy()

    for call in range(2):
        q = dev(S.f16_bits(rng.standard_normal((B, Hq, 128)) * (1 + call)))
        want = run(q, use_workspace=True)
        got = run(q, use_workspace=False)
        assert np.all(np.isfinite(got))
        assert np.array_equal(got, want), (call, np.abs(got - want).max())
    assert int(status.item()) == 0


@pytest.mark.parametrize("batch,d", [(187, 128), (64, 256), (427, 64)])
def test_noalloc_rejects_problems_beyond_its_scratch(batch, d):
    """batch x 128 query heads just beyond the 16 MiB scratch at each head
    dimension (23887 / 8033 / 54530 pairs fit at d = 128 / 256 / 64); the
    call is rejected on the host before any launch."""
    import compressed_decode_attention_b200 as tq
    FAKE = 1 << 20
    assert tq.tq_attend_workspace_size(batch, 128, 1024, d) > 16 << 20
    st = tq.lib().tq_attend_noalloc(FAKE, 0, FAKE, FAKE, FAKE, FAKE, FAKE, batch, 128, 4,
                                    d, 4, 2, 0, 1024, 0.0, 0, None, None, FAKE, 2, None)
    assert st == tq.TQ_ERR_UNSUPPORTED
