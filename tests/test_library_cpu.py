"""Host-side checks of libtq.so that need no GPU: it loads, exports every
entry point include/tq.h declares, its Lloyd-Max solver agrees with the
oracle's (two independent implementations), and bad arguments are rejected
on the host before any CUDA call."""
import ctypes
import os
import re

import numpy as np
import pytest

import compressed_decode_attention_b200 as tq
from oracle import codebook as ocb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(tq_\w+)\s*\(", src))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    names = _declared_functions()
    assert {"tq_build_codebook", "tq_encode", "tq_dequant", "tq_attend",
            "tq_attend_workspace_size"} <= set(names)
    lib = ctypes.CDLL(tq.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
        assert hasattr(tq, n), f"binding lacks {n}"


@pytest.mark.parametrize("variant", ["libtq_debug.so", "libtq_waittest.so"])
def test_checked_and_test_builds_export_the_same_abi(variant):
    """The bounds-checked (TQ_DEBUG) and wait-fault test builds are the same
    library: every declared symbol, the same ABI version."""
    path = os.path.join(os.path.dirname(tq.LIB_PATH), variant)
    if not os.path.exists(path):
        pytest.skip(f"{variant} not built (build() of __graft_entry__ builds it)")
    lib = ctypes.CDLL(path)
    for n in _declared_functions():
        assert hasattr(lib, n), n
    lib.tq_abi_version.restype = ctypes.c_int
    assert lib.tq_abi_version() == tq.tq_abi_version()


def test_abi_version_and_status_strings():
    hdr = open(os.path.join(ROOT, "include", "tq.h")).read()
    assert tq.tq_abi_version() == int(re.search(r"#define TQ_ABI_VERSION (\d+)", hdr).group(1))
    assert tq.tq_abi_version() == 8
    assert tq.status_string(0) == "TQ_OK"
    assert tq.status_string(2) == "TQ_ERR_UNSUPPORTED"


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5])
@pytest.mark.parametrize("d", [1, 64, 128])
def test_host_codebook_matches_oracle(bits, d):
    c, t, mse = tq.tq_build_codebook(bits, d)
    oc, ot = ocb.lloyd_max_normal(bits)
    np.testing.assert_allclose(c * np.sqrt(d), oc, atol=1e-12)
    np.testing.assert_allclose(t * np.sqrt(d), ot, atol=1e-12)
    assert mse == pytest.approx(ocb.quantizer_mse(oc, ot), abs=1e-12)


def test_codebook_rejects_bad_arguments():
    for bits, d in [(0, 128), (9, 128), (4, 0)]:
        with pytest.raises(tq.TQError) as e:
            tq.tq_build_codebook(bits, d)
        assert e.value.status == tq.TQ_ERR_INVALID_ARG


FAKE = 1 << 20  # 16-byte aligned dummy address; never dereferenced


def _encode(**kw):
    args = dict(kv=FAKE, dtype=tq.TQ_F16, n_tok=4, n_kv_heads=2, d=128, bits_k=4,
                bits_v=2, seed=0, packed_k=FAKE, packed_v=FAKE, norms_k=FAKE,
                norms_v=FAKE, cap_tok=8, tok_offset=0, dev_status=None, stream=0)
    args.update(kw)
    return tq.lib().tq_encode(args["kv"], args["dtype"], args["n_tok"], args["n_kv_heads"],
                              args["d"], args["bits_k"], args["bits_v"], args["seed"],
                              args["packed_k"], args["packed_v"], args["norms_k"],
                              args["norms_v"], args["cap_tok"], args["tok_offset"],
                              args["dev_status"], args["stream"])


@pytest.mark.parametrize("kw,want", [
    (dict(kv=None), tq.TQ_ERR_INVALID_ARG),
    (dict(packed_v=None), tq.TQ_ERR_INVALID_ARG),
    (dict(kv=FAKE + 2), tq.TQ_ERR_INVALID_ARG),           # misaligned
    (dict(bits_k=5), tq.TQ_ERR_INVALID_ARG),
    (dict(bits_v=1), tq.TQ_ERR_INVALID_ARG),
    (dict(d=96), tq.TQ_ERR_INVALID_ARG),                  # not a power of two
    (dict(d=32), tq.TQ_ERR_INVALID_ARG),                  # below the supported 64..256
    (dict(d=512), tq.TQ_ERR_INVALID_ARG),
    (dict(dtype=tq.TQ_F32), tq.TQ_ERR_INVALID_ARG),
    (dict(tok_offset=5), tq.TQ_ERR_INVALID_ARG),          # 5 + 4 > 8
    (dict(n_tok=-1), tq.TQ_ERR_INVALID_ARG),
    (dict(n_kv_heads=0), tq.TQ_ERR_INVALID_ARG),
    (dict(n_tok=0), tq.TQ_OK),                            # no-op, no launch
])
def test_encode_validation(kw, want):
    assert _encode(**kw) == want


def _attend(**kw):
    a = dict(q=FAKE, q_dtype=tq.TQ_F16, pk=FAKE, nk=FAKE, pv=FAKE, nv=FAKE, ctx=FAKE,
             batch=2, hq=8, gqa=4, d=128, bk=4, bv=2, seed=0, cap=256, tau=0.0,
             ctas=0, ws=FAKE, wsb=1 << 30, status=None, skipped=None, out=FAKE,
             out_dtype=tq.TQ_F32, stream=0)
    a.update(kw)
    return tq.lib().tq_attend(a["q"], a["q_dtype"], a["pk"], a["nk"], a["pv"], a["nv"],
                              a["ctx"], a["batch"], a["hq"], a["gqa"], a["d"], a["bk"],
                              a["bv"], a["seed"], a["cap"], a["tau"], a["ctas"], a["ws"],
                              a["wsb"], a["status"], a["skipped"], a["out"], a["out_dtype"],
                              a["stream"])


@pytest.mark.parametrize("kw,want", [
    (dict(q=None), tq.TQ_ERR_INVALID_ARG),
    (dict(ws=None), tq.TQ_ERR_INVALID_ARG),
    (dict(gqa=3), tq.TQ_ERR_INVALID_ARG),                 # 8 % 3 != 0
    (dict(hq=16, gqa=16), tq.TQ_ERR_UNSUPPORTED),         # group wider than 8
    (dict(ctas=-1), tq.TQ_ERR_INVALID_ARG),
    (dict(ctas=1025), tq.TQ_ERR_INVALID_ARG),             # more CTAs than slots
    (dict(cap=260), tq.TQ_ERR_UNSUPPORTED),               # capacity not a multiple of 8
    (dict(out=FAKE + 4), tq.TQ_ERR_INVALID_ARG),          # misaligned output
    (dict(nk=FAKE + 2), tq.TQ_ERR_INVALID_ARG),
    (dict(wsb=16), tq.TQ_ERR_INVALID_ARG),                # workspace too small
    (dict(bk=1), tq.TQ_ERR_INVALID_ARG),
    (dict(d=512), tq.TQ_ERR_INVALID_ARG),
    (dict(d=100), tq.TQ_ERR_INVALID_ARG),
    (dict(tau=float("nan")), tq.TQ_ERR_INVALID_ARG),
    (dict(out_dtype=7), tq.TQ_ERR_INVALID_ARG),
    (dict(batch=0), tq.TQ_ERR_INVALID_ARG),
    (dict(pk=FAKE + 8), tq.TQ_ERR_INVALID_ARG),
])
def test_attend_validation(kw, want):
    assert _attend(**kw) == want


def test_workspace_size_formula():
    # counters (4·batch·heads bytes, rounded to 256) + slots of d + 2 floats for
    # 1024 CTAs x 8 heads plus one per (batch, query head)
    def want(b, h, d=128):
        return -(-4 * b * h // 256) * 256 + (1024 * 8 + b * h) * (d + 2) * 4
    assert tq.tq_attend_workspace_size(1, 32, 32768, 128) == want(1, 32)
    assert tq.tq_attend_workspace_size(64, 32, 16384, 128) == want(64, 32)
    assert tq.tq_attend_workspace_size(1, 1, 10, 128) == want(1, 1)
    assert tq.tq_attend_workspace_size(3, 8, 10, 64) == want(3, 8, 64)
    assert tq.tq_attend_workspace_size(3, 8, 10, 256) == want(3, 8, 256)
    assert tq.tq_attend_workspace_size(1, 1, 10, 96) == 0
    assert tq.tq_attend_workspace_size(1, 1, 10, 512) == 0


def _combine(**kw):
    a = dict(parts=FAKE, n=2, batch=2, hq=8, d=128, seed=0, status=None, out=FAKE,
             out_dtype=tq.TQ_F32, stream=0)
    a.update(kw)
    return tq.lib().tq_attend_combine(a["parts"], a["n"], a["batch"], a["hq"], a["d"],
                                      a["seed"], a["status"], a["out"], a["out_dtype"],
                                      a["stream"])


@pytest.mark.parametrize("kw,want", [
    (dict(parts=None), tq.TQ_ERR_INVALID_ARG),
    (dict(out=None), tq.TQ_ERR_INVALID_ARG),
    (dict(n=0), tq.TQ_ERR_INVALID_ARG),
    (dict(batch=0), tq.TQ_ERR_INVALID_ARG),
    (dict(hq=-1), tq.TQ_ERR_INVALID_ARG),
    (dict(d=96), tq.TQ_ERR_INVALID_ARG),
    (dict(d=512), tq.TQ_ERR_INVALID_ARG),
    (dict(parts=FAKE + 4), tq.TQ_ERR_INVALID_ARG),       # records need 8-byte alignment
    (dict(out=FAKE + 4), tq.TQ_ERR_INVALID_ARG),
    (dict(out_dtype=3), tq.TQ_ERR_INVALID_ARG),
    (dict(status=FAKE + 2), tq.TQ_ERR_INVALID_ARG),
])
def test_combine_validation(kw, want):
    assert _combine(**kw) == want


def _partial(**kw):
    a = dict(q=FAKE, pk=FAKE, ws=FAKE, wsb=1 << 30, part=FAKE, d=128, gqa=4, bk=4)
    a.update(kw)
    return tq.lib().tq_attend_partial(a["q"], tq.TQ_F16, a["pk"], FAKE, FAKE, FAKE, FAKE, 2, 8,
                                      a["gqa"], a["d"], a["bk"], 2, 0, 256, 0.0, 0, a["ws"],
                                      a["wsb"], None, None, a["part"], 0)


@pytest.mark.parametrize("kw,want", [
    (dict(part=None), tq.TQ_ERR_INVALID_ARG),
    (dict(part=FAKE + 4), tq.TQ_ERR_INVALID_ARG),         # records need 8-byte alignment
    (dict(q=None), tq.TQ_ERR_INVALID_ARG),
    (dict(ws=None), tq.TQ_ERR_INVALID_ARG),
    (dict(wsb=16), tq.TQ_ERR_INVALID_ARG),
    (dict(gqa=3), tq.TQ_ERR_INVALID_ARG),
    (dict(d=100), tq.TQ_ERR_INVALID_ARG),
    (dict(bk=5), tq.TQ_ERR_INVALID_ARG),
])
def test_partial_validation(kw, want):
    assert _partial(**kw) == want


def _qjl_encode(**kw):
    a = dict(k=FAKE, dtype=tq.TQ_F16, n=4, H=2, d=128, bits=4, S=FAKE, pk=FAKE, nk=FAKE,
             sk=FAKE, g=FAKE, cap=8, off=0)
    a.update(kw)
    return tq.lib().tq_qjl_encode(a["k"], a["dtype"], a["n"], a["H"], a["d"], a["bits"], 0,
                                  a["S"], a["pk"], a["nk"], a["sk"], a["g"], a["cap"],
                                  a["off"], None, 0)


@pytest.mark.parametrize("kw,want", [
    (dict(S=None), tq.TQ_ERR_INVALID_ARG),
    (dict(sk=None), tq.TQ_ERR_INVALID_ARG),
    (dict(k=FAKE + 2), tq.TQ_ERR_INVALID_ARG),
    (dict(S=FAKE + 4), tq.TQ_ERR_INVALID_ARG),
    (dict(bits=5), tq.TQ_ERR_INVALID_ARG),
    (dict(d=96), tq.TQ_ERR_INVALID_ARG),
    (dict(dtype=tq.TQ_F32), tq.TQ_ERR_INVALID_ARG),
    (dict(off=5), tq.TQ_ERR_INVALID_ARG),                 # 5 + 4 > 8
    (dict(n=0), tq.TQ_OK),                                # no-op, no launch
])
def test_qjl_encode_validation(kw, want):
    assert _qjl_encode(**kw) == want


def _qjl_scores(**kw):
    a = dict(q=FAKE, pk=FAKE, sk=FAKE, g=FAKE, S=FAKE, ctx=FAKE, B=2, hq=8, gqa=4, d=128,
             bits=4, cap=256, with_sketch=1, out=FAKE)
    a.update(kw)
    return tq.lib().tq_qjl_scores(a["q"], tq.TQ_F16, a["pk"], FAKE, a["sk"], a["g"], a["S"],
                                  a["ctx"], a["B"], a["hq"], a["gqa"], a["d"], a["bits"], 0,
                                  a["cap"], a["with_sketch"], None, a["out"], 0)


@pytest.mark.parametrize("kw,want", [
    (dict(S=None), tq.TQ_ERR_INVALID_ARG),                # the sketch term needs S
    (dict(sk=None), tq.TQ_ERR_INVALID_ARG),
    (dict(out=None), tq.TQ_ERR_INVALID_ARG),
    (dict(gqa=3), tq.TQ_ERR_INVALID_ARG),
    (dict(hq=16, gqa=16), tq.TQ_ERR_UNSUPPORTED),
    (dict(with_sketch=2), tq.TQ_ERR_INVALID_ARG),
    (dict(sk=FAKE + 4), tq.TQ_ERR_INVALID_ARG),          # sketch rows need 8-byte alignment
    (dict(out=FAKE + 2), tq.TQ_ERR_INVALID_ARG),
    (dict(d=32), tq.TQ_ERR_INVALID_ARG),
    (dict(bits=1), tq.TQ_ERR_INVALID_ARG),
    (dict(B=0), tq.TQ_ERR_INVALID_ARG),
])
def test_qjl_scores_validation(kw, want):
    assert _qjl_scores(**kw) == want


def _prefill_split(**kw):
    a = dict(q=FAKE, n=2, ws=FAKE, wsb=1 << 30, d=128, ntok=16)
    a.update(kw)
    return tq.lib().tq_prefill_attend_split(a["q"], tq.TQ_F16, FAKE, FAKE, FAKE, FAKE, FAKE, 1,
                                            a["ntok"], 8, 4, a["d"], 4, 2, 0, 256, a["n"],
                                            a["ws"], a["wsb"], None, FAKE, tq.TQ_F32, 0)


@pytest.mark.parametrize("kw,want", [
    (dict(n=0), tq.TQ_ERR_INVALID_ARG),
    (dict(n=9), tq.TQ_ERR_INVALID_ARG),                  # at most 8 splits
    (dict(ws=None), tq.TQ_ERR_INVALID_ARG),              # splits need a workspace
    (dict(ws=FAKE + 8), tq.TQ_ERR_INVALID_ARG),          # 16-byte aligned
    (dict(wsb=1024), tq.TQ_ERR_INVALID_ARG),             # too small
    (dict(d=64), tq.TQ_ERR_UNSUPPORTED),                 # prefill is built for d = 128
    (dict(q=None), tq.TQ_ERR_INVALID_ARG),
])
def test_prefill_split_validation(kw, want):
    assert _prefill_split(**kw) == want


def test_prefill_workspace_size_and_split_choice():
    assert tq.tq_prefill_workspace_size(2, 16, 8, 128, 3) == 3 * 2 * 16 * 8 * 130 * 4
    assert tq.tq_prefill_workspace_size(2, 16, 8, 128, 1) == 0
    assert tq.tq_prefill_workspace_size(2, 16, 8, 96, 3) == 0
    assert 1 <= tq.tq_prefill_splits(1, 1024, 32, 4, 8192) <= 8
    assert tq.tq_prefill_splits(0, 1024, 32, 4, 8192) == 1


def test_prefill_split_choice_follows_the_measured_sweep():
    """On a 148-SM device (the host default without a GPU) the split count
    is the fastest one measured for these chunk shapes (8 kv heads, GQA 4):
    1 for 1024 tokens over 8192 (256 tiles already fill the SMs), 4 for 128
    tokens over 8192 (32 tiles), 1 for 4096 tokens over 16384."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("the choice depends on the device's SM count")
    assert tq.tq_prefill_splits(1, 1024, 32, 4, 8192) == 1
    assert tq.tq_prefill_splits(1, 128, 32, 4, 8192) == 4
    assert tq.tq_prefill_splits(1, 4096, 32, 4, 16384) == 1
    # a short context leaves little to split: one chunk per tile
    assert tq.tq_prefill_splits(1, 128, 32, 4, 128) == 1


@pytest.mark.parametrize("head_skipped,want", [
    (None, tq.TQ_ERR_INVALID_ARG),          # the counts array is required
    (FAKE + 2, tq.TQ_ERR_INVALID_ARG),      # not 4-byte aligned
])
def test_gate_counts_rejects_bad_count_array(head_skipped, want):
    """tq_attend_gate_counts checks its per-head count array on the host,
    before any CUDA call; every other argument is valid."""
    ws = tq.tq_attend_workspace_size(1, 8, 64, 128)
    st = tq.lib().tq_attend_gate_counts(FAKE, tq.TQ_F16, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 8, 4,
                                         128, 4, 2, 0, 64, 1e-3, 0, FAKE, ws, None, None,
                                         head_skipped, FAKE, tq.TQ_F32, None)
    assert st == want
