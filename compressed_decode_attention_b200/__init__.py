"""Python binding of the compressed decode-attention library (libtq.so).

Thin ctypes marshalling around the C ABI declared in include/tq.h: every
function here has the name of the C entry point it calls, accepts torch
tensors (device buffers) or raw integer addresses for the pointer arguments,
and raises TQError on a non-zero status. All computation runs in the CUDA
kernels of libtq.so; there is no fallback — if the library is not built,
importing any entry point raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq.so")

TQ_OK, TQ_ERR_INVALID_ARG, TQ_ERR_UNSUPPORTED, TQ_ERR_CUDA, TQ_ERR_NO_CONVERGENCE = range(5)
TQ_F16, TQ_BF16, TQ_F32 = 0, 1, 2
TQ_DEV_CTX_CLAMPED, TQ_DEV_NORM_SATURATED, TQ_DEV_CTX_EMPTY = 1, 2, 4
TQ_SPARSE_V_BLOCK = 64

_lib = None


class TQError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} returned {status_string(status)} ({status})")


def lib() -> ctypes.CDLL:
    """The loaded libtq.so (built in-tree). Raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is not built; run "
                              "`python -m compressed_decode_attention_b200.build`")
        _lib = load_library(LIB_PATH)
    return _lib


def load_library(path: str) -> ctypes.CDLL:
    """Open a build of the library at `path` with the C ABI's argument types
    declared (lib() uses it for libtq.so; tests use it for test builds)."""
    L = ctypes.CDLL(path)
    P, I, U64, SZ, F, D = (ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64,
                           ctypes.c_size_t, ctypes.c_float, ctypes.POINTER(ctypes.c_double))
    L.tq_abi_version.restype = I
    L.tq_abi_version.argtypes = []
    L.tq_status_string.restype = ctypes.c_char_p
    L.tq_status_string.argtypes = [I]
    L.tq_build_codebook.restype = I
    L.tq_build_codebook.argtypes = [I, I, D, D, D]
    L.tq_encode.restype = I
    L.tq_encode.argtypes = [P, I, I, I, I, I, I, U64, P, P, P, P, I, I, P, P]
    L.tq_dequant.restype = I
    L.tq_dequant.argtypes = [P, P, I, I, I, I, U64, I, I, P, P]
    L.tq_attend_workspace_size.restype = SZ
    L.tq_attend_workspace_size.argtypes = [I, I, I, I]
    L.tq_attend.restype = I
    L.tq_attend.argtypes = [P, I, P, P, P, P, P, I, I, I, I, I, I, U64, I, F, I,
                            P, SZ, P, P, P, I, P]
    L.tq_attend_gate_counts.restype = I
    L.tq_attend_gate_counts.argtypes = [P, I, P, P, P, P, P, I, I, I, I, I, I, U64, I, F, I,
                                        P, SZ, P, P, P, P, I, P]
    L.tq_attend_append.restype = I
    L.tq_attend_append.argtypes = [P, I, P, I, P, P, P, P, P, I, I, I, I, I, I, U64, I, F,
                                   I, P, SZ, P, P, P, I, P]
    L.tq_prefill_attend.restype = I
    L.tq_prefill_attend.argtypes = [P, I, P, P, P, P, P, I, I, I, I, I, I, I, U64, I, P, P,
                                    I, P]
    L.tq_prefill_attend_split.restype = I
    L.tq_prefill_attend_split.argtypes = [P, I, P, P, P, P, P, I, I, I, I, I, I, I, U64, I,
                                          I, P, SZ, P, P, I, P]
    L.tq_prefill_workspace_size.restype = SZ
    L.tq_prefill_workspace_size.argtypes = [I, I, I, I, I]
    L.tq_prefill_splits.restype = I
    L.tq_prefill_splits.argtypes = [I, I, I, I, I]
    L.tq_attend_partial.restype = I
    L.tq_attend_partial.argtypes = [P, I, P, P, P, P, P, I, I, I, I, I, I, U64, I, F, I,
                                    P, SZ, P, P, P, P]
    L.tq_attend_combine.restype = I
    L.tq_attend_combine.argtypes = [P, I, I, I, I, U64, P, P, I, P]
    L.tq_qjl_encode.restype = I
    L.tq_qjl_encode.argtypes = [P, I, I, I, I, I, U64, P, P, P, P, P, I, I, P, P]
    L.tq_qjl_scores.restype = I
    L.tq_qjl_scores.argtypes = [P, I, P, P, P, P, P, P, I, I, I, I, I, U64, I, I, P, P, P]
    L.tq_attend_noalloc.restype = I
    L.tq_attend_noalloc.argtypes = [P, I, P, P, P, P, P, I, I, I, I, I, I, U64, I, F, I,
                                    P, P, P, I, P]
    return L


def _ptr(x):
    """Device address of a torch tensor, an int address, or None (NULL)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(fn, st):
    if st != TQ_OK:
        raise TQError(fn, st)


def tq_status_string(status: int) -> str:
    return lib().tq_status_string(status).decode()


status_string = tq_status_string


def tq_abi_version() -> int:
    return lib().tq_abi_version()


def tq_build_codebook(bits: int, d: int):
    """(centroids[2^bits], thresholds[2^bits-1], mse) of the N(0,1/d) codebook."""
    n = 1 << bits
    c = np.zeros(n, dtype=np.float64)
    t = np.zeros(max(n - 1, 1), dtype=np.float64)
    m = ctypes.c_double()
    dp = ctypes.POINTER(ctypes.c_double)
    _check("tq_build_codebook", lib().tq_build_codebook(
        bits, d, c.ctypes.data_as(dp), t.ctypes.data_as(dp), ctypes.byref(m)))
    return c, t[:n - 1], m.value


def tq_encode(kv, dtype, n_tok, n_kv_heads, d, bits_k, bits_v, seed, packed_k,
              packed_v, norms_k, norms_v, cap_tok, tok_offset, dev_status=None,
              stream=None):
    _check("tq_encode", lib().tq_encode(
        _ptr(kv), dtype, n_tok, n_kv_heads, d, bits_k, bits_v, seed,
        _ptr(packed_k), _ptr(packed_v), _ptr(norms_k), _ptr(norms_v), cap_tok,
        tok_offset, _ptr(dev_status), _stream(stream)))


def tq_dequant(packed, norms, n_tok, n_kv_heads, d, bits, seed, cap_tok, domain,
               out, stream=None):
    _check("tq_dequant", lib().tq_dequant(
        _ptr(packed), _ptr(norms), n_tok, n_kv_heads, d, bits, seed, cap_tok,
        domain, _ptr(out), _stream(stream)))


def tq_attend_workspace_size(batch, n_q_heads, cap_tok, d) -> int:
    return lib().tq_attend_workspace_size(batch, n_q_heads, cap_tok, d)


def tq_attend(q, q_dtype, packed_k, norms_k, packed_v, norms_v, ctx_lens, batch,
              n_q_heads, gqa_ratio, d, bits_k, bits_v, seed, cap_tok,
              sparse_v_thresh, n_ctas, workspace, workspace_bytes, out,
              out_dtype, dev_status=None, sparse_v_skipped=None, stream=None):
    """Decode attention. The workspace's counter region must be zero before
    its first use (allocate it with torch.zeros); calls keep it zero."""
    _check("tq_attend", lib().tq_attend(
        _ptr(q), q_dtype, _ptr(packed_k), _ptr(norms_k), _ptr(packed_v),
        _ptr(norms_v), _ptr(ctx_lens), batch, n_q_heads, gqa_ratio, d, bits_k,
        bits_v, seed, cap_tok, float(sparse_v_thresh), n_ctas,
        _ptr(workspace), workspace_bytes, _ptr(dev_status),
        _ptr(sparse_v_skipped), _ptr(out), out_dtype, _stream(stream)))


def tq_attend_gate_counts(q, q_dtype, packed_k, norms_k, packed_v, norms_v, ctx_lens, batch,
                          n_q_heads, gqa_ratio, d, bits_k, bits_v, seed, cap_tok,
                          sparse_v_thresh, n_ctas, workspace, workspace_bytes, head_skipped,
                          out, out_dtype, dev_status=None, sparse_v_skipped=None,
                          stream=None):
    """tq_attend plus per (sequence, query head) sparse-V gate counts added
    into head_skipped (uint32 [batch][n_q_heads], zeroed by the caller)."""
    _check("tq_attend_gate_counts", lib().tq_attend_gate_counts(
        _ptr(q), q_dtype, _ptr(packed_k), _ptr(norms_k), _ptr(packed_v),
        _ptr(norms_v), _ptr(ctx_lens), batch, n_q_heads, gqa_ratio, d, bits_k,
        bits_v, seed, cap_tok, float(sparse_v_thresh), n_ctas,
        _ptr(workspace), workspace_bytes, _ptr(dev_status),
        _ptr(sparse_v_skipped), _ptr(head_skipped), _ptr(out), out_dtype, _stream(stream)))


def tq_attend_append(q, q_dtype, new_kv, kv_dtype, packed_k, norms_k, packed_v, norms_v,
                     ctx_lens, batch, n_q_heads, gqa_ratio, d, bits_k, bits_v, seed,
                     cap_tok, sparse_v_thresh, n_ctas, workspace, workspace_bytes, out,
                     out_dtype, dev_status=None, sparse_v_skipped=None, stream=None):
    """One decode step: encode new_kv [2][batch][n_kv_heads][d] into cache row
    ctx_lens[b] - 1 of every sequence, then attend over ctx_lens[b]
    positions (the workspace contract of tq_attend)."""
    _check("tq_attend_append", lib().tq_attend_append(
        _ptr(q), q_dtype, _ptr(new_kv), kv_dtype, _ptr(packed_k), _ptr(norms_k),
        _ptr(packed_v), _ptr(norms_v), _ptr(ctx_lens), batch, n_q_heads, gqa_ratio, d,
        bits_k, bits_v, seed, cap_tok, float(sparse_v_thresh), n_ctas,
        _ptr(workspace), workspace_bytes, _ptr(dev_status), _ptr(sparse_v_skipped),
        _ptr(out), out_dtype, _stream(stream)))


def tq_prefill_attend(q, q_dtype, packed_k, norms_k, packed_v, norms_v, ctx_lens, batch,
                      n_tok, n_q_heads, gqa_ratio, d, bits_k, bits_v, seed, cap_tok, out,
                      out_dtype, dev_status=None, stream=None):
    """Causal attention of n_tok new query tokens per sequence over the cache
    (q, out: [batch][n_tok][n_q_heads][d]; token i sits at position
    ctx_lens[b] - n_tok + i)."""
    _check("tq_prefill_attend", lib().tq_prefill_attend(
        _ptr(q), q_dtype, _ptr(packed_k), _ptr(norms_k), _ptr(packed_v), _ptr(norms_v),
        _ptr(ctx_lens), batch, n_tok, n_q_heads, gqa_ratio, d, bits_k, bits_v, seed, cap_tok,
        _ptr(dev_status), _ptr(out), out_dtype, _stream(stream)))


def tq_attend_partial(q, q_dtype, packed_k, norms_k, packed_v, norms_v, ctx_lens, batch,
                      n_q_heads, gqa_ratio, d, bits_k, bits_v, seed, cap_tok,
                      sparse_v_thresh, n_ctas, workspace, workspace_bytes, partial,
                      dev_status=None, sparse_v_skipped=None, stream=None):
    """Attention over one context slice, leaving log-sum-exp records
    (float [batch][n_q_heads][d + 2]) in `partial` for tq_attend_combine."""
    _check("tq_attend_partial", lib().tq_attend_partial(
        _ptr(q), q_dtype, _ptr(packed_k), _ptr(norms_k), _ptr(packed_v),
        _ptr(norms_v), _ptr(ctx_lens), batch, n_q_heads, gqa_ratio, d, bits_k,
        bits_v, seed, cap_tok, float(sparse_v_thresh), n_ctas,
        _ptr(workspace), workspace_bytes, _ptr(dev_status),
        _ptr(sparse_v_skipped), _ptr(partial), _stream(stream)))


def tq_attend_combine(partials, n_parts, batch, n_q_heads, d, seed, out, out_dtype,
                      dev_status=None, stream=None):
    """Merge n_parts slices' records ([n_parts][batch][n_q_heads][d + 2])
    into the attention output."""
    _check("tq_attend_combine", lib().tq_attend_combine(
        _ptr(partials), n_parts, batch, n_q_heads, d, seed, _ptr(dev_status), _ptr(out),
        out_dtype, _stream(stream)))


def tq_qjl_encode(k, dtype, n_tok, n_kv_heads, d, bits_k, seed, projection, packed_k, norms_k,
                  sketch, gamma, cap_tok, tok_offset, dev_status=None, stream=None):
    """Residual sketch rows (d/8 bytes) and fp16 residual norms of n_tok keys
    ([n_tok][n_kv_heads][d]) whose stage-1 rows are in packed_k / norms_k."""
    _check("tq_qjl_encode", lib().tq_qjl_encode(
        _ptr(k), dtype, n_tok, n_kv_heads, d, bits_k, seed, _ptr(projection), _ptr(packed_k),
        _ptr(norms_k), _ptr(sketch), _ptr(gamma), cap_tok, tok_offset, _ptr(dev_status),
        _stream(stream)))


def tq_qjl_scores(q, q_dtype, packed_k, norms_k, sketch, gamma, projection, ctx_lens, batch,
                  n_q_heads, gqa_ratio, d, bits_k, seed, cap_tok, with_sketch, scores,
                  dev_status=None, stream=None):
    """Estimated scores [batch][n_q_heads][cap_tok] (float) of the first
    ctx_lens[b] keys; with_sketch adds the unbiased residual correction."""
    _check("tq_qjl_scores", lib().tq_qjl_scores(
        _ptr(q), q_dtype, _ptr(packed_k), _ptr(norms_k), _ptr(sketch), _ptr(gamma),
        _ptr(projection), _ptr(ctx_lens), batch, n_q_heads, gqa_ratio, d, bits_k, seed, cap_tok,
        int(with_sketch), _ptr(dev_status), _ptr(scores), _stream(stream)))


def tq_prefill_attend_split(q, q_dtype, packed_k, norms_k, packed_v, norms_v, ctx_lens, batch,
                            n_tok, n_q_heads, gqa_ratio, d, bits_k, bits_v, seed, cap_tok,
                            n_splits, workspace, workspace_bytes, out, out_dtype,
                            dev_status=None, stream=None):
    """tq_prefill_attend with each query tile's context split n_splits ways
    (records in the workspace, merged into out by a second launch)."""
    _check("tq_prefill_attend_split", lib().tq_prefill_attend_split(
        _ptr(q), q_dtype, _ptr(packed_k), _ptr(norms_k), _ptr(packed_v), _ptr(norms_v),
        _ptr(ctx_lens), batch, n_tok, n_q_heads, gqa_ratio, d, bits_k, bits_v, seed, cap_tok,
        n_splits, _ptr(workspace), workspace_bytes, _ptr(dev_status), _ptr(out), out_dtype,
        _stream(stream)))


def tq_prefill_workspace_size(batch, n_tok, n_q_heads, d, n_splits) -> int:
    return lib().tq_prefill_workspace_size(batch, n_tok, n_q_heads, d, n_splits)


def tq_prefill_splits(batch, n_tok, n_q_heads, gqa_ratio, max_ctx=0) -> int:
    return lib().tq_prefill_splits(batch, n_tok, n_q_heads, gqa_ratio, max_ctx)


def tq_attend_noalloc(q, q_dtype, packed_k, norms_k, packed_v, norms_v, ctx_lens,
                      batch, n_q_heads, gqa_ratio, d, bits_k, bits_v, seed, cap_tok,
                      sparse_v_thresh, n_ctas, out, out_dtype, dev_status=None,
                      sparse_v_skipped=None, stream=None):
    """tq_attend with the library's fixed internal scratch instead of a
    workspace (for callers that cannot allocate). Calls on one device must
    not overlap on the GPU; the first call per device must precede any
    stream capture."""
    _check("tq_attend_noalloc", lib().tq_attend_noalloc(
        _ptr(q), q_dtype, _ptr(packed_k), _ptr(norms_k), _ptr(packed_v),
        _ptr(norms_v), _ptr(ctx_lens), batch, n_q_heads, gqa_ratio, d, bits_k,
        bits_v, seed, cap_tok, float(sparse_v_thresh), n_ctas, _ptr(dev_status),
        _ptr(sparse_v_skipped), _ptr(out), out_dtype, _stream(stream)))
