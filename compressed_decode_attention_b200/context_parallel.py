"""Context-parallel decode attention: one process per GPU, each holding a
contiguous slice of every sequence's compressed cache.

Each rank runs tq_attend_partial over its slice, the ranks exchange their
log-sum-exp records (a few KB: batch x query heads x (d + 2) floats) with one
all-gather over the process group (NCCL over NVLink between GPUs), and every
rank merges them with tq_attend_combine. The merge is exact, so the result
is single-pass attention over the whole context to rounding.

Slices consist of whole TQ_SPARSE_V_BLOCK-position blocks, so the sparse-V
gate's blocks are the same as in one pass. All arithmetic runs in the CUDA
kernels of libtq.so; this module only computes slice bounds and moves the
records.
"""
from __future__ import annotations

from . import (TQ_SPARSE_V_BLOCK, tq_attend_combine, tq_attend_partial)


def slice_bounds(n_positions: int, world: int, rank: int) -> tuple[int, int]:
    """Positions [start, stop) of `rank`'s slice of a context of
    n_positions: the blocks are dealt in `world` contiguous runs of
    ceil(blocks / world), so a slice starts on a block boundary; the last
    ranks may get fewer positions, or none."""
    if world < 1 or not 0 <= rank < world or n_positions < 0:
        raise ValueError("bad slice arguments")
    blocks = -(-n_positions // TQ_SPARSE_V_BLOCK)
    per = -(-blocks // world) * TQ_SPARSE_V_BLOCK
    return min(rank * per, n_positions), min((rank + 1) * per, n_positions)


def local_ctx_lens(ctx_lens, start: int, stop: int):
    """Positions each sequence has in the slice [start, stop) (numpy array or
    torch tensor in, same type out): clamp(ctx - start, 0, stop - start)."""
    return (ctx_lens - start).clip(0, stop - start)


def gather_records(partial, gathered, group=None):
    """All-gather every rank's records [batch][heads][d + 2] into gathered
    [world][batch][heads][d + 2] (rank order)."""
    import torch.distributed as dist
    # the concatenated form [world * batch][heads][d + 2] of the same memory,
    # which every backend accepts
    dist.all_gather_into_tensor(gathered.view((-1,) + tuple(partial.shape[1:])), partial,
                                group=group)
    return gathered


def attend_context_parallel(q, q_dtype, packed_k, norms_k, packed_v, norms_v, local_lens,
                            batch, n_q_heads, gqa_ratio, d, bits_k, bits_v, seed, cap_tok,
                            sparse_v_thresh, workspace, workspace_bytes, partial, gathered,
                            out, out_dtype, group=None, dev_status=None,
                            sparse_v_skipped=None):
    """This rank's slice (cache rows from the slice's first position,
    local_lens from local_ctx_lens) -> records -> all-gather -> merged
    output in `out` on every rank. partial: float32 [batch][n_q_heads][d + 2];
    gathered: float32 [world][batch][n_q_heads][d + 2]. Runs on torch's
    current stream, which the process group's collective is ordered with."""
    tq_attend_partial(q, q_dtype, packed_k, norms_k, packed_v, norms_v, local_lens, batch,
                      n_q_heads, gqa_ratio, d, bits_k, bits_v, seed, cap_tok,
                      sparse_v_thresh, 0, workspace, workspace_bytes, partial,
                      dev_status=dev_status, sparse_v_skipped=sparse_v_skipped)
    gather_records(partial, gathered, group)
    tq_attend_combine(gathered, gathered.shape[0], batch, n_q_heads, d, seed, out, out_dtype,
                      dev_status=dev_status)
    return out
