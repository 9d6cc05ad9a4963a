#!/usr/bin/env python3
"""Benchmark: decode attention over the packed KV cache, and bulk encode.

One step = one decode step of a 32-layer Llama-3-8B-shaped model (batch 1,
32 query heads, 8 kv heads, d = 128, 32768 cached tokens, K4/V2, fp16): for
every layer, one tq_attend_append launch appends the new token's K/V to that
layer's packed cache and attends over all 32768 positions. The 32 layer
caches (839 MB) are distinct, so successive reads of a layer are far apart
and the 126 MB L2 cannot hold them. Steps are CUDA-graph replays.

  value   packed-KV GB/s: algorithmic bytes of the step (packed K/V rows,
          fp16 norms, q and out, plus the appended token's input/output) /
          step time
  roofline  the attention kernel alone (tq_attend over the same caches): a
          CUDA graph of the 32 layer launches, time / 32 per launch
  e2e     the same bytes over a step that also copies the step's inputs from
          pinned host memory and its output back
  encode  bulk prefill encode of the same 32 x 8 x 32768 K/V (4.29 GB of fp16
          input): Mtok/s (model tokens/s and token-head vectors/s)
  prefill causal attention of a 1024-token chunk over an 8192-token
          compressed context (tensor cores): TFLOP/s
  qjl     the stage-2 residual sketch of the keys (tq_qjl_encode) and the
          estimated scores of 32 query heads (tq_qjl_scores), 8 layer caches
  batched attention at serving scale: 64 sequences of 1024-16384 positions
          (K4/V3, ~0.5 GB per call)
  context_parallel  the same attention split into 4 slices of the context,
          emulated on one GPU: 4 tq_attend_partial launches + tq_attend_combine
          per layer, against the one-pass launch

`--impl reference` times the CPU oracle (float64 numpy) on a bounded sample
of the same workload instead.

Multi-GPU (torchrun, one process per GPU): every rank runs its own replica of
the workload (weak scaling, no collective on the data path); the step time is
the maximum over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic as S  # noqa: E402

METRIC = "decode-attn packed-KV GB/s & % HBM roofline; encode Mtok/s (1×B200)"
WORKLOAD = "llama3_8b_decode"
ENCODE_WORKLOAD = "bulk_prefill_encode"
BATCHED_WORKLOAD = "batched_serving"
QWEN_WORKLOAD = "qwen14b_decode"
QWEN_LAYERS = 8          # long-context measurement: distinct layer caches (705 MB > L2)
# The pages' codec figures for random vectors (TQAI §The CLI), beside ours.
PAGES_CODEC = {"k4": {"nmse": 0.009287, "snr_db": 20.3, "cos": 0.9954},
               "v2": {"nmse": 0.115653, "snr_db": 9.4, "cos": 0.9408}}
LAYERS = 32
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
CP_SLICES = 4            # context-parallel measurement: slices per sequence
QJL_LAYERS = 8           # residual-sketch measurement: distinct layer caches
FP32_FMA_TFLOPS = 74.45  # 148 SMs x 128 FMA/clock x 2 FLOP x 1.965 GHz (nominal)
PREFILL_CTX = 8192       # prefill measurement: context length after the chunk
PREFILL_TOKENS = 1024    # tokens in the chunk


# ------------------------------------------------------------------ helpers
def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    """Dense bf16 tensor TFLOP/s measured on this machine (burst: the prefill
    kernel is timed on its own)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"])
    except Exception:
        return FALLBACK_BF16_TFLOPS


def attend_bytes(w, ctx_total, q_bytes=2, out_bytes=2):
    """Algorithmic bytes of one tq_attend call: packed rows + norms + q + out."""
    row = w.d * w.bits_k // 8 + w.d * w.bits_v // 8 + 4
    return ctx_total * w.n_kv_heads * row + w.batch * w.n_q_heads * w.d * (q_bytes + out_bytes)


def prefill_flops(w, ctx, n_tok):
    """Algorithmic FLOPs of one tq_prefill_attend call: 2·d for q·k and 2·d
    for the weighted V sum per (query token, head, visible position); token
    i of the chunk sees ctx - n_tok + i + 1 positions."""
    visible = sum(ctx - n_tok + i + 1 for i in range(n_tok))
    return 4 * w.d * w.n_q_heads * visible


def encode_bytes(w, n_vec_pairs):
    """Algorithmic bytes of tq_encode over n (token, kv head) K/V pairs."""
    return n_vec_pairs * (2 * w.d * 2 + w.d * w.bits_k // 8 + w.d * w.bits_v // 8 + 4)


def kernel_source_sha():
    h = hashlib.sha256()
    for fn in ("attend_kernel.cuh", "encode_common.cuh", "device_common.cuh", "tq_internal.h"):
        with open(os.path.join(ROOT, "compressed_decode_attention_b200", "csrc", fn), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic():
    """dram bytes per launch from the last ncu capture, if the kernel source
    is unchanged since (profiles/traffic.json), else None."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
        if t.get("kernel_source_sha") == kernel_source_sha():
            return t
    except Exception:
        pass
    return None


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled through NVML in a
    background thread while the timed region runs (read-only queries)."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device_index, period_s=0.002):
        self.dev = torch_device_index
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self._stop = None

    def __enter__(self):
        import threading
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report no samples
            self.error = repr(e)
            return self
        self._stop = threading.Event()

        def run():
            while not self._stop.is_set():
                try:
                    sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                    rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((sm, rs))
                except Exception:
                    pass
                self._stop.wait(self.period)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._stop is not None:
            self._stop.set()
            self._thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "note": getattr(self, "error", "no samples")}
        reasons = set()
        for _, rs in self.samples:
            for bit, name in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s for s, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
                "samples": len(self.samples)}


# ------------------------------------------------------------------ distributed
def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init_dist(world, backend):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def reduce_max(x: float, device=None) -> float:
    """Maximum of a per-rank float over all ranks (identity on one rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and str(device).startswith("cuda"):
            dist.barrier(device_ids=[int(str(device).split(":")[1])])
        else:
            dist.barrier()


# ------------------------------------------------------------------ GPU arm
class LayerCaches:
    """Device buffers of the 32-layer decode workload."""

    def __init__(self, w, layers, stream):
        import torch
        self.w = w
        d, H, cap = w.d, w.n_kv_heads, w.cap_tok
        dev = "cuda"
        self.rk, self.rv = d * w.bits_k // 8, d * w.bits_v // 8
        self.pk = [torch.empty((1, H, cap, self.rk), dtype=torch.uint8, device=dev) for _ in range(layers)]
        self.pv = [torch.empty((1, H, cap, self.rv), dtype=torch.uint8, device=dev) for _ in range(layers)]
        self.nk = [torch.empty((1, H, cap), dtype=torch.int16, device=dev) for _ in range(layers)]
        self.nv = [torch.empty((1, H, cap), dtype=torch.int16, device=dev) for _ in range(layers)]
        self.stream = stream


def device_kv(w, layer, n_tok, gen):
    """K/V [2][n][H][d] as 16-bit patterns of the workload's dtype on the
    device: N(0,1), with the workload's outlier K channels (x20, or values
    replaced by Laplace(0,1) draws); the recipe of synthetic.kv_f32 drawn
    with torch's generator."""
    import torch
    x = torch.randn((2, n_tok, w.n_kv_heads, w.d), generator=gen, device="cuda",
                    dtype=torch.float32)
    ch = S.outlier_channels(w, layer)
    for h in range(w.n_kv_heads):
        idx = torch.as_tensor(ch[h], device="cuda")
        if w.outlier == "x20":
            x[0, :, h, idx] *= 20.0
        elif w.outlier == "laplace":        # inverse CDF of Laplace(0, 1), u in (-1/2, 1/2)
            u = torch.rand((n_tok, len(ch[h])), generator=gen, device="cuda") * (1 - 2.0 ** -23) \
                + (2.0 ** -24 - 0.5)
            x[0, :, h, idx] = -torch.sign(u) * torch.log1p(-2.0 * u.abs())
    return (x.bfloat16() if w.dtype == "bf16" else x.half()).view(torch.int16)


class Nvtx:
    """NVTX range around a timed region (visible in profilers; no effect
    on the timing)."""

    def __init__(self, name):
        self.name = name

    def __enter__(self):
        import torch
        torch.cuda.nvtx.range_push(self.name)
        return self

    def __exit__(self, *exc):
        import torch
        torch.cuda.nvtx.range_pop()


def codec_quality(x16, dtype, xhat, nhat):
    """Sums over vectors of the codec's errors, on the device.

    x16: [n][H][d] 16-bit patterns of the encoder input; xhat: [H][n][d]
    float32 from tq_dequant (original domain); nhat: [H][n] stored fp16 norms.
    Returns (rotated-domain squared error ||y - y^||^2 with y = R x/||x||
    and y^ the codebook point, which equals ||x/||x|| - x^/n^||^2 since R is
    orthonormal; NMSE ||x - x^||^2/||x||^2; cosine) summed over vectors."""
    import torch
    x = (x16.view(torch.bfloat16) if dtype == "bf16" else x16.view(torch.float16)).float()
    x = x.permute(1, 0, 2)
    nx = x.norm(dim=-1, keepdim=True)
    nh = nhat.view(torch.float16).float().unsqueeze(-1)
    rot = ((x / nx - xhat / nh) ** 2).sum(-1)
    nmse = ((x - xhat) ** 2).sum(-1) / (nx.squeeze(-1) ** 2)
    cos = (x * xhat).sum(-1) / (nx.squeeze(-1) * xhat.norm(dim=-1))
    return float(rot.double().sum()), float(nmse.double().sum()), float(cos.double().sum())


def run_gpu(args, rank, world, local_rank):
    import torch
    import compressed_decode_attention_b200 as tq

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    w = S.WORKLOADS[WORKLOAD]
    we = S.WORKLOADS[ENCODE_WORKLOAD]
    assert (we.n_kv_heads, we.ctx, we.bits_k, we.bits_v) == (w.n_kv_heads, w.ctx, w.bits_k, w.bits_v)
    L = args.layers
    stream = torch.cuda.Stream(device)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(S.DATA_SEED + 7919 * rank)
    seed = S.SIGN_SEED
    caches = LayerCaches(w, L, stream)
    H, d, ctx, cap = w.n_kv_heads, w.d, w.ctx, w.cap_tok
    launches = 0

    # ---------------- bulk encode (prefill) of every layer: the encode metric
    kv_all = [device_kv(we, l, ctx, gen) for l in range(L)]
    status = torch.zeros(1, dtype=torch.int32, device=device)
    section_status = {}

    def take_status(name):
        """The device status bits the section just run set (then cleared)."""
        section_status[name] = int(status.item())
        status.zero_()


    def encode_all():
        for l in range(L):
            tq.tq_encode(kv_all[l], tq.TQ_F16, ctx, H, d, w.bits_k, w.bits_v, seed,
                         caches.pk[l], caches.pv[l], caches.nk[l], caches.nv[l], cap, 0,
                         status, stream)

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            encode_all()
    torch.cuda.synchronize()
    enc_steps = max(3, min(args.steps, 10))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(device)
    torch.cuda.synchronize()
    e0.record(stream)
    with Nvtx("encode"), torch.cuda.stream(stream):
        for _ in range(enc_steps):
            encode_all()
    e1.record(stream)
    torch.cuda.synchronize()
    enc_ms = reduce_max(e0.elapsed_time(e1) / enc_steps, device)
    enc_launches = enc_steps * L

    take_status("encode")
    # ---------------- encode -> dequant round trip of the bulk workload: every
    # layer's K and V dequantized to the original domain (tq_dequant, timed)
    # and compared with the encoder input: the codec's quality
    dq = torch.empty((H, ctx, d), dtype=torch.float32, device=device)
    quality = {"k": [0.0, 0.0, 0.0], "v": [0.0, 0.0, 0.0]}
    streams_ = (("k", 0, w.bits_k, caches.pk, caches.nk), ("v", 1, w.bits_v, caches.pv, caches.nv))
    for l in range(L):
        for name, which, bits, pks, nks in streams_:
            with torch.cuda.stream(stream):
                tq.tq_dequant(pks[l], nks[l], ctx, H, d, bits, seed, cap, 0, dq, stream)
            stream.synchronize()
            r = codec_quality(kv_all[l][which], we.dtype, dq, nks[l][0])
            quality[name] = [a_ + b_ for a_, b_ in zip(quality[name], r)]

    def dequant_all():
        for l in range(L):
            for name, which, bits, pks, nks in streams_:
                tq.tq_dequant(pks[l], nks[l], ctx, H, d, bits, seed, cap, 0, dq, stream)

    with torch.cuda.stream(stream):
        dequant_all()
    torch.cuda.synchronize()
    dq0, dq1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(device)
    torch.cuda.synchronize()
    dq0.record(stream)
    with Nvtx("dequant"), torch.cuda.stream(stream):
        dequant_all()
    dq1.record(stream)
    torch.cuda.synchronize()
    dq_ms = reduce_max(dq0.elapsed_time(dq1) / L, device)     # per layer, K and V
    launches += 2 * L
    n_vec = L * ctx * H
    round_trip = {"workload": ENCODE_WORKLOAD, "vectors_per_stream": n_vec,
                  "note": "rotated_mse = mean ||y - y^||^2 with y = R x/||x|| (per-coordinate "
                          "MSE in N(0,1) units); K has 4 outlier channels x20 per head, so its "
                          "rotated coordinates are not N(0,1) and its MSE departs from the "
                          "codebook's; V is plain N(0,1)"}
    for name, bits in (("k", w.bits_k), ("v", w.bits_v)):
        rot, nmse, cos = (v_ / n_vec for v_ in quality[name])
        dmse = tq.tq_build_codebook(bits, 1)[2]
        round_trip[name] = {"bits": bits, "rotated_mse": round(rot, 6),
                            "codebook_mse": round(dmse, 6), "ratio": round(rot / dmse, 4),
                            "nmse": round(nmse, 6), "snr_db": round(-10 * np.log10(nmse), 2),
                            "cos": round(cos, 5)}
    round_trip["pages_random_vectors"] = dict(PAGES_CODEC, source="TQAI §The CLI")
    round_trip["dequant_us_per_layer"] = round(dq_ms * 1e3, 2)
    round_trip["dequant_gbs"] = round(H * ctx * ((w.d * (w.bits_k + w.bits_v)) // 8 + 4 + 2 * w.d * 4)
                                      / (dq_ms * 1e-3) / 1e9, 1)
    del dq

    take_status("round_trip")
    # ---------------- stage-2 residual sketch (QJL) of the keys of QJL_LAYERS
    # layer caches, and the estimated scores of 32 query heads over them
    QL = min(QJL_LAYERS, L)
    proj = torch.from_numpy(S.projection_matrix(d)).to(device)
    qsk = [torch.empty((1, H, cap, d // 8), dtype=torch.uint8, device=device) for _ in range(QL)]
    qgm = [torch.empty((1, H, cap), dtype=torch.int16, device=device) for _ in range(QL)]
    qq = [torch.randn((1, w.n_q_heads, d), generator=gen, device=device).half() for _ in range(QL)]
    qsc = [torch.empty((1, w.n_q_heads, cap), dtype=torch.float32, device=device) for _ in range(QL)]
    qctx = torch.full((1,), ctx, dtype=torch.int32, device=device)

    def qjl_encode_all():
        for l in range(QL):
            tq.tq_qjl_encode(kv_all[l][0], tq.TQ_F16, ctx, H, d, w.bits_k, seed, proj,
                             caches.pk[l], caches.nk[l], qsk[l], qgm[l], cap, 0, status, stream)

    def qjl_scores_all():
        for l in range(QL):
            tq.tq_qjl_scores(qq[l], tq.TQ_F16, caches.pk[l], caches.nk[l], qsk[l], qgm[l], proj,
                             qctx, 1, w.n_q_heads, w.gqa, d, w.bits_k, seed, cap, 1, qsc[l],
                             dev_status=status, stream=stream)

    qjl_ms = {}
    for name, fn in (("encode", qjl_encode_all), ("scores", qjl_scores_all)):
        with torch.cuda.stream(stream):
            fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        for _ in range(max(3, args.warmup)):
            g.replay()
        torch.cuda.synchronize()
        q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        qsteps = max(3, min(args.steps, 10))
        barrier(device)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            q0.record(stream)
            for _ in range(qsteps):
                g.replay()
            q1.record(stream)
        torch.cuda.synchronize()
        qjl_ms[name] = reduce_max(q0.elapsed_time(q1) / (qsteps * QL), device)
        launches += qsteps * QL
        del g
    n_keys = ctx * H
    qjl_enc_flops = n_keys * 2 * d * d
    qjl_enc_bytes = n_keys * (2 * d + d * w.bits_k // 8 + 2 + d // 8 + 2)
    qjl_sc_flops = ctx * w.n_q_heads * 4 * d
    qjl_sc_bytes = n_keys * (d * w.bits_k // 8 + 2 + d // 8 + 2) + ctx * w.n_q_heads * 4 + \
        w.n_q_heads * d * 2
    del qsk, qgm, qq, qsc
    del kv_all
    torch.cuda.empty_cache()

    take_status("qjl")
    # ---------------- prefill attention: a 1024-token chunk at the end of an
    # 8192-token context (the chunk's rows are in the cache), 4 layers
    pf_layers, pf_ctx, pf_T = 4, PREFILL_CTX, PREFILL_TOKENS
    pf = LayerCaches(dataclasses.replace(w, ctx=pf_ctx, cap_tok=pf_ctx), pf_layers, stream)
    for l in range(pf_layers):
        kv_pf = device_kv(w, l, pf_ctx, gen)
        tq.tq_encode(kv_pf, tq.TQ_F16, pf_ctx, H, d, w.bits_k, w.bits_v, seed, pf.pk[l], pf.pv[l],
                     pf.nk[l], pf.nv[l], pf_ctx, 0, status, stream)
        torch.cuda.synchronize()       # the input's memory is reused on another stream
        del kv_pf
    pf_q = [torch.randn((1, pf_T, w.n_q_heads, d), generator=gen, device=device).half()
            for _ in range(pf_layers)]
    pf_out = [torch.empty((1, pf_T, w.n_q_heads, d), dtype=torch.float16, device=device)
              for _ in range(pf_layers)]
    pf_ctx_dev = torch.full((1,), pf_ctx, dtype=torch.int32, device=device)

    pf_splits = tq.tq_prefill_splits(1, pf_T, w.n_q_heads, w.gqa, pf_ctx)
    pf_wsb = tq.tq_prefill_workspace_size(1, pf_T, w.n_q_heads, d, pf_splits)
    pf_ws = torch.empty(max(pf_wsb, 16), dtype=torch.uint8, device=device)

    def prefill_all():
        for l in range(pf_layers):
            tq.tq_prefill_attend_split(pf_q[l], tq.TQ_F16, pf.pk[l], pf.nk[l], pf.pv[l],
                                       pf.nv[l], pf_ctx_dev, 1, pf_T, w.n_q_heads, w.gqa, d,
                                       w.bits_k, w.bits_v, seed, pf_ctx, pf_splits, pf_ws,
                                       pf_wsb, pf_out[l], tq.TQ_F16, dev_status=status,
                                       stream=stream)

    with torch.cuda.stream(stream):
        prefill_all()
    torch.cuda.synchronize()
    pf_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(pf_graph, stream=stream):
        prefill_all()
    for _ in range(max(3, args.warmup)):
        pf_graph.replay()
    torch.cuda.synchronize()
    pf_steps = max(3, min(args.steps, 10))
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(device)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        p0.record(stream)
        for _ in range(pf_steps):
            pf_graph.replay()
        p1.record(stream)
    torch.cuda.synchronize()
    pf_ms = reduce_max(p0.elapsed_time(p1) / (pf_steps * pf_layers), device)
    pf_flops = prefill_flops(w, pf_ctx, pf_T)
    del pf_graph, pf, pf_q, pf_out, pf_ws
    torch.cuda.empty_cache()

    take_status("prefill")
    # ---------------- decode step graphs
    # per-layer queries, new K/V and outputs are views of three contiguous
    # buffers, so that the end-to-end step moves each with one copy
    # the step's inputs (every layer's query, then every layer's new K/V)
    # share one device buffer of 16-bit words
    nq16, nkv16 = L * w.n_q_heads * d, L * 2 * H * d
    inputs = torch.empty(nq16 + nkv16, dtype=torch.int16, device=device)
    q_all = inputs[:nq16].view(torch.float16).view(L, 1, w.n_q_heads, d)
    kv_all_new = inputs[nq16:].view(L, 2, 1, H, d)
    q_all.copy_(torch.randn((L, 1, w.n_q_heads, d), generator=gen, device=device).half())
    kv_all_new.copy_(torch.stack([device_kv(w, l, 1, gen) for l in range(L)]))
    outs_all = torch.empty((L, 1, w.n_q_heads, d), dtype=torch.float16, device=device)
    q = [q_all[l] for l in range(L)]
    kv_new = [kv_all_new[l] for l in range(L)]
    outs = [outs_all[l] for l in range(L)]
    ctx_dev = torch.full((1,), ctx, dtype=torch.int32, device=device)
    ws_bytes = tq.tq_attend_workspace_size(1, w.n_q_heads, cap, d)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=device)

    def attend_layer(l):
        tq.tq_attend(q[l], tq.TQ_F16, caches.pk[l], caches.nk[l], caches.pv[l], caches.nv[l],
                     ctx_dev, 1, w.n_q_heads, w.gqa, d, w.bits_k, w.bits_v, seed, cap, 0.0, 0,
                     ws, ws_bytes, outs[l], tq.TQ_F16, dev_status=status, stream=stream)

    def step():
        # one decode step: per layer, the new token is appended to the
        # compressed cache and attention runs over ctx positions, one launch
        for l in range(L):
            tq.tq_attend_append(q[l], tq.TQ_F16, kv_new[l], tq.TQ_F16, caches.pk[l],
                                caches.nk[l], caches.pv[l], caches.nv[l], ctx_dev, 1,
                                w.n_q_heads, w.gqa, d, w.bits_k, w.bits_v, seed, cap, 0.0, 0,
                                ws, ws_bytes, outs[l], tq.TQ_F16, dev_status=status,
                                stream=stream)

    kernels_per_step = L       # one tq_attend_append per layer

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        return g

    with torch.cuda.stream(stream):
        step()                       # eager warm-up of the exact sequence
    torch.cuda.synchronize()
    step_graph = capture(step)
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        step_graph.replay()
    torch.cuda.synchronize()

    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(device)
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk, Nvtx("decode_step"):
        with torch.cuda.stream(stream):
            t0.record(stream)
            for _ in range(args.steps):
                step_graph.replay()
            t1.record(stream)
        torch.cuda.synchronize()
    ms_total = t0.elapsed_time(t1)
    ms_step = reduce_max(ms_total / args.steps, device)
    launches += kernels_per_step * args.steps

    take_status("decode_step")
    # ---------------- the attention kernel alone: per-launch time = a graph
    # of the L layers' launches (distinct caches, larger than L2) / L
    def attend_all():
        for l in range(L):
            attend_layer(l)

    attend_graph = capture(attend_all)
    for _ in range(args.warmup):
        attend_graph.replay()
    torch.cuda.synchronize()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(device)
    torch.cuda.synchronize()
    with Nvtx("attend"), torch.cuda.stream(stream):
        a0.record(stream)
        for _ in range(args.steps):
            attend_graph.replay()
        a1.record(stream)
    torch.cuda.synchronize()
    attend_ms_mean = reduce_max(a0.elapsed_time(a1) / (args.steps * L), device)
    launches += L * args.steps

    take_status("attend")
    # ---------------- context parallelism, P slices emulated on this GPU: per
    # layer, one tq_attend_partial per slice of whole 64-position blocks
    # (views into the layer cache: row offset, cap_tok kept as the head
    # stride), then tq_attend_combine of the P records. On P GPUs the
    # partials run concurrently and an all-gather of the records precedes
    # the combine; here they run back to back.
    from compressed_decode_attention_b200.context_parallel import slice_bounds
    P = CP_SLICES
    spans = [slice_bounds(ctx, P, r) for r in range(P)]
    cp_lens = [torch.full((1,), b - a, dtype=torch.int32, device=device) for a, b in spans]
    rec = torch.empty((P, 1, w.n_q_heads, d + 2), dtype=torch.float32, device=device)
    rk, rv = d * w.bits_k // 8, d * w.bits_v // 8

    def cp_partials(l):
        for r, (a, _) in enumerate(spans):
            tq.tq_attend_partial(q[l], tq.TQ_F16, caches.pk[l].data_ptr() + a * rk,
                                 caches.nk[l].data_ptr() + 2 * a,
                                 caches.pv[l].data_ptr() + a * rv,
                                 caches.nv[l].data_ptr() + 2 * a, cp_lens[r], 1, w.n_q_heads,
                                 w.gqa, d, w.bits_k, w.bits_v, seed, cap, 0.0, 0, ws, ws_bytes,
                                 rec[r], dev_status=status, stream=stream)

    def cp_combine(l):
        tq.tq_attend_combine(rec, P, 1, w.n_q_heads, d, seed, outs[l], tq.TQ_F16,
                             dev_status=status, stream=stream)

    def cp_all():
        for l in range(L):
            cp_partials(l)
            cp_combine(l)

    def combine_all():
        for l in range(L):
            cp_combine(l)

    cp_times = {}
    for name, fn, per in (("layer", cp_all, P + 1), ("combine", combine_all, 1)):
        g = capture(fn)
        for _ in range(args.warmup):
            g.replay()
        torch.cuda.synchronize()
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(device)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            c0.record(stream)
            for _ in range(args.steps):
                g.replay()
            c1.record(stream)
        torch.cuda.synchronize()
        cp_times[name] = reduce_max(c0.elapsed_time(c1) / (args.steps * L), device)
        launches += per * L * args.steps
        del g

    take_status("context_parallel")
    # ---------------- attention at serving scale: the batched workload (64
    # sequences of U{1024..16384} positions, K4/V3, sparse-V gate 1e-6), two
    # layer caches alternating (2 x 0.97 GB of capacity, > L2), each encoded
    # by tq_encode from the workload's recipe (N(0,1) fp16 K/V)
    wb = S.WORKLOADS[BATCHED_WORKLOAD]
    bctx_h = S.ctx_lens(wb)
    bctx = torch.from_numpy(bctx_h).to(device)
    bH, bcap, bHq = wb.n_kv_heads, wb.cap_tok, wb.n_q_heads
    brk, brv = d * wb.bits_k // 8, d * wb.bits_v // 8
    bcache = []
    for _ in range(2):
        bpk = torch.zeros((wb.batch, bH, bcap, brk), dtype=torch.uint8, device=device)
        bpv = torch.zeros((wb.batch, bH, bcap, brv), dtype=torch.uint8, device=device)
        bnk = torch.zeros((wb.batch, bH, bcap), dtype=torch.int16, device=device)
        bnv = torch.zeros((wb.batch, bH, bcap), dtype=torch.int16, device=device)
        for b in range(wb.batch):
            kvb = device_kv(wb, 0, int(bctx_h[b]), gen)
            tq.tq_encode(kvb, tq.TQ_F16, int(bctx_h[b]), bH, d, wb.bits_k, wb.bits_v, seed,
                         bpk[b], bpv[b], bnk[b], bnv[b], bcap, 0, status, stream)
            torch.cuda.synchronize()   # the input's memory is reused on another stream
        bcache.append((bpk, bnk, bpv, bnv))
    skipped = torch.zeros(1, dtype=torch.int64, device=device)
    bq = [torch.randn((wb.batch, bHq, d), generator=gen, device=device).half() for _ in range(2)]
    bout = torch.empty((wb.batch, bHq, d), dtype=torch.float16, device=device)
    bws_bytes = tq.tq_attend_workspace_size(wb.batch, bHq, bcap, d)
    bws = torch.zeros(bws_bytes, dtype=torch.uint8, device=device)

    def batched_all():
        for i in range(2):
            bpk, bnk, bpv, bnv = bcache[i]
            tq.tq_attend(bq[i], tq.TQ_F16, bpk, bnk, bpv, bnv, bctx, wb.batch, bHq, wb.gqa, d,
                         wb.bits_k, wb.bits_v, seed, bcap, wb.tau, 0, bws, bws_bytes, bout,
                         tq.TQ_F16, dev_status=status, sparse_v_skipped=skipped, stream=stream)

    bgraph = capture(batched_all)
    for _ in range(args.warmup):
        bgraph.replay()
    torch.cuda.synchronize()
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(device)
    torch.cuda.synchronize()
    skipped.zero_()
    with Nvtx("batched"), torch.cuda.stream(stream):
        b0.record(stream)
        for _ in range(args.steps):
            bgraph.replay()
        b1.record(stream)
    torch.cuda.synchronize()
    batched_ms = reduce_max(b0.elapsed_time(b1) / (2 * args.steps), device)
    launches += 2 * args.steps
    batched_skipped = int(skipped.item()) // args.steps
    batched_bytes = int(bctx_h.astype(np.int64).sum()) * bH * (brk + brv + 4) + \
        wb.batch * bHq * d * (2 + 2)
    del bgraph, bcache, bq, bout, bws
    torch.cuda.empty_cache()

    take_status("batched")
    # ---------------- the Qwen-14B-shaped long-context layer (40 q / 8 kv
    # heads, GQA 5, ctx 131072, K3/V2, bf16 with Laplace(0,1) values on 3 K
    # channels per head): QWEN_LAYERS layer caches encoded by tq_encode from
    # the recipe, a CUDA graph of their tq_attend launches (time / layers)
    wq = S.WORKLOADS[QWEN_WORKLOAD]
    QLAY = min(QWEN_LAYERS, L)
    qcache = LayerCaches(wq, QLAY, stream)
    for l in range(QLAY):
        kvq = device_kv(wq, l, wq.ctx, gen)
        tq.tq_encode(kvq, tq.TQ_BF16, wq.ctx, wq.n_kv_heads, d, wq.bits_k, wq.bits_v, seed,
                     qcache.pk[l], qcache.pv[l], qcache.nk[l], qcache.nv[l], wq.cap_tok, 0,
                     status, stream)
        torch.cuda.synchronize()
        del kvq
    qw_q = torch.randn((QLAY, 1, wq.n_q_heads, d), generator=gen, device=device).bfloat16()
    qw_out = torch.empty((QLAY, 1, wq.n_q_heads, d), dtype=torch.bfloat16, device=device)
    qw_ctx = torch.full((1,), wq.ctx, dtype=torch.int32, device=device)
    qw_wsb = tq.tq_attend_workspace_size(1, wq.n_q_heads, wq.cap_tok, d)
    qw_ws = torch.zeros(qw_wsb, dtype=torch.uint8, device=device)

    def qwen_all():
        for l in range(QLAY):
            tq.tq_attend(qw_q[l], tq.TQ_BF16, qcache.pk[l], qcache.nk[l], qcache.pv[l],
                         qcache.nv[l], qw_ctx, 1, wq.n_q_heads, wq.gqa, d, wq.bits_k, wq.bits_v,
                         seed, wq.cap_tok, 0.0, 0, qw_ws, qw_wsb, qw_out[l], tq.TQ_BF16,
                         dev_status=status, stream=stream)

    qgraph = capture(qwen_all)
    for _ in range(args.warmup):
        qgraph.replay()
    torch.cuda.synchronize()
    w0_, w1_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(device)
    torch.cuda.synchronize()
    with Nvtx("qwen14b"), torch.cuda.stream(stream):
        w0_.record(stream)
        for _ in range(args.steps):
            qgraph.replay()
        w1_.record(stream)
    torch.cuda.synchronize()
    qwen_ms = reduce_max(w0_.elapsed_time(w1_) / (QLAY * args.steps), device)
    launches += QLAY * args.steps
    qwen_bytes = attend_bytes(wq, wq.ctx)
    del qgraph, qcache, qw_q, qw_out, qw_ws
    torch.cuda.empty_cache()

    take_status("qwen14b")
    # ---------------- end to end: host inputs in, host output back, every step
    in_host = torch.empty(nq16 + nkv16, dtype=torch.int16).pin_memory()
    out_host = torch.empty((L, 1, w.n_q_heads, d), dtype=torch.float16).pin_memory()
    in_host.copy_(inputs.cpu())
    e2e_graph = capture(step)
    torch.cuda.synchronize()

    def e2e_step():
        # one host-to-device copy of every layer's query and new K/V, the
        # step's launches, one device-to-host copy of every output
        inputs.copy_(in_host, non_blocking=True)
        e2e_graph.replay()
        out_host.copy_(outs_all, non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            e2e_step()
    torch.cuda.synchronize()
    barrier(device)
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Nvtx("e2e"), torch.cuda.stream(stream):
        x0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        x1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(x0.elapsed_time(x1) / args.steps, device)
    launches += kernels_per_step * args.steps
    take_status("e2e")
    st = 0
    for v_ in section_status.values():
        st |= v_

    per_layer_attend = attend_bytes(w, ctx)
    per_layer_encode = encode_bytes(w, H)
    step_bytes = L * (per_layer_attend + per_layer_encode)
    peak, peak_kind = measured_peak()
    achieved = per_layer_attend / (attend_ms_mean * 1e-3) / 1e9
    enc_bytes = L * encode_bytes(we, ctx * H)
    enc_gbs = enc_bytes / (enc_ms * 1e-3) / 1e9
    traffic = recorded_traffic()
    res = {
        "metric": METRIC,
        "value": round(world * step_bytes / (ms_step * 1e-3) / 1e9, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16",
        "dtype_detail": "tensor-core mma.sync with fp16 operands and fp32 accumulation: scores "
                        "from fp16 high+low pairs of the query and of the K codebook (~22 "
                        "significant bits), P.V with fp16 weights x V norm and fp16 V levels; "
                        "softmax, merges and the inverse rotation in fp32",
        "data": "synthetic (seeded N(0,1) fp16 K/V with x20 outlier K channels; torch generator on device)",
        "config": config_of(w, L),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                     "frac_of_nominal_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
                     "kernel": "tq_attend (attend_kernel): per-launch time from a CUDA graph of "
                               f"{L} back-to-back launches over distinct layer caches, / {L}",
                     "bytes_per_launch": per_layer_attend,
                     "launch_ms": round(attend_ms_mean, 5),
                     "traffic": traffic["traffic_bytes_per_launch"] if traffic else None},
        "e2e": {"value": round(world * step_bytes / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 4),
                "h2d_bytes_per_step": int(in_host.numel() * 2),
                "d2h_bytes_per_step": int(out_host.numel() * 2)},
        "gpu_launches": launches,
        "clocks": clk.summary(),
        "encode": {"workload": ENCODE_WORKLOAD, "metric": "encode Mtok/s",
                   "value": round(world * L * ctx / (enc_ms * 1e-3) / 1e6, 3), "unit": "Mtok/s",
                   "token_head_vectors_per_s": round(world * L * ctx * H / (enc_ms * 1e-3), 0),
                   "ms_per_step": round(enc_ms, 4), "steps": enc_steps,
                   "roofline": {"bound": "hbm", "achieved": round(enc_gbs, 1), "peak": peak,
                                "unit": "GB/s", "frac": round(enc_gbs / peak, 4),
                                "frac_of_nominal_8tbs": round(enc_gbs / NOMINAL_HBM_GBS, 4),
                                "bytes_per_step": enc_bytes},
                   "gpu_launches": enc_launches},
        "prefill": {"workload": f"{WORKLOAD} prefill chunk: {pf_T} tokens at the end of a "
                                f"{pf_ctx}-token context (32 q / 8 kv heads, d=128, "
                                f"K{w.bits_k}/V{w.bits_v}), {pf_layers} layer caches",
                    "metric": "prefill attention TFLOP/s", "unit": "TFLOP/s",
                    "value": round(world * pf_flops / (pf_ms * 1e-3) / 1e12, 2),
                    "ms_per_call": round(pf_ms, 4),
                    "roofline": {"bound": "tensor", "achieved": round(pf_flops / (pf_ms * 1e-3) / 1e12, 2),
                                 "peak": measured_tensor_peak(), "unit": "TFLOP/s",
                                 "frac": round(pf_flops / (pf_ms * 1e-3) / 1e12 / measured_tensor_peak(), 4),
                                 "peak_kind": "measured dense bf16 (fp16 mma runs at the same rate)",
                                 "flops_per_call": pf_flops},
                    "context_splits": pf_splits,
                    "gpu_launches": pf_steps * pf_layers * (2 if pf_splits > 1 else 1)},
        "qjl": {
            "workload": f"{WORKLOAD} keys: {H} kv heads x {ctx} positions, K{w.bits_k}, d={d}; "
                        f"scores of {w.n_q_heads} query heads; {QL} distinct layer caches",
            "encode": {"us_per_layer": round(qjl_ms["encode"] * 1e3, 2),
                       "mkeys_per_s": round(n_keys / (qjl_ms["encode"] * 1e-3) / 1e6, 1),
                       "gbs": round(qjl_enc_bytes / (qjl_ms["encode"] * 1e-3) / 1e9, 1),
                       "roofline": {"bound": "tensor",
                                    "achieved": round(qjl_enc_flops / (qjl_ms["encode"] * 1e-3) / 1e12, 2),
                                    "peak": measured_tensor_peak(), "unit": "TFLOP/s",
                                    "frac": round(qjl_enc_flops / (qjl_ms["encode"] * 1e-3) / 1e12 / measured_tensor_peak(), 4),
                                    "peak_kind": "measured dense bf16 (fp16 mma runs at the same rate)",
                                    "flops_per_layer": qjl_enc_flops,
                                    "mma_flops_per_layer": 3 * qjl_enc_flops}},
            "scores": {"us_per_layer": round(qjl_ms["scores"] * 1e3, 2),
                       "gbs": round(qjl_sc_bytes / (qjl_ms["scores"] * 1e-3) / 1e9, 1),
                       "bytes_per_layer": qjl_sc_bytes,
                       "roofline": {"bound": "fp32 fma",
                                    "achieved": round(qjl_sc_flops / (qjl_ms["scores"] * 1e-3) / 1e12, 2),
                                    "peak": FP32_FMA_TFLOPS, "unit": "TFLOP/s",
                                    "frac": round(qjl_sc_flops / (qjl_ms["scores"] * 1e-3) / 1e12 / FP32_FMA_TFLOPS, 4),
                                    "hbm_frac": round(qjl_sc_bytes / (qjl_ms["scores"] * 1e-3) / 1e9 / peak, 4),
                                    "flops_per_layer": qjl_sc_flops}}},
        "batched": {
            "workload": f"{BATCHED_WORKLOAD}: {wb.batch} sequences, ctx U{{{wb.ctx_range[0]}.."
                        f"{wb.ctx_range[1]}}}, {bHq} q / {bH} kv heads, d={d}, "
                        f"K{wb.bits_k}/V{wb.bits_v}, sparse-V gate {wb.tau}; 2 layer caches "
                        "alternating, each encoded by tq_encode from seeded N(0,1) fp16 K/V",
            "sparse_v_skipped_per_call": batched_skipped,
            "us_per_call": round(batched_ms * 1e3, 2),
            "bytes_per_call": batched_bytes,
            "gbs": round(batched_bytes / (batched_ms * 1e-3) / 1e9, 1),
            "frac": round(batched_bytes / (batched_ms * 1e-3) / 1e9 / peak, 4),
            "frac_of_nominal_8tbs": round(batched_bytes / (batched_ms * 1e-3) / 1e9 / NOMINAL_HBM_GBS, 4)},
        "qwen14b": {
            "workload": f"{QWEN_WORKLOAD}: batch 1, {wq.n_q_heads} q / {wq.n_kv_heads} kv heads "
                        f"(GQA {wq.gqa}), d={d}, ctx {wq.ctx}, K{wq.bits_k}/V{wq.bits_v}, bf16 "
                        f"q/K/V, Laplace(0,1) values on {wq.n_outlier} K channels per head; "
                        f"{QLAY} distinct layer caches ({QLAY * qwen_bytes / 1e6:.0f} MB > L2), "
                        "CUDA graph of their tq_attend launches",
            "us_per_launch": round(qwen_ms * 1e3, 2),
            "bytes_per_launch": qwen_bytes,
            "roofline": {"bound": "hbm", "achieved": round(qwen_bytes / (qwen_ms * 1e-3) / 1e9, 1),
                         "peak": peak, "unit": "GB/s",
                         "frac": round(qwen_bytes / (qwen_ms * 1e-3) / 1e9 / peak, 4),
                         "frac_of_nominal_8tbs": round(qwen_bytes / (qwen_ms * 1e-3) / 1e9 / NOMINAL_HBM_GBS, 4)}},
        "round_trip": round_trip,
        "context_parallel": {
            "slices": P, "emulated_on_one_gpu": True,
            "per_layer": f"{P} x tq_attend_partial over {ctx // P}-position slices + "
                         "tq_attend_combine of the records (no all-gather on one GPU)",
            "layer_ms": round(cp_times["layer"], 5),
            "one_pass_layer_ms": round(attend_ms_mean, 5),
            "achieved_gbs": round(per_layer_attend / (cp_times["layer"] * 1e-3) / 1e9, 1),
            "combine_ms": round(cp_times["combine"], 5),
            "record_bytes_per_slice": int(w.n_q_heads * (d + 2) * 4)},
        "device_status": st,
        "device_status_by_section": section_status,
    }
    del step_graph, attend_graph, e2e_graph
    return res


# ------------------------------------------------------------------ CPU oracle arm
def config_of(w, layers):
    """The `config` object of the bench line (shared by both arms)."""
    return {"workload": WORKLOAD, "layers": layers, "batch": w.batch, "n_q_heads": w.n_q_heads,
            "n_kv_heads": w.n_kv_heads, "d": w.d, "ctx": w.ctx,
            "bits": f"K{w.bits_k}/V{w.bits_v}", "kv_dtype": "fp16", "q_out_dtype": "fp16",
            "per_gpu": "one model replica",
            "l2": f"inputs larger than L2: {layers} distinct layer caches, "
                  f"{layers * attend_bytes(w, w.ctx) / 1e6:.0f} MB per step",
            "step": "per layer: tq_attend_append (append the new token, attend over "
                    "ctx positions; one launch), CUDA graph"}


def oracle_sample(budget_s=12.0, threads=None):
    """Time the oracle on a bounded sample of the decode workload: whole
    (kv head, query group) units of one layer at full context, plus a block of
    encode vectors. `threads` caps numpy's BLAS pool (None: its default).
    Returns GB/s on the bench's byte basis, the units and seconds timed."""
    import threadpoolctl
    from oracle import attention, codec
    w = S.WORKLOADS[WORKLOAD]
    with threadpoolctl.threadpool_limits(threads):
        info = threadpoolctl.threadpool_info()
        cores = max((i.get("num_threads", 1) for i in info), default=1)
        # inputs (not timed): one kv head's K/V at full context
        kv = S.kv_bits(w, 0, w.ctx)[:, :, :1]
        x_k = codec.promote(kv[0, :, 0], w.dtype)
        x_v = codec.promote(kv[1, :, 0], w.dtype)
        t = time.perf_counter()
        rk, nk = codec.encode_rows(x_k, w.bits_k, S.SIGN_SEED)
        rv, nv = codec.encode_rows(x_v, w.bits_v, S.SIGN_SEED)
        enc_s = time.perf_counter() - t
        enc_vecs = 2 * w.ctx
        qb = S.query_bits(w)[:, :w.gqa]
        q64 = codec.promote(qb, w.dtype)
        units, att_s = 0, 0.0
        while units < 1 or (att_s < budget_s and units < 64):
            t = time.perf_counter()
            attention.attend(q64, rk[None, None], nk[None, None], rv[None, None], nv[None, None],
                             np.array([w.ctx]), w.gqa, w.bits_k, w.bits_v, S.SIGN_SEED)
            att_s += time.perf_counter() - t
            units += 1
    unit_bytes = w.ctx * (w.d * w.bits_k // 8 + w.d * w.bits_v // 8 + 4) + w.gqa * w.d * 4
    return {"attend_gbs": units * unit_bytes / att_s / 1e9, "attend_units": units,
            "attend_s": att_s, "encode_s": enc_s,
            "encode_mtoks": (enc_vecs / 2 / w.n_kv_heads) / enc_s / 1e6,
            "encode_vectors_per_s": enc_vecs / enc_s, "cores": cores,
            "sample": f"{units} x (1 kv head + its {w.gqa} query heads, ctx {w.ctx}) attention; "
                      f"{enc_vecs} vector encodes"}


def cpu_baseline_both(budget_s):
    """The oracle timed single-threaded and with numpy's default thread pool."""
    one = oracle_sample(budget_s / 2, threads=1)
    allc = oracle_sample(budget_s / 2)
    return {"value": round(allc["attend_gbs"], 4), "unit": "GB/s", "cores": allc["cores"],
            "nproc": os.cpu_count(), "kind": "oracle", "sample": allc["sample"],
            "encode_mtoks": round(allc["encode_mtoks"], 6),
            "single_thread": {"value": round(one["attend_gbs"], 4), "unit": "GB/s", "threads": 1,
                              "sample": one["sample"],
                              "encode_mtoks": round(one["encode_mtoks"], 6)}}


def run_reference(args, rank, world):
    """The oracle as the reference arm. A step is one bounded sample of the
    workload (see oracle_sample); value is GB/s over the timed samples and
    ms_per_step the measured wall time of one sample step."""
    if rank != 0:
        return None
    w = S.WORKLOADS[WORKLOAD]
    per_step = []
    o = None
    for i in range(args.warmup + args.steps):
        t = time.perf_counter()
        o = oracle_sample(budget_s=1.0)
        o["step_s"] = time.perf_counter() - t
        if i >= args.warmup:
            per_step.append(o)
    att_bytes = sum(p["attend_units"] for p in per_step) * \
        (w.ctx * (w.d * w.bits_k // 8 + w.d * w.bits_v // 8 + 4) + w.gqa * w.d * 4)
    att_s = sum(p["attend_s"] for p in per_step)
    gbs = att_bytes / att_s / 1e9
    step_ms = 1e3 * float(np.mean([p["step_s"] for p in per_step]))
    full_step_bytes = LAYERS * (attend_bytes(w, w.ctx) + encode_bytes(w, w.n_kv_heads))
    return {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(step_ms, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, LAYERS),
        "step": "one bounded sample per step: " + o["sample"] + " (timed wall clock, host cores)",
        "units_timed_per_step": {"attention_units": round(float(np.mean([p["attend_units"] for p in per_step])), 2),
                                 "encode_vectors": 2 * w.ctx},
        "projection_ms_per_full_decode_step": round(full_step_bytes / (gbs * 1e9) * 1e3, 1),
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": o["cores"],
                         "nproc": os.cpu_count(), "kind": "oracle",
                         "sample": "per step: " + o["sample"]},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def profile_case(name, reps):
    """A few eager launches of one kernel's workload for an ncu capture
    (prints no bench line): 'llama' = tq_attend over 8 Llama-3-8B-shaped
    layer caches, 'batched' = one serving-scale call, 'qwen' = tq_attend over
    2 Qwen-14B-shaped layers, 'encode' = tq_encode of 4 bulk-prefill layers,
    'dequant' = tq_dequant (original domain) of one bulk-prefill layer's K,
    'prefill' = tq_prefill_attend of the prefill leg's chunk on one layer.
    Caches hold tq_encode'd seeded data."""
    import torch
    import compressed_decode_attention_b200 as tq
    torch.cuda.set_device(0)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(S.DATA_SEED)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    seed = S.SIGN_SEED
    if name == "encode":
        w = S.WORKLOADS[ENCODE_WORKLOAD]
        caches = LayerCaches(w, 4, None)
        kvs = [device_kv(w, l, w.ctx, gen) for l in range(4)]
        for _ in range(reps):
            for l in range(4):
                tq.tq_encode(kvs[l], tq.TQ_F16, w.ctx, w.n_kv_heads, w.d, w.bits_k, w.bits_v, seed,
                             caches.pk[l], caches.pv[l], caches.nk[l], caches.nv[l], w.cap_tok, 0,
                             status)
        torch.cuda.synchronize()
        return
    if name == "dequant":
        w = S.WORKLOADS[ENCODE_WORKLOAD]
        caches = LayerCaches(w, 1, None)
        kv = device_kv(w, 0, w.ctx, gen)
        tq.tq_encode(kv, tq.TQ_F16, w.ctx, w.n_kv_heads, w.d, w.bits_k, w.bits_v, seed,
                     caches.pk[0], caches.pv[0], caches.nk[0], caches.nv[0], w.cap_tok, 0, status)
        del kv
        out = torch.empty((w.n_kv_heads, w.ctx, w.d), dtype=torch.float32, device="cuda")
        for _ in range(reps):
            tq.tq_dequant(caches.pk[0], caches.nk[0], w.ctx, w.n_kv_heads, w.d, w.bits_k, seed,
                          w.cap_tok, 0, out)
        torch.cuda.synchronize()
        return
    if name == "prefill":
        w = S.WORKLOADS[WORKLOAD]
        ctx, T, H, d = PREFILL_CTX, PREFILL_TOKENS, w.n_kv_heads, w.d
        caches = LayerCaches(dataclasses.replace(w, ctx=ctx, cap_tok=ctx), 1, None)
        kv = device_kv(w, 0, ctx, gen)
        tq.tq_encode(kv, tq.TQ_F16, ctx, H, d, w.bits_k, w.bits_v, seed, caches.pk[0],
                     caches.pv[0], caches.nk[0], caches.nv[0], ctx, 0, status)
        del kv
        q = torch.randn((1, T, w.n_q_heads, d), generator=gen, device="cuda").half()
        out = torch.empty_like(q)
        ctx_dev = torch.full((1,), ctx, dtype=torch.int32, device="cuda")
        splits = tq.tq_prefill_splits(1, T, w.n_q_heads, w.gqa, ctx)
        wsb = tq.tq_prefill_workspace_size(1, T, w.n_q_heads, d, splits)
        ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device="cuda")
        for _ in range(reps):
            tq.tq_prefill_attend_split(q, tq.TQ_F16, caches.pk[0], caches.nk[0], caches.pv[0],
                                       caches.nv[0], ctx_dev, 1, T, w.n_q_heads, w.gqa, d,
                                       w.bits_k, w.bits_v, seed, ctx, splits, ws, wsb, out,
                                       tq.TQ_F16, dev_status=status)
        torch.cuda.synchronize()
        return
    w = S.WORKLOADS[{"llama": WORKLOAD, "batched": BATCHED_WORKLOAD, "qwen": QWEN_WORKLOAD}[name]]
    layers = {"llama": 8, "batched": 1, "qwen": 2}[name]
    ctx_h = S.ctx_lens(w)
    B, H, d, cap = w.batch, w.n_kv_heads, w.d, w.cap_tok
    rk, rv = d * w.bits_k // 8, d * w.bits_v // 8
    kvdt = tq.TQ_BF16 if w.dtype == "bf16" else tq.TQ_F16
    cs = []
    for _ in range(layers):
        pk = torch.zeros((B, H, cap, rk), dtype=torch.uint8, device="cuda")
        pv = torch.zeros((B, H, cap, rv), dtype=torch.uint8, device="cuda")
        nk = torch.zeros((B, H, cap), dtype=torch.int16, device="cuda")
        nv = torch.zeros((B, H, cap), dtype=torch.int16, device="cuda")
        for b in range(B):
            kvb = device_kv(w, 0, int(ctx_h[b]), gen)
            tq.tq_encode(kvb, kvdt, int(ctx_h[b]), H, d, w.bits_k, w.bits_v, seed, pk[b], pv[b],
                         nk[b], nv[b], cap, 0, status)
        cs.append((pk, nk, pv, nv))
    q = torch.randn((B, w.n_q_heads, d), generator=gen, device="cuda")
    q = q.bfloat16() if w.dtype == "bf16" else q.half()
    out = torch.empty_like(q)
    ctx = torch.from_numpy(ctx_h).cuda()
    wsb = tq.tq_attend_workspace_size(B, w.n_q_heads, cap, d)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    for _ in range(reps):
        for pk, nk, pv, nv in cs:
            tq.tq_attend(q, kvdt, pk, nk, pv, nv, ctx, B, w.n_q_heads, w.gqa, d, w.bits_k,
                         w.bits_v, seed, cap, w.tau, 0, ws, wsb, out, kvdt, dev_status=status)
    torch.cuda.synchronize()


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--layers", type=int, default=LAYERS)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", choices=["llama", "batched", "qwen", "encode",
                                                      "dequant", "prefill"],
                    help="only launch one kernel's workload a few times (for ncu captures)")
    args = ap.parse_args(argv)
    if args.profile_case:
        profile_case(args.profile_case, args.steps)
        return 0
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, world, local_rank = dist_env()
    if args.gpus > 1 and world == 1:
        ap.error("--gpus N > 1 runs under torch.distributed.run (one process per GPU)")

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0

    init_dist(world, "nccl")
    res = run_gpu(args, rank, world, local_rank)
    if rank == 0:
        if not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline_both(16.0)
        print(json.dumps(res), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
