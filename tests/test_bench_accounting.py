"""The algorithmic bytes and FLOPs behind bench.py's roofline figures (CPU).

The per-position figures are the byte accounting of the packed cache
("We Built a Python Library That Cuts LLM Memory Usage by 80%", section
"Compression numbers": 100 bytes per token and kv head at K4/V2 against 512
for fp16 K and V); the totals are written out here from the workload
shapes, independently of the functions under test.
"""
import bench
import synthetic as S


def test_decode_layer_bytes():
    w = S.WORKLOADS["llama3_8b_decode"]
    # 8 kv heads x 32768 positions x (64 + 32 + 2 + 2) bytes, plus the fp16
    # query and output of 32 heads x 128
    assert bench.attend_bytes(w, 32768) == 8 * 32768 * 100 + 32 * 128 * 2 * 2
    assert bench.attend_bytes(w, 32768) == 26_230_784


def test_long_context_layer_bytes():
    w = S.WORKLOADS["qwen14b_decode"]
    # K3/V2: 48 + 32 + 4 = 84 bytes per position and kv head
    assert bench.attend_bytes(w, 131072) == 8 * 131072 * 84 + 40 * 128 * 4


def test_serving_bytes_per_position():
    w = S.WORKLOADS["batched_serving"]
    # K4/V3: 64 + 48 + 4 = 116 bytes per position and kv head
    ctx_total = 1000
    assert bench.attend_bytes(w, ctx_total) == ctx_total * 8 * 116 + 64 * 32 * 128 * 4


def test_encode_bytes():
    w = S.WORKLOADS["llama3_8b_decode"]
    # fp16 K and V in (2 x 256 bytes), packed rows and norms out (100 bytes)
    assert bench.encode_bytes(w, 1) == 612
    assert bench.encode_bytes(w, 32768 * 8) == 160_432_128


def test_prefill_flops():
    w = S.WORKLOADS["llama3_8b_decode"]
    ctx, T = 8192, 1024
    # token i of the chunk sees ctx - T + i + 1 positions: sum over i is
    # T·(ctx - T) + T·(T + 1)/2; 4·d FLOPs per (token, head, position)
    visible = T * (ctx - T) + T * (T + 1) // 2
    assert bench.prefill_flops(w, ctx, T) == 4 * 128 * 32 * visible
    assert bench.prefill_flops(w, ctx, T) == 128_857_407_488
