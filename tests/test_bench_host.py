"""Host-side logic of bench.py: the roofline classification per kernel kind."""
import numpy as np

import bench
import tt_inputs

PEAKS = {"hbm_gbs": 6531.3, "bf16_tflops": 1632.8, "bf16_tflops_sustained": 1361.8}


def test_vocab_gemm_bound_follows_rows():
    d = tt_inputs.workload("mid")
    inp = {"ctx_len": np.full(d.B, d.L_cap, np.int32)}
    b, per, unit, t = bench.algorithmic("gemm_vocab", d, inp, [128] * 16, 16, PEAKS)
    assert b == "hbm" and unit == "GB/s"
    assert per == d.V * d.H * 2 + 128 * (d.H * 2 + (-(-d.V // 224)) * 16)
    assert abs(t - 16 * per / (PEAKS["hbm_gbs"] * 1e9)) < 1e-12
    b, per, unit, t = bench.algorithmic("gemm_vocab", d, inp, [1024] * 4, 4, PEAKS)
    assert b == "tensor" and unit == "TFLOP/s" and per == 2.0 * 1024 * d.V * d.H


def test_vocab_roofline_time_sums_each_launch_floor():
    d = tt_inputs.workload("loop64")
    inp = {"ctx_len": np.full(d.B, d.L_cap, np.int32)}
    ms = [1024 - 64 * k for k in range(16)]
    _, _, _, t = bench.algorithmic("gemm_vocab", d, inp, ms, 16, PEAKS)
    floors = [max((d.V * d.H * 2 + m * (d.H * 2 + (-(-d.V // 224)) * 16)) / 6531.3e9,
                  2.0 * m * d.V * d.H / 1361.8e12) for m in ms]
    assert abs(t - sum(floors)) < 1e-12


def test_attention_counts_context_and_block_bytes_and_flops():
    d = tt_inputs.workload("long")
    inp = {"ctx_len": np.full(d.B, d.L_cap, np.int32)}
    b, per, unit, t = bench.algorithmic("attn", d, inp, [], 1, PEAKS)
    kv = 2 * d.Hkv * d.dh * 2 * d.B * d.L_cap
    flops = 4.0 * d.S * d.Hq * d.dh * d.B * (d.L_cap + d.S)
    blk = d.B * d.S * (d.Hq + 2 * d.Hkv) * d.dh * 2 + d.B * d.S * d.H * 2
    assert abs(t - max((kv + blk) / 6531.3e9, flops / 1361.8e12)) < 1e-12
    # at S = 16, G = 16 the kernel sits at the ridge; against the sustained
    # tensor peak the FLOPs dominate
    assert b == "tensor" and per == flops
    assert bench.algorithmic("commit", d, inp, [], 1, PEAKS)[0] is None
