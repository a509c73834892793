"""Host-side logic of bench.py: the roofline classification per kernel kind
and the attention kernel's exponential (MUFU) roof."""
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


def test_attention_exponential_roof():
    d = tt_inputs.workload("long")
    inp = {"ctx_len": np.full(d.B, d.L_cap, np.int32)}
    e = bench.attn_exp_per_launch(d, inp)
    # one exponential per (query row, key): B * Hq * S * (L + S); 0.134e9 here
    assert e == d.B * d.Hq * d.S * (d.L_cap + d.S)
    assert abs(e - 0.134e9) < 0.001e9
    ragged = {"ctx_len": np.array([0, 100, 5], np.int32)}
    assert bench.attn_exp_per_launch(d, ragged) == d.Hq * d.S * (0 + 100 + 5 + 3 * d.S)
    r = bench.exp_roof(e, 100e-6, 148, {"sm_mhz": 1500.0})
    peak = 16 * 148 * 1500e6
    assert abs(r["frac"] - round(e / 100e-6 / peak, 4)) < 1e-12
    assert abs(r["peak_T_per_s"] - round(peak / 1e12, 3)) < 1e-12
    assert "median under load" in r["peak_source"]
    for clk in (None, {}, {"sm_mhz": None}):
        r = bench.exp_roof(e, 100e-6, 148, clk)
        assert r["peak_T_per_s"] == round(16 * 148 * 1965e6 / 1e12, 3)
        assert "nominal" in r["peak_source"]


def _reference_line(capsys, monkeypatch, *extra):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "2",
                       "--warmup", "3", *extra]) == 0
    out = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(out) == 1
    import json
    return json.loads(out[0])


def test_reference_arm_prints_the_contract_line(capsys, monkeypatch):
    """The reference arm times the oracle on the host: one JSON line with the
    same metric, unit and config as the GPU arm, its own cpu_baseline and an
    e2e block with no host<->device bytes."""
    j = _reference_line(capsys, monkeypatch)
    assert j["impl"] == "reference" and j["metric"] == "committed tokens/s"
    assert j["unit"] == "tokens/s" and j["higher_is_better"] is True
    assert j["value"] > 0 and j["steps"] == 2 and j["warmup"] == 3 and j["n_gpus"] == 1
    assert j["config"]["workload"].startswith("tiny-block-loop")
    # a sample is the first REF_SAMPLE_STEPS denoise steps of one sequence's
    # block; at unit logit scale each commits one position
    n = bench.REF_SAMPLE_STEPS
    assert abs(j["ms_per_step"] * 1e-3 * j["value"] - n) < 1e-6 * n
    assert j["denoise_steps_per_s"] == j["value"]
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == j["value"] and cb["cores"] >= 1
    assert "1 of 1 sequences" in cb["sample"] and f"first {n} denoise steps" in cb["sample"]
    assert j["e2e"] == {"value": j["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_quietly(capsys, monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")
    assert bench.main(["--impl", "reference", "--gpus", "2", "--workload", "tiny"]) == 0
    assert capsys.readouterr().out == ""


def test_both_roofs_reports_each_view():
    d = tt_inputs.workload("loop64")
    inp = {"ctx_len": np.full(d.B, d.L_cap, np.int32)}
    r = bench.both_roofs("attn", d, inp, [], 16, 100e-6, PEAKS)
    by, fl = bench.per_launch("attn", d, inp, [], 16)
    assert r["hbm"]["bytes_per_launch"] == by[0] and r["tensor"]["flops_per_launch"] == fl[0]
    assert abs(r["hbm"]["achieved_GB_per_s"] - round(by[0] / 100e-6 / 1e9, 1)) < 1e-9
    assert r["hbm"]["frac_of_8TBps"] == round(by[0] / 100e-6 / 1e9 / 8000.0, 4)
    assert r["tensor"]["frac_of_sustained"] == round(fl[0] / 100e-6 / 1e12 / 1361.8, 4)
    ms = [1024 - 64 * k for k in range(16)]
    v = bench.both_roofs("gemm_vocab", d, inp, ms, 16, 450e-6, PEAKS)
    assert v["tensor"]["flops_per_launch"] == sum(2.0 * m * d.V * d.H for m in ms) / 16


def test_clock_sampler_keeps_the_samples_of_the_timed_region():
    """The sampler starts before the warm-up; only samples stamped inside the
    timed region count (the nearest one on each side when it is shorter than
    the sampling period), and throttle reasons are read from those."""
    s = bench.ClockSampler(None)   # no nvidia-smi: fill in stamped lines by hand
    line = "{mhz}, 1965, {w}, Not Active, Not Active, Not Active, {cap}\n"
    s.lines = [(10.0, line.format(mhz=1965, w=300, cap="Not Active")),   # warm-up
               (10.2, line.format(mhz=1500, w=990, cap="Active")),       # timed
               (10.4, line.format(mhz=1520, w=995, cap="Active")),       # timed
               (10.6, line.format(mhz=1965, w=150, cap="Not Active"))]   # after
    s.proc = type("P", (), {"terminate": lambda self: None, "wait": lambda self, timeout=None: 0,
                            "kill": lambda self: None})()
    got = s.stop(10.1, 10.45)
    assert got["samples"] == 2 and got["sm_mhz"] == 1510.0
    assert got["reasons"] == ["sw_power_cap"] and got["sm_max_mhz"] == 1965.0
    # a region between two samples: the samples on either side
    got = s.stop(10.25, 10.3)
    assert got["samples"] == 2 and got["sm_mhz"] == 1510.0
