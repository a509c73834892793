#!/usr/bin/env python
"""Benchmark of the block-wise diffusion denoise loop on B200.

One step = one tt_denoise_block_loop call: a block of S masked positions per
sequence is refined (re-embed + linear update -> block-denoise attention ->
adaLN -> vocab GEMM with fused confidence -> commit) until every position is
committed.  Default workload: the full block loop of 64 sequences, 32 query /
2 KV heads (GQA 16), d_head 128, hidden 4096, context 8192, S = 16,
V = 131072, gamma 0.8, unit logit scale; synthetic seeded inputs resident in
HBM (``--workload`` picks the other shapes).

Metric: committed tokens/s (whole job), with denoise steps/s alongside.
Timing: CUDA events on the library's stream around each call, an L2 flush
(256 MiB write) between calls outside the events, max over ranks.
`--impl reference` times the float64 CPU oracle on a bounded sample instead.
`--stage attn|vocab|blocks` times one other entry point on its own (for
profilers; prints a plain line, not the benchmark record).

Launch: python bench.py [--gpus N --steps K --warmup W].  N > 1 runs one
independent replica per GPU (weak scaling); under torch.distributed.run each
process is one rank, and without a launcher bench.py starts N ranks itself.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import tt_inputs  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")
KERNEL_SOURCES = {
    "gemm_vocab": ["tt_gemm.cu", "tt_ptx.cuh", "tt_internal.h"],
    "gemm_qkv": ["tt_gemm.cu", "tt_ptx.cuh", "tt_internal.h"],
    "attn": ["tt_attn.cu", "tt_ptx.cuh", "tt_internal.h"],
}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="loop64", choices=sorted(tt_inputs.WORKLOADS))
    p.add_argument("--stage", default="loop", choices=["loop", "attn", "vocab", "blocks"],
                   help="loop: the benchmark; attn / vocab / blocks: time one entry point "
                        "alone (tt_block_denoise_attn, tt_vocab_confidence_commit with every "
                        "position masked, tt_decode_blocks) for profilers")
    p.add_argument("--B", type=int, default=None, help="--stage runs: override the batch")
    p.add_argument("--V", type=int, default=None, help="--stage runs: override the vocabulary")
    p.add_argument("--calls", type=int, default=2, help="--stage runs: timed calls")
    p.add_argument("--n-blocks", type=int, default=4, help="--stage blocks: blocks per call")
    p.add_argument("--gamma", type=float, default=0.8)
    p.add_argument("--logit-scale", type=float, default=1.0)
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--n-layers", type=int, default=1,
                   help="denoiser layers per step (each with its own context KV)")
    a = p.parse_args(argv)
    if a.warmup < 3:
        p.error("--warmup must be >= 3")
    return a


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_seed(seed: int, rank: int) -> int:
    """Each replica draws its own batch (independent sequences)."""
    return seed + 1000 * rank


def reduce_max(x: float, world: int, device=None) -> float:
    """Max of a host float over all ranks (identity for one rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def workload_config(d, args, world):
    return {
        "workload": (f"{args.workload}-block-loop: B={d.B} S={d.S} Hq={d.Hq} Hkv={d.Hkv} "
                     f"dh={d.dh} H={d.H} V={d.V} ctx={d.ctx} gamma={args.gamma} "
                     f"logit_scale={args.logit_scale}"
                     + (f" layers={args.n_layers}" if args.n_layers > 1 else "")),
        "global_batch": d.B * world,
        "seq_len": d.L_cap,
        "block_size": d.S,
        "l2": "flushed between timed steps (256 MiB write, outside the events)",
        "parallelism": "replicas" if world == 1 else f"dp{world} independent replicas",
    }


# ------------------------------------------------------------------ peaks
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return {k: float(pk[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def source_sha(kind: str) -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES.get(kind, []):
        with open(os.path.join(ROOT, "block_wise_diffusion_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def committed_traffic(kind: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if still current."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
        e = t[kind]
        if e.get("src_sha") == source_sha(kind) and e.get("workload") == workload:
            return float(e["bytes_per_launch"])
    except Exception:
        pass
    return None


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling SM clocks, power and throttle reasons every 200 ms.

    nvidia-smi's start-up (NVML initialisation) competes with kernel launches
    for the driver for up to a second, so the sampler is started and waited
    for (first sample seen) before the warm-up; a reader thread stamps each
    sample with the host clock on arrival, and window(t0, t1) keeps those
    taken during the timed region (the nearest one on each side when the
    region is shorter than the sampling period)."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.proc = None
        self.lines = []
        self.thread = None
        if gpu_id is None:
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        import threading

        def read():
            for line in self.proc.stdout:
                self.lines.append((time.time(), line))
        self.thread = threading.Thread(target=read, daemon=True)
        self.thread.start()

    def wait_ready(self, timeout_s: float = 10.0):
        t_end = time.time() + timeout_s
        while self.proc is not None and not self.lines and time.time() < t_end:
            time.sleep(0.05)

    def stop(self, t0: float | None = None, t1: float | None = None):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)
        stamped = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 7:
                continue
            try:
                stamped.append((ts, (float(parts[0]), float(parts[1]), float(parts[2]), parts[3:])))
            except ValueError:
                continue
        if t0 is not None and t1 is not None and stamped:
            inside = [r for ts, r in stamped if t0 <= ts <= t1 + 0.05]
            if not inside:  # region shorter than the period: the samples around it
                before = [r for ts, r in stamped if ts < t0][-1:]
                after = [r for ts, r in stamped if ts > t1][:1]
                inside = before + after
            rows = inside
        else:
            rows = [r for _, r in stamped]
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v == "Active"})
        loaded = [r for r in rows if r[2] > 200.0] or rows
        return {"sm_mhz": statistics.median(r[0] for r in loaded),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


def gpu_uuid(torch, idx):
    try:
        u = str(torch.cuda.get_device_properties(idx).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return None


# -------------------------------------------------------- CPU oracle arm
def sample_inputs(inp, bsel):
    """The loop inputs restricted to the sequences ``bsel``."""
    one = dict(inp)
    for k in ("k_ctx", "v_ctx", "ctx_len", "tokens", "masked"):
        one[k] = inp[k][bsel]
    for k in ("k_ctx_l", "v_ctx_l"):
        if k in inp:
            one[k] = inp[k][:, bsel]
    return one


def oracle_sample(d, inp, gamma, logit_scale, n_seq=1, max_steps=None):
    """Run the oracle's block loop on the first n_seq sequences of the workload
    (all its steps, or the first max_steps): a bounded sample.  Returns
    (seconds, committed positions, steps, n_seq)."""
    from oracle import twotower_oracle as O
    n_seq = min(n_seq, d.B)
    one = sample_inputs(inp, slice(0, n_seq))
    t0 = time.perf_counter()
    r = O.denoise_block_loop(one, gamma, logit_scale, max_steps=max_steps)
    dt = time.perf_counter() - t0
    committed = int((one["masked"].astype(bool) & ~r["masked"]).sum())
    return dt, committed, len(r["trace"]), n_seq


def oracle_check(d, inp, gamma, logit_scale, g_tokens, g_commit_step, bsel):
    """The CPU-baseline leg: the oracle's block loop on the sequences ``bsel``,
    teacher-forced on the GPU's trajectory of the timed call, timed on the
    host cores; its comparison with the GPU's committed tokens gives the
    parity counts (oracle.parity.compare_loop: compared and excluded
    sequence-steps, literal-rule exclusions, near-tie top-2 flips,
    disagreements outside the exclusions).  Returns (seconds, committed
    positions, counts)."""
    from oracle import parity as P
    one = sample_inputs(inp, bsel)
    t0 = time.perf_counter()
    cnt, problems = P.compare_loop(one, g_tokens[bsel], g_commit_step[bsel], gamma, logit_scale)
    dt = time.perf_counter() - t0
    cnt["mismatches"] = len(problems)
    if problems:
        log("parity: " + "; ".join(problems[:5]))
    return dt, int(one["masked"].sum()), cnt


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


# denoise steps of one sequence's block that one reference-arm step runs
# (the whole block when it has at most this many), so that the driver's
# --steps 20 --warmup 5 run stays within a few minutes at the large shapes
REF_SAMPLE_STEPS = 4


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    d = tt_inputs.workload(args.workload)
    inp = tt_inputs.generate(d, seed=rank_seed(args.seed, 0), n_layers=args.n_layers)
    times, tokens, steps = [], 0, 0
    for i in range(args.warmup + args.steps):
        dt, c, s, _ = oracle_sample(d, inp, args.gamma, args.logit_scale, n_seq=1,
                                    max_steps=REF_SAMPLE_STEPS)
        if i >= args.warmup:
            times.append(dt)
            tokens += c
            steps += s
    total = sum(times)
    value = tokens / total
    sample = (f"1 of {d.B} sequences of the workload per step, the first "
              f"{steps // max(1, args.steps)} denoise steps of its block "
              f"({tokens // max(1, args.steps)} committed positions), float64 NumPy oracle")
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": "committed tokens/s", "value": value,
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": workload_config(d, args, 1),
        "denoise_steps_per_s": steps / total,
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------ GPU arm
def per_launch(kind, d, inp, m_per_launch, launches):
    """Algorithmic bytes and FLOPs of each launch of a kernel kind (lists), or
    (None, None) for a kind without a roofline model.  ``m_per_launch`` lists
    the vocabulary GEMM's rows per launch (the still-masked positions of each
    step)."""
    if kind == "gemm_vocab":
        n_vt = -(-d.V // 224)
        ms = list(m_per_launch)[:launches] or [0]
        by = [d.V * d.H * 2 + m * (d.H * 2 + n_vt * 16) for m in ms]
        fl = [2.0 * m * d.V * d.H for m in ms]
    elif kind == "attn":
        L = np.asarray(inp["ctx_len"], dtype=np.float64)
        kv = 2 * d.Hkv * d.dh * 2 * float(L.sum())
        blk = d.B * d.S * (d.Hq + 2 * d.Hkv) * d.dh * 2 + d.B * d.S * d.H * 2
        by = [kv + blk] * launches
        fl = [4.0 * d.S * d.Hq * d.dh * float((L + d.S).sum())] * launches
    elif kind == "gemm_qkv":
        n_qkv = d.H + 2 * d.Hkv * d.dh
        by = [n_qkv * d.H * 2 + d.B * d.S * (d.H + n_qkv) * 2] * launches
        fl = [2.0 * d.B * d.S * d.H * n_qkv] * launches
    else:
        return None, None
    return by, fl


def algorithmic(kind, d, inp, m_per_launch, launches, peaks):
    """(bound, algorithmic bytes or FLOPs per launch, unit, roofline time s) of a
    kernel kind over its launches.

    Each launch has algorithmic bytes and FLOPs; its floor is the larger of
    bytes / HBM peak and FLOPs / sustained bf16 peak.  The bound reported is
    the one whose floors dominate the sum over launches (the vocabulary GEMM
    is HBM-bound at a few hundred rows and tensor-bound above; attention sits
    at the ridge).
    """
    by, fl = per_launch(kind, d, inp, m_per_launch, launches)
    if by is None:
        return None, None, None, None
    hbm = peaks["hbm_gbs"] * 1e9
    tc = peaks["bf16_tflops_sustained"] * 1e12
    t_h = sum(b / hbm for b in by)
    t_t = sum(f / tc for f in fl)
    t_roof = sum(max(b / hbm, f / tc) for b, f in zip(by, fl))
    if t_t > t_h:
        return "tensor", sum(fl) / len(fl), "TFLOP/s", t_roof
    return "hbm", sum(by) / len(by), "GB/s", t_roof


# ex2.approx retires 16 results per clock per SM on B200 in its f32, f16x2 and
# bf16x2 forms alike (micro-benchmarked: one 1024-thread CTA per SM, eight
# independent chains per thread).
MUFU_EX2_PER_CLK_SM = 16
NOMINAL_MAX_SM_MHZ = 1965.0


SPEC_HBM_GBS = 8000.0  # the B200 spec sheet's ~8 TB/s, for context beside the measured copy


def both_roofs(kind, d, inp, m_per_launch, launches, avg_s, peaks):
    """A kernel's standing against both roofs, whichever bounds it: achieved
    HBM GB/s (algorithmic bytes per launch / time) against the measured copy
    bandwidth and against the spec sheet's 8 TB/s, and achieved TFLOP/s
    against the sustained and burst dense-bf16 peaks (the tensor-pipe share
    the algorithmic FLOPs need)."""
    bl, fll = per_launch(kind, d, inp, m_per_launch, launches)
    by, fl = sum(bl) / len(bl), sum(fll) / len(fll)
    gbs = by / avg_s / 1e9
    tfs = fl / avg_s / 1e12
    return {"hbm": {"achieved_GB_per_s": round(gbs, 1), "bytes_per_launch": by,
                    "frac_of_measured": round(gbs / peaks["hbm_gbs"], 4),
                    "frac_of_8TBps": round(gbs / SPEC_HBM_GBS, 4)},
            "tensor": {"achieved_TFLOP_per_s": round(tfs, 1), "flops_per_launch": fl,
                       "frac_of_sustained": round(tfs / peaks["bf16_tflops_sustained"], 4),
                       "frac_of_burst": round(tfs / peaks["bf16_tflops"], 4)}}


def attn_exp_per_launch(d, inp):
    """Exponentials one attention launch must evaluate: one per (query row,
    key), i.e. sum over b of Hq * S * (L_b + S)."""
    L = np.asarray(inp["ctx_len"], dtype=np.float64)
    return float(d.Hq * d.S * (L + d.S).sum())


def exp_roof(exps, avg_s, n_sm, clk):
    """The attention kernel's third roof: exponentials per second against the
    MUFU rate at the SM clock sampled under load (the nominal maximum clock
    when no sample was taken)."""
    mhz = float(clk["sm_mhz"]) if clk and clk.get("sm_mhz") else NOMINAL_MAX_SM_MHZ
    peak = MUFU_EX2_PER_CLK_SM * n_sm * mhz * 1e6
    ach = exps / avg_s
    return {"per_launch": exps, "achieved_T_per_s": round(ach / 1e12, 3),
            "peak_T_per_s": round(peak / 1e12, 3), "frac": round(ach / peak, 4),
            "peak_source": f"{MUFU_EX2_PER_CLK_SM} ex2/clk/SM x {n_sm} SMs x {mhz:.0f} MHz "
                           + ("(median under load)" if clk and clk.get("sm_mhz") else
                              "(nominal max clock)")}


def run_ours(args, rank, world, local):
    import torch
    import block_wise_diffusion_b200 as tt

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
    tt.lib()
    d = tt_inputs.workload(args.workload)
    D = tt.dims(d)
    t0 = time.time()
    nl = args.n_layers
    inp = tt_inputs.generate(d, seed=rank_seed(args.seed, rank), n_layers=nl)
    log(f"[rank {rank}] inputs generated in {time.time() - t0:.1f}s")

    def bf(k):
        return torch.from_numpy(inp[k].view(np.int16)).to(dev).view(torch.bfloat16)

    names = ["k_ctx", "v_ctx", "emb", "e_mask", "u_t", "shift_scale", "w"]
    # with several layers the per-layer tensors are the stacked ones
    X = {k: bf(k + "_l" if nl > 1 and k in tt_inputs.LAYER_NAMES else k) for k in names}
    ctx_len = torch.from_numpy(inp["ctx_len"]).to(dev)
    tokens0 = torch.from_numpy(inp["tokens"]).to(dev)
    masked0 = torch.from_numpy(inp["masked"]).to(dev)
    tokens, masked = tokens0.clone(), masked0.clone()
    steps_taken = torch.empty(d.B, dtype=torch.int32, device=dev)
    commit_step = torch.empty((d.B, d.S), dtype=torch.int32, device=dev)
    ws = tt.workspace(D, tt.TT_WS_LOOP, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    n_masked0 = int(inp["masked"].sum())

    def call(kc=None, vc=None, cl=None, tk=None, mk=None):
        a = (kc if kc is not None else X["k_ctx"], vc if vc is not None else X["v_ctx"],
             cl if cl is not None else ctx_len, X["emb"], X["e_mask"], X["u_t"],
             X["shift_scale"], X["w"], args.gamma, args.logit_scale, d.S,
             tk if tk is not None else tokens, mk if mk is not None else masked,
             steps_taken, commit_step, ws, stream)
        if nl > 1:
            return tt.tt_denoise_block_loop_layers(D, nl, *a)
        return tt.tt_denoise_block_loop(D, *a)

    def reset():
        tokens.copy_(tokens0)
        masked.copy_(masked0)
        flush.zero_()

    # the clock sampler runs from before the warm-up (see ClockSampler)
    clocks = ClockSampler(gpu_uuid(torch, local))
    clocks.wait_ready()

    # warm-up
    for _ in range(args.warmup):
        reset()
        call()
    torch.cuda.synchronize(dev)

    # timed region
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    launches0 = tt.tt_launch_count()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    denoise_steps = 0
    for i in range(args.steps):
        reset()
        ev[i][0].record(stream)
        denoise_steps += call()
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    gpu_launches = tt.tt_launch_count() - launches0
    t_wall1 = time.time()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    clk = clocks.stop(t_wall0, t_wall1)
    ms_local = sum(a.elapsed_time(b) for a, b in ev)
    assert not masked.any().item(), "block not committed"
    ms = reduce_max(ms_local, world, dev)
    tokens_all = reduce_sum(float(n_masked0 * args.steps), world, dev)
    steps_all = reduce_sum(float(denoise_steps), world, dev)
    value = tokens_all / (ms / 1e3)

    # End to end through the public API with host buffers: every step copies
    # its block's inputs (context K/V, lengths, tokens, mask) from pinned host
    # memory and reads its results back (weights stay resident).  The copies
    # are pipelined as a server would: step i+1's inputs go up on a copy
    # stream into the other of two device buffer sets while step i computes.
    # The timed region runs from the first copy to the last result read.
    h_in = {"k_ctx": X["k_ctx"].cpu().pin_memory(), "v_ctx": X["v_ctx"].cpu().pin_memory(),
            "ctx_len": ctx_len.cpu().pin_memory(), "tokens": tokens0.cpu().pin_memory(),
            "masked": masked0.cpu().pin_memory()}
    h_out = {"tokens": torch.empty_like(tokens0, device="cpu").pin_memory(),
             "masked": torch.empty_like(masked0, device="cpu").pin_memory(),
             "steps_taken": torch.empty_like(steps_taken, device="cpu").pin_memory(),
             "commit_step": torch.empty_like(commit_step, device="cpu").pin_memory()}
    d_in = [{k: torch.empty_like(v, device=dev) for k, v in h_in.items()} for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in h_in.values())
    d2h = sum(v.numel() * v.element_size() for v in h_out.values())
    copy_stream = torch.cuda.Stream(dev)
    ready = [torch.cuda.Event() for _ in range(2)]     # a buffer set's inputs are up
    free = [torch.cuda.Event() for _ in range(2)]      # a buffer set's step is done

    def upload(i):
        buf = d_in[i % 2]
        copy_stream.wait_event(free[i % 2])            # step i - 2 is done with it
        with torch.cuda.stream(copy_stream):
            for k in h_in:
                buf[k].copy_(h_in[k], non_blocking=True)
        ready[i % 2].record(copy_stream)

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(copy_stream)
    upload(0)
    for i in range(args.steps):
        if i + 1 < args.steps:
            upload(i + 1)
        buf = d_in[i % 2]
        stream.wait_event(ready[i % 2])
        call(buf["k_ctx"], buf["v_ctx"], buf["ctx_len"], buf["tokens"], buf["masked"])
        h_out["tokens"].copy_(buf["tokens"], non_blocking=True)
        h_out["masked"].copy_(buf["masked"], non_blocking=True)
        h_out["steps_taken"].copy_(steps_taken, non_blocking=True)
        h_out["commit_step"].copy_(commit_step, non_blocking=True)
        free[i % 2].record(stream)
    e_end.record(stream)
    e_end.synchronize()
    e2e_ms = e_start.elapsed_time(e_end)
    assert not h_out["masked"].any().item()
    e2e_ms = reduce_max(e2e_ms, world, dev)
    e2e_value = tokens_all / (e2e_ms / 1e3)

    # per-kernel profile (one extra call, outside the timed region)
    reset()
    tt.tt_profile_enable(True)
    call()
    table = tt.profile_table()
    tt.tt_profile_enable(False)
    cs = commit_step.cpu().numpy()
    m0 = inp["masked"].astype(bool)
    # rows of the vocabulary GEMM at step k: positions still masked at its start
    m_per_step = [int((m0 & (cs >= k)).sum()) for k in range(int(cs.max()) + 1)]
    peaks, peak_src = load_peaks()
    n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
    kernels = {}
    for kind, (kms, n) in sorted(table.items(), key=lambda kv: -kv[1][0]):
        e = {"launches": n, "total_ms": round(kms, 4), "avg_us": round(1e3 * kms / n, 2)}
        bound, per, unit, t_roof = algorithmic(kind, d, inp, m_per_step, n, peaks)
        if bound is not None:
            ach = per / (kms / n / 1e3) / (1e9 if unit == "GB/s" else 1e12)
            pk = peaks["hbm_gbs"] if bound == "hbm" else peaks["bf16_tflops_sustained"]
            e.update(bound=bound, achieved=round(ach, 2), unit=unit, frac=round(ach / pk, 4),
                     roofline_time_frac=round(t_roof / (kms / 1e3), 4))
        if kind == "attn":
            e["exp"] = exp_roof(attn_exp_per_launch(d, inp), kms / n / 1e3, n_sm, clk)
            # the loop keeps a context cache of at most 48 MiB in L2 across
            # its steps (evict-last), so the HBM figure then counts bytes that
            # L2 mostly serves
            kv_bytes = 2.0 * d.B * d.Hkv * d.L_cap * d.dh * 2
            e["kv_l2_resident"] = bool(kv_bytes <= 48.0 * (1 << 20))
        kernels[kind] = e
    for kind in ("attn", "gemm_vocab"):
        if kind in kernels:
            kms, n = table[kind]
            kernels[kind].update(both_roofs(kind, d, inp, m_per_step, n, kms / n / 1e3, peaks))
    dom = max(table, key=lambda k: table[k][0])
    bound, per, unit, t_roof = algorithmic(dom, d, inp, m_per_step, table[dom][1], peaks)
    roofline = None
    if bound is not None:
        avg_s = table[dom][0] / table[dom][1] / 1e3
        ach = per / avg_s / (1e9 if unit == "GB/s" else 1e12)
        pk = peaks["hbm_gbs"] if bound == "hbm" else peaks["bf16_tflops_sustained"]
        roofline = {"kernel": dom, "bound": bound, "achieved": round(ach, 2), "peak": pk,
                    "unit": unit, "frac": round(ach / pk, 4),
                    "traffic": committed_traffic(dom, args.workload),
                    "peak_source": f"{peak_src} ({'hbm_gbs' if bound == 'hbm' else 'bf16_tflops_sustained'})",
                    "algorithmic_per_launch": per,
                    "roofline_time_frac": round(t_roof / (table[dom][0] / 1e3), 4)}

    cpu = parity = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the first and the last sequence of the timed batch (its last call)
        bsel = np.array(sorted({0, d.B - 1}))
        dt, c, cnt = oracle_check(d, inp, args.gamma, args.logit_scale,
                                  tokens.cpu().numpy(), commit_step.cpu().numpy(), bsel)
        cpu = {"value": c / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"sequences {bsel.tolist()} of {d.B}, full block loop ({dt:.1f} s), "
                         "float64 NumPy oracle, teacher-forced on the timed call's trajectory"}
        parity = dict(cnt, sample=f"sequences {bsel.tolist()} of the last timed call, end to end "
                                  "against the float64 oracle; exclusions as oracle/parity.py")

    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": "committed tokens/s", "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1)/sqrt(fan-in), bf16)",
        "config": workload_config(d, args, world),
        "denoise_steps_per_s": steps_all / (ms / 1e3),
        "gpu_launches": gpu_launches,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "note": "every step's inputs copied from pinned host memory and results read "
                        "back; the next step's copy overlaps this step's compute (copy stream, "
                        "two device buffer sets)"},
        "roofline": roofline,
        "kernels": kernels,
        "cpu_baseline": cpu,
        "parity": parity,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------- single-stage runs
def _dev_bf16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def stage_attn(d):
    """(call, check) for tt_block_denoise_attn on seeded inputs."""
    import torch
    import block_wise_diffusion_b200 as tt
    inp = tt_inputs.generate(d, seed=0, names=["q_blk", "k_blk", "v_blk", "k_ctx", "v_ctx"])
    q, kb, vb, kc, vc = (_dev_bf16(inp[k]) for k in ("q_blk", "k_blk", "v_blk", "k_ctx", "v_ctx"))
    cl = torch.from_numpy(inp["ctx_len"]).cuda()
    D = tt.dims(d)
    out = torch.empty((d.B, d.S, d.Hq, d.dh), dtype=torch.bfloat16, device="cuda")
    ws = tt.workspace(D, tt.TT_WS_ATTN)

    def call():
        tt.tt_block_denoise_attn(D, q, kb, vb, kc, vc, cl, out, ws)

    return call, lambda: tt.tt_device_status(ws)


def stage_vocab(d):
    """(call, check) for tt_vocab_confidence_commit with every position masked
    (all B*S rows go through the GEMM)."""
    import torch
    import block_wise_diffusion_b200 as tt
    inp = tt_inputs.generate(d, seed=0, names=["w"])
    rng = np.random.default_rng(0)
    y = _dev_bf16(tt_inputs.bf16_bits(rng.standard_normal((d.B * d.S, d.H)).astype(np.float32)))
    w = _dev_bf16(inp["w"])
    D = tt.dims(d)
    ws = tt.workspace(D, tt.TT_WS_VOCAB)
    tok = torch.full((d.B, d.S), -1, dtype=torch.int32, device="cuda")
    msk0 = torch.ones((d.B, d.S), dtype=torch.uint8, device="cuda")
    msk = msk0.clone()
    conf = torch.empty((d.B, d.S), dtype=torch.float32, device="cuda")
    am = torch.empty((d.B, d.S), dtype=torch.int32, device="cuda")
    nc = torch.empty((d.B,), dtype=torch.int32, device="cuda")

    def call():
        msk.copy_(msk0)  # the call commits positions: start every call fully masked
        tt.tt_vocab_confidence_commit(D, y, w, 0.8, 1.0, tok, msk, conf, am, nc, ws)

    return call, lambda: tt.tt_device_status(ws)


def stage_blocks(d, n_blocks, logit_scale):
    """(call, check) for tt_decode_blocks over n_blocks blocks (the context is
    reset before each call)."""
    import torch
    import block_wise_diffusion_b200 as tt
    inp = tt_inputs.generate(d, seed=0)
    kc0, vc0 = _dev_bf16(inp["k_ctx"]), _dev_bf16(inp["v_ctx"])
    kc, vc = kc0.clone(), vc0.clone()
    cl0 = torch.from_numpy(inp["ctx_len"]).cuda()
    cl = cl0.clone()
    X = {k: _dev_bf16(inp[k]) for k in ("emb", "e_mask", "u_t", "shift_scale", "w", "u_ctx")}
    D = tt.dims(d)
    tok = torch.empty((n_blocks, d.B, d.S), dtype=torch.int32, device="cuda")
    steps = torch.empty((n_blocks, d.B), dtype=torch.int32, device="cuda")
    cs = torch.empty((n_blocks, d.B, d.S), dtype=torch.int32, device="cuda")
    ws = tt.workspace(D, tt.TT_WS_LOOP)

    def call():
        kc.copy_(kc0)
        vc.copy_(vc0)
        cl.copy_(cl0)
        tt.tt_decode_blocks(D, n_blocks, kc, vc, cl, X["emb"], X["e_mask"], X["u_t"],
                            X["shift_scale"], X["w"], X["u_ctx"], 0.8, logit_scale, tok, steps,
                            cs, ws)

    return call, lambda: tt.tt_device_status(ws)


def run_stage(args) -> int:
    """One entry point on its own: a warm-up call, then --calls calls timed
    together with CUDA events (no L2 flush), then the device status word."""
    import dataclasses
    import torch
    import block_wise_diffusion_b200 as tt
    tt.lib()
    over = {k: v for k, v in (("B", args.B), ("V", args.V)) if v is not None}
    d = tt_inputs.workload(args.workload, **over)
    if args.stage == "blocks":
        d = dataclasses.replace(d, L_cap=d.L_cap + args.n_blocks * d.S)  # room for the blocks
        call, check = stage_blocks(d, args.n_blocks, args.logit_scale)
    else:
        call, check = (stage_attn if args.stage == "attn" else stage_vocab)(d)
    call()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record()
    for _ in range(args.calls):
        call()
    ev[1].record()
    torch.cuda.synchronize()
    if check() != 0:
        raise RuntimeError("device reported an error")
    us = ev[0].elapsed_time(ev[1]) * 1e3 / args.calls
    msg = f"ok {args.stage} {d}: {us:.1f} us per call (mean of {args.calls}, no L2 flush)"
    if args.stage == "blocks":
        msg += f", {args.n_blocks * d.B * d.S / (us * 1e-6):.0f} committed tokens/s"
    print(msg, flush=True)
    return 0


# ----------------------------------------------------------------- launch
def free_port() -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def spawn_ranks(n: int, argv) -> int:
    """Run this script as n local ranks under torch.distributed.run (one per
    GPU, rendezvous on 127.0.0.1) and return its exit status; rank 0 prints
    the record."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr=127.0.0.1", f"--master-port={free_port()}",
           os.path.abspath(__file__), *argv]
    log("launching: " + " ".join(cmd))
    return subprocess.call(cmd)


def main(argv=None):
    argv = list(sys.argv[1:] if argv is None else argv)
    args = parse_args(argv)
    rank, world, local = dist_env()
    if args.stage != "loop":
        return run_stage(args)
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # no launcher: start the ranks here rather than run one replica
        if args.impl == "ours":
            import torch
            n = torch.cuda.device_count()
            if n < args.gpus:
                log(f"error: --gpus {args.gpus} but this host has {n} visible GPU(s)")
                return 2
        return spawn_ranks(args.gpus, argv)
    if world > 1 and args.gpus != world:
        log(f"error: --gpus {args.gpus} but WORLD_SIZE={world}")
        return 2
    if args.impl == "reference":
        return run_reference(args, rank, world)
    return run_ours(args, rank, world, local)


if __name__ == "__main__":
    sys.exit(main())
