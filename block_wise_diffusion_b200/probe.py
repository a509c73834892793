"""Run one library entry point a few times on seeded synthetic inputs.

For profilers (ncu) and quick timing of a single stage outside the block loop:

    python -m block_wise_diffusion_b200.probe attn --workload long --B 2
    python -m block_wise_diffusion_b200.probe vocab --workload mid --V 65536

The entry point runs once, then ``--calls`` more times on the current stream
(``--time`` reports their mean with CUDA events), then the device status word
is checked.  Inputs come from ``tt_inputs`` (the same seeded
generator the tests and the benchmark use); nothing here computes a reference.
"""
from __future__ import annotations

import argparse
import dataclasses
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _dev(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def setup_attn(d):
    """Upload seeded inputs; return (call, check) for tt_block_denoise_attn."""
    import torch
    import tt_inputs
    import block_wise_diffusion_b200 as tt
    inp = tt_inputs.generate(d, seed=0, names=["q_blk", "k_blk", "v_blk", "k_ctx", "v_ctx"])
    q, kb, vb, kc, vc = (_dev(inp[k]) for k in ("q_blk", "k_blk", "v_blk", "k_ctx", "v_ctx"))
    cl = torch.from_numpy(inp["ctx_len"]).cuda()
    D = tt.dims(d)
    out = torch.empty((d.B, d.S, d.Hq, d.dh), dtype=torch.bfloat16, device="cuda")
    ws = tt.workspace(D, tt.TT_WS_ATTN)

    def call():
        tt.tt_block_denoise_attn(D, q, kb, vb, kc, vc, cl, out, ws)

    return call, lambda: tt.tt_device_status(ws)


def setup_vocab(d):
    """Upload seeded inputs; return (call, check) for tt_vocab_confidence_commit
    with every position masked (all B*S rows go through the GEMM)."""
    import torch
    import tt_inputs
    import block_wise_diffusion_b200 as tt
    inp = tt_inputs.generate(d, seed=0, names=["w"])
    rng = np.random.default_rng(0)
    y = _dev(tt_inputs.bf16_bits(rng.standard_normal((d.B * d.S, d.H)).astype(np.float32)))
    w = _dev(inp["w"])
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


def setup_blocks(d, n_blocks: int, logit_scale: float):
    """Upload seeded inputs; return (call, check) for tt_decode_blocks over
    n_blocks blocks (the context is reset before each call)."""
    import torch
    import tt_inputs
    import block_wise_diffusion_b200 as tt
    inp = tt_inputs.generate(d, seed=0)
    kc0, vc0 = _dev(inp["k_ctx"]), _dev(inp["v_ctx"])
    kc, vc = kc0.clone(), vc0.clone()
    cl0 = torch.from_numpy(inp["ctx_len"]).cuda()
    cl = cl0.clone()
    X = {k: _dev(inp[k]) for k in ("emb", "e_mask", "u_t", "shift_scale", "w", "u_ctx")}
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


def main(argv=None) -> int:
    import torch
    import tt_inputs
    p = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    p.add_argument("stage", choices=["attn", "vocab", "blocks"])
    p.add_argument("--n-blocks", type=int, default=4,
                   help="blocks stage: blocks per call (the cache grows to hold them)")
    p.add_argument("--logit-scale", type=float, default=1.0)
    p.add_argument("--workload", default="mid", choices=sorted(tt_inputs.WORKLOADS))
    p.add_argument("--B", type=int, default=None, help="override the batch")
    p.add_argument("--V", type=int, default=None, help="override the vocabulary (vocab stage)")
    p.add_argument("--calls", type=int, default=2)
    p.add_argument("--time", action="store_true",
                   help="report the mean time of the calls after the first (CUDA events)")
    a = p.parse_args(argv)
    over = {}
    if a.B is not None:
        over["B"] = a.B
    if a.V is not None:
        over["V"] = a.V
    d = tt_inputs.workload(a.workload, **over)
    if a.stage == "blocks":
        # room for the blocks behind the context
        d = dataclasses.replace(d, L_cap=d.L_cap + a.n_blocks * d.S)
        call, check = setup_blocks(d, a.n_blocks, a.logit_scale)
    else:
        call, check = (setup_attn if a.stage == "attn" else setup_vocab)(d)
    call()  # warm-up
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record()
    for _ in range(a.calls):
        call()
    ev[1].record()
    torch.cuda.synchronize()
    if check() != 0:
        raise RuntimeError("device reported an error")
    msg = f"ok {a.stage} {d}"
    if a.time:
        us = ev[0].elapsed_time(ev[1]) * 1e3 / a.calls
        msg += f": {us:.1f} us per call (no L2 flush)"
        if a.stage == "blocks":
            msg += f", {a.n_blocks * d.B * d.S / (us * 1e-6):.0f} committed tokens/s"
    print(msg)
    return 0

if __name__ == "__main__":
    sys.exit(main())
