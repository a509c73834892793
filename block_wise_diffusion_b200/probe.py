"""Run one library entry point a few times on seeded synthetic inputs.

For profilers (ncu) and quick timing of a single stage outside the block loop:

    python -m block_wise_diffusion_b200.probe attn --workload long --B 2
    python -m block_wise_diffusion_b200.probe vocab --workload mid --V 65536

Each call runs ``--calls`` times on the current stream, then checks the
device status word.  Inputs come from ``tt_inputs`` (the same seeded
generator the tests and the benchmark use); nothing here computes a reference.
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _dev(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def run_attn(d, calls: int) -> None:
    import torch
    import tt_inputs
    import block_wise_diffusion_b200 as tt
    inp = tt_inputs.generate(d, seed=0, names=["q_blk", "k_blk", "v_blk", "k_ctx", "v_ctx"])
    q, kb, vb, kc, vc = (_dev(inp[k]) for k in ("q_blk", "k_blk", "v_blk", "k_ctx", "v_ctx"))
    cl = torch.from_numpy(inp["ctx_len"]).cuda()
    D = tt.dims(d)
    out = torch.empty((d.B, d.S, d.Hq, d.dh), dtype=torch.bfloat16, device="cuda")
    ws = tt.workspace(D, tt.TT_WS_ATTN)
    for _ in range(calls):
        tt.tt_block_denoise_attn(D, q, kb, vb, kc, vc, cl, out, ws)
    if tt.tt_device_status(ws) != 0:
        raise RuntimeError("device reported an error")


def run_vocab(d, calls: int) -> None:
    import torch
    import tt_inputs
    import block_wise_diffusion_b200 as tt
    inp = tt_inputs.generate(d, seed=0, names=["w"])
    rng = np.random.default_rng(0)
    y = _dev(tt_inputs.bf16_bits(rng.standard_normal((d.B * d.S, d.H)).astype(np.float32)))
    w = _dev(inp["w"])
    D = tt.dims(d)
    ws = tt.workspace(D, tt.TT_WS_VOCAB)
    for _ in range(calls):
        tok = torch.full((d.B, d.S), -1, dtype=torch.int32, device="cuda")
        msk = torch.ones((d.B, d.S), dtype=torch.uint8, device="cuda")
        conf = torch.empty((d.B, d.S), dtype=torch.float32, device="cuda")
        am = torch.empty((d.B, d.S), dtype=torch.int32, device="cuda")
        nc = torch.empty((d.B,), dtype=torch.int32, device="cuda")
        tt.tt_vocab_confidence_commit(D, y, w, 0.8, 1.0, tok, msk, conf, am, nc, ws)
    if tt.tt_device_status(ws) != 0:
        raise RuntimeError("device reported an error")


def main(argv=None) -> int:
    import torch
    import tt_inputs
    p = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    p.add_argument("stage", choices=["attn", "vocab"])
    p.add_argument("--workload", default="mid", choices=sorted(tt_inputs.WORKLOADS))
    p.add_argument("--B", type=int, default=None, help="override the batch")
    p.add_argument("--V", type=int, default=None, help="override the vocabulary (vocab stage)")
    p.add_argument("--calls", type=int, default=2)
    a = p.parse_args(argv)
    over = {}
    if a.B is not None:
        over["B"] = a.B
    if a.V is not None:
        over["V"] = a.V
    d = tt_inputs.workload(a.workload, **over)
    (run_attn if a.stage == "attn" else run_vocab)(d, a.calls)
    torch.cuda.synchronize()
    print(f"ok {a.stage} {d}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
