"""Failure detection on the device without faulting the GPU.

tt_selftest_timeout runs one kernel whose bounded wait can never be
satisfied (an mbarrier nothing arrives on); the wait gives up after the given
limit, records TT_ERR_TIMEOUT in the workspace control block and the kernel
returns.  The host then reads the status and the context stays usable.
"""
import numpy as np
import pytest
import torch

import block_wise_diffusion_b200 as tt
import tt_inputs
from oracle import twotower_oracle as O
from tests import _gpu as G


@pytest.mark.gpu
def test_bounded_wait_times_out_and_context_survives():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    tt.tt_selftest_timeout(ws, 5000)                 # 5 ms limit
    assert tt.tt_device_status(ws) == 5              # TT_ERR_TIMEOUT
    assert tt.tt_device_status(ws) == 0              # read once, then cleared
    # the context still works: a small attention call stays parity-green
    d = tt_inputs.workload("tiny")
    inp = tt_inputs.generate(d, seed=2, names=["q_blk", "k_blk", "v_blk", "k_ctx", "v_ctx"])
    D = tt.dims(d)
    out = torch.empty((d.B, d.S, d.Hq, d.dh), dtype=torch.bfloat16, device="cuda")
    wsa = G.workspace(D, tt.TT_WS_ATTN)
    tt.tt_block_denoise_attn(D, *(G.dev_bf16(inp[k]) for k in ("q_blk", "k_blk", "v_blk", "k_ctx",
                                                             "v_ctx")),
                             G.dev(inp["ctx_len"]), out, wsa)
    assert tt.tt_device_status(wsa) == 0
    f = O.from_bf16
    ref = O.round_bf16(O.block_attention(f(inp["q_blk"]), f(inp["k_blk"]), f(inp["v_blk"]),
                                         f(inp["k_ctx"]), f(inp["v_ctx"]), inp["ctx_len"]))
    G.assert_close_bf16(G.host_f64(out), ref, "after timeout")


def test_selftest_rejects_bad_limits():
    tt.lib()
    with pytest.raises(tt.TTError):
        tt.tt_selftest_timeout(1 << 20, 0, stream=0)
    with pytest.raises(tt.TTError):
        tt.tt_selftest_timeout(1 << 20, 2_000_000, stream=0)
