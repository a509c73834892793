"""The allocation-free vocab confidence / commit entry point.

tt_vocab_confidence_commit_noalloc serves callers that cannot allocate
device memory (no workspace to give); its scratch is a 16 MiB array built
into the library.  Its results must equal those of
tt_vocab_confidence_commit on the same inputs, on two calls in a row (the
second call starts from the array as the first one left it).  This file is
collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_wise_diffusion_b200 as tt
import tt_inputs



def _case(d, seed, frac_masked):
    rng = np.random.default_rng(seed)
    w = tt_inputs.generate(d, seed=seed, names=["w"])["w"]
    y = tt_inputs.bf16_bits(rng.standard_normal((d.B * d.S, d.H)).astype(np.float32))
    masked = (rng.random((d.B, d.S)) < frac_masked).astype(np.uint8)
    masked[0, 0] = 1
    tokens = np.where(masked == 1, -1, rng.integers(0, d.V, (d.B, d.S))).astype(np.int32)
    to_bf = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return to_bf(y), to_bf(w), tokens, masked


def _outputs(d):
    return (torch.full((d.B, d.S), -5.0, device="cuda"),
            torch.full((d.B, d.S), -5, dtype=torch.int32, device="cuda"),
            torch.full((d.B,), -5, dtype=torch.int32, device="cuda"))


def _with_workspace(D, d, y, w, gamma, scale, tokens, masked):
    tk, mk = torch.from_numpy(tokens).cuda(), torch.from_numpy(masked).cuda()
    conf, amax, ncom = _outputs(d)
    ws = tt.workspace(D, tt.TT_WS_VOCAB)
    tt.tt_vocab_confidence_commit(D, y, w, gamma, scale, tk, mk, conf, amax, ncom, ws)
    assert tt.tt_device_status(ws) == 0
    return [t.cpu().numpy() for t in (tk, mk, conf, amax, ncom)]


def _no_alloc(D, d, y, w, gamma, scale, tokens, masked):
    """One call, with every buffer allocated beforehand; returns its outputs
    and the device's free memory just before and just after the call."""
    tk, mk = torch.from_numpy(tokens).cuda(), torch.from_numpy(masked).cuda()
    conf, amax, ncom = _outputs(d)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    tt.tt_vocab_confidence_commit_noalloc(D, y, w, gamma, scale, tk, mk, conf, amax, ncom)
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    return [t.cpu().numpy() for t in (tk, mk, conf, amax, ncom)], (free0, free1)


@pytest.mark.gpu
@pytest.mark.parametrize("wl,B,scale,frac", [("tiny", 4, 12.0, 0.7), ("mid", 8, 8.0, 1.0)])
def test_no_alloc_matches_workspace_entry_point_twice(wl, B, scale, frac):
    d = tt_inputs.workload(wl, B=B)
    D = tt.dims(d)
    gamma = 0.8
    runs = []
    for seed in (1, 2):                       # two calls in a row, different inputs
        y, w, tokens, masked = _case(d, seed, frac)
        ref = _with_workspace(D, d, y, w, gamma, scale, tokens, masked)
        got, (free0, free1) = _no_alloc(D, d, y, w, gamma, scale, tokens, masked)
        if seed == 2:
            # the array and the kernels are loaded by now: a call takes no
            # device memory at all
            assert free1 == free0, (free0, free1)
        for name, a, b in zip(("tokens", "masked", "conf", "argmax", "n_committed"), got, ref):
            if name == "conf":
                np.testing.assert_allclose(a, b, rtol=2e-4, err_msg=f"seed {seed}: {name}")
            else:
                np.testing.assert_array_equal(a, b, err_msg=f"seed {seed}: {name}")
        assert (got[4][masked.any(axis=1)] >= 1).all()
        runs.append(got)
    assert not np.array_equal(runs[0][0], runs[1][0])


def test_no_alloc_rejects_problems_beyond_its_scratch():
    # host-side check: returns before any CUDA call, so it runs without a GPU
    d = tt_inputs.workload("ragged32")          # 4096 rows: about 69 MiB of scratch
    D = tt.dims(d)
    fake = 1 << 20                              # never dereferenced: rejected before launch
    L = tt.lib()
    r = L.tt_vocab_confidence_commit_noalloc(ctypes.byref(D), fake, fake, ctypes.c_float(0.8),
                                             ctypes.c_float(1.0), fake, fake, fake, fake, fake,
                                             None)
    assert r == 3
    assert "maximum is 16777216 bytes" in tt.tt_last_error()
