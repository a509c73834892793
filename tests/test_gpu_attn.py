"""Parity of tt_block_denoise_attn against the float64 oracle.

Element by element at sizes the oracle finishes in seconds (several key tiles,
ragged tails, empty contexts, both head sizes, S = 16 and 32, forced split
counts), and on whole sequences at the full mid-size decode shape.
Tolerance: max-abs 2e-2 and relative L2 1e-2 (bf16 inputs, fp32 accumulation).
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import block_wise_diffusion_b200 as tt
import tt_inputs
from oracle import twotower_oracle as O
from tests import _gpu as G

pytestmark = pytest.mark.gpu


def run_attn(d, inp, ctx_len=None, splits=0):
    D = tt.dims(d)
    tt.tt_set_attn_splits(splits)
    try:
        q = G.dev_bf16(inp["q_blk"])
        kb = G.dev_bf16(inp["k_blk"])
        vb = G.dev_bf16(inp["v_blk"])
        kc = G.dev_bf16(inp["k_ctx"])
        vc = G.dev_bf16(inp["v_ctx"])
        cl = G.dev(inp["ctx_len"] if ctx_len is None else ctx_len.astype(np.int32))
        out = torch.full((d.B, d.S, d.Hq, d.dh), float("nan"), dtype=torch.bfloat16, device="cuda")
        ws = G.workspace(D, tt.TT_WS_ATTN)
        tt.tt_block_denoise_attn(D, q, kb, vb, kc, vc, cl, out, ws)
        assert tt.tt_device_status(ws) == 0
        return G.host_f64(out)
    finally:
        tt.tt_set_attn_splits(0)


def oracle_attn(inp, ctx_len=None, bsel=None):
    f = O.from_bf16
    cl = inp["ctx_len"] if ctx_len is None else ctx_len
    sl = slice(None) if bsel is None else bsel
    return O.block_attention(f(inp["q_blk"][sl]), f(inp["k_blk"][sl]), f(inp["v_blk"][sl]),
                             f(inp["k_ctx"][sl]), f(inp["v_ctx"][sl]), cl[sl])


CASES = [
    # name, dims overrides, ctx lengths (None = workload's), sharp
    ("tiny", tt_inputs.workload("tiny"), None, False),
    ("tiny-sharp", tt_inputs.workload("tiny"), None, True),
    ("gqa16-ragged", tt_inputs.workload("mid", B=3, L_cap=1000, ctx=("fixed", 1000), V=1024),
     np.array([1000, 777, 0]), True),
    ("gqa16-S32", tt_inputs.workload("mid", B=2, S=32, L_cap=300, ctx=("fixed", 300), V=1024),
     np.array([300, 65]), True),
    ("dh64-gqa8", tt_inputs.Dims(B=2, S=16, Hq=16, Hkv=2, dh=64, V=512, L_cap=513,
                                 ctx=("fixed", 513)), np.array([513, 129]), True),
    ("mha-like-g2", tt_inputs.Dims(B=2, S=16, Hq=4, Hkv=2, dh=128, V=512, L_cap=200,
                                   ctx=("fixed", 200)), np.array([1, 200]), False),
    # autoregressive baseline step: one block position, M = G query rows
    ("ar-S1", tt_inputs.workload("mid", B=3, S=1, L_cap=700, ctx=("fixed", 700), V=1024),
     np.array([700, 129, 0]), True),
    # larger blocks: S = 128 is a whole key tile of block keys and 8 query tiles
    ("block-S128", tt_inputs.workload("mid", B=2, S=128, L_cap=500, ctx=("fixed", 500), V=1024),
     np.array([500, 77]), True),
    ("block-S64-g4", tt_inputs.Dims(B=2, S=64, Hq=8, Hkv=2, dh=64, V=512, L_cap=300,
                                    ctx=("fixed", 300)), np.array([300, 0]), True),
    # the top of the accepted envelope: G = 32, 64 and 128 query heads per KV
    # head (a 128-row half holds 4, 2 or 1 block positions), H = 8192
    ("gqa32", tt_inputs.Dims(B=2, S=16, Hq=32, Hkv=1, dh=64, V=512, L_cap=300,
                             ctx=("fixed", 300)), np.array([300, 45]), True),
    ("gqa64-H8192", tt_inputs.Dims(B=1, S=16, Hq=64, Hkv=1, dh=128, V=512, L_cap=150,
                                   ctx=("fixed", 150)), np.array([150]), True),
    ("gqa128-H8192", tt_inputs.Dims(B=2, S=32, Hq=128, Hkv=1, dh=64, V=512, L_cap=200,
                                    ctx=("fixed", 200)), np.array([200, 3]), True),
    # the rest of the envelope's edges: one query head per KV head (G = 1), a
    # batch of 200 sequences, a context longer than 65536 keys
    ("g1", tt_inputs.Dims(B=2, S=16, Hq=4, Hkv=4, dh=64, V=512, L_cap=300,
                          ctx=("fixed", 300)), np.array([300, 17]), True),
    ("batch200", tt_inputs.Dims(B=200, S=16, Hq=4, Hkv=1, dh=64, V=512, L_cap=130,
                                ctx=("uniform", 0, 130)), None, False),
    ("L70000", tt_inputs.Dims(B=1, S=16, Hq=4, Hkv=1, dh=64, V=512, L_cap=70000,
                              ctx=("fixed", 70000)), None, False),
]


@pytest.mark.parametrize("name,d,cl,sharp", CASES, ids=[c[0] for c in CASES])
def test_attention_matches_oracle(name, d, cl, sharp):
    inp = tt_inputs.generate(d, seed=11, sharp=sharp,
                             names=["q_blk", "k_blk", "v_blk", "k_ctx", "v_ctx"])
    got = run_attn(d, inp, cl)
    ref = O.round_bf16(oracle_attn(inp, cl))
    G.assert_close_bf16(got, ref, name)


@pytest.mark.parametrize("splits", [1, 2, 5, 16])
def test_attention_independent_of_split_count(splits):
    d = tt_inputs.workload("mid", B=2, L_cap=2000, ctx=("fixed", 2000), V=1024)
    inp = tt_inputs.generate(d, seed=12, sharp=True,
                             names=["q_blk", "k_blk", "v_blk", "k_ctx", "v_ctx"])
    cl = np.array([2000, 1111])
    got = run_attn(d, inp, cl, splits=splits)
    ref = O.round_bf16(oracle_attn(inp, cl))
    G.assert_close_bf16(got, ref, f"splits={splits}")


def test_attention_block_permutation_equivariance_on_gpu():
    d = tt_inputs.workload("mid", B=1, L_cap=256, ctx=("fixed", 256), V=1024)
    inp = tt_inputs.generate(d, seed=13, sharp=True,
                             names=["q_blk", "k_blk", "v_blk", "k_ctx", "v_ctx"])
    perm = np.random.default_rng(0).permutation(d.S)
    inp2 = dict(inp, q_blk=inp["q_blk"][:, perm], k_blk=inp["k_blk"][:, perm],
                v_blk=inp["v_blk"][:, perm])
    a = run_attn(d, inp)
    b = run_attn(d, inp2)
    # the block keys form one tile, so permuting them only reorders fp32 sums
    G.assert_close_bf16(b, a[:, perm], "permuted block")


def test_attention_full_mid_shape_sampled_sequences():
    d = tt_inputs.workload("mid")
    inp = tt_inputs.generate(d, seed=0, names=["q_blk", "k_blk", "v_blk", "k_ctx", "v_ctx"])
    got = run_attn(d, inp)
    for b in (0, 5):
        ref = O.round_bf16(oracle_attn(inp, bsel=slice(b, b + 1)))
        G.assert_close_bf16(got[b:b + 1], ref, f"mid b={b}")


def test_attention_long_context_sampled():
    d = tt_inputs.workload("long", B=1)
    inp = tt_inputs.generate(d, seed=3, sharp=True,
                             names=["q_blk", "k_blk", "v_blk", "k_ctx", "v_ctx"])
    got = run_attn(d, inp)
    ref = O.round_bf16(oracle_attn(inp))
    G.assert_close_bf16(got, ref, "long")


def test_attention_rejects_bad_ctx_len_on_device():
    d = tt_inputs.workload("tiny")
    inp = tt_inputs.generate(d, seed=1, names=["q_blk", "k_blk", "v_blk", "k_ctx", "v_ctx"])
    D = tt.dims(d)
    q, kb, vb = (G.dev_bf16(inp[k]) for k in ("q_blk", "k_blk", "v_blk"))
    kc, vc = G.dev_bf16(inp["k_ctx"]), G.dev_bf16(inp["v_ctx"])
    out = torch.empty((d.B, d.S, d.Hq, d.dh), dtype=torch.bfloat16, device="cuda")
    ws = G.workspace(D, tt.TT_WS_ATTN)
    tt.tt_block_denoise_attn(D, q, kb, vb, kc, vc, G.dev(np.array([d.L_cap + 5], np.int32)),
                             out, ws)
    assert tt.tt_device_status(ws) == 1          # TT_ERR_INVALID_ARG recorded, clamped
    assert tt.tt_device_status(ws) == 0          # and cleared
