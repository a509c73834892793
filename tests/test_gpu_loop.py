"""Parity of tt_denoise_block_loop with the oracle's loop, step by step.

Two comparisons, both teacher-forced (every oracle step starts from the
GPU's state, so one excluded near tie cannot cascade):

* stage-wise (bit-exact): the loop is driven one step per call and
  tt_loop_last_step hands out the adaLN rows the step fed the vocabulary
  projection.  The oracle's projection, confidence and commit rule run on
  those very bytes; the compacted row list, every argmax and every
  sequence's commit set and tokens must match bit for bit outside the
  near-tie exclusions of tests/_gpu.py, and the confidences within the fp32
  merge's rounding.  The literal exclusion rule's counts are reported.
* end-to-end: the oracle recomputes attention and adaLN in float64 from the
  GPU's tokens and mask; commit sets must match, and a committed token may be
  the oracle's runner-up only at a near tie (tests/_gpu.py LOOP_TIE_LOGIT).
  Such flips are counted, reported and bounded.

The step-at-a-time run must end in exactly the state of one uninterrupted
call (the launch configuration the benchmark times).
"""
import numpy as np
import pytest
import torch

import block_wise_diffusion_b200 as tt
import tt_inputs
from oracle import parity as P
from oracle import twotower_oracle as O
from tests import _gpu as G

pytestmark = pytest.mark.gpu

LOOP_INPUTS = ["k_ctx", "v_ctx", "shift_scale", "w", "emb", "e_mask", "u_t"]


def run_loop_gpu(d, inp, gamma, logit_scale, max_steps=None):
    D = tt.dims(d)
    dv = {k: G.dev_bf16(inp[k]) for k in LOOP_INPUTS}
    tokens = G.dev(inp["tokens"])
    masked = G.dev(inp["masked"])
    steps_taken = torch.full((d.B,), -7, dtype=torch.int32, device="cuda")
    commit_step = torch.full((d.B, d.S), -7, dtype=torch.int32, device="cuda")
    ws = G.workspace(D, tt.TT_WS_LOOP)
    n = tt.tt_denoise_block_loop(D, dv["k_ctx"], dv["v_ctx"], G.dev(inp["ctx_len"]), dv["emb"],
                                 dv["e_mask"], dv["u_t"], dv["shift_scale"], dv["w"], gamma,
                                 logit_scale, max_steps or d.S, tokens, masked, steps_taken,
                                 commit_step, ws)
    return dict(tokens=tokens.cpu().numpy(), masked=masked.cpu().numpy(),
                steps_taken=steps_taken.cpu().numpy(), commit_step=commit_step.cpu().numpy(),
                steps_run=n)


def run_loop_layers_gpu(d, inp, n_layers, gamma, logit_scale, max_steps=None):
    D = tt.dims(d)
    dv = {k: G.dev_bf16(inp[k + "_l"] if n_layers > 1 else inp[k][None])
          for k in ("k_ctx", "v_ctx", "shift_scale", "u_t")}
    dv.update({k: G.dev_bf16(inp[k]) for k in ("w", "emb", "e_mask")})
    tokens = G.dev(inp["tokens"])
    masked = G.dev(inp["masked"])
    steps_taken = torch.full((d.B,), -7, dtype=torch.int32, device="cuda")
    commit_step = torch.full((d.B, d.S), -7, dtype=torch.int32, device="cuda")
    ws = G.workspace(D, tt.TT_WS_LOOP)
    n = tt.tt_denoise_block_loop_layers(
        D, n_layers, dv["k_ctx"], dv["v_ctx"], G.dev(inp["ctx_len"]), dv["emb"], dv["e_mask"],
        dv["u_t"], dv["shift_scale"], dv["w"], gamma, logit_scale, max_steps or d.S, tokens,
        masked, steps_taken, commit_step, ws)
    return dict(tokens=tokens.cpu().numpy(), masked=masked.cpu().numpy(),
                steps_taken=steps_taken.cpu().numpy(), commit_step=commit_step.cpu().numpy(),
                steps_run=n)


def run_loop_stepwise(d, inp, gamma, logit_scale, n_layers=1, limit=None):
    """Drive the loop one step per call; after each call copy out the step's
    vocabulary rows with tt_loop_last_step.  Returns (steps, final) where each
    step holds the state before and after it and the step's rows."""
    D = tt.dims(d)
    if n_layers > 1:
        dv = {k: G.dev_bf16(inp[k + "_l"]) for k in ("k_ctx", "v_ctx", "shift_scale", "u_t")}
    else:
        dv = {k: G.dev_bf16(inp[k]) for k in ("k_ctx", "v_ctx", "shift_scale", "u_t")}
    dv.update({k: G.dev_bf16(inp[k]) for k in ("w", "emb", "e_mask")})
    cl = G.dev(inp["ctx_len"])
    tokens = G.dev(inp["tokens"])
    masked = G.dev(inp["masked"])
    steps_taken = torch.empty((d.B,), dtype=torch.int32, device="cuda")
    commit_step = torch.empty((d.B, d.S), dtype=torch.int32, device="cuda")
    ws = G.workspace(D, tt.TT_WS_LOOP)
    rows = d.B * d.S
    y_rows = torch.empty((rows, d.H), dtype=torch.bfloat16, device="cuda")
    row_ids = torch.empty((rows,), dtype=torch.int32, device="cuda")
    conf = torch.empty((rows,), dtype=torch.float32, device="cuda")
    amax = torch.empty((rows,), dtype=torch.int32, device="cuda")
    steps = []
    for k in range(limit or d.S):
        before = (tokens.cpu().numpy(), masked.cpu().numpy())
        if not before[1].any():
            break
        n = tt.tt_denoise_block_loop_layers(
            D, n_layers, dv["k_ctx"], dv["v_ctx"], cl, dv["emb"], dv["e_mask"], dv["u_t"],
            dv["shift_scale"], dv["w"], gamma, logit_scale, 1, tokens, masked, steps_taken,
            commit_step, ws)
        assert n == 1
        M = tt.tt_loop_last_step(D, ws, y_rows, row_ids, conf, amax)
        steps.append(dict(tokens0=before[0], masked0=before[1], tokens1=tokens.cpu().numpy(),
                          masked1=masked.cpu().numpy(), M=M,
                          y=G.bits_of(y_rows[:M]), row_ids=row_ids[:M].cpu().numpy(),
                          conf=conf.cpu().numpy().reshape(d.B, d.S),
                          argmax=amax.cpu().numpy().reshape(d.B, d.S)))
    cs = np.full((d.B, d.S), -1, np.int32)
    for k, st in enumerate(steps):
        cs[(st["masked0"] == 1) & (st["masked1"] == 0)] = k
    final = dict(tokens=tokens.cpu().numpy(), masked=masked.cpu().numpy(), commit_step=cs)
    return steps, final


def check_stagewise(d, steps, w_bits, gamma, logit_scale, bsel=None):
    """The oracle's vocabulary projection and commit rule on each step's GPU
    rows, bit-exact outside near ties.  ``bsel``: the sequences to check
    (all by default).  Returns the counts (dict)."""
    w64 = O.from_bf16(w_bits)
    bsel = np.arange(d.B) if bsel is None else np.asarray(bsel)
    cnt = dict(steps=len(steps), seq_steps=0, seq_steps_excluded=0, positions=0,
               argmax_excluded=0, spec_excluded=0)
    for k, st in enumerate(steps):
        m0 = st["masked0"].astype(bool)
        # the compacted row list is exact integer work: all masked rows, in order
        np.testing.assert_array_equal(st["row_ids"], np.flatnonzero(m0.reshape(-1)),
                                      err_msg=f"step {k}: row list")
        pos = {int(r): j for j, r in enumerate(st["row_ids"])}
        sel_rows = [b * d.S + s for b in bsel for s in range(d.S) if m0[b, s]]
        y = O.from_bf16(st["y"][[pos[r] for r in sel_rows]]) if sel_rows else np.zeros((0, d.H))
        c, tk, gl, gp = O.vocab_confidence(y, w64, logit_scale)
        nb = len(bsel)
        conf_o = np.full((nb, d.S), np.nan)
        tok_o = np.full((nb, d.S), -1, np.int64)
        gl_o = np.full((nb, d.S), np.inf)
        gp_o = np.full((nb, d.S), np.inf)
        bi = {int(b): i for i, b in enumerate(bsel)}
        for j, r in enumerate(sel_rows):
            i, s = bi[r // d.S], r % d.S
            conf_o[i, s], tok_o[i, s], gl_o[i, s], gp_o[i, s] = c[j], tk[j], gl[j], gp[j]
        mb = m0[bsel]
        # per-position results the commit used: argmax bit-exact outside near
        # ties, confidence within the fp32 merge's rounding
        g_conf, g_tok = st["conf"][bsel], st["argmax"][bsel]
        assert np.all(g_conf[~mb] == -1) and np.all(g_tok[~mb] == -1), f"step {k}"
        np.testing.assert_allclose(g_conf[mb], conf_o[mb], rtol=2e-4, err_msg=f"step {k}: conf")
        ex_arg = mb & G.derived_excluded_argmax(gl_o)
        np.testing.assert_array_equal(g_tok[mb & ~ex_arg], tok_o[mb & ~ex_arg],
                                      err_msg=f"step {k}: argmax")
        cnt["argmax_excluded"] += int(ex_arg.sum())
        cnt["spec_excluded"] += int((mb & G.spec_excluded(conf_o, gp_o, gamma)).sum())
        cnt["positions"] += int(mb.sum())
        # the commit rule on the oracle's values, from the state before the step
        t2, m2, committed, fb = O.commit(conf_o, tok_o, st["tokens0"][bsel], mb, gamma)
        for i, b in enumerate(bsel):
            if not mb[i].any():
                continue
            cnt["seq_steps"] += 1
            skip = (mb[i] & G.derived_excluded_threshold(conf_o[i], gamma)).any()
            skip |= (ex_arg[i] & committed[i]).any()
            if fb[i]:
                skip |= G.fallback_near_tie(conf_o[i][mb[i]])
            if skip:
                cnt["seq_steps_excluded"] += 1
                continue
            np.testing.assert_array_equal(st["masked1"][b], m2[i].astype(np.uint8),
                                          err_msg=f"step {k} seq {b}: commit set")
            np.testing.assert_array_equal(st["tokens1"][b], t2[i], err_msg=f"step {k} seq {b}: tokens")
    print(f"stage-wise: {cnt}")
    return cnt


def stepwise_equals_single_call(d, inp, gamma, logit_scale, single, n_layers=1, bsel=None,
                                 max_seq_steps_excluded=2):
    """Step-at-a-time run: the same final state as the uninterrupted call
    ``single``, and the stage-wise comparison on it."""
    steps, final = run_loop_stepwise(d, inp, gamma, logit_scale, n_layers=n_layers)
    np.testing.assert_array_equal(final["tokens"], single["tokens"])
    np.testing.assert_array_equal(final["commit_step"], single["commit_step"])
    cnt = check_stagewise(d, steps, inp["w"], gamma, logit_scale, bsel=bsel)
    assert cnt["seq_steps"] > 0
    assert cnt["seq_steps_excluded"] <= max_seq_steps_excluded, cnt
    return steps


def slice_batch(inp, bsel):
    out = dict(inp)
    for k in ("k_ctx", "v_ctx", "ctx_len", "tokens", "masked"):
        out[k] = inp[k][bsel]
    for k in ("k_ctx_l", "v_ctx_l"):
        if k in inp:
            out[k] = inp[k][:, bsel]
    return out


def rows_by_position(steps, S, bsel=None):
    """The stepwise run's vocabulary rows as {(b, s): float64 row} per step,
    b counted within ``bsel`` (all sequences by default)."""
    out = []
    for st in steps:
        rows = {}
        for j, rid in enumerate(st["row_ids"]):
            b, s = divmod(int(rid), S)
            if bsel is None:
                rows[(b, s)] = st["y"][j]
            elif b in bsel:
                rows[(bsel.index(b), s)] = st["y"][j]
        out.append({k: O.from_bf16(v) for k, v in rows.items()})
    return out


def compare_teacher_forced(inp, g, gamma, logit_scale, bsel=None, steps=None):
    """End-to-end comparison (oracle.parity.compare_loop) on the sequences
    ``bsel``; every disagreement outside the exclusions fails, near-tie top-2
    flips are reported and bounded.  With ``steps`` (the step-at-a-time run of
    the same trajectory) the kernel's rows are compared with the oracle's
    (relative L2 within oracle.parity.Y_REL_L2) and decisions that the
    oracle itself takes differently on the two sets of rows are excluded and
    counted.  Returns the compared sequence-steps and those excluded as near
    ties (the decisions explained by the rows' difference are reported in
    the printed counts)."""
    S = inp["masked"].shape[1]
    g_rows = None
    if steps is not None:
        g_rows = rows_by_position(steps, S, None if bsel is None else [int(b) for b in bsel])
    if bsel is not None:
        inp = slice_batch(inp, bsel)
        g = {k: (v[bsel] if isinstance(v, np.ndarray) else v) for k, v in g.items()}
    cnt, problems = P.compare_loop(inp, g["tokens"], g["commit_step"], gamma, logit_scale,
                                   g_rows=g_rows)
    print(f"end-to-end: {cnt}")
    assert not problems, problems[:5]
    # a flip needs the oracle's top-2 logit gap below the attention-error
    # band; with these inputs that is a minority of the committed tokens
    assert cnt["top2_flips"] <= max(1, cnt["tokens"] // 4), cnt
    if g_rows is not None:
        # The numerical bar of the end-to-end comparison: the rows.  A
        # decision the oracle takes differently on the kernel's rows than on
        # its own is explained by their difference (counted, not bounded):
        # the stage-wise comparison holds the kernel to the oracle on those
        # very rows bit for bit.  At unit logit scale every step is a
        # fallback between masked positions that are equal in exact
        # arithmetic; where the kernels compute them with different
        # summation orders (different query tiles of one sequence) the
        # last bits pick the position, so such counts can be large there.
        assert cnt["y_rel_l2_max"] <= P.Y_REL_L2, cnt
    return cnt["seq_steps"], cnt["seq_steps_excluded"] - cnt.get("y_explained", 0)


def check_invariants(d, inp, g):
    m0 = inp["masked"].astype(bool)
    assert not g["masked"].any()
    np.testing.assert_array_equal(g["tokens"][~m0], inp["tokens"][~m0])     # never change
    assert np.all(g["commit_step"][~m0] == -1)
    assert np.all(g["commit_step"][m0] >= 0)
    assert np.all((g["tokens"] >= 0) & (g["tokens"] < d.V))
    n0 = m0.sum(axis=1)
    assert np.all(g["steps_taken"] <= n0)
    assert np.all((g["steps_taken"] >= 1) | (n0 == 0))
    # every step commits at least one position of every sequence still masked
    for b in range(d.B):
        if n0[b]:
            steps = set(g["commit_step"][b][m0[b]].tolist())
            assert steps == set(range(g["steps_taken"][b]))
    assert g["steps_run"] == g["steps_taken"].max()


@pytest.mark.parametrize("gamma,logit_scale", [(0.8, 1.0), (0.5, 12.0), (0.95, 40.0)])
def test_loop_tiny(gamma, logit_scale):
    d = tt_inputs.workload("tiny", B=3, precommit=("uniform", 0.0, 0.75))
    inp = tt_inputs.generate(d, seed=31)
    g = run_loop_gpu(d, inp, gamma, logit_scale)
    check_invariants(d, inp, g)
    steps = stepwise_equals_single_call(d, inp, gamma, logit_scale, g)
    n_cmp, n_ex = compare_teacher_forced(inp, g, gamma, logit_scale, steps=steps)
    assert n_cmp > 0 and n_ex <= 2, (n_cmp, n_ex)


@pytest.mark.parametrize("gamma,logit_scale", [(0.8, 1.0), (0.8, 12.0), (0.5, 40.0)])
def test_loop_tiny_block_of_32(gamma, logit_scale):
    """S = 32 (the ragged serving batch's second block size) at tiny shapes."""
    d = tt_inputs.workload("tiny", B=3, S=32, precommit=("uniform", 0.0, 0.75))
    inp = tt_inputs.generate(d, seed=34)
    g = run_loop_gpu(d, inp, gamma, logit_scale)
    check_invariants(d, inp, g)
    steps = stepwise_equals_single_call(d, inp, gamma, logit_scale, g)
    n_cmp, n_ex = compare_teacher_forced(inp, g, gamma, logit_scale, steps=steps)
    assert n_cmp > 0 and n_ex <= 2, (n_cmp, n_ex)


@pytest.mark.parametrize("logit_scale", [1.0, 12.0])
def test_loop_autoregressive_step_s1(logit_scale):
    """S = 1: every call commits the block's single position in one step."""
    d = tt_inputs.workload("mid", B=4, S=1, L_cap=300, ctx=("fixed", 300), V=1024)
    inp = tt_inputs.generate(d, seed=41)
    g = run_loop_gpu(d, inp, 0.8, logit_scale)
    check_invariants(d, inp, g)
    assert g["steps_run"] == 1 and np.all(g["steps_taken"] == 1)
    steps = stepwise_equals_single_call(d, inp, 0.8, logit_scale, g, max_seq_steps_excluded=1)
    n_cmp, n_ex = compare_teacher_forced(inp, g, 0.8, logit_scale, steps=steps)
    assert n_cmp + n_ex == d.B and n_ex <= 1, (n_cmp, n_ex)


@pytest.mark.parametrize("S,logit_scale", [(128, 1.0), (128, 40.0), (64, 12.0)])
def test_loop_larger_blocks(S, logit_scale):
    d = tt_inputs.workload("tiny", B=2, S=S, precommit=("uniform", 0.0, 0.75))
    inp = tt_inputs.generate(d, seed=43)
    g = run_loop_gpu(d, inp, 0.8, logit_scale)
    check_invariants(d, inp, g)
    steps = stepwise_equals_single_call(d, inp, 0.8, logit_scale, g)
    n_cmp, n_ex = compare_teacher_forced(inp, g, 0.8, logit_scale, steps=steps)
    assert n_cmp > 0 and n_ex <= 2, (n_cmp, n_ex)


@pytest.mark.parametrize("logit_scale", [1.0, 12.0])
def test_loop_widest_hidden_and_group(logit_scale):
    """H = 8192 (the largest hidden size accepted) with G = 32 query heads per
    KV head."""
    d = tt_inputs.Dims(B=2, S=16, Hq=64, Hkv=2, dh=128, V=1024, L_cap=256, ctx=("fixed", 256),
                       precommit=("uniform", 0.0, 0.75))
    inp = tt_inputs.generate(d, seed=44)
    g = run_loop_gpu(d, inp, 0.8, logit_scale)
    check_invariants(d, inp, g)
    steps = stepwise_equals_single_call(d, inp, 0.8, logit_scale, g)
    n_cmp, n_ex = compare_teacher_forced(inp, g, 0.8, logit_scale, steps=steps)
    assert n_cmp > 0 and n_ex <= 2, (n_cmp, n_ex)


@pytest.mark.parametrize("wl,logit_scale", [("tiny", 12.0), ("mid", 1.0)])
def test_loop_graph_replay_equals_direct_launches(wl, logit_scale):
    """The loop replays one captured CUDA graph per argument set: the first
    call captures and replays, later calls with the same buffers replay.  All
    give bitwise the state of direct launches, and each call counts the same
    kernels."""
    d = tt_inputs.workload(wl, precommit=("uniform", 0.0, 0.75)) if wl == "tiny" else \
        tt_inputs.workload(wl, B=2, L_cap=512, ctx=("fixed", 512))
    inp = tt_inputs.generate(d, seed=46)
    D = tt.dims(d)
    dv = {k: G.dev_bf16(inp[k]) for k in LOOP_INPUTS}
    cl = G.dev(inp["ctx_len"])
    tok0, msk0 = G.dev(inp["tokens"]), G.dev(inp["masked"])
    tokens, masked = tok0.clone(), msk0.clone()
    steps_taken = torch.empty((d.B,), dtype=torch.int32, device="cuda")
    commit_step = torch.empty((d.B, d.S), dtype=torch.int32, device="cuda")
    ws = G.workspace(D, tt.TT_WS_LOOP)

    def call():
        tokens.copy_(tok0)
        masked.copy_(msk0)
        n0 = tt.tt_launch_count()
        n = tt.tt_denoise_block_loop(D, dv["k_ctx"], dv["v_ctx"], cl, dv["emb"], dv["e_mask"],
                                     dv["u_t"], dv["shift_scale"], dv["w"], 0.8, logit_scale, d.S,
                                     tokens, masked, steps_taken, commit_step, ws)
        return (n, tt.tt_launch_count() - n0, tokens.cpu().numpy(), masked.cpu().numpy(),
                steps_taken.cpu().numpy(), commit_step.cpu().numpy())

    def same(got, ref):
        assert got[0] == ref[0] and got[1] == ref[1], (got[:2], ref[:2])
        for a, b in zip(got[2:], ref[2:]):
            np.testing.assert_array_equal(a, b)

    tt.tt_set_loop_graphs(0)
    try:
        direct = call()
    finally:
        tt.tt_set_loop_graphs(1)
    first, second, third = call(), call(), call()
    for got in (first, second, third):
        same(got, direct)
    assert not direct[3].any()
    # the same buffers with another logit scale, or another attention CTA
    # count, are other argument sets: no stale graph may be replayed
    logit_scale, saved = logit_scale * 3.0, logit_scale
    tt.tt_set_loop_graphs(0)
    try:
        direct2 = call()
    finally:
        tt.tt_set_loop_graphs(1)
    same(call(), direct2)
    logit_scale = saved
    tt.tt_set_attn_splits(37)
    try:
        tt.tt_set_loop_graphs(0)
        try:
            direct3 = call()
        finally:
            tt.tt_set_loop_graphs(1)
        same(call(), direct3)
    finally:
        tt.tt_set_attn_splits(0)
    same(call(), direct)


def test_loop_canonical_scale_commits_in_position_order():
    d = tt_inputs.workload("tiny", B=2)
    inp = tt_inputs.generate(d, seed=32)
    g = run_loop_gpu(d, inp, 0.8, 1.0)
    check_invariants(d, inp, g)
    # identical masked positions tie; the lowest position commits first
    np.testing.assert_array_equal(g["commit_step"], np.tile(np.arange(16), (2, 1)))
    compare_teacher_forced(inp, g, 0.8, 1.0)


def test_loop_resume_equals_single_call():
    d = tt_inputs.workload("tiny", B=2)
    inp = tt_inputs.generate(d, seed=33)
    # unit logit scale: one commit per sequence per step, so a 3-step call
    # leaves 13 masked positions to resume from
    full = run_loop_gpu(d, inp, 0.8, 1.0)
    part = run_loop_gpu(d, inp, 0.8, 1.0, max_steps=3)
    assert part["masked"].sum(axis=1).tolist() == [13, 13]
    inp2 = dict(inp, tokens=part["tokens"], masked=part["masked"])
    rest = run_loop_gpu(d, inp2, 0.8, 1.0)
    np.testing.assert_array_equal(rest["tokens"], full["tokens"])
    assert rest["steps_run"] == 13


@pytest.mark.parametrize("logit_scale", [1.0, 8.0])
def test_loop_full_mid_shape_sampled_sequences(logit_scale):
    d = tt_inputs.workload("mid")
    inp = tt_inputs.generate(d, seed=0)
    g = run_loop_gpu(d, inp, 0.8, logit_scale)
    check_invariants(d, inp, g)
    if logit_scale == 1.0:
        assert g["steps_run"] == 16
    steps = stepwise_equals_single_call(d, inp, 0.8, logit_scale, g)
    n_cmp, n_ex = compare_teacher_forced(inp, g, 0.8, logit_scale, bsel=np.array([0, 5]),
                                      steps=steps)
    print(f"mid loop scale={logit_scale}: compared {n_cmp} sequence-steps, excluded {n_ex}")
    assert n_cmp > 0 and n_ex <= 2


@pytest.mark.parametrize("n_layers,logit_scale", [(2, 1.0), (3, 40.0), (2, 12.0)])
def test_loop_layers_tiny(n_layers, logit_scale):
    d = tt_inputs.workload("tiny", B=3, precommit=("uniform", 0.0, 0.75))
    inp = tt_inputs.generate(d, seed=47, n_layers=n_layers)
    g = run_loop_layers_gpu(d, inp, n_layers, 0.8, logit_scale)
    check_invariants(d, inp, g)
    steps = stepwise_equals_single_call(d, inp, 0.8, logit_scale, g, n_layers=n_layers)
    n_cmp, n_ex = compare_teacher_forced(inp, g, 0.8, logit_scale, steps=steps)
    assert n_cmp > 0 and n_ex <= 2, (n_cmp, n_ex)


def test_loop_layers_one_layer_is_the_single_layer_call():
    d = tt_inputs.workload("tiny", B=2, precommit=("uniform", 0.0, 0.75))
    inp = tt_inputs.generate(d, seed=48)
    a = run_loop_gpu(d, inp, 0.5, 40.0)
    b = run_loop_layers_gpu(d, inp, 1, 0.5, 40.0)
    for k in ("tokens", "masked", "steps_taken", "commit_step"):
        np.testing.assert_array_equal(a[k], b[k])


def test_loop_layers_mid_shape_sampled_sequences():
    d = tt_inputs.workload("mid")
    inp = tt_inputs.generate(d, seed=2, n_layers=2)
    g = run_loop_layers_gpu(d, inp, 2, 0.8, 8.0)
    check_invariants(d, inp, g)
    steps = stepwise_equals_single_call(d, inp, 0.8, 8.0, g, n_layers=2, bsel=[1, 6])
    n_cmp, n_ex = compare_teacher_forced(inp, g, 0.8, 8.0, bsel=np.array([1, 6]), steps=steps)
    print(f"mid 2-layer loop: compared {n_cmp} sequence-steps, excluded {n_ex}")
    assert n_cmp > 0 and n_ex <= 2


@pytest.mark.parametrize("logit_scale", [1.0, 12.0])
def test_decode_blocks_block_after_block(logit_scale):
    """Three blocks one after the other: each committed block joins the
    context.  The oracle follows the GPU's committed tokens block by block;
    appended K/V rows agree within one bf16 unit, each block's steps are
    compared teacher-forced as in the single-block loop."""
    nb = 3
    d = tt_inputs.Dims(B=2, S=16, Hq=4, Hkv=1, dh=64, V=1024, L_cap=256 + nb * 16,
                       ctx=("fixed", 256))
    inp = tt_inputs.generate(d, seed=51)
    D = tt.dims(d)
    kc, vc = G.dev_bf16(inp["k_ctx"]), G.dev_bf16(inp["v_ctx"])
    cl = G.dev(inp["ctx_len"])
    dv = {k: G.dev_bf16(inp[k]) for k in ("emb", "e_mask", "u_t", "shift_scale", "w", "u_ctx")}
    tokens = torch.empty((nb, d.B, d.S), dtype=torch.int32, device="cuda")
    steps = torch.empty((nb, d.B), dtype=torch.int32, device="cuda")
    cstep = torch.empty((nb, d.B, d.S), dtype=torch.int32, device="cuda")
    ws = G.workspace(D, tt.TT_WS_LOOP)
    n = tt.tt_decode_blocks(D, nb, kc, vc, cl, dv["emb"], dv["e_mask"], dv["u_t"],
                            dv["shift_scale"], dv["w"], dv["u_ctx"], 0.8, logit_scale, tokens,
                            steps, cstep, ws)
    np.testing.assert_array_equal(cl.cpu().numpy(), [256 + nb * 16] * d.B)
    gt, gs, gc = tokens.cpu().numpy(), steps.cpu().numpy(), cstep.cpu().numpy()
    assert n == int(gs.max(axis=1).sum())
    f = O.from_bf16
    k64, v64, u = f(inp["k_ctx"]), f(inp["v_ctx"]), f(inp["u_ctx"])
    L = np.array(inp["ctx_len"], dtype=np.int64)
    n_cmp = n_ex = 0
    for j in range(nb):
        blk = dict(inp, k_ctx=O._to_bits(k64), v_ctx=O._to_bits(v64), ctx_len=L.astype(np.int32),
                   tokens=np.full((d.B, d.S), -1, np.int32), masked=np.ones((d.B, d.S), np.uint8))
        g = dict(tokens=gt[j], masked=np.zeros((d.B, d.S), np.uint8), steps_taken=gs[j],
                 commit_step=gc[j], steps_run=int(gs[j].max()))
        check_invariants(d, blk, g)
        c, e = compare_teacher_forced(blk, g, 0.8, logit_scale)
        n_cmp, n_ex = n_cmp + c, n_ex + e
        L = O.append_block(k64, v64, L, gt[j].astype(np.int64), inp["emb"], u)
    assert n_cmp > 0 and n_ex <= 3, (n_cmp, n_ex)
    for got, ref in ((G.host_f64(kc), k64), (G.host_f64(vc), v64)):
        new = got[:, :, 256:], ref[:, :, 256:]
        np.testing.assert_allclose(new[0], new[1], rtol=2 ** -8, atol=1e-6)
        np.testing.assert_array_equal(got[:, :, :256], ref[:, :, :256])
