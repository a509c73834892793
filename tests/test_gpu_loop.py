"""Parity of tt_denoise_block_loop with the oracle's loop, step by step.

The oracle is teacher-forced: at every step it starts from the GPU's state
(rebuilt from commit_step and the final tokens), so one excluded near tie
cannot cascade.  Each step's commit set and committed tokens must then match
bit for bit, outside the near-tie exclusions of tests/_gpu.py.
"""
import numpy as np
import pytest
import torch

import block_wise_diffusion_b200 as tt
import tt_inputs
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


def slice_batch(inp, bsel):
    out = dict(inp)
    for k in ("k_ctx", "v_ctx", "ctx_len", "tokens", "masked"):
        out[k] = inp[k][bsel]
    for k in ("k_ctx_l", "v_ctx_l"):
        if k in inp:
            out[k] = inp[k][:, bsel]
    return out


def compare_teacher_forced(inp, g, gamma, logit_scale, bsel=None):
    """Re-run the oracle from the GPU's state at every step; return counts."""
    if bsel is not None:
        inp = slice_batch(inp, bsel)
        g = {k: (v[bsel] if isinstance(v, np.ndarray) else v) for k, v in g.items()}
    m0 = inp["masked"].astype(bool)
    cs = g["commit_step"]

    def state(step):
        done = (cs >= 0) & (cs < step)
        tok = np.where(done, g["tokens"], inp["tokens"])
        return tok, m0 & ~done

    r = O.denoise_block_loop(inp, gamma, logit_scale, max_steps=int(cs.max()) + 1, teacher=state)
    n_cmp = n_ex = 0
    n_flip = [0]
    for k, st in enumerate(r["trace"]):
        tok_k, m_k = state(k)
        for b in range(m_k.shape[0]):
            if not m_k[b].any():
                continue
            gpu_c = cs[b] == k
            ora_c = st["committed"][b]
            conf = st["conf"][b]
            ex = (m_k[b] & G.derived_excluded_threshold(conf, gamma)).any()
            ex |= (ora_c & G.derived_excluded_argmax(st["gap_l"][b])).any()
            if st["fallback"][b]:
                cb = np.sort(conf[m_k[b]])[::-1]
                ex |= len(cb) > 1 and cb[0] != cb[1] and (cb[0] - cb[1]) / cb[0] < G.TIE_FALLBACK_REL
            if ex:
                n_ex += 1
                continue
            n_cmp += 1
            np.testing.assert_array_equal(gpu_c, ora_c, err_msg=f"step {k} seq {b}")
            for s in np.flatnonzero(ora_c):
                got, want = int(g["tokens"][b][s]), int(st["tok"][b][s])
                if got == want:
                    continue
                # a flip between the oracle's two best tokens at a near tie
                lg = O.logits(st["y"][b, s][None], O.from_bf16(inp["w"]), logit_scale)[0]
                top2 = np.argsort(-lg, kind="stable")[:2]
                gap = lg[top2[0]] - lg[top2[1]]
                assert got in top2 and gap < G.LOOP_TIE_LOGIT * logit_scale, (
                    f"step {k} seq {b} pos {s}: token {got}, oracle top-2 {top2} gap {gap:.3g}")
                n_flip[0] += 1
    if n_flip[0]:
        print(f"near-tie top-2 flips: {n_flip[0]} of {n_cmp} compared sequence-steps")
    return n_cmp, n_ex


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
    n_cmp, n_ex = compare_teacher_forced(inp, g, gamma, logit_scale)
    assert n_cmp > 0 and n_ex <= 2, (n_cmp, n_ex)


@pytest.mark.parametrize("logit_scale", [1.0, 12.0])
def test_loop_autoregressive_step_s1(logit_scale):
    """S = 1: every call commits the block's single position in one step."""
    d = tt_inputs.workload("mid", B=4, S=1, L_cap=300, ctx=("fixed", 300), V=1024)
    inp = tt_inputs.generate(d, seed=41)
    g = run_loop_gpu(d, inp, 0.8, logit_scale)
    check_invariants(d, inp, g)
    assert g["steps_run"] == 1 and np.all(g["steps_taken"] == 1)
    n_cmp, n_ex = compare_teacher_forced(inp, g, 0.8, logit_scale)
    assert n_cmp + n_ex == d.B and n_ex <= 1, (n_cmp, n_ex)


@pytest.mark.parametrize("S,logit_scale", [(128, 1.0), (128, 40.0), (64, 12.0)])
def test_loop_larger_blocks(S, logit_scale):
    d = tt_inputs.workload("tiny", B=2, S=S, precommit=("uniform", 0.0, 0.75))
    inp = tt_inputs.generate(d, seed=43)
    g = run_loop_gpu(d, inp, 0.8, logit_scale)
    check_invariants(d, inp, g)
    n_cmp, n_ex = compare_teacher_forced(inp, g, 0.8, logit_scale)
    assert n_cmp > 0 and n_ex <= 2, (n_cmp, n_ex)


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
    n_cmp, n_ex = compare_teacher_forced(inp, g, 0.8, logit_scale, bsel=np.array([0, 5]))
    print(f"mid loop scale={logit_scale}: compared {n_cmp} sequence-steps, excluded {n_ex}")
    assert n_cmp > 0 and n_ex <= 2


@pytest.mark.parametrize("n_layers,logit_scale", [(2, 1.0), (3, 40.0), (2, 12.0)])
def test_loop_layers_tiny(n_layers, logit_scale):
    d = tt_inputs.workload("tiny", B=3, precommit=("uniform", 0.0, 0.75))
    inp = tt_inputs.generate(d, seed=47, n_layers=n_layers)
    g = run_loop_layers_gpu(d, inp, n_layers, 0.8, logit_scale)
    check_invariants(d, inp, g)
    n_cmp, n_ex = compare_teacher_forced(inp, g, 0.8, logit_scale)
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
    n_cmp, n_ex = compare_teacher_forced(inp, g, 0.8, 8.0, bsel=np.array([1, 6]))
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
