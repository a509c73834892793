"""Pins of the float64 oracle against things other than itself.

Closed forms, explicit-loop brute force, invariants, library routines
(scipy softmax, torch's bf16 conversion) and the hand-worked commit example
in tests/golden/.  No GPU needed.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

from oracle import twotower_oracle as O
import tt_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# ---------------------------------------------------------------- bf16 format
def test_round_bf16_ties_and_specials():
    one = 1.0
    ulp = 2.0 ** -7
    assert O.round_bf16(np.array([one + ulp / 2]))[0] == one                # tie -> even (1.0)
    assert O.round_bf16(np.array([one + 1.5 * ulp]))[0] == one + 2 * ulp    # tie -> even
    assert O.round_bf16(np.array([one + 0.51 * ulp]))[0] == one + ulp
    assert O.round_bf16(np.array([-3.0]))[0] == -3.0
    assert O.round_bf16(np.array([0.0]))[0] == 0.0
    assert O.round_bf16(np.array([1e39]))[0] == np.inf
    assert O.round_bf16(np.array([2.0 ** -130]))[0] == 2.0 ** -130          # subnormal, exact
    # bf16 subnormals are spaced 2^-133 (7 stored bits below 2^-126): ties go to even
    sub = 2.0 ** -133
    assert O.round_bf16(np.array([1.5 * sub]))[0] == 2 * sub
    assert O.round_bf16(np.array([2.5 * sub]))[0] == 2 * sub
    assert O.round_bf16(np.array([0.75 * sub]))[0] == sub
    assert O.round_bf16(np.array([0.5 * sub]))[0] == 0.0                   # tie -> even (0)
    assert O.round_bf16(np.array([2.0 ** -126 + 0.5 * sub]))[0] == 2.0 ** -126


def test_round_bf16_matches_torch_and_input_module():
    x32 = (rnd(20000, 1) * np.exp(rnd(20000, 2) * 8)).astype(np.float32)
    mine = O.round_bf16(x32.astype(np.float64))
    ref_torch = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    ref_inputs = O.from_bf16(tt_inputs.bf16_bits(x32))
    np.testing.assert_array_equal(mine, ref_torch)
    np.testing.assert_array_equal(mine, ref_inputs)
    # float32 values around and below the smallest normal bf16 (2^-126)
    tiny = (np.sign(rnd(20000, 3)) * 2.0 ** (-150 + 30 * np.random.default_rng(4).random(20000))
            ).astype(np.float32)
    ref_tiny = torch.from_numpy(tiny).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.round_bf16(tiny.astype(np.float64)), ref_tiny)


def test_from_bf16_exact():
    bits = np.array([0x3F80, 0xBF80, 0x4000, 0x0000, 0x3F81, 0x7F80], dtype=np.uint16)
    np.testing.assert_array_equal(O.from_bf16(bits), [1.0, -1.0, 2.0, 0.0, 1.0 + 2 ** -7, np.inf])


# ------------------------------------------------------------------ attention
def _attn_inputs(B, S, Hq, Hkv, dh, L, seed=0, scale=1.0):
    q = rnd((B, S, Hq, dh), seed, scale)
    kb = rnd((B, S, Hkv, dh), seed + 1, scale)
    vb = rnd((B, S, Hkv, dh), seed + 2)
    kc = rnd((B, Hkv, L, dh), seed + 3, scale)
    vc = rnd((B, Hkv, L, dh), seed + 4)
    return q, kb, vb, kc, vc


def test_attention_matches_explicit_loops():
    q, kb, vb, kc, vc = _attn_inputs(2, 3, 4, 2, 5, 6, seed=10)
    ctx_len = np.array([4, 0])
    a = O.block_attention(q, kb, vb, kc, vc, ctx_len)
    b = O.block_attention_loops(q, kb, vb, kc, vc, ctx_len)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


def test_attention_hand_example_joint_softmax_and_scale():
    # dh = 4: one context key with score 2*1/sqrt(4) = 1, one block key with
    # score 0.  Joint softmax gives weights e/(e+1) and 1/(e+1).
    q = np.zeros((1, 1, 1, 4)); q[0, 0, 0, 0] = 2.0
    kc = np.zeros((1, 1, 1, 4)); kc[0, 0, 0, 0] = 1.0
    kb = np.zeros((1, 1, 1, 4))
    vc = np.zeros((1, 1, 1, 4)); vc[0, 0, 0, 0] = 1.0
    vb = np.zeros((1, 1, 1, 4)); vb[0, 0, 0, 1] = 1.0
    o = O.block_attention(q, kb, vb, kc, vc, np.array([1]))
    e = math.e
    np.testing.assert_allclose(o[0, 0, 0], [e / (e + 1), 1 / (e + 1), 0, 0], rtol=1e-14)


def test_attention_closed_forms():
    # no context, one block position: the only key is the block's own -> o = v
    q, kb, vb, kc, vc = _attn_inputs(1, 1, 4, 2, 8, 3, seed=3)
    o = O.block_attention(q, kb, vb, kc, vc, np.array([0]))
    for h in range(4):
        np.testing.assert_allclose(o[0, 0, h], vb[0, 0, h // 2], rtol=1e-14)
    # all keys equal -> uniform weights -> mean of the values
    q, kb, vb, kc, vc = _attn_inputs(1, 4, 2, 1, 8, 5, seed=4)
    kb[:] = 0.3
    kc[:] = 0.3
    o = O.block_attention(q, kb, vb, kc, vc, np.array([5]))
    allv = np.concatenate([vc[0, 0], vb[0, :, 0]])
    np.testing.assert_allclose(o[0, 2, 1], allv.mean(axis=0), rtol=1e-12)


def test_attention_block_permutation_equivariance():
    q, kb, vb, kc, vc = _attn_inputs(2, 6, 4, 2, 8, 7, seed=5, scale=2.0)
    ctx_len = np.array([7, 3])
    o = O.block_attention(q, kb, vb, kc, vc, ctx_len)
    perm = np.random.default_rng(0).permutation(6)
    o2 = O.block_attention(q[:, perm], kb[:, perm], vb[:, perm], kc, vc, ctx_len)
    np.testing.assert_allclose(o2, o[:, perm], rtol=1e-12, atol=1e-13)


def test_attention_context_permutation_and_tail_ignored():
    q, kb, vb, kc, vc = _attn_inputs(1, 4, 4, 2, 8, 9, seed=6, scale=2.0)
    o = O.block_attention(q, kb, vb, kc, vc, np.array([6]))
    perm = np.random.default_rng(1).permutation(6)
    kc2, vc2 = kc.copy(), vc.copy()
    kc2[:, :, :6] = kc[:, :, perm]
    vc2[:, :, :6] = vc[:, :, perm]
    kc2[:, :, 6:] = 1e3        # rows past ctx_len must not matter
    vc2[:, :, 6:] = np.nan
    o2 = O.block_attention(q, kb, vb, kc2, vc2, np.array([6]))
    np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-13)


def test_attention_gqa_grouping_and_own_layer_only():
    B, S, Hq, Hkv, dh, L = 1, 3, 8, 2, 4, 5
    q, kb, vb, kc, vc = _attn_inputs(B, S, Hq, Hkv, dh, L, seed=7)
    o = O.block_attention(q, kb, vb, kc, vc, np.array([L]))
    kc2, vb2 = kc.copy(), vb.copy()
    kc2[:, 1] += 1.0
    vb2[:, :, 1] -= 0.5
    o2 = O.block_attention(q, kb, vb2, kc2, vc, np.array([L]))
    np.testing.assert_array_equal(o2[:, :, :4], o[:, :, :4])   # heads 0..3 read KV head 0
    assert np.all(np.abs(o2[:, :, 4:] - o[:, :, 4:]).max(axis=-1) > 1e-6)
    # two layers: layer 0's output depends on layer 0's K/V only
    layers = [_attn_inputs(B, S, Hq, Hkv, dh, L, seed=s) for s in (20, 30)]
    ref = O.block_attention(*layers[0], np.array([L]))
    pert = [a.copy() for a in layers[1]]
    pert[3] *= -1
    _ = O.block_attention(*pert, np.array([L]))
    np.testing.assert_array_equal(O.block_attention(*layers[0], np.array([L])), ref)


# ----------------------------------------------------------------------- adaLN
def test_timestep_embedding_closed_form():
    H = 64
    t = 0.37
    phi = O.timestep_embedding(t, H)
    assert phi.shape == (2 * H,)
    assert phi[0] == pytest.approx(math.sin(t))
    assert phi[H] == pytest.approx(math.cos(t))
    assert phi[H // 2] == pytest.approx(math.sin(t * 0.01))          # 10000^(-1/2)
    assert phi[H + H // 4] == pytest.approx(math.cos(t * 0.1))       # 10000^(-1/4)
    z = O.timestep_embedding(0.0, H)
    np.testing.assert_array_equal(z[:H], 0.0)
    np.testing.assert_array_equal(z[H:], 1.0)


def test_adaln_closed_forms():
    H = 256
    x = rnd((5, H), 11, 3.0) + 2.0
    E = np.zeros((2, H))
    y = O.adaln_modulate(x, E, np.zeros(5))       # t = 0: shift 0, scale 1 -> 2 LN(x)
    ln = y / 2
    np.testing.assert_allclose(ln.mean(axis=1), 0, atol=1e-12)
    var = x.var(axis=1)
    np.testing.assert_allclose((ln ** 2).mean(axis=1), var / (var + O.LN_EPS), rtol=1e-12)
    # affine invariance of LN: a*x + c gives the same output (up to eps)
    y2 = O.adaln_modulate(4.0 * x - 7.0, E, np.zeros(5))
    np.testing.assert_allclose(y2, y, atol=1e-6)
    # constant row: LN = 0 so y = shift = E0 + sin(t w)
    E = rnd((2, H), 12)
    t = np.array([0.25])
    yc = O.adaln_modulate(np.full((1, H), 1.5), E, t)
    phi = O.timestep_embedding(0.25, H)
    np.testing.assert_allclose(yc[0], E[0] + phi[:H], rtol=1e-12, atol=1e-12)
    # shift and scale rows are not swapped: scale multiplies, shift adds
    x1 = rnd((1, H), 13)
    y1 = O.adaln_modulate(x1, E, np.array([0.0]))
    n = (x1 - x1.mean()) / np.sqrt(x1.var() + O.LN_EPS)
    np.testing.assert_allclose(y1, n * (2.0 + E[1]) + E[0], rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------ confidence/argmax
def test_confidence_matches_scipy_and_ties():
    lg = rnd((7, 300), 14, 3.0)
    conf, tok = O.confidence(lg)
    p = scipy.special.softmax(lg, axis=-1)
    np.testing.assert_allclose(conf, p.max(axis=-1), rtol=1e-13)
    np.testing.assert_array_equal(tok, p.argmax(axis=-1))
    lg2 = np.zeros((1, 10)); lg2[0, [3, 7]] = 2.0
    c2, t2 = O.confidence(lg2)
    assert t2[0] == 3
    np.testing.assert_allclose(c2[0], math.e ** 2 / (2 * math.e ** 2 + 8))
    c3, _ = O.confidence(np.zeros((1, 1024)))
    assert c3[0] == pytest.approx(1 / 1024)


def test_logits_orientation_and_scale():
    V, H = 50, 16
    w = rnd((V, H), 15)
    y = np.zeros((1, H)); y[0, 5] = 1.0
    np.testing.assert_allclose(O.logits(y, w, 2.5)[0], 2.5 * w[:, 5])
    wb = tt_inputs.bf16_bits(w.astype(np.float32))
    yr = rnd((3, H), 16)
    conf, tok, gl, gp = O.vocab_confidence(yr, wb, 3.0, rows_per_block=2)
    p = scipy.special.softmax(3.0 * yr @ O.from_bf16(wb).T, axis=-1)
    np.testing.assert_allclose(conf, p.max(axis=-1), rtol=1e-12)
    ps = np.sort(p, axis=-1)
    np.testing.assert_allclose(gp, ps[:, -1] - ps[:, -2], rtol=1e-9, atol=1e-15)
    ls = np.sort(3.0 * yr @ O.from_bf16(wb).T, axis=-1)
    np.testing.assert_allclose(gl, ls[:, -1] - ls[:, -2], rtol=1e-12, atol=1e-15)
    assert (gl >= 0).all()


# --------------------------------------------------------------------- commit
def _golden():
    with open(os.path.join(GOLDEN, "commit_example.json")) as f:
        return json.load(f)


def test_commit_golden_example():
    g = _golden()
    tokens = np.array([[-1, -1]])
    masked = np.array([[1, 1]], dtype=bool)
    for st in g["steps"]:
        np.testing.assert_array_equal(masked[0].astype(int), st["masked_before"])
        lg = np.array(st["logits"])
        conf, tok = O.confidence(lg)
        for s in range(2):
            if st["probs"][s] is not None:
                np.testing.assert_allclose(scipy.special.softmax(lg[s]), st["probs"][s], atol=1e-6)
                assert conf[s] == pytest.approx(st["conf"][s], abs=1e-6)
                assert tok[s] == st["tok"][s]
        conf = np.where(masked[0], conf, np.nan)
        tokens, masked, committed, fb = O.commit(conf[None], tok[None], tokens, masked, g["gamma"])
        np.testing.assert_array_equal(committed[0].astype(int), st["committed"])
        assert bool(fb[0]) == st["fallback"]
    np.testing.assert_array_equal(tokens[0], g["final_tokens"])
    assert not masked.any()


def test_commit_golden_variants():
    g = _golden()
    lg = np.array(g["steps"][0]["logits"])
    conf, tok = O.confidence(lg)
    v = g["variant_gamma_0_7"]
    t, m, c, _ = O.commit(conf[None], tok[None], np.array([[-1, -1]]), np.ones((1, 2), bool), v["gamma"])
    np.testing.assert_array_equal(t[0], v["final_tokens_step1"])
    np.testing.assert_array_equal(c[0].astype(int), v["committed_step1"])
    v = g["variant_fallback"]
    _, _, c, fb = O.commit(np.array([v["conf"]]), np.array([[0, 0]]), np.array([[-1, -1]]),
                           np.ones((1, 2), bool), v["gamma"])
    assert fb[0] and c[0, v["chosen"]] and c.sum() == 1
    v = g["variant_tie"]
    conf, tok = O.confidence(np.array([v["logits"]]))
    assert tok[0] == v["tok"] and conf[0] == pytest.approx(v["p_top"], abs=1e-6)
    _, gp = O.top2_margin(np.array([v["logits"]]))
    assert gp[0] == pytest.approx(v["top2_prob_gap"], abs=1e-15)


def test_commit_invariants_random():
    rng = np.random.default_rng(17)
    for trial in range(200):
        B, S = 3, 8
        masked = rng.random((B, S)) < 0.6
        tokens = np.where(masked, -1, rng.integers(0, 100, (B, S)))
        conf = rng.random((B, S))
        if trial % 3 == 0:
            conf[:, :4] = conf[:, :1]                     # planted ties
        tok = rng.integers(0, 100, (B, S))
        gamma = rng.choice([0.5, 0.8, 0.95])
        if trial % 4 == 1:
            conf[:, 4:6] = gamma                          # exactly at the threshold: commits
        t2, m2, c, fb = O.commit(conf, tok, tokens, masked, gamma)
        assert not np.any(c & ~masked)                      # only masked positions commit
        np.testing.assert_array_equal(t2[~masked], tokens[~masked])   # committed never change
        for b in range(B):
            if masked[b].any():
                assert c[b].sum() >= 1                      # progress every step
                if (conf[b][masked[b]] >= gamma).any():
                    np.testing.assert_array_equal(c[b], masked[b] & (conf[b] >= gamma))
                else:
                    cand = np.where(masked[b])[0]
                    best = cand[np.argmax(conf[b][cand])]   # first max = lowest position
                    assert c[b].sum() == 1 and c[b, best]
        np.testing.assert_array_equal(m2, masked & ~c)


# ------------------------------------------------------------ embed / update
def test_embed_and_linear_update_orientation():
    B, S, Hq, Hkv, dh = 1, 3, 2, 1, 4
    H = Hq * dh
    n_qkv = H + 2 * Hkv * dh
    emb = tt_inputs.bf16_bits(rnd((10, H), 18).astype(np.float32))
    e_mask = tt_inputs.bf16_bits(rnd((H,), 19).astype(np.float32))
    tokens = np.array([[4, -1, 7]])
    masked = np.array([[0, 1, 0]], dtype=bool)
    e = O.embed_block(tokens, masked, emb, e_mask)
    np.testing.assert_array_equal(e[0, 0], O.from_bf16(emb[4]))
    np.testing.assert_array_equal(e[0, 1], O.from_bf16(e_mask))
    # u_t rows pick coordinates: output column j of [q|k|v] = e[:, j % H]
    u_t = np.zeros((n_qkv, H))
    for j in range(n_qkv):
        u_t[j, j % H] = 1.0
    q, k, v = O.linear_update(e, u_t, Hq, Hkv, dh)
    np.testing.assert_array_equal(q.reshape(B, S, H), e)
    np.testing.assert_array_equal(k.reshape(B, S, -1), e[..., :Hkv * dh])
    np.testing.assert_array_equal(v.reshape(B, S, -1), e[..., Hkv * dh:2 * Hkv * dh])


# ----------------------------------------------------------------------- loop
def _tiny_loop_inputs(seed=0, **kw):
    d = tt_inputs.workload("tiny", **kw)
    return d, tt_inputs.generate(d, seed)


def test_loop_invariants_canonical_scale():
    d, inp = _tiny_loop_inputs(B=2)
    r = O.denoise_block_loop(inp, gamma=0.8)
    assert not r["masked"].any()
    prev_tok, prev_m = inp["tokens"], inp["masked"].astype(bool)
    for st in r["trace"]:
        # at V = 1024 and unit logit scale no confidence gets near 0.8, so the
        # fallback commits exactly one position per sequence per step
        assert np.nanmax(st["conf"]) < 0.5
        np.testing.assert_array_equal(st["committed"].sum(axis=1), prev_m.any(axis=1).astype(int))
        np.testing.assert_array_equal(st["tokens"][~prev_m], prev_tok[~prev_m])
        prev_tok, prev_m = st["tokens"], st["masked"]
    np.testing.assert_array_equal(r["steps_taken"], [16, 16])
    # with nothing to tell masked positions apart (no positional signal) they
    # tie, and the lowest position commits first
    np.testing.assert_array_equal(r["commit_step"], np.tile(np.arange(16), (2, 1)))


def test_loop_multi_commit_and_resume():
    d, inp = _tiny_loop_inputs(B=2, precommit=("uniform", 0.0, 0.75))
    r = O.denoise_block_loop(inp, gamma=0.5, logit_scale=40.0)
    n0 = inp["masked"].sum(axis=1)
    assert np.all(r["steps_taken"] <= n0)
    assert np.all(r["steps_taken"] >= 1)
    assert any(st["committed"].sum() > 2 for st in r["trace"])  # several commits in one step
    pre = ~inp["masked"].astype(bool)
    np.testing.assert_array_equal(r["tokens"][pre], inp["tokens"][pre])
    np.testing.assert_array_equal(r["commit_step"][pre], -1)
    # resume: stop after 1 step, restart from that state, same final tokens
    r1 = O.denoise_block_loop(inp, gamma=0.5, logit_scale=40.0, max_steps=1)
    inp2 = dict(inp, tokens=r1["tokens"], masked=r1["masked"].astype(np.uint8))
    r2 = O.denoise_block_loop(inp2, gamma=0.5, logit_scale=40.0)
    np.testing.assert_array_equal(r2["tokens"], r["tokens"])


def test_loop_autoregressive_s1_single_step():
    """S = 1 (the autoregressive baseline): the loop takes exactly one step,
    t = 1, and commits the argmax of that step's logits, whose attention is
    one softmax over the context keys and the position's own key."""
    d = tt_inputs.Dims(B=3, S=1, Hq=4, Hkv=1, dh=64, V=1024, L_cap=64, ctx=("fixed", 64))
    inp = tt_inputs.generate(d, seed=5)
    r = O.denoise_block_loop(inp, gamma=0.8)
    assert len(r["trace"]) == 1
    st = r["trace"][0]
    np.testing.assert_array_equal(r["steps_taken"], [1, 1, 1])
    np.testing.assert_array_equal(r["commit_step"], np.zeros((3, 1), dtype=r["commit_step"].dtype))
    np.testing.assert_array_equal(st["t"], [1.0, 1.0, 1.0])
    np.testing.assert_array_equal(r["tokens"][:, 0], st["tok"][:, 0])
    # the attention of that step, by explicit loops over the L + 1 keys
    f = O.from_bf16
    e = O.embed_block(inp["tokens"], inp["masked"], inp["emb"], inp["e_mask"])
    q, k, v = O.linear_update(e, f(inp["u_t"]), d.Hq, d.Hkv, d.dh)
    kc, vc = f(inp["k_ctx"]), f(inp["v_ctx"])
    for b in range(d.B):
        for h in range(d.Hq):
            keys = [kc[b, 0, j] for j in range(d.L_cap)] + [k[b, 0, 0]]
            vals = [vc[b, 0, j] for j in range(d.L_cap)] + [v[b, 0, 0]]
            sc = [float(np.dot(q[b, 0, h], kk)) / np.sqrt(d.dh) for kk in keys]
            mx = max(sc)
            w = [np.exp(x - mx) for x in sc]
            o = sum(wi * vi for wi, vi in zip(w, vals)) / sum(w)
            np.testing.assert_allclose(st["o"][b, 0, h * d.dh:(h + 1) * d.dh],
                                       O.round_bf16(o), rtol=0, atol=2 ** -8 * np.abs(o).max())


def _stack_one_layer(inp):
    out = dict(inp)
    for n in tt_inputs.LAYER_NAMES:
        out[n + "_l"] = inp[n][None]
    return out


def test_layers_one_layer_stack_equals_single_layer_loop():
    d, inp = _tiny_loop_inputs(B=2, precommit=("uniform", 0.0, 0.75))
    a = O.denoise_block_loop(inp, 0.5, 40.0)
    b = O.denoise_block_loop(_stack_one_layer(inp), 0.5, 40.0)
    np.testing.assert_array_equal(a["tokens"], b["tokens"])
    np.testing.assert_array_equal(a["commit_step"], b["commit_step"])


def test_layers_depend_only_on_their_own_context():
    d = tt_inputs.workload("tiny", B=2)
    inp = tt_inputs.generate(d, seed=7, n_layers=2)
    f = O.from_bf16
    layers = [tuple(f(inp[n + "_l"][i]) for n in ("u_t", "k_ctx", "v_ctx", "shift_scale"))
              for i in range(2)]
    e = O.embed_block(inp["tokens"], inp["masked"], inp["emb"], inp["e_mask"])
    t = inp["masked"].sum(axis=1) / d.S
    x1 = O.denoiser_layers(e, layers[:1], inp["ctx_len"], t, d.Hq, d.Hkv, d.dh)
    # layer 1's context has no effect on layer 0's output ...
    bumped = list(layers)
    bumped[1] = (layers[1][0], layers[1][1] + 1.0, layers[1][2] - 1.0, layers[1][3])
    np.testing.assert_array_equal(
        x1, O.denoiser_layers(e, bumped[:1], inp["ctx_len"], t, d.Hq, d.Hkv, d.dh))
    # ... and layer 0's context beyond ctx_len has none either
    kc = layers[0][1].copy()
    kc[:, :, d.L_cap // 2:] = 0.0
    short = np.full(d.B, d.L_cap // 2, dtype=np.int32)
    half = [(layers[0][0], kc, layers[0][2], layers[0][3])]
    np.testing.assert_array_equal(
        O.denoiser_layers(e, layers[:1], short, t, d.Hq, d.Hkv, d.dh),
        O.denoiser_layers(e, half, short, t, d.Hq, d.Hkv, d.dh))
    # while the last layer's context does move the final confidences
    r = O.denoise_block_loop(inp, 0.8, max_steps=1)
    inp2 = dict(inp, v_ctx_l=inp["v_ctx_l"].copy())
    inp2["v_ctx_l"][1] = tt_inputs.bf16_bits(-O.from_bf16(inp["v_ctx_l"][1]).astype(np.float32))
    r2 = O.denoise_block_loop(inp2, 0.8, max_steps=1)
    assert not np.allclose(r["trace"][0]["conf"], r2["trace"][0]["conf"])


def test_step_sequences_are_independent():
    """One step over a batch whose sequences differ in mask (hence t), context
    length and tokens gives, per sequence, what that sequence gives alone."""
    d = tt_inputs.workload("tiny", B=3)
    inp = tt_inputs.generate(d, seed=6)
    f = O.from_bf16
    masked = np.ones((d.B, d.S), dtype=bool)
    masked[1, :5] = False
    masked[2, 3:15] = False
    tokens = np.where(masked, -1, 9)
    cl = np.array([256, 100, 17])
    e = O.embed_block(tokens, masked, inp["emb"], inp["e_mask"])
    q, k, v = O.linear_update(e, f(inp["u_t"]), d.Hq, d.Hkv, d.dh)
    kc, vc, E, w = f(inp["k_ctx"]), f(inp["v_ctx"]), f(inp["shift_scale"]), f(inp["w"])
    args = (E, w)
    both = O.denoise_step(q, k, v, kc, vc, cl, *args, tokens, masked, 0.8, 12.0)
    for b in range(d.B):
        sl = slice(b, b + 1)
        one = O.denoise_step(q[sl], k[sl], v[sl], kc[sl], vc[sl], cl[sl], *args, tokens[sl],
                             masked[sl], 0.8, 12.0)
        for key in ("o", "y", "conf", "tok", "tokens", "masked", "committed"):
            np.testing.assert_array_equal(both[key][sl], one[key], err_msg=f"{key} of {b}")


def test_layers_sequences_are_independent():
    """A batch of sequences with different times t gives, row for row, what
    each sequence gives alone: a row is modulated by its own sequence's t."""
    d = tt_inputs.workload("tiny", B=3)
    inp = tt_inputs.generate(d, seed=5, n_layers=2)
    f = O.from_bf16
    layers = [tuple(f(inp[n + "_l"][i]) for n in ("u_t", "k_ctx", "v_ctx", "shift_scale"))
              for i in range(1)]
    masked = np.ones((d.B, d.S), dtype=bool)
    masked[1, :5] = False
    masked[2, :12] = False
    tokens = np.where(masked, -1, 3)
    e = O.embed_block(tokens, masked, inp["emb"], inp["e_mask"])
    t = masked.sum(axis=1) / d.S
    assert len(set(t)) == 3
    cl = np.array([256, 100, 17])
    both = O.denoiser_layers(e, layers, cl, t, d.Hq, d.Hkv, d.dh)
    for b in range(d.B):
        one = [(u, kc[b:b + 1], vc[b:b + 1], E) for u, kc, vc, E in layers]
        np.testing.assert_array_equal(
            both[b:b + 1], O.denoiser_layers(e[b:b + 1], one, cl[b:b + 1], t[b:b + 1],
                                             d.Hq, d.Hkv, d.dh))


def test_loop_wires_each_layer_to_its_own_tables():
    """Step 0 of a two-layer loop is layer 0 (its own U, context and adaLN
    table) followed by the single-layer step on layer 1's tables; layer 0's
    context moves the result."""
    d = tt_inputs.workload("tiny", B=2)
    inp = tt_inputs.generate(d, seed=11, n_layers=2)
    f = O.from_bf16
    per = [{n: f(inp[n + "_l"][i]) for n in ("u_t", "k_ctx", "v_ctx", "shift_scale")}
           for i in range(2)]
    r = O.denoise_block_loop(inp, 0.8, 8.0, max_steps=1)
    e = O.embed_block(inp["tokens"], inp["masked"], inp["emb"], inp["e_mask"])
    t = inp["masked"].sum(axis=1) / d.S
    l0 = per[0]
    x = O.denoiser_layers(e, [(l0["u_t"], l0["k_ctx"], l0["v_ctx"], l0["shift_scale"])],
                          inp["ctx_len"], t, d.Hq, d.Hkv, d.dh)
    l1 = per[1]
    q, k, v = O.linear_update(x, l1["u_t"], d.Hq, d.Hkv, d.dh)
    st = O.denoise_step(q, k, v, l1["k_ctx"], l1["v_ctx"], inp["ctx_len"], l1["shift_scale"],
                        f(inp["w"]), inp["tokens"], inp["masked"], 0.8, 8.0)
    np.testing.assert_array_equal(r["trace"][0]["conf"], st["conf"])
    np.testing.assert_array_equal(r["tokens"], st["tokens"])
    inp2 = dict(inp, v_ctx_l=inp["v_ctx_l"].copy())
    inp2["v_ctx_l"][0] = tt_inputs.bf16_bits(-f(inp["v_ctx_l"][0]).astype(np.float32))
    r2 = O.denoise_block_loop(inp2, 0.8, 8.0, max_steps=1)
    assert not np.allclose(r["trace"][0]["conf"], r2["trace"][0]["conf"], equal_nan=True)


def test_layer_by_explicit_loops():
    """One denoiser layer (all rows) against explicit loops: scores, softmax,
    LayerNorm and the sinusoidal modulation written out element by element."""
    d = tt_inputs.Dims(B=1, S=2, Hq=2, Hkv=1, dh=4, V=8, L_cap=3, ctx=("fixed", 3))
    inp = tt_inputs.generate(d, seed=9, n_layers=2)
    f = O.from_bf16
    u, kc, vc, E = (f(inp[n + "_l"][0]) for n in ("u_t", "k_ctx", "v_ctx", "shift_scale"))
    inp["masked"][0, 1] = 0
    inp["tokens"][0, 1] = 5
    e = O.embed_block(inp["tokens"], inp["masked"], inp["emb"], inp["e_mask"])
    t = np.array([0.5])
    got = O.denoiser_layers(e, [(u, kc, vc, E)], inp["ctx_len"], t, d.Hq, d.Hkv, d.dh)
    H, dh = d.H, d.dh
    for s in range(d.S):
        row = [O.round_bf16(sum(e[0, s, i] * u[j, i] for i in range(H))) for j in range(u.shape[0])]
        o = []
        for h in range(d.Hq):
            q = row[h * dh:(h + 1) * dh]
            keys = [list(kc[0, 0, j]) for j in range(3)]
            vals = [list(vc[0, 0, j]) for j in range(3)]
            for s2 in range(d.S):
                r2 = [O.round_bf16(sum(e[0, s2, i] * u[jj, i] for i in range(H)))
                      for jj in range(u.shape[0])]
                keys.append(r2[H:H + dh])
                vals.append(r2[H + dh:H + 2 * dh])
            sc = [sum(q[c] * kv[c] for c in range(dh)) / np.sqrt(dh) for kv in keys]
            mx = max(sc)
            w = [np.exp(x - mx) for x in sc]
            o += [O.round_bf16(sum(w[j] * vals[j][c] for j in range(len(w))) / sum(w))
                  for c in range(dh)]
        mean = sum(o) / H
        var = sum((x - mean) ** 2 for x in o) / H
        for i in range(H):
            om = 10000.0 ** (-i / H)
            y = (o[i] - mean) / np.sqrt(var + 1e-6) * (1 + E[1, i] + np.cos(0.5 * om)) \
                + E[0, i] + np.sin(0.5 * om)
            assert abs(got[0, s, i] - O.round_bf16(y)) <= 2 ** -7 * max(1.0, abs(y)), (s, i)


def _blocks_inputs(seed=3, B=2, n_room=3):
    d = tt_inputs.Dims(B=B, S=16, Hq=4, Hkv=1, dh=64, V=1024, L_cap=256 + 16 * n_room,
                       ctx=("fixed", 256))
    return d, tt_inputs.generate(d, seed=seed)


def test_append_block_writes_the_projection_and_nothing_else():
    d, inp = _blocks_inputs()
    f = O.from_bf16
    kc, vc, u = f(inp["k_ctx"]), f(inp["v_ctx"]), f(inp["u_ctx"])
    kc0, vc0 = kc.copy(), vc.copy()
    L = np.array([256, 100])
    tok = np.arange(d.B * d.S).reshape(d.B, d.S) * 7 % d.V
    new = O.append_block(kc, vc, L, tok, inp["emb"], u)
    np.testing.assert_array_equal(new, L + d.S)
    for b in range(d.B):
        for s in (0, d.S - 1):
            e = f(inp["emb"][tok[b, s]])
            for c in (0, 17, d.dh - 1):
                kk = sum(e[i] * u[c, i] for i in range(d.H))
                vv = sum(e[i] * u[d.Hkv * d.dh + c, i] for i in range(d.H))
                assert kc[b, 0, L[b] + s, c] == O.round_bf16(kk)
                assert vc[b, 0, L[b] + s, c] == O.round_bf16(vv)
    # outside [L_b, L_b + S) the cache is untouched
    for b in range(d.B):
        keep = np.ones(d.L_cap, bool)
        keep[L[b]:L[b] + d.S] = False
        np.testing.assert_array_equal(kc[b, :, keep], kc0[b, :, keep])
        np.testing.assert_array_equal(vc[b, :, keep], vc0[b, :, keep])
    with pytest.raises(ValueError):
        O.append_block(kc, vc, np.array([d.L_cap - 3, 0]), tok, inp["emb"], u)


def test_decode_blocks_first_block_is_the_block_loop_and_contexts_grow():
    d, inp = _blocks_inputs()
    r = O.decode_blocks(inp, 3, 0.8)
    single = O.denoise_block_loop(inp, 0.8)
    np.testing.assert_array_equal(r["tokens"][0], single["tokens"])
    np.testing.assert_array_equal(r["ctx_len"], [256 + 3 * 16] * 2)
    # block 1 saw block 0: its first step's attention over the grown context
    b1 = r["blocks"][1]["trace"][0]
    kc = O.from_bf16(inp["k_ctx"]).copy()
    vc = O.from_bf16(inp["v_ctx"]).copy()
    L = O.append_block(kc, vc, inp["ctx_len"], r["tokens"][0], inp["emb"], O.from_bf16(inp["u_ctx"]))
    o = O.round_bf16(O.block_attention(b1["q"], b1["k"], b1["v"], kc, vc, L))
    np.testing.assert_array_equal(b1["o"], o.reshape(b1["o"].shape))
