"""Parity of tt_adaln_modulate and tt_vocab_confidence_commit with the oracle.

The vocabulary step is compared stage-wise: the oracle is fed the same bf16
y bytes as the kernel, computes logits in float64 and applies the commit
rule; committed token ids and masks must match bit for bit outside near ties
(see tests/_gpu.py for the exclusion rules; both the literal and the applied
exclusion counts are reported).
"""
import numpy as np
import pytest
import torch

import block_wise_diffusion_b200 as tt
import tt_inputs
from oracle import twotower_oracle as O
from tests import _gpu as G

pytestmark = pytest.mark.gpu


# ---------------------------------------------------------------- adaLN
@pytest.mark.parametrize("wl,B", [("tiny", 1), ("mid", 8), ("ragged32", 3)])
def test_adaln_matches_oracle(wl, B):
    d = tt_inputs.workload(wl, B=B)
    inp = tt_inputs.generate(d, seed=5, names=["shift_scale"])
    rng = np.random.default_rng(5)
    x32 = (rng.standard_normal((d.B * d.S, d.H)) * 0.7 + 0.3).astype(np.float32)
    xb = tt_inputs.bf16_bits(x32)
    t = np.array([0.0, 0.5, 1.0, 0.3125, 0.9][:d.B] + [0.25] * max(0, d.B - 5), np.float32)
    D = tt.dims(d)
    x = G.dev_bf16(xb)
    y = torch.full_like(x, float("nan"))
    ws = G.workspace(D, tt.TT_WS_ADALN)
    tt.tt_adaln_modulate(D, x, G.dev_bf16(inp["shift_scale"]), G.dev(t), y, ws)
    got = G.host_f64(y)
    ref = O.round_bf16(O.adaln_modulate(O.from_bf16(xb), O.from_bf16(inp["shift_scale"]),
                                        np.repeat(t.astype(np.float64), d.S)))
    err = np.abs(got - ref)
    # one bf16 ulp of the result plus fp32 rounding of the statistics
    assert (err <= 2.0 ** -7 * np.maximum(np.abs(ref), 1.0) + 1e-3).all(), err.max()
    assert G.rel_l2(got, ref) < 4e-3


# ---------------------------------------------------- vocab + commit
def _vocab_case(d, seed, logit_scale, gamma, y_scale=1.0, masked=None, w_override=None):
    inp = tt_inputs.generate(d, seed=seed, names=[] if w_override is not None else ["w"])
    wb = w_override if w_override is not None else inp["w"]
    rng = np.random.default_rng(seed)
    rows = d.B * d.S
    yb = tt_inputs.bf16_bits((rng.standard_normal((rows, d.H)) * y_scale).astype(np.float32))
    if masked is None:
        masked = np.ones((d.B, d.S), np.uint8)
    tokens = np.where(masked == 1, -1, rng.integers(0, d.V, (d.B, d.S))).astype(np.int32)
    D = tt.dims(d)
    t_tok, t_m = G.dev(tokens), G.dev(masked)
    conf = torch.empty((d.B, d.S), dtype=torch.float32, device="cuda")
    amax = torch.empty((d.B, d.S), dtype=torch.int32, device="cuda")
    ncom = torch.empty((d.B,), dtype=torch.int32, device="cuda")
    ws = G.workspace(D, tt.TT_WS_VOCAB)
    tt.tt_vocab_confidence_commit(D, G.dev_bf16(yb), G.dev_bf16(wb), gamma, logit_scale,
                                  t_tok, t_m, conf, amax, ncom, ws)
    assert tt.tt_device_status(ws) == 0
    got = dict(tokens=t_tok.cpu().numpy(), masked=t_m.cpu().numpy(), conf=conf.cpu().numpy(),
               tok=amax.cpu().numpy(), ncom=ncom.cpu().numpy())
    # oracle on the same y bytes (only masked rows are predicted)
    sel = masked.reshape(-1) == 1
    c, tk, gl, gp = O.vocab_confidence(O.from_bf16(yb)[sel], wb, logit_scale)
    conf_o = np.full(rows, np.nan)
    tok_o = np.full(rows, -1, np.int64)
    gl_o = np.full(rows, np.inf)
    gp_o = np.full(rows, np.inf)
    conf_o[sel], tok_o[sel], gl_o[sel], gp_o[sel] = c, tk, gl, gp
    ref = dict(conf=conf_o.reshape(d.B, d.S), tok=tok_o.reshape(d.B, d.S),
               gap_l=gl_o.reshape(d.B, d.S), gap_p=gp_o.reshape(d.B, d.S))
    t2, m2, committed, fb = O.commit(ref["conf"], ref["tok"], tokens, masked.astype(bool), gamma)
    ref.update(tokens=t2, masked=m2, committed=committed, fallback=fb)
    return got, ref, masked, tokens


def _check_commit(got, ref, masked, tokens, gamma):
    m = masked.astype(bool)
    # confidences: relative agreement of the fp32 merge with float64
    np.testing.assert_allclose(got["conf"][m], ref["conf"][m], rtol=2e-4)
    assert np.all(got["conf"][~m] == -1) and np.all(got["tok"][~m] == -1)
    ex_arg = m & G.derived_excluded_argmax(ref["gap_l"])
    ok_arg = m & ~ex_arg
    np.testing.assert_array_equal(got["tok"][ok_arg], ref["tok"][ok_arg])
    # committed positions never change
    np.testing.assert_array_equal(got["tokens"][~m], tokens[~m])
    assert np.all(got["masked"][~m] == 0)
    n_spec = int((m & G.spec_excluded(ref["conf"], ref["gap_p"], gamma)).sum())
    n_der = 0
    for b in range(m.shape[0]):
        if not m[b].any():
            assert got["ncom"][b] == 0
            continue
        assert got["ncom"][b] >= 1                          # progress
        thr = m[b] & G.derived_excluded_threshold(ref["conf"][b], gamma)
        fbk = False
        if ref["fallback"][b]:
            cb = np.sort(ref["conf"][b][m[b]])[::-1]
            fbk = len(cb) > 1 and (cb[0] - cb[1]) / cb[0] < G.TIE_FALLBACK_REL and cb[0] != cb[1]
        skip = thr.any() or fbk or (ex_arg[b] & ref["committed"][b]).any()
        if skip:
            n_der += 1
            continue
        np.testing.assert_array_equal(got["masked"][b], ref["masked"][b].astype(np.uint8))
        np.testing.assert_array_equal(got["tokens"][b], ref["tokens"][b])
        assert got["ncom"][b] == ref["committed"][b].sum()
    return n_spec, n_der


@pytest.mark.parametrize("logit_scale,gamma", [(1.0, 0.8), (8.0, 0.8), (12.0, 0.5), (40.0, 0.95)])
def test_vocab_commit_tiny(logit_scale, gamma):
    d = tt_inputs.workload("tiny", B=4)
    got, ref, m, tok = _vocab_case(d, 21, logit_scale, gamma)
    n_spec, n_der = _check_commit(got, ref, m, tok, gamma)
    print(f"tiny scale={logit_scale}: spec-excluded {n_spec}, test-excluded sequences {n_der}")
    assert n_der <= 1, n_der                      # at most one of the 4 sequences skipped


def test_vocab_commit_ragged_vocab_and_partial_mask():
    d = tt_inputs.Dims(B=5, S=32, Hq=4, Hkv=1, dh=64, V=1000, L_cap=0)   # V not a tile multiple
    rng = np.random.default_rng(3)
    masked = (rng.random((5, 32)) < 0.5).astype(np.uint8)
    masked[2] = 0                                                        # fully committed sequence
    got, ref, m, tok = _vocab_case(d, 22, 6.0, 0.7, masked=masked)
    n_spec, n_der = _check_commit(got, ref, m, tok, 0.7)
    print(f"ragged vocab: spec-excluded {n_spec}, test-excluded sequences {n_der}")
    assert n_der <= 1, n_der                      # at most one of the 4 masked sequences


@pytest.mark.parametrize("V", [2, 3])
def test_vocab_commit_smallest_vocabularies(V):
    """The bottom of the accepted envelope: a vocabulary of 2 or 3 tokens, one
    224-wide tile almost all past V."""
    d = tt_inputs.Dims(B=4, S=16, Hq=4, Hkv=1, dh=64, V=V, L_cap=0)
    got, ref, m, tok = _vocab_case(d, 24, 3.0, 0.6)
    n_spec, n_der = _check_commit(got, ref, m, tok, 0.6)
    print(f"V={V}: spec-excluded {n_spec}, test-excluded sequences {n_der}")
    assert n_der <= 1, n_der
    assert np.all((got["tok"][m.astype(bool)] >= 0) & (got["tok"][m.astype(bool)] < V))


def test_vocab_planted_argmax_ties_pick_lowest_id():
    d = tt_inputs.workload("tiny", B=2)
    inp = tt_inputs.generate(d, seed=23, names=["w"])
    wb = inp["w"].copy()
    wb[700] = wb[3]       # token 3 and 700 give identical logits for every y
    wb[900] = wb[3]
    got, ref, m, tok = _vocab_case(d, 23, 30.0, 0.9, w_override=wb)
    hit = ref["tok"] == 3
    assert np.all(got["tok"][hit] == 3)
    _check_commit(got, ref, m, tok, 0.9)


@pytest.mark.parametrize("logit_scale", [1.0, 8.0])
def test_vocab_commit_full_mid_shape(logit_scale):
    d = tt_inputs.workload("mid")
    got, ref, m, tok = _vocab_case(d, 0, logit_scale, 0.8)
    n_spec, n_der = _check_commit(got, ref, m, tok, 0.8)
    print(f"mid scale={logit_scale}: spec-excluded positions {n_spec}, "
          f"test-excluded sequences {n_der}")
    assert n_der <= 2
