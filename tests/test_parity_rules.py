"""The comparison machinery itself (oracle/parity.py), on the CPU.

The GPU tests and the benchmark's sampled check trust compare_loop to find
every disagreement outside the near-tie exclusions; here it is fed the
oracle's own trajectory (nothing to find) and trajectories with one planted
mistake each (each must be found), and the exclusion rules are checked on
hand-made values.
"""
import numpy as np

import tt_inputs
from oracle import parity as P
from oracle import twotower_oracle as O


def _tiny_run(scale):
    d = tt_inputs.workload("tiny", B=2, precommit=("uniform", 0.0, 0.75))
    inp = tt_inputs.generate(d, seed=71)
    r = O.denoise_block_loop(inp, 0.8, scale)
    return d, inp, r["tokens"].astype(np.int64), r["commit_step"].astype(np.int64)


def test_oracle_trajectory_compares_clean():
    d, inp, tok, cs = _tiny_run(12.0)
    cnt, problems = P.compare_loop(inp, tok, cs, 0.8, 12.0)
    assert problems == []
    assert cnt["seq_steps"] > 0 and cnt["tokens"] > 0 and cnt["top2_flips"] == 0
    if cnt["seq_steps_excluded"] == 0:       # then every committed token was compared
        assert cnt["tokens"] == int((inp["masked"] == 1).sum())


def test_planted_wrong_token_is_found():
    d, inp, tok, cs = _tiny_run(12.0)
    m0 = inp["masked"].astype(bool)
    b, s = np.argwhere(m0)[0]
    bad = tok.copy()
    bad[b, s] = (bad[b, s] + 517) % d.V                  # far from any near tie
    _, problems = P.compare_loop(inp, bad, cs, 0.8, 12.0)
    assert any(f"pos {s}" in p for p in problems), problems


def test_planted_wrong_commit_step_is_found():
    d, inp, tok, cs = _tiny_run(1.0)                      # one commit per step
    m0 = inp["masked"].astype(bool)
    b = int(np.flatnonzero(m0.sum(axis=1) >= 2)[0])
    s0, s1 = [s for s in range(d.S) if m0[b, s]][:2]
    bad = cs.copy()
    bad[b, s0], bad[b, s1] = cs[b, s1], cs[b, s0]         # commit order swapped
    _, problems = P.compare_loop(inp, tok, bad, 0.8, 1.0)
    assert any("commit set" in p for p in problems), problems


def test_exclusion_rules_on_hand_values():
    conf = np.array([0.8005, 0.7, 0.9, 0.5])
    gap_p = np.array([0.5, 0.0005, 0.5, 0.5])
    np.testing.assert_array_equal(P.spec_excluded(conf, gap_p, 0.8), [True, True, False, False])
    np.testing.assert_array_equal(P.derived_excluded_threshold(conf, 0.8),
                                  [True, False, False, False])
    np.testing.assert_array_equal(P.derived_excluded_argmax(np.array([1e-3, 3e-3])), [True, False])
    assert P.fallback_near_tie([0.30000, 0.299999, 0.1])
    assert not P.fallback_near_tie([0.3, 0.3, 0.1])        # exact tie: compared (lowest s wins)
    assert not P.fallback_near_tie([0.3, 0.2])
    assert not P.fallback_near_tie([0.3])


def test_rows_supplied_compare_clean_and_measure_the_row_difference():
    """With the kernel's rows at hand the comparison measures them against
    the oracle's; the oracle's own rows give zero difference and nothing to
    explain, slightly perturbed rows a small difference."""
    d, inp, tok, cs = _tiny_run(12.0)
    m0 = inp["masked"].astype(bool)

    def state(step):
        done = (cs >= 0) & (cs < step)
        return np.where(done, tok, inp["tokens"]), m0 & ~done

    r = O.denoise_block_loop(inp, 0.8, 12.0, max_steps=int(cs.max()) + 1, teacher=state)
    rows = [{(b, s): st["y"][b, s] for b in range(d.B) for s in range(d.S) if state(k)[1][b, s]}
            for k, st in enumerate(r["trace"])]
    cnt, problems = P.compare_loop(inp, tok, cs, 0.8, 12.0, g_rows=rows)
    assert problems == [] and cnt["y_rel_l2_max"] == 0.0 and cnt["y_explained"] == 0
    rng = np.random.default_rng(1)
    noisy = [{k: v * (1 + 1e-3 * rng.standard_normal(v.shape)) for k, v in st.items()}
             for st in rows]
    cnt, _ = P.compare_loop(inp, tok, cs, 0.8, 12.0, g_rows=noisy)
    assert 5e-4 < cnt["y_rel_l2_max"] < 2e-3
