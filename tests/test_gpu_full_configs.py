"""Full-size parity of the block loop and the attention at the remaining
workload shapes: the batch-64 loop (all 1024 positions masked at step 0, so
the vocabulary GEMM runs tensor-bound) with gamma swept, the long-context
batch (4 sequences of 65536 keys), and the ragged serving batch (context
lengths U[512, 32768], pre-committed positions) at S = 16 and S = 32.  The
GPU runs the whole batch in the launch configuration the benchmark times,
then again one step per call; the float64 oracle checks sampled sequences
(the shortest and the longest context among them) stage-wise on the GPU's
own rows and end to end, teacher-forced as in test_gpu_loop.py.
"""
import numpy as np
import pytest

import tt_inputs
from oracle import twotower_oracle as O
from tests import _gpu as G
from tests.test_gpu_loop import (check_invariants, compare_teacher_forced, run_loop_gpu,
                                 stepwise_equals_single_call)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def loop64():
    d = tt_inputs.workload("loop64")
    return d, tt_inputs.generate(d, seed=0)


@pytest.mark.parametrize("gamma,logit_scale", [(0.8, 1.0), (0.5, 8.0), (0.95, 8.0)])
def test_loop64_gamma_sweep_sampled_sequences(loop64, gamma, logit_scale):
    d, inp = loop64
    g = run_loop_gpu(d, inp, gamma, logit_scale)
    check_invariants(d, inp, g)
    if logit_scale == 1.0:
        assert g["steps_run"] == 16          # nothing reaches gamma: one commit per step
    steps = stepwise_equals_single_call(d, inp, gamma, logit_scale, g, bsel=[0, 63])
    n_cmp, n_ex = compare_teacher_forced(inp, g, gamma, logit_scale, bsel=np.array([0, 63]),
                                      steps=steps)
    print(f"loop64 gamma={gamma} scale={logit_scale}: steps {g['steps_run']}, "
          f"compared {n_cmp} sequence-steps, excluded {n_ex}")
    assert n_cmp > 0 and n_ex <= 3


@pytest.fixture(scope="module")
def ragged16():
    d = tt_inputs.workload("ragged16")
    return d, tt_inputs.generate(d, seed=0)


def test_loop_ragged16_sampled_sequences(ragged16):
    d, inp = ragged16
    g = run_loop_gpu(d, inp, 0.8, 8.0)
    check_invariants(d, inp, g)
    cl = inp["ctx_len"]
    sel = np.array(sorted({int(np.argmin(cl)), int(np.argmax(cl)), 7}))
    steps = stepwise_equals_single_call(d, inp, 0.8, 8.0, g, bsel=sel)
    n_cmp, n_ex = compare_teacher_forced(inp, g, 0.8, 8.0, bsel=sel, steps=steps)
    print(f"ragged16 loop: sequences {sel.tolist()} (ctx {cl[sel].tolist()}), "
          f"compared {n_cmp} sequence-steps, excluded {n_ex}")
    assert n_cmp > 0 and n_ex <= 3


@pytest.mark.parametrize("logit_scale", [1.0, 8.0])
def test_loop_ragged32_sampled_sequences(logit_scale):
    """The ragged serving batch with blocks of 32 positions."""
    d = tt_inputs.workload("ragged32")
    inp = tt_inputs.generate(d, seed=0)
    g = run_loop_gpu(d, inp, 0.8, logit_scale)
    check_invariants(d, inp, g)
    cl = inp["ctx_len"]
    sel = np.array(sorted({int(np.argmin(cl)), int(np.argmax(cl)), 11}))
    steps = stepwise_equals_single_call(d, inp, 0.8, logit_scale, g, bsel=sel)
    n_cmp, n_ex = compare_teacher_forced(inp, g, 0.8, logit_scale, bsel=sel, steps=steps)
    print(f"ragged32 loop scale={logit_scale}: sequences {sel.tolist()} "
          f"(ctx {cl[sel].tolist()}), compared {n_cmp} sequence-steps, excluded {n_ex}")
    assert n_cmp > 0 and n_ex <= 3


@pytest.mark.parametrize("logit_scale", [1.0, 12.0])
def test_loop_long_context_full_batch(logit_scale):
    """4 sequences of 65536 context keys: stage-wise on every sequence, end to
    end on the first and the last."""
    d = tt_inputs.workload("long")
    inp = tt_inputs.generate(d, seed=0)
    g = run_loop_gpu(d, inp, 0.8, logit_scale)
    check_invariants(d, inp, g)
    if logit_scale == 1.0:
        assert g["steps_run"] == 16
    steps = stepwise_equals_single_call(d, inp, 0.8, logit_scale, g)
    n_cmp, n_ex = compare_teacher_forced(inp, g, 0.8, logit_scale, bsel=np.array([0, 3]),
                                      steps=steps)
    print(f"long loop scale={logit_scale}: compared {n_cmp} sequence-steps, excluded {n_ex}")
    assert n_cmp > 0 and n_ex <= 2


def test_attention_ragged32_sampled_sequences():
    from tests.test_gpu_attn import oracle_attn, run_attn
    d = tt_inputs.workload("ragged32")
    inp = tt_inputs.generate(d, seed=1, sharp=True,
                             names=["q_blk", "k_blk", "v_blk", "k_ctx", "v_ctx"])
    got = run_attn(d, inp)
    cl = inp["ctx_len"]
    for b in sorted({int(np.argmin(cl)), int(np.argmax(cl)), 100}):
        ref = O.round_bf16(oracle_attn(inp, bsel=slice(b, b + 1)))
        G.assert_close_bf16(got[b:b + 1], ref, f"ragged32 b={b} L={cl[b]}")
