"""The seeded input generator follows its documented recipe.

Shapes, scales (N(0,1)/sqrt(fan-in), ``sharp`` Q/K at unit scale), the
context-length and pre-committed-fraction laws, determinism, and the
independence of every tensor's bytes from the subset requested and the
thread count.  No GPU needed.
"""
import numpy as np
import pytest

import tt_inputs
from tt_inputs import Dims


def _f32(bits):
    return tt_inputs.bf16_bits_to_f32(bits).astype(np.float64)


def test_bf16_bits_round_trip_and_rounding():
    x = np.array([1.0, -2.5, 3.140625, 0.0, 65536.0], np.float32)   # all exact in bf16
    np.testing.assert_array_equal(tt_inputs.bf16_bits_to_f32(tt_inputs.bf16_bits(x)), x)
    one_plus_half_ulp = np.float32(1.0 + 2.0 ** -8)                  # tie -> even (1.0)
    assert tt_inputs.bf16_bits(np.array([one_plus_half_ulp]))[0] == 0x3F80


def test_shapes_and_dtypes_follow_the_recipe():
    d = Dims(B=2, S=16, Hq=4, Hkv=1, dh=64, V=1024, L_cap=300, ctx=("fixed", 300))
    inp = tt_inputs.generate(d, seed=0)
    H, n_qkv = d.H, d.H + 2 * d.Hkv * d.dh
    want = {"q_blk": (2, 16, 4, 64), "k_blk": (2, 16, 1, 64), "v_blk": (2, 16, 1, 64),
            "k_ctx": (2, 1, 300, 64), "v_ctx": (2, 1, 300, 64), "shift_scale": (2, H),
            "w": (1024, H), "emb": (1024, H), "e_mask": (H,), "u_t": (n_qkv, H),
            "u_ctx": (2 * d.Hkv * d.dh, H)}
    for k, shape in want.items():
        assert inp[k].shape == shape and inp[k].dtype == np.uint16, k
        assert np.isfinite(_f32(inp[k])).all(), k
    assert inp["ctx_len"].dtype == np.int32 and (inp["ctx_len"] == 300).all()
    assert inp["tokens"].dtype == np.int32 and (inp["tokens"] == -1).all()
    assert inp["masked"].dtype == np.uint8 and (inp["masked"] == 1).all()


def test_scales_are_one_over_sqrt_fan_in():
    d = Dims(B=4, S=16, Hq=8, Hkv=2, dh=64, V=2048, L_cap=512, ctx=("fixed", 512))
    inp = tt_inputs.generate(d, seed=1)
    fan = {"q_blk": d.dh, "k_blk": d.dh, "v_blk": d.dh, "k_ctx": d.dh, "v_ctx": d.dh,
           "shift_scale": d.H, "w": d.H, "emb": d.H, "e_mask": d.H, "u_t": d.H, "u_ctx": d.H}
    for k, n in fan.items():
        x = _f32(inp[k])
        sd = 1.0 / np.sqrt(n)
        tol = 0.05 if x.size > 4000 else 0.2     # the sample sd's error is ~1/sqrt(2 n)
        assert abs(x.std() / sd - 1.0) < tol, k
        assert abs(x.mean()) < 5 * sd / np.sqrt(x.size), k
    sharp = tt_inputs.generate(d, seed=1, sharp=True, names=["q_blk", "k_blk", "k_ctx", "v_ctx"])
    for k in ("q_blk", "k_blk", "k_ctx"):
        assert abs(_f32(sharp[k]).std() - 1.0) < 0.05, k
    # sharp changes the scale of Q and K only; the draws are the same
    np.testing.assert_array_equal(sharp["v_ctx"], inp["v_ctx"])


def test_deterministic_and_independent_of_subset_and_threads():
    d = Dims(B=1, S=16, Hq=4, Hkv=1, dh=64, V=20000, L_cap=64, ctx=("fixed", 64))
    a = tt_inputs.generate(d, seed=5, threads=1)
    b = tt_inputs.generate(d, seed=5, threads=4)      # w has two 4 Mi-element chunks
    assert a["w"].size > 1 << 22
    for k in a:
        np.testing.assert_array_equal(a[k], b[k], err_msg=k)
    only = tt_inputs.generate(d, seed=5, names=["e_mask", "u_ctx"])
    assert set(only) >= {"e_mask", "u_ctx"} and "w" not in only
    np.testing.assert_array_equal(only["e_mask"], a["e_mask"])
    np.testing.assert_array_equal(only["u_ctx"], a["u_ctx"])
    c = tt_inputs.generate(d, seed=6, names=["e_mask"])
    assert not np.array_equal(c["e_mask"], a["e_mask"])


def test_ragged_context_lengths_are_uniform_integers_in_range():
    d = tt_inputs.workload("ragged16")
    cl = tt_inputs.generate(d, seed=0, names=[])["ctx_len"]
    assert cl.shape == (128,) and cl.dtype == np.int32
    assert cl.min() >= 512 and cl.max() <= 32768
    # mean and spread of U[512, 32768]: 16640 and 9312
    assert abs(cl.mean() - 16640) < 4 * 9312 / np.sqrt(128)
    assert abs(cl.std() - 9312) < 0.2 * 9312
    big = Dims(B=4000, S=16, Hq=4, Hkv=1, dh=64, V=64, L_cap=32768, ctx=("uniform", 512, 32768))
    many = tt_inputs.generate(big, seed=2, names=[])["ctx_len"]
    assert many.min() >= 512 and many.max() <= 32768
    assert abs(many.mean() - 16640) < 4 * 9312 / np.sqrt(4000)


def test_precommitted_fraction_law():
    S, V = 16, 1000
    d = Dims(B=6000, S=S, Hq=4, Hkv=1, dh=64, V=V, L_cap=0, precommit=("uniform", 0.0, 0.75))
    inp = tt_inputs.generate(d, seed=3, names=[])
    tok, m = inp["tokens"], inp["masked"].astype(bool)
    assert (tok[m] == -1).all()
    assert ((tok[~m] >= 0) & (tok[~m] < V)).all()
    k = (~m).sum(axis=1)                     # floor(f*S) with f ~ U[0, 0.75): 0..11
    assert k.min() == 0 and k.max() == 11
    counts = np.bincount(k, minlength=12)[:12]
    expect = len(k) / 12
    assert (np.abs(counts - expect) < 5 * np.sqrt(expect)).all(), counts
    # committed positions are spread over the block, not packed at its start
    per_pos = (~m).mean(axis=0)
    assert np.ptp(per_pos) < 0.05, per_pos
    # committed tokens are uniform over the vocabulary
    t = tok[~m]
    assert abs(t.mean() - (V - 1) / 2) < 4 * V / np.sqrt(12 * t.size)


def test_layer_stacks():
    d = tt_inputs.workload("tiny", B=2)
    one = tt_inputs.generate(d, seed=4)
    three = tt_inputs.generate(d, seed=4, n_layers=3)
    for name in tt_inputs.LAYER_NAMES:
        st = three[name + "_l"]
        assert st.shape == (3,) + one[name].shape
        np.testing.assert_array_equal(st[0], one[name])           # layer 0 = the single draw
        assert not np.array_equal(st[1], st[0]) and not np.array_equal(st[2], st[1])
        np.testing.assert_array_equal(three[name], one[name])


def test_rejects_inconsistent_dims():
    with pytest.raises(ValueError):
        tt_inputs.generate(Dims(B=1, S=16, Hq=3, Hkv=2, dh=64, V=8, L_cap=0), names=[])
    with pytest.raises(ValueError):
        tt_inputs.generate(Dims(B=1, S=16, Hq=4, Hkv=1, dh=64, V=8, L_cap=10,
                                ctx=("fixed", 11)), names=[])
