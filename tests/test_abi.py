"""The C-ABI library loads, exports every declared symbol, and its host-side
argument checks reject bad calls before anything reaches a GPU.

No GPU needed: validation runs on the host and returns before any CUDA call,
so fake (never dereferenced) pointers are enough here.
"""
import ctypes
import os
import re

import pytest

import block_wise_diffusion_b200 as tt
import tt_inputs
from block_wise_diffusion_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "twotower.h")
FAKE = 1 << 20  # 16-byte aligned, never dereferenced


@pytest.fixture(scope="module")
def L():
    build.build()
    return tt.lib()


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"TT_API\s+[\w\s\*]+?\b(tt_\w+)\s*\(", src)))


def test_header_and_binding_agree():
    syms = declared_symbols()
    assert len(syms) >= 10
    assert sorted(tt.EXPORTS) == syms


def test_library_exports_every_declared_symbol(L):
    for name in declared_symbols():
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


def test_status_strings(L):
    for code, name in tt.STATUS.items():
        assert tt.tt_status_string(code) == name
    assert tt.tt_status_string(99) == "TT_ERR_UNKNOWN"


def _d(**kw):
    base = dict(B=8, S=16, Hq=32, Hkv=2, dh=128, V=131072, L_cap=4096)
    base.update(kw)
    return tt.Dims(base["B"], base["S"], base["Hq"], base["Hkv"], base["dh"],
                   base.get("H", base["Hq"] * base["dh"]), base["V"], base["L_cap"])


def test_workspace_sizes(L):
    d = _d()
    attn = tt.tt_workspace_bytes(d, tt.TT_WS_ATTN)
    vocab = tt.tt_workspace_bytes(d, tt.TT_WS_VOCAB)
    loop = tt.tt_workspace_bytes(d, tt.TT_WS_LOOP)
    assert tt.tt_workspace_bytes(d, tt.TT_WS_ADALN) == 256
    assert loop >= vocab and loop >= attn
    # vocab: 128 rows of y (1 MiB) + 512 tiles x 128 rows x 12 B of tile statistics
    assert vocab >= 128 * 4096 * 2 + 512 * 128 * 12
    # all positions of all sequences fit one query tile when S*G <= 256
    tiny = tt.dims(tt_inputs.workload("tiny"))
    assert tt.tt_workspace_bytes(tiny, tt.TT_WS_LOOP) > 0


@pytest.mark.parametrize("kw,code", [
    (dict(S=8), 2), (dict(S=2), 2), (dict(dh=96), 2), (dict(Hkv=3), 1), (dict(Hq=24, Hkv=2), 2),
    (dict(H=1000), 1), (dict(B=0), 1), (dict(V=1), 1), (dict(L_cap=-1), 1),
])
def test_bad_dims_rejected(L, kw, code):
    d = _d(**kw)
    assert L.tt_workspace_bytes(ctypes.byref(d), 0) == 0
    r = L.tt_block_denoise_attn(ctypes.byref(d), *([FAKE] * 7), FAKE, 1 << 40, None)
    assert r == code, tt.tt_last_error()
    assert tt.tt_last_error()


def test_pointer_and_workspace_checks(L):
    d = _d()
    ws_need = tt.tt_workspace_bytes(d, tt.TT_WS_ATTN)
    args = [FAKE] * 7
    r = L.tt_block_denoise_attn(ctypes.byref(d), *args, FAKE, ws_need - 1, None)
    assert r == 3 and "workspace" in tt.tt_last_error()
    bad = list(args)
    bad[0] = None
    assert L.tt_block_denoise_attn(ctypes.byref(d), *bad, FAKE, ws_need, None) == 1
    assert "q_blk" in tt.tt_last_error()
    bad[0] = FAKE + 2                          # misaligned for TMA
    assert L.tt_block_denoise_attn(ctypes.byref(d), *bad, FAKE, ws_need, None) == 1
    assert "aligned" in tt.tt_last_error()
    assert L.tt_block_denoise_attn(ctypes.byref(d), *args, FAKE + 16, ws_need, None) == 1
    assert L.tt_adaln_modulate(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, 256, None) == 1


def test_commit_and_loop_argument_checks(L):
    d = _d()
    wsb = tt.tt_workspace_bytes(d, tt.TT_WS_VOCAB)
    call = lambda g, s: L.tt_vocab_confidence_commit(
        ctypes.byref(d), FAKE, FAKE, ctypes.c_float(g), ctypes.c_float(s), FAKE, FAKE, FAKE,
        FAKE, FAKE, FAKE, wsb, None)
    assert call(0.0, 1.0) == 1
    assert call(1.5, 1.0) == 1
    assert call(0.8, 0.0) == 1
    assert call(0.8, float("inf")) == 1
    wsl = tt.tt_workspace_bytes(d, tt.TT_WS_LOOP)
    loop = lambda ms: L.tt_denoise_block_loop(
        ctypes.byref(d), *([FAKE] * 8), ctypes.c_float(0.8), ctypes.c_float(1.0), ms,
        *([FAKE] * 4), None, FAKE, wsl, None)
    assert loop(0) == 1
    assert loop(2000) == 1
    layers = lambda n: L.tt_denoise_block_loop_layers(
        ctypes.byref(d), n, *([FAKE] * 8), ctypes.c_float(0.8), ctypes.c_float(1.0), 4,
        *([FAKE] * 4), None, FAKE, wsl, None)
    assert layers(0) == 1 and "n_layers" in tt.tt_last_error()
    assert layers(65) == 1
    blocks = lambda n: L.tt_decode_blocks(
        ctypes.byref(d), n, *([FAKE] * 9), ctypes.c_float(0.8), ctypes.c_float(1.0),
        *([FAKE] * 3), None, FAKE, wsl, None)
    assert blocks(0) == 1 and "n_blocks" in tt.tt_last_error()
    assert blocks(4097) == 1
    n_rows = ctypes.c_int32(-3)
    last = lambda ws_bytes, out: L.tt_loop_last_step(
        ctypes.byref(d), FAKE, ws_bytes, FAKE, FAKE, FAKE, FAKE, out, None)
    assert last(wsl, None) == 1 and "n_rows" in tt.tt_last_error()
    assert last(wsl - 1, ctypes.addressof(n_rows)) == 3
    assert last(tt.tt_workspace_bytes(d, tt.TT_WS_VOCAB), ctypes.addressof(n_rows)) == 3
    assert n_rows.value == -3                               # nothing written on refusal


def test_loop_graph_knob(L):
    with pytest.raises(tt.TTError):
        tt.tt_set_loop_graphs(2)
    tt.tt_set_loop_graphs(0)
    tt.tt_set_loop_graphs(1)


def test_split_knob(L):
    with pytest.raises(tt.TTError):
        tt.tt_set_attn_splits(1025)
    d = _d(B=1, L_cap=65536)
    tt.tt_set_attn_splits(1)
    one = tt.tt_workspace_bytes(d, tt.TT_WS_ATTN)
    tt.tt_set_attn_splits(8)
    eight = tt.tt_workspace_bytes(d, tt.TT_WS_ATTN)
    tt.tt_set_attn_splits(0)
    # a partial slot per (unit, CTA) boundary: units + CTAs - 1 slots of 256
    # rows x (dh + 4) floats
    slot = 256 * (128 + 4) * 4
    assert eight - one == 7 * slot


def test_binding_refuses_cpu_tensors(L):
    import torch
    d = _d()
    x = torch.zeros(4)
    with pytest.raises(ValueError):
        tt.tt_adaln_modulate(d, x, x, x, x, x)


# ------------------------------------------- binding: buffer sizes vs the header
def _documented_bytes(B, S, Hq, Hkv, dh, V, L_cap, n_layers, n_blocks):
    """Bytes of every buffer argument, from the shapes include/twotower.h
    documents for each entry point."""
    H = Hq * dh
    R = B * S
    ctx = B * Hkv * L_cap * dh * 2
    u_t = (H + 2 * Hkv * dh) * H * 2
    vocab = dict(y=R * H * 2, w=V * H * 2, tokens=R * 4, masked=R, conf_out=R * 4,
                 argmax_out=R * 4, n_committed=B * 4)
    loop_in = dict(k_ctx=ctx, v_ctx=ctx, ctx_len=B * 4, emb=V * H * 2, e_mask=H * 2, u_t=u_t,
                   shift_scale=2 * H * 2, w=V * H * 2)
    state = dict(tokens=R * 4, masked=R, steps_taken=B * 4, commit_step=R * 4)
    layers = dict(loop_in, **state)
    for k in ("k_ctx", "v_ctx", "u_t", "shift_scale"):
        layers[k] *= n_layers
    return {
        "tt_block_denoise_attn": dict(q_blk=R * Hq * dh * 2, k_blk=R * Hkv * dh * 2,
                                      v_blk=R * Hkv * dh * 2, k_ctx=ctx, v_ctx=ctx,
                                      ctx_len=B * 4, out=R * Hq * dh * 2),
        "tt_adaln_modulate": dict(x=R * H * 2, shift_scale=2 * H * 2, t=B * 4, y=R * H * 2),
        "tt_vocab_confidence_commit": vocab,
        "tt_vocab_confidence_commit_noalloc": vocab,
        "tt_denoise_block_loop": dict(loop_in, **state),
        "tt_denoise_block_loop_layers": layers,
        "tt_decode_blocks": dict(loop_in, u_ctx=2 * Hkv * dh * H * 2, tokens=n_blocks * R * 4,
                                 steps_taken=n_blocks * B * 4, commit_step=n_blocks * R * 4),
        "tt_loop_last_step": dict(y_rows=R * H * 2, row_ids=R * 4, conf=R * 4, argmax=R * 4),
    }


SCALARS = dict(gamma=0.8, logit_scale=1.0, max_steps=4, n_layers=3, n_blocks=2, stream=0)


@pytest.mark.parametrize("fn", sorted(_documented_bytes(1, 1, 1, 1, 1, 1, 1, 1, 1)))
def test_binding_checks_every_buffer_size(L, fn):
    import inspect
    import torch
    shape = dict(B=2, S=16, Hq=4, Hkv=1, dh=64, V=1024, L_cap=40)
    d = tt.Dims(shape["B"], shape["S"], shape["Hq"], shape["Hkv"], shape["dh"],
                shape["Hq"] * shape["dh"], shape["V"], shape["L_cap"])
    need = _documented_bytes(**shape, n_layers=SCALARS["n_layers"],
                             n_blocks=SCALARS["n_blocks"])[fn]
    wrapper = getattr(tt, fn)
    params = [p for p in inspect.signature(wrapper).parameters if p != "d"]
    buffers = [p for p in params if p not in SCALARS and p != "ws"]
    assert sorted(buffers) == sorted(need), fn
    for name in buffers:
        for nbytes, message in ((need[name], "CUDA tensors only"), (need[name] - 1, "holds")):
            kw = {p: SCALARS.get(p, FAKE) for p in params}
            kw[name] = torch.zeros(nbytes, dtype=torch.uint8)      # a CPU buffer of that size
            with pytest.raises(ValueError, match=message):
                wrapper(d, **kw)
