"""Every entry point writes only its outputs.

Each tensor handed to the library sits inside a larger buffer.  Guard bands
of a known byte pattern surround it on both sides.  The guards are 512 bytes
each, so every tensor keeps the 512-byte alignment of a fresh allocation.
After the call, every guard band must still hold the pattern.  Every input
must be unchanged bit for bit, and the outputs must be written only where the
header says: for block-after-block decoding, only the appended context rows.
"""
import numpy as np
import pytest
import torch

import block_wise_diffusion_b200 as tt
import tt_inputs

pytestmark = pytest.mark.gpu

DEVICE = "cuda"
PAD_BYTES = 512
PATTERN = 0xA5


class Guarded:
    """A tensor of `shape` inside a buffer with PAD_BYTES of PATTERN on each side."""

    def __init__(self, shape, dtype, init=None):
        esz = torch.empty((), dtype=dtype).element_size()
        self.n = int(np.prod(shape))
        self.pad = PAD_BYTES // esz
        self.buf = torch.empty(self.n + 2 * self.pad, dtype=dtype, device=DEVICE)
        self.buf.view(torch.uint8).fill_(PATTERN)
        self.t = self.buf[self.pad:self.pad + self.n].view(shape)
        if init is not None:
            self.t.copy_(init)
        self.before = self.t.clone()

    def guards_intact(self) -> bool:
        u = self.buf.view(torch.uint8)
        b = PAD_BYTES
        return bool((u[:b] == PATTERN).all()) and bool((u[-b:] == PATTERN).all())

    def unchanged(self) -> bool:
        return bool(torch.equal(self.t.view(torch.uint8), self.before.view(torch.uint8)))


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def _g_bf16(bits):
    return Guarded(bits.shape, torch.bfloat16, _bf16(bits).to(DEVICE))


def _g(arr, dtype):
    return Guarded(arr.shape, dtype, torch.from_numpy(np.ascontiguousarray(arr)).to(DEVICE))


def _ws(D, which):
    return Guarded((tt.tt_workspace_bytes(D, which),), torch.uint8)


def _check(inputs, outputs):
    if DEVICE == "cuda":
        torch.cuda.synchronize()
    for name, g in {**inputs, **outputs}.items():
        assert g.guards_intact(), f"{name}: a guard band was overwritten"
    for name, g in inputs.items():
        assert g.unchanged(), f"{name}: an input was modified"


@pytest.mark.parametrize("wl,over,cl", [
    ("tiny", {}, None),                                               # one split, 64 rows per KV head
    ("mid", dict(B=3, L_cap=1000, ctx=("fixed", 1000), V=1024), [1000, 377, 0]),   # splits + merge
])
def test_attention_writes_only_its_output(wl, over, cl):
    d = tt_inputs.workload(wl, **over)
    inp = tt_inputs.generate(d, seed=61, names=["q_blk", "k_blk", "v_blk", "k_ctx", "v_ctx"])
    D = tt.dims(d)
    ins = {k: _g_bf16(inp[k]) for k in ("q_blk", "k_blk", "v_blk", "k_ctx", "v_ctx")}
    ins["ctx_len"] = _g(np.array(cl if cl is not None else inp["ctx_len"], np.int32), torch.int32)
    outs = {"out": Guarded((d.B, d.S, d.Hq, d.dh), torch.bfloat16),
            "ws": _ws(D, tt.TT_WS_ATTN)}
    tt.tt_block_denoise_attn(D, *(ins[k].t for k in ("q_blk", "k_blk", "v_blk", "k_ctx", "v_ctx",
                                                     "ctx_len")), outs["out"].t, outs["ws"].t)
    assert tt.tt_device_status(outs["ws"].t) == 0
    _check(ins, outs)
    assert bool(torch.isfinite(outs["out"].t.float()).all())


def test_adaln_writes_only_y():
    d = tt_inputs.workload("tiny", B=3)
    inp = tt_inputs.generate(d, seed=62, names=["shift_scale"])
    rng = np.random.default_rng(62)
    D = tt.dims(d)
    x = tt_inputs.bf16_bits(rng.standard_normal((d.B * d.S, d.H)).astype(np.float32))
    ins = {"x": _g_bf16(x), "shift_scale": _g_bf16(inp["shift_scale"]),
           "t": _g(np.array([0.25, 0.5, 1.0], np.float32), torch.float32)}
    outs = {"y": Guarded((d.B * d.S, d.H), torch.bfloat16), "ws": _ws(D, tt.TT_WS_ADALN)}
    tt.tt_adaln_modulate(D, ins["x"].t, ins["shift_scale"].t, ins["t"].t, outs["y"].t,
                         outs["ws"].t)
    assert tt.tt_device_status(outs["ws"].t) == 0
    _check(ins, outs)


def test_vocab_commit_writes_only_its_outputs():
    d = tt_inputs.Dims(B=3, S=32, Hq=4, Hkv=1, dh=64, V=1000, L_cap=0)   # ragged vocabulary
    inp = tt_inputs.generate(d, seed=63, names=["w"])
    rng = np.random.default_rng(63)
    D = tt.dims(d)
    y = tt_inputs.bf16_bits((rng.standard_normal((d.B * d.S, d.H)) * 2).astype(np.float32))
    masked = (rng.random((d.B, d.S)) < 0.6).astype(np.uint8)
    masked[1] = 0                                          # a fully committed sequence
    tokens = np.where(masked == 1, -1, rng.integers(0, d.V, (d.B, d.S))).astype(np.int32)
    ins = {"y": _g_bf16(y), "w": _g_bf16(inp["w"])}
    outs = {"tokens": _g(tokens, torch.int32), "masked": _g(masked, torch.uint8),
            "conf": Guarded((d.B, d.S), torch.float32),
            "argmax": Guarded((d.B, d.S), torch.int32),
            "n_committed": Guarded((d.B,), torch.int32), "ws": _ws(D, tt.TT_WS_VOCAB)}
    tt.tt_vocab_confidence_commit(D, ins["y"].t, ins["w"].t, 0.8, 6.0, outs["tokens"].t,
                                  outs["masked"].t, outs["conf"].t, outs["argmax"].t,
                                  outs["n_committed"].t, outs["ws"].t)
    assert tt.tt_device_status(outs["ws"].t) == 0
    _check(ins, outs)
    # the fully committed sequence is left as it was
    assert bool(torch.equal(outs["tokens"].t[1], outs["tokens"].before[1]))
    assert int(outs["n_committed"].t[1]) == 0


def test_loop_writes_only_its_state():
    d = tt_inputs.workload("tiny", B=2, precommit=("uniform", 0.0, 0.75))
    inp = tt_inputs.generate(d, seed=64)
    D = tt.dims(d)
    names = ("k_ctx", "v_ctx", "emb", "e_mask", "u_t", "shift_scale", "w")
    ins = {k: _g_bf16(inp[k]) for k in names}
    ins["ctx_len"] = _g(inp["ctx_len"], torch.int32)
    outs = {"tokens": _g(inp["tokens"], torch.int32), "masked": _g(inp["masked"], torch.uint8),
            "steps_taken": Guarded((d.B,), torch.int32),
            "commit_step": Guarded((d.B, d.S), torch.int32), "ws": _ws(D, tt.TT_WS_LOOP)}
    tt.tt_denoise_block_loop(D, ins["k_ctx"].t, ins["v_ctx"].t, ins["ctx_len"].t, ins["emb"].t,
                             ins["e_mask"].t, ins["u_t"].t, ins["shift_scale"].t, ins["w"].t,
                             0.8, 12.0, d.S, outs["tokens"].t, outs["masked"].t,
                             outs["steps_taken"].t, outs["commit_step"].t, outs["ws"].t)
    _check(ins, outs)
    assert not bool(outs["masked"].t.any())


def test_decode_blocks_writes_only_the_appended_rows():
    nb = 2
    d = tt_inputs.Dims(B=2, S=16, Hq=4, Hkv=1, dh=64, V=1024, L_cap=256 + nb * 16 + 32,
                       ctx=("fixed", 256))
    inp = tt_inputs.generate(d, seed=65)
    D = tt.dims(d)
    names = ("emb", "e_mask", "u_t", "shift_scale", "w", "u_ctx")
    ins = {k: _g_bf16(inp[k]) for k in names}
    cache = {"k_ctx": _g_bf16(inp["k_ctx"]), "v_ctx": _g_bf16(inp["v_ctx"])}
    cl = np.array([256, 100], np.int32)
    outs = {**cache, "ctx_len": _g(cl, torch.int32),
            "tokens": Guarded((nb, d.B, d.S), torch.int32),
            "steps_taken": Guarded((nb, d.B), torch.int32),
            "commit_step": Guarded((nb, d.B, d.S), torch.int32), "ws": _ws(D, tt.TT_WS_LOOP)}
    tt.tt_decode_blocks(D, nb, cache["k_ctx"].t, cache["v_ctx"].t, outs["ctx_len"].t,
                        ins["emb"].t, ins["e_mask"].t, ins["u_t"].t, ins["shift_scale"].t,
                        ins["w"].t, ins["u_ctx"].t, 0.8, 12.0, outs["tokens"].t,
                        outs["steps_taken"].t, outs["commit_step"].t, outs["ws"].t)
    _check(ins, outs)
    assert outs["ctx_len"].t.cpu().tolist() == (cl + nb * d.S).tolist()
    for name, g in cache.items():
        now, before = g.t.view(torch.int16).cpu(), g.before.view(torch.int16).cpu()
        for b in range(d.B):
            lo, hi = int(cl[b]), int(cl[b]) + nb * d.S
            assert torch.equal(now[b, :, :lo], before[b, :, :lo]), f"{name}[{b}] before ctx_len"
            assert torch.equal(now[b, :, hi:], before[b, :, hi:]), f"{name}[{b}] past the blocks"
            assert not torch.equal(now[b, :, lo:hi], before[b, :, lo:hi]), f"{name}[{b}] appended"
