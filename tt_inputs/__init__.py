"""Seeded synthetic inputs for the block-wise diffusion denoise step.

This module is the one piece shared by the CPU oracle and the CUDA path: it
draws random numbers and rounds them to bf16 bit patterns, and nothing else.
It holds none of the method's arithmetic (no attention, normalisation,
softmax or commit logic), so the two implementations stay independent.

Every tensor is drawn from its own child of ``numpy.random.SeedSequence(seed)``
in a fixed order (``_STREAMS``); large tensors are cut into fixed-size chunks,
each from its own grandchild seed, so the bytes do not depend on the number
of threads used to produce them.

Shapes, layouts and distributions (workload recipe)
---------------------------------------------------
* ``q_blk``  bf16 [B, S, Hq, dh]      N(0,1)/sqrt(dh)   (``sharp``: N(0,1))
* ``k_blk``  bf16 [B, S, Hkv, dh]     N(0,1)/sqrt(dh)   (``sharp``: N(0,1))
* ``v_blk``  bf16 [B, S, Hkv, dh]     N(0,1)/sqrt(dh)
* ``k_ctx``  bf16 [B, Hkv, L_cap, dh] N(0,1)/sqrt(dh)   (``sharp``: N(0,1))
* ``v_ctx``  bf16 [B, Hkv, L_cap, dh] N(0,1)/sqrt(dh)
* ``shift_scale`` bf16 [2, H]         N(0,1)/sqrt(H)    (row 0 shift, row 1 scale)
* ``w``      bf16 [V, H]              N(0,1)/sqrt(H)    (vocab projection, one row per token)
* ``emb``    bf16 [V, H]              N(0,1)/sqrt(H)    (token embedding table)
* ``e_mask`` bf16 [H]                 N(0,1)/sqrt(H)    (embedding of the MASK state)
* ``u_t``    bf16 [H + 2*Hkv*dh, H]   N(0,1)/sqrt(H)    (linear update, output-major)
* ``ctx_len`` int32 [B]               fixed L, or uniform integers in [lo, hi]
* ``tokens`` int32 [B, S], ``masked`` uint8 [B, S]: all masked, or a per-
  sequence pre-committed fraction f ~ U[0, 0.75] (floor(f*S) positions drawn
  without replacement, tokens uniform in [0, V)).  Masked positions hold -1.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace

import numpy as np

__all__ = [
    "Dims", "WORKLOADS", "workload", "bf16_bits", "bf16_bits_to_f32", "generate",
    "INPUT_NAMES",
]

# Order in which SeedSequence children are handed out.  Never reorder: the
# bytes of every stored expectation depend on it.
_STREAMS = (
    "q_blk", "k_blk", "v_blk", "k_ctx", "v_ctx", "shift_scale", "w", "emb",
    "e_mask", "u_t", "ctx_len", "precommit", "u_ctx",
)
INPUT_NAMES = tuple(n for n in _STREAMS if n not in ("ctx_len", "precommit"))

_CHUNK = 1 << 22  # elements per independently seeded chunk


@dataclass(frozen=True)
class Dims:
    """Problem sizes.  ``H`` must equal ``Hq * dh``."""

    B: int
    S: int
    Hq: int
    Hkv: int
    dh: int
    V: int
    L_cap: int
    # context-length law: ("fixed", L) or ("uniform", lo, hi)
    ctx: tuple = ("fixed", 0)
    # pre-committed fraction law: None (all masked) or ("uniform", lo, hi)
    precommit: tuple | None = None

    @property
    def H(self) -> int:
        return self.Hq * self.dh

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def n_qkv(self) -> int:
        return self.H + 2 * self.Hkv * self.dh


def _fixed(B, S, Hq, Hkv, dh, V, L, **kw):
    return Dims(B=B, S=S, Hq=Hq, Hkv=Hkv, dh=dh, V=V, L_cap=L, ctx=("fixed", L), **kw)


# The five synthetic workloads of the denoise step (sizes as named).
WORKLOADS = {
    # tiny single step: 1 seq, 4 q heads / 1 kv head, d_head 64, hidden 256, ctx 256, V 1024
    "tiny": _fixed(1, 16, 4, 1, 64, 1024, 256),
    # mid decode step: 8 seqs, 32/2 heads (GQA 16), d_head 128, hidden 4096, ctx 4096, V 131072
    "mid": _fixed(8, 16, 32, 2, 128, 131072, 4096),
    # full block loop: 64 seqs, mid shapes, ctx 8192
    "loop64": _fixed(64, 16, 32, 2, 128, 131072, 8192),
    # long context: 4 seqs, ctx 65536
    "long": _fixed(4, 16, 32, 2, 128, 131072, 65536),
    # ragged serving batch: 128 seqs, ctx ~ U[512, 32768], S 16 (or 32), pre-committed fraction U[0, .75]
    "ragged16": Dims(B=128, S=16, Hq=32, Hkv=2, dh=128, V=131072, L_cap=32768,
                     ctx=("uniform", 512, 32768), precommit=("uniform", 0.0, 0.75)),
    "ragged32": Dims(B=128, S=32, Hq=32, Hkv=2, dh=128, V=131072, L_cap=32768,
                     ctx=("uniform", 512, 32768), precommit=("uniform", 0.0, 0.75)),
    # autoregressive baseline at the mid shapes: one position per block (S = 1),
    # the same denoiser step; the denominator of a block-vs-AR throughput ratio
    "mid_ar": _fixed(8, 1, 32, 2, 128, 131072, 4096),
}


def workload(name: str, **overrides) -> Dims:
    d = WORKLOADS[name]
    return replace(d, **overrides) if overrides else d


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + r) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal_bf16(ss: np.random.SeedSequence, shape, scale: float, threads: int) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    n_chunks = max(1, -(-n // _CHUNK))
    kids = ss.spawn(n_chunks)

    def fill(i):
        lo = i * _CHUNK
        hi = min(n, lo + _CHUNK)
        g = np.random.Generator(np.random.PCG64(kids[i]))
        buf = g.standard_normal(hi - lo, dtype=np.float32)
        if scale != 1.0:
            buf *= np.float32(scale)
        out[lo:hi] = bf16_bits(buf)

    if n_chunks == 1 or threads <= 1:
        for i in range(n_chunks):
            fill(i)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(fill, range(n_chunks)))
    return out.reshape(shape)


LAYER_NAMES = ("k_ctx", "v_ctx", "shift_scale", "u_t")


def generate(d: Dims, seed: int = 0, *, sharp: bool = False, names=None,
             threads: int | None = None, n_layers: int = 1) -> dict:
    """Draw the inputs of one denoise-step problem.

    ``names`` restricts which large tensors are produced (the others are
    skipped but still consume their seed slot, so the bytes of every tensor
    are the same whatever subset is asked for).  ``sharp`` draws Q and K
    (block and context) unscaled, which makes attention far from uniform.

    ``n_layers`` > 1 adds ``<name>_l`` arrays for the per-layer tensors
    (context K/V, adaLN table, linear update) with a leading layer dimension;
    layer 0 is the single-layer draw, layer i > 0 comes from its own
    ``SeedSequence([seed, i])``.
    """
    if d.Hq % d.Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    threads = threads or min(16, os.cpu_count() or 1)
    kids = dict(zip(_STREAMS, np.random.SeedSequence(seed).spawn(len(_STREAMS))))
    want = set(names) if names is not None else set(INPUT_NAMES)
    s_dh = 1.0 / np.sqrt(d.dh)
    s_h = 1.0 / np.sqrt(d.H)
    qk = 1.0 if sharp else s_dh
    shapes = {
        "q_blk": ((d.B, d.S, d.Hq, d.dh), qk),
        "k_blk": ((d.B, d.S, d.Hkv, d.dh), qk),
        "v_blk": ((d.B, d.S, d.Hkv, d.dh), s_dh),
        "k_ctx": ((d.B, d.Hkv, d.L_cap, d.dh), qk),
        "v_ctx": ((d.B, d.Hkv, d.L_cap, d.dh), s_dh),
        "shift_scale": ((2, d.H), s_h),
        "w": ((d.V, d.H), s_h),
        "emb": ((d.V, d.H), s_h),
        "e_mask": ((d.H,), s_h),
        "u_t": ((d.n_qkv, d.H), s_h),
        # stand-in for the frozen context tower when a committed block joins
        # the context: [k | v] = Emb[token] . U_ctx^T
        "u_ctx": ((2 * d.Hkv * d.dh, d.H), s_h),
    }
    out = {}
    for name, (shape, scale) in shapes.items():
        if name in want:
            out[name] = _normal_bf16(kids[name], shape, float(scale), threads)

    g = np.random.Generator(np.random.PCG64(kids["ctx_len"]))
    if d.ctx[0] == "fixed":
        ctx_len = np.full(d.B, d.ctx[1], dtype=np.int32)
    else:
        lo, hi = d.ctx[1], d.ctx[2]
        ctx_len = g.integers(lo, hi, size=d.B, endpoint=True).astype(np.int32)
    if int(ctx_len.max(initial=0)) > d.L_cap:
        raise ValueError("context length above L_cap")
    out["ctx_len"] = ctx_len

    tokens = np.full((d.B, d.S), -1, dtype=np.int32)
    masked = np.ones((d.B, d.S), dtype=np.uint8)
    if d.precommit is not None:
        g = np.random.Generator(np.random.PCG64(kids["precommit"]))
        _, lo, hi = d.precommit
        for b in range(d.B):
            f = g.uniform(lo, hi)
            k = int(np.floor(f * d.S))
            pos = g.choice(d.S, size=k, replace=False)
            toks = g.integers(0, d.V, size=k)
            tokens[b, pos] = toks
            masked[b, pos] = 0
    out["tokens"] = tokens
    out["masked"] = masked
    if n_layers > 1:
        for name in LAYER_NAMES:
            if name not in want:
                continue
            shape, scale = shapes[name]
            stack = np.empty((n_layers,) + shape, dtype=np.uint16)
            stack[0] = out[name]
            for i in range(1, n_layers):
                lk = dict(zip(_STREAMS, np.random.SeedSequence([seed, i]).spawn(len(_STREAMS))))
                stack[i] = _normal_bf16(lk[name], shape, float(scale), threads)
            out[name + "_l"] = stack
    return out
