"""Plain float64 CPU oracle of the block-wise diffusion denoise step.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's ``smoke()`` check and
the benchmark's CPU-baseline and reference arms may import this module.  The CUDA library
never calls it, and it shares no code with the CUDA library: the only module
both sides use is ``tt_inputs`` (seeded random draws, no method arithmetic).

What the method computes (sources: "Nemotron-TwoTower: Diffusion Language
Modeling with Pretrained Autoregressive Context", gist.science technical
summary, sections Architecture / Generation Process / Training and
Conditioning; snilld.dk article on TwoTower, sections "Hvad TwoTower ændrer
teknisk" and "Blockwise generering i praksis"):

* the denoiser attends, at every attention layer, to the frozen context
  tower's K/V cache of the same layer *and* to the current block's own K/V
  with no mask inside the block (Architecture; Generation Process);
* it is conditioned on the diffusion time t through adaptive layer norm
  ("adaLN-single" per layer, snilld.dk "Hvad TwoTower ændrer teknisk");
* all masked positions are predicted in parallel and those whose confidence
  reaches the threshold gamma commit, the rest stay masked (Training and
  Conditioning, "Sampling"); the block is refined over T steps until it is
  committed (Generation Process).

Where the pages leave a step open, this file takes the library's stated
reading; each one is a named constant or a sentence in the docstring of the
function that uses it:

* attention scale 1/sqrt(dh); no positional encoding; contiguous GQA
  grouping (query head h reads KV head h // G); one joint softmax over
  [context keys ; block keys]; context positions >= ctx_len are ignored.
* adaLN: LayerNorm without affine parameters (biased variance, eps 1e-6);
  [shift ; scale] = E + phi(t) with phi(t) = [sin(t w_i) || cos(t w_i)],
  w_i = 10000^(-i/H), i < H;  y = LN(x) * (1 + scale) + shift.
* confidence = max softmax probability of (logit_scale * y @ W^T); token =
  argmax, lowest id on ties.  logit_scale is an inverse temperature (1 in the
  canonical runs).
* commit rule: among still-masked positions, every one with conf >= gamma
  commits its argmax token; if none does, the single masked position with the
  highest conf commits (lowest position on ties).  Committed tokens never
  change.
* loop: t_b = (masked count of sequence b) / S at the start of each step; a
  masked position is embedded as e_MASK, a committed one as Emb[token]; the
  block's q|k|v come from one linear map u_t (output-major) of that
  embedding; the context K/V do not change inside a block.
* storage precision: the library stores q|k|v, the attention output and the
  adaLN output as bf16, so the oracle rounds (round-to-nearest-even) at those
  same three points; everything else is float64.

Every function here is pinned by tests/test_oracle_pins.py against closed
forms, brute force, invariants, a library softmax and the hand-worked commit
example in tests/golden/.  tests/test_oracle_mutations.py checks the pins
themselves: it plants plausible mistakes in a copy of this file, one at a
time, and each one must make a pin fail.
"""
from __future__ import annotations

import math

import numpy as np

# ---- readings (named constants) -------------------------------------------
LN_EPS = 1e-6            # LayerNorm epsilon (reading: pages give no value)
ROPE = False             # no positional encoding (pages mention none)
TIME_BASE = 10000.0      # sinusoidal timestep base (reading)


# ---- number formats --------------------------------------------------------
def from_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (ties to even).

    bf16 keeps 8 significant bits.  Written with frexp so that the rounding is
    done once, directly from float64 (no float32 intermediate).
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                     # x = m * 2**e, 0.5 <= |m| < 1
    # values below the bf16 normal range keep the fixed exponent of -125
    e = np.maximum(e, -125)
    scaled = np.ldexp(x, 8 - e)            # |scaled| in [128, 256) for normals
    r = np.round(scaled)                   # numpy rounds half to even
    out = np.ldexp(r, e - 8)
    big = np.abs(out) > 3.3895313892515355e38
    if np.any(big):
        out = np.where(big, np.sign(out) * np.inf, out)
    return out


# ---- a1: block-denoise attention -------------------------------------------
def block_attention(q_blk, k_blk, v_blk, k_ctx, v_ctx, ctx_len):
    """Denoiser attention of one layer (Architecture; Generation Process).

    q_blk [B,S,Hq,dh], k_blk/v_blk [B,S,Hkv,dh], k_ctx/v_ctx [B,Hkv,L,dh],
    ctx_len [B]; all float64.  Query head h uses KV head h // (Hq // Hkv).
    Keys of sequence b are the first ctx_len[b] context rows followed by the
    S block rows; one softmax with scale 1/sqrt(dh) runs over all of them and
    no key is masked inside the block.  Returns float64 [B,S,Hq,dh].
    """
    B, S, Hq, dh = q_blk.shape
    Hkv = k_blk.shape[2]
    G = Hq // Hkv
    out = np.zeros((B, S, Hq, dh))
    scale = 1.0 / math.sqrt(dh)
    for b in range(B):
        L = int(ctx_len[b])
        for g in range(Hkv):
            keys = np.concatenate([k_ctx[b, g, :L], k_blk[b, :, g]], axis=0)
            vals = np.concatenate([v_ctx[b, g, :L], v_blk[b, :, g]], axis=0)
            q = q_blk[b, :, g * G:(g + 1) * G, :]              # [S, G, dh]
            sc = np.einsum("sjd,kd->sjk", q, keys) * scale     # [S, G, L+S]
            sc -= sc.max(axis=-1, keepdims=True)
            p = np.exp(sc)
            p /= p.sum(axis=-1, keepdims=True)
            out[b, :, g * G:(g + 1) * G, :] = np.einsum("sjk,kd->sjd", p, vals)
    return out


def block_attention_loops(q_blk, k_blk, v_blk, k_ctx, v_ctx, ctx_len):
    """The same attention written as explicit scalar loops (tiny shapes only).

    Used to pin ``block_attention``: every score, weight and output element is
    formed one term at a time from the definition softmax(q.k/sqrt(dh)) v.
    """
    B, S, Hq, dh = q_blk.shape
    Hkv = k_blk.shape[2]
    G = Hq // Hkv
    out = np.zeros((B, S, Hq, dh))
    for b in range(B):
        L = int(ctx_len[b])
        for h in range(Hq):
            g = h // G
            for s in range(S):
                keys = [k_ctx[b, g, i] for i in range(L)] + [k_blk[b, j, g] for j in range(S)]
                vals = [v_ctx[b, g, i] for i in range(L)] + [v_blk[b, j, g] for j in range(S)]
                scores = []
                for k in keys:
                    acc = 0.0
                    for d in range(dh):
                        acc += q_blk[b, s, h, d] * k[d]
                    scores.append(acc / math.sqrt(dh))
                mx = max(scores)
                ws = [math.exp(x - mx) for x in scores]
                tot = sum(ws)
                for d in range(dh):
                    acc = 0.0
                    for w, v in zip(ws, vals):
                        acc += w * v[d]
                    out[b, s, h, d] = acc / tot
    return out


# ---- a2: adaLN-single modulation -------------------------------------------
def timestep_embedding(t: float, H: int) -> np.ndarray:
    """phi(t) in R^{2H}: [sin(t*w_i) for i<H] || [cos(t*w_i) for i<H].

    w_i = TIME_BASE^(-i/H).  The pages name adaLN time conditioning but give
    no embedding; this is the library's reading (sinusoidal, no MLP).
    """
    i = np.arange(H, dtype=np.float64)
    w = TIME_BASE ** (-i / H)
    return np.concatenate([np.sin(t * w), np.cos(t * w)])


def layer_norm(x: np.ndarray) -> np.ndarray:
    """LayerNorm over the last axis, no affine parameters, biased variance."""
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + LN_EPS)


def adaln_modulate(x: np.ndarray, shift_scale: np.ndarray, t_rows: np.ndarray) -> np.ndarray:
    """y = LN(x) * (1 + scale) + shift with [shift; scale] = E + phi(t).

    x [R, H] float64, shift_scale (E) [2, H] float64, t_rows [R] (time of the
    sequence each row belongs to).  Training and Conditioning, "Time
    Conditioning"; snilld.dk, adaLN-single block per layer.
    """
    R, H = x.shape
    y = np.empty_like(x)
    n = layer_norm(x)
    for r in range(R):
        phi = timestep_embedding(float(t_rows[r]), H)
        shift = shift_scale[0] + phi[:H]
        scale = shift_scale[1] + phi[H:]
        y[r] = n[r] * (1.0 + scale) + shift
    return y


# ---- a3: vocab projection and confidence -----------------------------------
def logits(y: np.ndarray, w: np.ndarray, logit_scale: float = 1.0) -> np.ndarray:
    """logit_scale * y @ W^T.  y [R, H], W [V, H] (one row per token)."""
    return logit_scale * (y @ w.T)


def confidence(lg: np.ndarray):
    """Per row: (max softmax probability, argmax token with lowest id on ties).

    conf = 1 / sum_j exp(l_j - max_j l_j); np.argmax returns the first index
    of the maximum, i.e. the lowest token id.
    """
    mx = lg.max(axis=-1, keepdims=True)
    z = np.exp(lg - mx).sum(axis=-1)
    conf = 1.0 / z
    tok = np.argmax(lg, axis=-1).astype(np.int64)
    return conf, tok


def top2_margin(lg: np.ndarray):
    """Per row: (gap between the two largest logits, top-2 probability gap)."""
    part = np.partition(lg, -2, axis=-1)
    l1, l2 = part[..., -1], part[..., -2]
    mx = l1[..., None]
    z = np.exp(lg - mx).sum(axis=-1)
    return l1 - l2, (1.0 - np.exp(l2 - l1)) / z


def vocab_confidence(y: np.ndarray, w_bits: np.ndarray, logit_scale: float = 1.0,
                     rows_per_block: int = 128):
    """conf, token and top-2 margins for each row of y against bf16 W.

    Rows are independent; they are processed a block at a time only to bound
    memory.  ``w_bits`` may also be W already widened to float64.
    """
    w = w_bits if w_bits.dtype == np.float64 else from_bf16(w_bits)
    R = y.shape[0]
    conf = np.empty(R)
    tok = np.empty(R, dtype=np.int64)
    gap_l = np.empty(R)
    gap_p = np.empty(R)
    for r0 in range(0, R, rows_per_block):
        lg = logits(y[r0:r0 + rows_per_block], w, logit_scale)
        c, t = confidence(lg)
        gl, gp = top2_margin(lg)
        conf[r0:r0 + len(c)] = c
        tok[r0:r0 + len(c)] = t
        gap_l[r0:r0 + len(c)] = gl
        gap_p[r0:r0 + len(c)] = gp
    return conf, tok, gap_l, gap_p


# ---- a4: commit (confidence unmasking) --------------------------------------
def commit(conf: np.ndarray, tok: np.ndarray, tokens: np.ndarray, masked: np.ndarray,
           gamma: float):
    """One confidence-unmasking decision for every sequence.

    conf/tok [B,S] (only masked entries are read), tokens int [B,S],
    masked bool/uint8 [B,S].  Returns (tokens', masked', committed [B,S] bool,
    fallback [B] bool).  Training and Conditioning, "Sampling": confident
    masked tokens commit, uncertain ones stay masked, so the number committed
    per step adapts; if no masked position reaches gamma the most confident
    one commits (lowest position on ties) so that every step makes progress.
    """
    tokens = np.array(tokens, copy=True)
    masked = np.array(masked, dtype=bool, copy=True)
    B, S = masked.shape
    committed = np.zeros((B, S), dtype=bool)
    fallback = np.zeros(B, dtype=bool)
    for b in range(B):
        cand = [s for s in range(S) if masked[b, s]]
        if not cand:
            continue
        chosen = [s for s in cand if conf[b, s] >= gamma]
        if not chosen:
            best = cand[0]
            for s in cand[1:]:
                if conf[b, s] > conf[b, best]:
                    best = s
            chosen = [best]
            fallback[b] = True
        for s in chosen:
            tokens[b, s] = tok[b, s]
            masked[b, s] = False
            committed[b, s] = True
    return tokens, masked, committed, fallback


# ---- a5: re-embedding and linear update -------------------------------------
def embed_block(tokens, masked, emb_bits, e_mask_bits) -> np.ndarray:
    """e[b,s] = e_MASK if masked else Emb[token]; float64 [B,S,H]."""
    B, S = masked.shape
    H = e_mask_bits.shape[0]
    e_mask = from_bf16(e_mask_bits)
    e = np.empty((B, S, H))
    for b in range(B):
        for s in range(S):
            e[b, s] = e_mask if masked[b, s] else from_bf16(emb_bits[int(tokens[b, s])])
    return e


def linear_update(e: np.ndarray, u_t: np.ndarray, Hq: int, Hkv: int, dh: int):
    """[q | k | v] = e @ U with U = u_t^T; each part rounded to bf16 (stored).

    e [B,S,H] float64, u_t [H + 2*Hkv*dh, H] float64.  Returns q [B,S,Hq,dh],
    k [B,S,Hkv,dh], v [B,S,Hkv,dh] (float64 values that are exactly bf16).
    """
    B, S, H = e.shape
    qkv = round_bf16(e @ u_t.T)
    q = qkv[..., :H].reshape(B, S, Hq, dh)
    k = qkv[..., H:H + Hkv * dh].reshape(B, S, Hkv, dh)
    v = qkv[..., H + Hkv * dh:].reshape(B, S, Hkv, dh)
    return q, k, v


# ---- one step and the loop --------------------------------------------------
def denoise_step(q, k, v, k_ctx, v_ctx, ctx_len, shift_scale, w_bits, tokens, masked,
                 gamma: float, logit_scale: float = 1.0):
    """a1 -> a2 -> a3 -> a4 for one step; q/k/v, contexts, E float64.

    Returns a dict with the bf16-rounded attention output ``o`` and adaLN
    output ``y`` (float64 [B,S,H]), per-position ``conf``/``tok`` (NaN/-1 for
    positions that were not masked), the margins, and the commit results.
    """
    B, S, Hq, dh = q.shape
    H = Hq * dh
    masked = np.asarray(masked, dtype=bool)
    o = round_bf16(block_attention(q, k, v, k_ctx, v_ctx, ctx_len)).reshape(B, S, H)
    t = masked.sum(axis=1) / S
    rows = [(b, s) for b in range(B) for s in range(S) if masked[b, s]]
    conf = np.full((B, S), np.nan)
    tok = np.full((B, S), -1, dtype=np.int64)
    gap_l = np.full((B, S), np.nan)
    gap_p = np.full((B, S), np.nan)
    y = np.full((B, S, H), np.nan)
    if rows:
        x = np.stack([o[b, s] for b, s in rows])
        tr = np.array([t[b] for b, s in rows])
        yr = round_bf16(adaln_modulate(x, shift_scale, tr))
        c, tk, gl, gp = vocab_confidence(yr, w_bits, logit_scale)
        for i, (b, s) in enumerate(rows):
            y[b, s] = yr[i]
            conf[b, s], tok[b, s], gap_l[b, s], gap_p[b, s] = c[i], tk[i], gl[i], gp[i]
    tokens2, masked2, committed, fallback = commit(conf, tok, tokens, masked, gamma)
    return dict(o=o, y=y, t=t, conf=conf, tok=tok, gap_l=gap_l, gap_p=gap_p,
                tokens=tokens2, masked=masked2, committed=committed, fallback=fallback)


def denoiser_layers(x, layers, ctx_len, t, Hq, Hkv, dh):
    """Every denoiser layer but the last, on all block rows (reading of the
    layer-aligned attention of the Architecture section: each denoiser layer
    attends to the context tower's KV of the same layer, with its own
    adaLN-single table).  Layer l: [q|k|v] = x.U_l, o = attention over
    [Kctx_l ; k], x <- adaLN_l(o, t), every stored tensor rounded to bf16.
    ``layers`` is a list of (u_t, k_ctx, v_ctx, E) float64 tuples; x is
    float64 [B,S,H]; t [B].  Returns the input of the last layer."""
    B, S, H = x.shape
    for u_t, kc, vc, E in layers:
        q, k, v = linear_update(x, u_t, Hq, Hkv, dh)
        o = round_bf16(block_attention(q, k, v, kc, vc, ctx_len)).reshape(B * S, H)
        x = round_bf16(adaln_modulate(o, E, np.repeat(t, S))).reshape(B, S, H)
    return x


def denoise_block_loop(inp: dict, gamma: float, logit_scale: float = 1.0,
                       max_steps: int | None = None, teacher=None):
    """Refine one block until every position is committed (Generation Process).

    ``inp`` holds the bf16 bit arrays of tt_inputs (k_ctx, v_ctx, shift_scale,
    w, emb, e_mask, u_t) plus ctx_len, tokens, masked.  Each step: embed ->
    linear update -> attention -> adaLN -> vocab confidence -> commit, with
    t_b recomputed from the mask.  With ``<name>_l`` arrays (several
    denoiser layers, tt_inputs.generate(n_layers=...)) the layers before the
    last run first (denoiser_layers) and the last one feeds the vocabulary.
    ``teacher`` (optional callable step -> (tokens, masked) or None) replaces
    the state at the start of a step, which lets a test follow another
    implementation's trajectory step by step.
    Returns dict(tokens, masked, steps_taken [B], commit_step [B,S], trace).
    """
    tokens = np.array(inp["tokens"], dtype=np.int64, copy=True)
    masked = np.array(inp["masked"], dtype=bool, copy=True)
    B, S = masked.shape
    Hkv, dh = inp["k_ctx"].shape[1], inp["k_ctx"].shape[3]
    H = inp["e_mask"].shape[0]
    Hq = H // dh
    if "k_ctx_l" in inp:
        n_layers = inp["k_ctx_l"].shape[0]
        per = [tuple(from_bf16(inp[n + "_l"][i]) for n in ("u_t", "k_ctx", "v_ctx", "shift_scale"))
               for i in range(n_layers)]
        early, (u_t, k_ctx, v_ctx, E) = per[:-1], per[-1]
    else:
        early = []
        k_ctx = from_bf16(inp["k_ctx"])
        v_ctx = from_bf16(inp["v_ctx"])
        E = from_bf16(inp["shift_scale"])
        u_t = from_bf16(inp["u_t"])
    w = from_bf16(inp["w"])
    steps_taken = np.zeros(B, dtype=np.int64)
    commit_step = np.full((B, S), -1, dtype=np.int64)
    max_steps = S if max_steps is None else max_steps
    trace = []
    for step in range(max_steps):
        if teacher is not None:
            st = teacher(step)
            if st is not None:
                tokens = np.array(st[0], dtype=np.int64, copy=True)
                masked = np.array(st[1], dtype=bool, copy=True)
        if not masked.any():
            break
        active = masked.any(axis=1)
        e = embed_block(tokens, masked, inp["emb"], inp["e_mask"])
        if early:
            e = denoiser_layers(e, early, inp["ctx_len"], masked.sum(axis=1) / S, Hq, Hkv, dh)
        q, k, v = linear_update(e, u_t, Hq, Hkv, dh)
        r = denoise_step(q, k, v, k_ctx, v_ctx, inp["ctx_len"], E, w, tokens, masked,
                         gamma, logit_scale)
        commit_step[r["committed"]] = step
        steps_taken[active] = step + 1
        tokens, masked = r["tokens"], r["masked"]
        r["q"], r["k"], r["v"] = q, k, v
        trace.append(r)
    return dict(tokens=tokens, masked=masked, steps_taken=steps_taken,
                commit_step=commit_step, trace=trace)


# ---- outer block loop (Generation Process: the context tower updates after
# each block commits, then the next block starts) ---------------------------
def append_block(k_ctx, v_ctx, ctx_len, tokens, emb_bits, u_ctx):
    """The committed block joins the context.  The frozen context tower is not
    modelled: a seeded projection stands in for it (reading), [k | v] of
    position s = Emb[token_s] . U_ctx^T, rounded to bf16 (stored), written at
    context positions ctx_len[b] + s.  k_ctx/v_ctx float64 [B,Hkv,L_cap,dh]
    (modified in place), u_ctx float64 [2*Hkv*dh, H].  Returns the new lengths.
    """
    B, S = tokens.shape
    Hkv, dh = k_ctx.shape[1], k_ctx.shape[3]
    e = np.stack([from_bf16(emb_bits[tokens[b]]) for b in range(B)])  # [B,S,H]
    kv = round_bf16(e @ u_ctx.T)                                       # [B,S,2*Hkv*dh]
    new_len = np.array(ctx_len, dtype=np.int64, copy=True)
    for b in range(B):
        L = int(ctx_len[b])
        if L + S > k_ctx.shape[2]:
            raise ValueError("context cache full")
        for s in range(S):
            k_ctx[b, :, L + s] = kv[b, s, :Hkv * dh].reshape(Hkv, dh)
            v_ctx[b, :, L + s] = kv[b, s, Hkv * dh:].reshape(Hkv, dh)
        new_len[b] = L + S
    return new_len


def decode_blocks(inp: dict, n_blocks: int, gamma: float, logit_scale: float = 1.0,
                  teacher=None):
    """n_blocks blocks one after the other (Generation Process): each block
    starts fully masked, is refined to completion by denoise_block_loop, then
    joins the context (append_block).  ``teacher`` (optional callable
    block -> tokens [B,S] or None) replaces a block's committed tokens before
    it joins the context, so a test can follow another implementation.
    Returns dict(tokens [n_blocks,B,S], ctx_len, k_ctx, v_ctx (float64),
    blocks: the per-block loop results)."""
    B, S = inp["tokens"].shape
    k_ctx = from_bf16(inp["k_ctx"])
    v_ctx = from_bf16(inp["v_ctx"])
    u_ctx = from_bf16(inp["u_ctx"])
    ctx_len = np.array(inp["ctx_len"], dtype=np.int64, copy=True)
    out_tokens, blocks = [], []
    for j in range(n_blocks):
        blk = dict(inp, k_ctx=_to_bits(k_ctx), v_ctx=_to_bits(v_ctx),
                   ctx_len=ctx_len.astype(np.int32),
                   tokens=np.full((B, S), -1, dtype=np.int32),
                   masked=np.ones((B, S), dtype=np.uint8))
        r = denoise_block_loop(blk, gamma, logit_scale)
        tok = r["tokens"]
        if teacher is not None:
            t = teacher(j)
            if t is not None:
                tok = np.asarray(t, dtype=np.int64)
        ctx_len = append_block(k_ctx, v_ctx, ctx_len, tok, inp["emb"], u_ctx)
        out_tokens.append(tok)
        blocks.append(r)
    return dict(tokens=np.stack(out_tokens), ctx_len=ctx_len, k_ctx=k_ctx, v_ctx=v_ctx,
                blocks=blocks)


def _to_bits(x: np.ndarray) -> np.ndarray:
    """float64 values that are exactly bf16 -> their bf16 bit patterns."""
    u = x.astype(np.float32).view(np.uint32)
    return (u >> 16).astype(np.uint16)
