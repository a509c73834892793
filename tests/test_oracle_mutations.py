"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's source: a dropped
term, a wrong sign, index or axis, a transposed or swapped operand, an
off-by-one, a tie broken the other way.  It then runs every pin in
test_oracle_pins against that copy, and at least one pin must fail.  The
unmodified source must pass them all.  Nothing here touches the GPU path,
and the mistakes are planted on the CPU only, in the copy.
"""
import inspect
import types

import pytest

from oracle import twotower_oracle
import test_oracle_pins as P

SRC = inspect.getsource(twotower_oracle)

# (name, text in the oracle, replacement, occurrences to replace)
MUTATIONS = [
    # bf16 format
    ("round-ties-away", "r = np.round(scaled)", "r = np.floor(scaled + 0.5)", 1),
    ("round-no-subnormal-floor", "e = np.maximum(e, -125)", "e = np.maximum(e, -126)", 1),
    ("from-bf16-shift", "<< np.uint32(16)", "<< np.uint32(15)", 1),
    # attention
    ("attn-no-scale", 'sc = np.einsum("sjd,kd->sjk", q, keys) * scale',
     'sc = np.einsum("sjd,kd->sjk", q, keys)', 1),
    ("attn-scale-1/dh", "scale = 1.0 / math.sqrt(dh)\n    for b", "scale = 1.0 / dh\n    for b", 1),
    ("attn-ctx-off-by-one", "[b, g, :L]", "[b, g, :L - 1]", 2),
    ("attn-no-block-keys", "keys = np.concatenate([k_ctx[b, g, :L], k_blk[b, :, g]], axis=0)",
     "keys = np.concatenate([k_ctx[b, g, :L], 0 * k_blk[b, :, g]], axis=0)", 1),
    ("attn-values-are-keys", "vals = np.concatenate([v_ctx[b, g, :L], v_blk[b, :, g]], axis=0)",
     "vals = np.concatenate([k_ctx[b, g, :L], k_blk[b, :, g]], axis=0)", 1),
    ("loops-no-scale", "scores.append(acc / math.sqrt(dh))", "scores.append(acc)", 1),
    ("attn-gqa-interleaved", "q_blk[b, :, g * G:(g + 1) * G, :]", "q_blk[b, :, g::Hkv, :]", 1),
    ("attn-softmax-wrong-axis", "p /= p.sum(axis=-1, keepdims=True)",
     "p /= p.sum(axis=0, keepdims=True)", 1),
    # adaLN
    ("time-sin-cos-swapped", "[np.sin(t * w), np.cos(t * w)]", "[np.cos(t * w), np.sin(t * w)]", 1),
    ("time-frequency-sign", "w = TIME_BASE ** (-i / H)", "w = TIME_BASE ** (i / H)", 1),
    ("time-frequency-doubled", "w = TIME_BASE ** (-i / H)", "w = TIME_BASE ** (-2 * i / H)", 1),
    ("ln-unbiased-variance", "var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)",
     "var = ((x - mu) ** 2).sum(axis=-1, keepdims=True) / (x.shape[-1] - 1)", 1),
    ("ln-no-sqrt", "(x - mu) / np.sqrt(var + LN_EPS)", "(x - mu) / (var + LN_EPS)", 1),
    ("ln-not-centred", "return (x - mu) / np.sqrt", "return x / np.sqrt", 1),
    ("adaln-no-one-plus", "n[r] * (1.0 + scale) + shift", "n[r] * scale + shift", 1),
    ("adaln-shift-scale-swapped", "shift = shift_scale[0] + phi[:H]",
     "shift = shift_scale[1] + phi[:H]", 1),
    # vocabulary and confidence
    ("logits-no-scale", "return logit_scale * (y @ w.T)", "return y @ w.T", 1),
    ("conf-is-z", "conf = 1.0 / z", "conf = z / z.max()", 1),
    ("argmax-highest-id-on-ties", "tok = np.argmax(lg, axis=-1).astype(np.int64)",
     "tok = (lg.shape[-1] - 1 - np.argmax(lg[..., ::-1], axis=-1)).astype(np.int64)", 1),
    ("margin-sign", "return l1 - l2, (1.0 - np.exp(l2 - l1)) / z",
     "return l2 - l1, (1.0 - np.exp(l2 - l1)) / z", 1),
    # commit
    ("commit-strict-gamma", "if conf[b, s] >= gamma]", "if conf[b, s] > gamma]", 1),
    ("commit-fallback-last-on-ties", "if conf[b, s] > conf[b, best]:",
     "if conf[b, s] >= conf[b, best]:", 1),
    ("commit-reconsiders-unmasked", "cand = [s for s in range(S) if masked[b, s]]",
     "cand = [s for s in range(S) if masked[b, s] or conf[b, s] == conf[b, s]]", 1),
    ("commit-no-fallback", "            chosen = [best]\n", "            chosen = []\n", 1),
    # re-embedding and the linear update
    ("embed-mask-inverted", "e_mask if masked[b, s] else", "e_mask if not masked[b, s] else", 1),
    ("qkv-k-v-swapped", "k = qkv[..., H:H + Hkv * dh]", "k = qkv[..., H + Hkv * dh:]", 1),
    ("qkv-dh-major-heads", "q = qkv[..., :H].reshape(B, S, Hq, dh)",
     "q = qkv[..., :H].reshape(B, S, dh, Hq).transpose(0, 1, 3, 2)", 1),
    ("qkv-not-rounded", "qkv = round_bf16(e @ u_t.T)", "qkv = e @ u_t.T", 1),
    # step and loop bookkeeping
    ("time-is-committed-fraction", "t = masked.sum(axis=1) / S", "t = 1.0 - masked.sum(axis=1) / S", 1),
    ("step-time-of-first-sequence", "tr = np.array([t[b] for b, s in rows])",
     "tr = np.array([t[0] for b, s in rows])", 1),
    ("attn-output-not-rounded",
     "o = round_bf16(block_attention(q, k, v, k_ctx, v_ctx, ctx_len)).reshape(B, S, H)",
     "o = block_attention(q, k, v, k_ctx, v_ctx, ctx_len).reshape(B, S, H)", 1),
    ("steps-taken-off-by-one", "steps_taken[active] = step + 1", "steps_taken[active] = step", 1),
    ("commit-step-off-by-one", "commit_step[r[\"committed\"]] = step",
     "commit_step[r[\"committed\"]] = step + 1", 1),
    # layers
    ("layers-time-tiled", "np.repeat(t, S)", "np.tile(t, S)", 1),
    ("layers-shared-context", "early, (u_t, k_ctx, v_ctx, E) = per[:-1], per[-1]",
     "early, (u_t, k_ctx, v_ctx, E) = [(l[0], per[-1][1], per[-1][2], l[3]) for l in per[:-1]], per[-1]",
     1),
    # block after block
    ("append-at-zero", "k_ctx[b, :, L + s] =", "k_ctx[b, :, s] =", 1),
    ("append-not-rounded", "kv = round_bf16(e @ u_ctx.T)", "kv = e @ u_ctx.T", 1),
    ("append-length-short", "new_len[b] = L + S", "new_len[b] = L + S - 1", 1),
    ("append-k-v-swapped", "k_ctx[b, :, L + s] = kv[b, s, :Hkv * dh]",
     "k_ctx[b, :, L + s] = kv[b, s, Hkv * dh:]", 1),
    ("decode-context-not-grown", "blk = dict(inp, k_ctx=_to_bits(k_ctx), v_ctx=_to_bits(v_ctx),",
     "blk = dict(inp, k_ctx=inp[\"k_ctx\"], v_ctx=inp[\"v_ctx\"],", 1),
    ("to-bits-shift", "return (u >> 16).astype(np.uint16)", "return (u >> 17).astype(np.uint16)", 1),
]


def _pins():
    return [(n, f) for n, f in sorted(vars(P).items())
            if n.startswith("test_") and callable(f)]


def _copy(src):
    mod = types.ModuleType("twotower_oracle_copy")
    mod.__file__ = twotower_oracle.__file__
    exec(compile(src, "<twotower_oracle copy>", "exec"), mod.__dict__)
    return mod


def _mutant(old, new, count):
    assert SRC.count(old) == count, f"{old!r} occurs {SRC.count(old)} times, expected {count}"
    return _copy(SRC.replace(old, new))


def _failing_pins(mod, monkeypatch):
    monkeypatch.setattr(P, "O", mod)
    failed = []
    for name, fn in _pins():
        try:
            fn()
        except Exception:  # noqa: BLE001 - any failure of a pin counts
            failed.append(name)
    return failed


def test_unmodified_copy_passes_every_pin(monkeypatch):
    assert _failing_pins(_copy(SRC), monkeypatch) == []


@pytest.mark.parametrize("name,old,new,count", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(monkeypatch, name, old, new, count):
    failed = _failing_pins(_mutant(old, new, count), monkeypatch)
    assert failed, f"no pin catches the planted mistake {name}"
