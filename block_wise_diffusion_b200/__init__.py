"""Python binding of libtwotower (argument marshalling only).

Every function with a ``tt_`` name calls the C entry point of the same name
in ``libtwotower.so`` (built in-tree by ``block_wise_diffusion_b200.build``)
with raw device pointers taken from torch tensors.  Nothing here computes:
torch provides device memory and streams; all arithmetic runs in the
library's sm_100a kernels.  There is no CPU path: if the library or a CUDA
device is missing, the calls raise.  Before a call, every tensor argument is
checked to hold at least the bytes of the shape include/twotower.h documents
for it, since the kernels address each buffer from the dims alone.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "TTError", "Dims", "lib", "lib_path", "dims", "workspace", "tt_workspace_bytes",
    "tt_block_denoise_attn", "tt_adaln_modulate", "tt_vocab_confidence_commit",
    "tt_denoise_block_loop", "tt_denoise_block_loop_layers", "tt_decode_blocks",
    "tt_vocab_confidence_commit_noalloc", "tt_loop_last_step",
    "tt_device_status", "tt_launch_count", "tt_set_attn_splits", "tt_set_loop_graphs",
    "tt_status_string", "tt_last_error", "EXPORTS", "tt_profile_enable", "tt_profile_read",
    "tt_selftest_timeout",
    "profile_table", "KERNEL_KINDS",
    "TT_WS_ATTN", "TT_WS_ADALN", "TT_WS_VOCAB", "TT_WS_LOOP",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libtwotower.so")

TT_WS_ATTN, TT_WS_ADALN, TT_WS_VOCAB, TT_WS_LOOP = 0, 1, 2, 3
STATUS = {0: "TT_OK", 1: "TT_ERR_INVALID_ARG", 2: "TT_ERR_UNSUPPORTED", 3: "TT_ERR_WORKSPACE",
          4: "TT_ERR_CUDA", 5: "TT_ERR_TIMEOUT", 6: "TT_ERR_INTERNAL"}

# Every symbol the header declares.
EXPORTS = (
    "tt_status_string", "tt_last_error", "tt_workspace_bytes", "tt_device_status",
    "tt_launch_count", "tt_set_attn_splits", "tt_set_loop_graphs", "tt_block_denoise_attn",
    "tt_adaln_modulate",
    "tt_vocab_confidence_commit", "tt_denoise_block_loop", "tt_profile_enable", "tt_profile_read",
    "tt_vocab_confidence_commit_noalloc", "tt_selftest_timeout", "tt_denoise_block_loop_layers",
    "tt_decode_blocks", "tt_loop_last_step",
)
KERNEL_KINDS = ("plan", "embed", "gemm_qkv", "attn", "merge", "adaln", "gemm_vocab", "commit",
                "gather", "init", "splitk_reduce", "append", "attn_plan")


class TTError(RuntimeError):
    def __init__(self, code: int, where: str, detail: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)}: {detail}")


class Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "S", "Hq", "Hkv", "dh", "H", "V", "L_cap")]


_P = ctypes.c_void_p
_lib = None


def lib() -> ctypes.CDLL:
    """Load libtwotower.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(lib_path):
            raise RuntimeError(
                f"{lib_path} is missing: build it with `python -m block_wise_diffusion_b200.build`")
        L = ctypes.CDLL(lib_path)
        L.tt_status_string.restype = ctypes.c_char_p
        L.tt_status_string.argtypes = [ctypes.c_int]
        L.tt_last_error.restype = ctypes.c_char_p
        L.tt_last_error.argtypes = []
        L.tt_workspace_bytes.restype = ctypes.c_size_t
        L.tt_workspace_bytes.argtypes = [ctypes.POINTER(Dims), ctypes.c_int]
        L.tt_device_status.restype = ctypes.c_int
        L.tt_device_status.argtypes = [_P, _P]
        L.tt_selftest_timeout.restype = ctypes.c_int
        L.tt_selftest_timeout.argtypes = [_P, ctypes.c_int32, _P]
        L.tt_launch_count.restype = ctypes.c_uint64
        L.tt_launch_count.argtypes = []
        L.tt_set_attn_splits.restype = ctypes.c_int
        L.tt_set_attn_splits.argtypes = [ctypes.c_int32]
        L.tt_set_loop_graphs.restype = ctypes.c_int
        L.tt_set_loop_graphs.argtypes = [ctypes.c_int32]
        L.tt_profile_enable.restype = ctypes.c_int
        L.tt_profile_enable.argtypes = [ctypes.c_int32]
        L.tt_profile_read.restype = ctypes.c_int
        L.tt_profile_read.argtypes = [ctypes.c_int32, ctypes.POINTER(ctypes.c_double),
                                      ctypes.POINTER(ctypes.c_int64)]
        L.tt_block_denoise_attn.restype = ctypes.c_int
        L.tt_block_denoise_attn.argtypes = [ctypes.POINTER(Dims)] + [_P] * 7 + [_P, ctypes.c_size_t, _P]
        L.tt_adaln_modulate.restype = ctypes.c_int
        L.tt_adaln_modulate.argtypes = [ctypes.POINTER(Dims), _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
        L.tt_vocab_confidence_commit.restype = ctypes.c_int
        L.tt_vocab_confidence_commit.argtypes = (
            [ctypes.POINTER(Dims), _P, _P, ctypes.c_float, ctypes.c_float] + [_P] * 5
            + [_P, ctypes.c_size_t, _P])
        L.tt_vocab_confidence_commit_noalloc.restype = ctypes.c_int
        L.tt_vocab_confidence_commit_noalloc.argtypes = (
            [ctypes.POINTER(Dims), _P, _P, ctypes.c_float, ctypes.c_float] + [_P] * 5 + [_P])
        L.tt_denoise_block_loop.restype = ctypes.c_int
        L.tt_denoise_block_loop.argtypes = (
            [ctypes.POINTER(Dims)] + [_P] * 8 + [ctypes.c_float, ctypes.c_float, ctypes.c_int32]
            + [_P] * 5 + [_P, ctypes.c_size_t, _P])
        L.tt_decode_blocks.restype = ctypes.c_int
        L.tt_decode_blocks.argtypes = (
            [ctypes.POINTER(Dims), ctypes.c_int32] + [_P] * 9
            + [ctypes.c_float, ctypes.c_float] + [_P] * 4 + [_P, ctypes.c_size_t, _P])
        L.tt_loop_last_step.restype = ctypes.c_int
        L.tt_loop_last_step.argtypes = [ctypes.POINTER(Dims), _P, ctypes.c_size_t] + [_P] * 5 + [_P]
        L.tt_denoise_block_loop_layers.restype = ctypes.c_int
        L.tt_denoise_block_loop_layers.argtypes = (
            [ctypes.POINTER(Dims), ctypes.c_int32] + [_P] * 8
            + [ctypes.c_float, ctypes.c_float, ctypes.c_int32] + [_P] * 5
            + [_P, ctypes.c_size_t, _P])
        _lib = L
    return _lib


def dims(d) -> Dims:
    """tt_dims from any object with B, S, Hq, Hkv, dh, V, L_cap (and H) fields."""
    H = getattr(d, "H", d.Hq * d.dh)
    return Dims(d.B, d.S, d.Hq, d.Hkv, d.dh, H, d.V, d.L_cap)


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if not x.is_cuda:
        raise ValueError("libtwotower takes CUDA tensors only (no CPU path)")
    if not x.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return x.data_ptr()


def _nbytes(x) -> int:
    return x.numel() * x.element_size() if hasattr(x, "numel") else 0


def _sized(x, name: str, nbytes: int) -> int | None:
    """_ptr(x) after checking that a tensor holds at least ``nbytes``: the
    shape include/twotower.h documents for the argument times its element
    size.  The kernels address these buffers from the dims alone, so a short
    tensor would be read or written past its end.  Raw integer addresses
    carry no size and pass unchecked."""
    if x is not None and not isinstance(x, int) and _nbytes(x) < nbytes:
        raise ValueError(f"{name} holds {_nbytes(x)} bytes; these dims need {nbytes}")
    return _ptr(x)


def _ctx_bytes(d: Dims) -> int:
    """bf16 [B, Hkv, L_cap, dh]: one context cache (K or V) of one layer."""
    return d.B * d.Hkv * d.L_cap * d.dh * 2


def _u_t_bytes(d: Dims) -> int:
    """bf16 [H + 2*Hkv*dh, H]: one layer's linear update."""
    return (d.H + 2 * d.Hkv * d.dh) * d.H * 2


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _check(code: int, where: str) -> None:
    if code != 0:
        raise TTError(code, where, lib().tt_last_error().decode())


def tt_status_string(code: int) -> str:
    return lib().tt_status_string(code).decode()


def tt_last_error() -> str:
    return lib().tt_last_error().decode()


def tt_launch_count() -> int:
    return int(lib().tt_launch_count())


def tt_set_attn_splits(n: int) -> None:
    _check(lib().tt_set_attn_splits(n), "tt_set_attn_splits")


def tt_set_loop_graphs(on: int) -> None:
    _check(lib().tt_set_loop_graphs(on), "tt_set_loop_graphs")


def tt_profile_enable(on: bool) -> None:
    _check(lib().tt_profile_enable(1 if on else 0), "tt_profile_enable")


def tt_profile_read(kind: int) -> tuple[float, int]:
    """(total ms, launches) of one kernel kind since profiling was enabled."""
    ms, n = ctypes.c_double(0), ctypes.c_int64(0)
    _check(lib().tt_profile_read(kind, ctypes.byref(ms), ctypes.byref(n)), "tt_profile_read")
    return ms.value, n.value


def profile_table() -> dict:
    """{kernel kind name: (total ms, launches)} for every kind that ran."""
    out = {}
    for k, name in enumerate(KERNEL_KINDS):
        ms, n = tt_profile_read(k)
        if n:
            out[name] = (ms, n)
    return out


def tt_workspace_bytes(d: Dims, which: int) -> int:
    n = lib().tt_workspace_bytes(ctypes.byref(d), which)
    if n == 0:
        raise TTError(1, "tt_workspace_bytes", tt_last_error())
    return int(n)


def workspace(d: Dims, which: int, device="cuda"):
    """A torch uint8 device buffer of tt_workspace_bytes(d, which) bytes."""
    import torch
    return torch.empty(tt_workspace_bytes(d, which), dtype=torch.uint8, device=device)


def tt_selftest_timeout(ws, limit_us: int, stream=None) -> None:
    """Make one bounded device wait run out on purpose (see the header)."""
    _check(lib().tt_selftest_timeout(_ptr(ws), int(limit_us), _stream(stream)),
           "tt_selftest_timeout")


def tt_device_status(ws, stream=None) -> int:
    """Synchronise and return (and clear) the device error code in `ws`."""
    return int(lib().tt_device_status(_ptr(ws), _stream(stream)))


def tt_block_denoise_attn(d: Dims, q_blk, k_blk, v_blk, k_ctx, v_ctx, ctx_len, out, ws,
                          stream=None) -> None:
    rows = d.B * d.S
    _check(lib().tt_block_denoise_attn(
        ctypes.byref(d), _sized(q_blk, "q_blk", rows * d.Hq * d.dh * 2),
        _sized(k_blk, "k_blk", rows * d.Hkv * d.dh * 2),
        _sized(v_blk, "v_blk", rows * d.Hkv * d.dh * 2), _sized(k_ctx, "k_ctx", _ctx_bytes(d)),
        _sized(v_ctx, "v_ctx", _ctx_bytes(d)), _sized(ctx_len, "ctx_len", d.B * 4),
        _sized(out, "out", rows * d.Hq * d.dh * 2), _ptr(ws), _nbytes(ws),
        _stream(stream)), "tt_block_denoise_attn")


def tt_adaln_modulate(d: Dims, x, shift_scale, t, y, ws, stream=None) -> None:
    rows = d.B * d.S
    _check(lib().tt_adaln_modulate(
        ctypes.byref(d), _sized(x, "x", rows * d.H * 2),
        _sized(shift_scale, "shift_scale", 2 * d.H * 2), _sized(t, "t", d.B * 4),
        _sized(y, "y", rows * d.H * 2), _ptr(ws), _nbytes(ws), _stream(stream)),
        "tt_adaln_modulate")


def tt_vocab_confidence_commit(d: Dims, y, w, gamma: float, logit_scale: float, tokens, masked,
                               conf_out, argmax_out, n_committed, ws, stream=None) -> None:
    _check(lib().tt_vocab_confidence_commit(
        ctypes.byref(d), *_vocab_args(d, y, w, gamma, logit_scale, tokens, masked, conf_out,
                                      argmax_out, n_committed),
        _ptr(ws), _nbytes(ws), _stream(stream)), "tt_vocab_confidence_commit")


def _vocab_args(d: Dims, y, w, gamma, logit_scale, tokens, masked, conf_out, argmax_out,
                n_committed) -> tuple:
    rows = d.B * d.S
    return (_sized(y, "y", rows * d.H * 2), _sized(w, "w", d.V * d.H * 2), float(gamma),
            float(logit_scale), _sized(tokens, "tokens", rows * 4),
            _sized(masked, "masked", rows), _sized(conf_out, "conf_out", rows * 4),
            _sized(argmax_out, "argmax_out", rows * 4),
            _sized(n_committed, "n_committed", d.B * 4))


def tt_vocab_confidence_commit_noalloc(d: Dims, y, w, gamma: float, logit_scale: float,
                                       tokens, masked, conf_out, argmax_out, n_committed,
                                       stream=None) -> None:
    """tt_vocab_confidence_commit without a workspace, for callers that cannot
    allocate device memory; its scratch is a 16 MiB array built into the
    library (calls that overlap on the GPU must be serialised)."""
    _check(lib().tt_vocab_confidence_commit_noalloc(
        ctypes.byref(d), *_vocab_args(d, y, w, gamma, logit_scale, tokens, masked, conf_out,
                                      argmax_out, n_committed), _stream(stream)),
        "tt_vocab_confidence_commit_noalloc")


def tt_denoise_block_loop(d: Dims, k_ctx, v_ctx, ctx_len, emb, e_mask, u_t, shift_scale, w,
                          gamma: float, logit_scale: float, max_steps: int, tokens, masked,
                          steps_taken, commit_step, ws, stream=None) -> int:
    """Runs the loop; returns the number of steps that did work."""
    steps_run = ctypes.c_int32(0)
    _check(lib().tt_denoise_block_loop(
        ctypes.byref(d), *_loop_args(d, 1, k_ctx, v_ctx, ctx_len, emb, e_mask, u_t, shift_scale,
                                     w),
        float(gamma), float(logit_scale), int(max_steps),
        *_state_args(d, tokens, masked, steps_taken, commit_step),
        ctypes.addressof(steps_run), _ptr(ws), _nbytes(ws), _stream(stream)),
        "tt_denoise_block_loop")
    return int(steps_run.value)


def _loop_args(d: Dims, n_layers: int, k_ctx, v_ctx, ctx_len, emb, e_mask, u_t, shift_scale,
               w) -> tuple:
    """Checked pointers of the loop's inputs; per-layer tensors hold n_layers
    stacked copies (layer outermost)."""
    nl = max(int(n_layers), 0)
    return (_sized(k_ctx, "k_ctx", nl * _ctx_bytes(d)), _sized(v_ctx, "v_ctx", nl * _ctx_bytes(d)),
            _sized(ctx_len, "ctx_len", d.B * 4), _sized(emb, "emb", d.V * d.H * 2),
            _sized(e_mask, "e_mask", d.H * 2), _sized(u_t, "u_t", nl * _u_t_bytes(d)),
            _sized(shift_scale, "shift_scale", nl * 2 * d.H * 2),
            _sized(w, "w", d.V * d.H * 2))


def _state_args(d: Dims, tokens, masked, steps_taken, commit_step) -> tuple:
    rows = d.B * d.S
    return (_sized(tokens, "tokens", rows * 4), _sized(masked, "masked", rows),
            _sized(steps_taken, "steps_taken", d.B * 4),
            _sized(commit_step, "commit_step", rows * 4))


def tt_decode_blocks(d: Dims, n_blocks: int, k_ctx, v_ctx, ctx_len, emb, e_mask, u_t,
                     shift_scale, w, u_ctx, gamma: float, logit_scale: float, tokens,
                     steps_taken, commit_step, ws, stream=None) -> int:
    """n_blocks blocks one after the other, each joining the context once
    committed (k_ctx, v_ctx and ctx_len are updated in place); returns the
    total number of steps that did work."""
    steps_run = ctypes.c_int32(0)
    nb = max(int(n_blocks), 0)
    rows = d.B * d.S
    _check(lib().tt_decode_blocks(
        ctypes.byref(d), int(n_blocks),
        *_loop_args(d, 1, k_ctx, v_ctx, ctx_len, emb, e_mask, u_t, shift_scale, w),
        _sized(u_ctx, "u_ctx", 2 * d.Hkv * d.dh * d.H * 2), float(gamma), float(logit_scale),
        _sized(tokens, "tokens", nb * rows * 4), _sized(steps_taken, "steps_taken", nb * d.B * 4),
        _sized(commit_step, "commit_step", nb * rows * 4),
        ctypes.addressof(steps_run), _ptr(ws), _nbytes(ws), _stream(stream)),
        "tt_decode_blocks")
    return int(steps_run.value)


def tt_denoise_block_loop_layers(d: Dims, n_layers: int, k_ctx, v_ctx, ctx_len, emb, e_mask,
                                 u_t, shift_scale, w, gamma: float, logit_scale: float,
                                 max_steps: int, tokens, masked, steps_taken, commit_step, ws,
                                 stream=None) -> int:
    """The loop over n_layers denoiser layers (per-layer tensors stacked with
    the layer outermost); returns the number of steps that did work."""
    steps_run = ctypes.c_int32(0)
    _check(lib().tt_denoise_block_loop_layers(
        ctypes.byref(d), int(n_layers),
        *_loop_args(d, n_layers, k_ctx, v_ctx, ctx_len, emb, e_mask, u_t, shift_scale, w),
        float(gamma), float(logit_scale), int(max_steps),
        *_state_args(d, tokens, masked, steps_taken, commit_step),
        ctypes.addressof(steps_run), _ptr(ws), _nbytes(ws), _stream(stream)),
        "tt_denoise_block_loop_layers")
    return int(steps_run.value)


def tt_loop_last_step(d: Dims, ws, y_rows, row_ids, conf, argmax, stream=None) -> int:
    """Copy out what the loop's last working step fed the vocabulary and the
    commit rule (data copies only): the compacted adaLN rows into y_rows
    [B*S, H] bf16, their row indices b*S+s into row_ids [B*S] int32, and the
    confidence / argmax of each position masked at the start of the step into
    conf [B*S] float32 and argmax [B*S] int32 (-1 elsewhere).  Returns the
    number of compacted rows."""
    rows = d.B * d.S
    n = ctypes.c_int32(0)
    _check(lib().tt_loop_last_step(
        ctypes.byref(d), _ptr(ws), _nbytes(ws), _sized(y_rows, "y_rows", rows * d.H * 2),
        _sized(row_ids, "row_ids", rows * 4), _sized(conf, "conf", rows * 4),
        _sized(argmax, "argmax", rows * 4), ctypes.addressof(n), _stream(stream)),
        "tt_loop_last_step")
    return int(n.value)
