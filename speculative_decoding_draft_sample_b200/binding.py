"""Thin Python binding of libdspark.so (include/dspark.h), via ctypes.

Argument marshalling only: every function takes PyTorch CUDA tensors, checks
that they are contiguous and on the device, and passes their data pointers and
sizes to the C entry point of the same name. All arithmetic happens in the
library's kernels; there is no fallback path. If the library is missing, every
call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdspark.so")

F32, BF16 = 0, 1
OP_DRAFT, OP_SCHEDULE, OP_VERIFY, OP_CALIB = 0, 1, 2, 3
CUT_COST, CUT_THRESHOLD, CUT_NONE = 0, 1, 2
STATUS_BAD_TOKEN, STATUS_BAD_ROW, STATUS_BAD_CUT, STATUS_BAD_TEMP, STATUS_TIMEOUT = 1, 2, 4, 8, 16
STATUS_INTERNAL = 32

_lib = None

_p = ctypes.c_void_p
_i = ctypes.c_int
_u64 = ctypes.c_uint64
_sz = ctypes.c_size_t
_f = ctypes.c_float

SIGNATURES = {
    "dspark_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "dspark_draft_sample": (_i, [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _u64, _u64,
                                 _p, _p, _p, _p, _p, _p, _sz, _p]),
    "dspark_prefix_schedule": (_i, [_p, _p, _p, _f, _i, _i, _i, _f, _p, _p, _p, _sz, _p]),
    "dspark_verify": (_i, [_p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _u64, _u64, _p, _p, _p,
                           _p, _sz, _p]),
    "dspark_verify_target_stats": (_i, [_p, _p, _p, _i, _i, _i, _i, _p, _sz, _p]),
    "dspark_verify_from_stats": (_i, [_p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _u64, _u64, _p,
                                      _p, _p, _p, _sz, _p]),
    "dspark_draft_logits": (_i, [_p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _p, _p,
                                 _sz, _p]),
    "dspark_draft_pick": (_i, [_p, _p, _p, _i, _i, _i, _i, _u64, _u64, _i, _p, _p, _p, _p, _p,
                               _sz, _p]),
    "dspark_draft_sample_recurrent": (_i, [_p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _u64,
                                           _u64, _p, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "dspark_draft_sample_beside": (_i, [_p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _u64,
                                        _u64, _p, _p, _p, _p, _p, _p, _i, _p, _sz, _p]),
    "dspark_draft_sample_static": (_i, [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _u64, _u64,
                                        _p, _p, _p, _p, _p, _p]),
    "dspark_sts_fit": (_i, [_p, _p, _i, _i, _p, _p, _p, _p, _p, _sz, _p]),
    "dspark_read_status": (_i, [_p, _p, ctypes.POINTER(ctypes.c_uint32),
                                ctypes.POINTER(ctypes.c_int32)]),
    "dspark_clear_status": (_i, [_p, _p]),
    "dspark_status_string": (ctypes.c_char_p, [_i]),
    "dspark_version": (_i, []),
    "dspark_selftest_waits": (_i, [_p, _p, _sz, _p]),
}


class DSparkError(RuntimeError):
    pass


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise DSparkError(f"{LIB_PATH} is missing: build it with "
                              "`python -m speculative_decoding_draft_sample_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(rc: int, what: str) -> None:
    if rc != 0:
        msg = lib().dspark_status_string(rc).decode()
        raise DSparkError(f"{what} failed ({rc}): {msg}")


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise DSparkError(f"unsupported logit dtype {t.dtype}")


def _ptr(t: Optional[torch.Tensor], name: str, dtype=None, shape=None,
         device=None) -> Optional[int]:
    """The tensor's device pointer after checking it against the call's shapes.

    The library sees only pointers and the sizes B, K, V, r; a tensor smaller
    than those sizes imply would be read or written past its end on the device,
    so every tensor's shape is checked here (`shape`), as are its dtype,
    layout and device (`device`: the device of the call's first tensor).
    """
    if t is None:
        return None
    if dtype is not None and t.dtype != dtype:
        raise DSparkError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise DSparkError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise DSparkError(f"{name} must be contiguous")
    if device is None:
        if not t.is_cuda:
            raise DSparkError(f"{name} must be a CUDA tensor")
    elif t.device != device:
        raise DSparkError(f"{name} is on {t.device}, the call's tensors on {device}")
    return t.data_ptr()


def _on_gpu(device: torch.device) -> None:
    """Every tensor of a call is on `device` (checked by _ptr); it must be a GPU."""
    if device.type != "cuda":
        raise DSparkError(f"the call's tensors must be CUDA tensors, not on {device}")


def _stream(stream, device: torch.device) -> int:
    """The handle of `stream`, or of `device`'s current stream; a stream of
    another device is refused (its kernels would run there with this
    device's pointers)."""
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    if stream.device != device:
        raise DSparkError(f"the stream is on {stream.device}, the call's tensors on {device}")
    return stream.cuda_stream


def _call(name: str, device: torch.device, args, stream) -> None:
    """Calls entry point `name` with `device` current: the library launches
    on the current device and looks up per-device state there, so it must be
    the device that holds the call's tensors."""
    _on_gpu(device)
    s = _stream(stream, device)
    with torch.cuda.device(device):
        rc = getattr(lib(), name)(*args, s)
    _check(rc, name)


def workspace_bytes(op: int, B: int, K: int, V: int, r: int, dtype: int) -> int:
    return int(lib().dspark_workspace_bytes(op, B, K, V, r, dtype))


def version() -> int:
    return int(lib().dspark_version())


def draft_sample(base, U, W, bias_scale, last_tok, temp, seed: int, round_id: int,
                 x, d, q_lse, q_tok, ws, stream=None, q_norm=None) -> None:
    """dspark_draft_sample: base [B,K,V], U [V,r], W [r,V] -> x, d, q_lse, q_tok
    (and q_norm [B,K,2] when given)."""
    B, K, V = base.shape
    r = U.shape[1]
    dt = _dtype_code(base)
    dev, f32, i32 = base.device, torch.float32, torch.int32
    args = (
        _ptr(base, "base", None, (B, K, V), dev), _ptr(U, "U", base.dtype, (V, r), dev),
        _ptr(W, "W", base.dtype, (r, V), dev), _ptr(bias_scale, "bias_scale", f32, (B,), dev),
        _ptr(last_tok, "last_tok", i32, (B,), dev), _ptr(temp, "temp", f32, (B,), dev),
        B, K, V, r, dt, seed, round_id,
        _ptr(x, "x", i32, (B, K), dev), _ptr(d, "d", base.dtype, (B, K, V), dev),
        _ptr(q_lse, "q_lse", f32, (B, K), dev), _ptr(q_tok, "q_tok", f32, (B, K), dev),
        _ptr(q_norm, "q_norm", f32, (B, K, 2), dev), _ptr(ws, "ws", None, None, dev),
        ws.numel() * ws.element_size())
    _call("dspark_draft_sample", dev, args, stream)


def draft_sample_recurrent(base, U, W, R, bias_scale, last_tok, temp, seed: int, round_id: int,
                           x, d, q_lse, q_tok, h, ws, stream=None, q_norm=None) -> None:
    """dspark_draft_sample_recurrent: the recurrent head (state matrix R [r,r]);
    the states come back in h [B,K,r]."""
    B, K, V = base.shape
    r = U.shape[1]
    dt = _dtype_code(base)
    dev, f32, i32 = base.device, torch.float32, torch.int32
    args = (
        _ptr(base, "base", None, (B, K, V), dev), _ptr(U, "U", base.dtype, (V, r), dev),
        _ptr(W, "W", base.dtype, (r, V), dev), _ptr(R, "R", base.dtype, (r, r), dev),
        _ptr(bias_scale, "bias_scale", f32, (B,), dev),
        _ptr(last_tok, "last_tok", i32, (B,), dev), _ptr(temp, "temp", f32, (B,), dev),
        B, K, V, r, dt, seed, round_id,
        _ptr(x, "x", i32, (B, K), dev), _ptr(d, "d", base.dtype, (B, K, V), dev),
        _ptr(q_lse, "q_lse", f32, (B, K), dev), _ptr(q_tok, "q_tok", f32, (B, K), dev),
        _ptr(q_norm, "q_norm", f32, (B, K, 2), dev), _ptr(h, "h", base.dtype, (B, K, r), dev),
        _ptr(ws, "ws", None, None, dev), ws.numel() * ws.element_size())
    _call("dspark_draft_sample_recurrent", dev, args, stream)


def draft_sample_beside(base, U, W, R, bias_scale, last_tok, temp, seed: int, round_id: int,
                        x, d, q_lse, q_tok, h, free_sms: int, ws, stream=None,
                        q_norm=None) -> None:
    """dspark_draft_sample_beside: the draft (Markov head when R is None, else
    the recurrent head with its states in h) leaving free_sms SMs to kernels of
    other streams; results identical to draft_sample / draft_sample_recurrent."""
    B, K, V = base.shape
    r = U.shape[1]
    dt = _dtype_code(base)
    dev, f32, i32 = base.device, torch.float32, torch.int32
    if R is not None and h is None:
        raise DSparkError("the recurrent head needs h [B,K,r]")
    args = (
        _ptr(base, "base", None, (B, K, V), dev), _ptr(U, "U", base.dtype, (V, r), dev),
        _ptr(W, "W", base.dtype, (r, V), dev), _ptr(R, "R", base.dtype, (r, r), dev),
        _ptr(bias_scale, "bias_scale", f32, (B,), dev),
        _ptr(last_tok, "last_tok", i32, (B,), dev), _ptr(temp, "temp", f32, (B,), dev),
        B, K, V, r, dt, seed, round_id,
        _ptr(x, "x", i32, (B, K), dev), _ptr(d, "d", base.dtype, (B, K, V), dev),
        _ptr(q_lse, "q_lse", f32, (B, K), dev), _ptr(q_tok, "q_tok", f32, (B, K), dev),
        _ptr(q_norm, "q_norm", f32, (B, K, 2), dev),
        _ptr(h if R is not None else None, "h", base.dtype, (B, K, r), dev), int(free_sms),
        _ptr(ws, "ws", None, None, dev), ws.numel() * ws.element_size())
    _call("dspark_draft_sample_beside", dev, args, stream)


def draft_logits(base, U, W, bias_scale, last_tok, x, temp, k: int, d, ws, stream=None) -> None:
    """dspark_draft_logits: position k's draft logits d[:, k-1] and the chunk
    partials (in ws) that dspark_draft_pick(k) reads."""
    B, K, V = base.shape
    r = U.shape[1]
    dt = _dtype_code(base)
    dev, f32, i32 = base.device, torch.float32, torch.int32
    args = (
        _ptr(base, "base", None, (B, K, V), dev), _ptr(U, "U", base.dtype, (V, r), dev),
        _ptr(W, "W", base.dtype, (r, V), dev), _ptr(bias_scale, "bias_scale", f32, (B,), dev),
        _ptr(last_tok, "last_tok", i32, (B,), dev), _ptr(x, "x", i32, (B, K), dev),
        _ptr(temp, "temp", f32, (B,), dev), B, K, V, r, dt, int(k),
        _ptr(d, "d", base.dtype, (B, K, V), dev), _ptr(ws, "ws", None, None, dev),
        ws.numel() * ws.element_size())
    _call("dspark_draft_logits", dev, args, stream)


def draft_pick(d, last_tok, temp, seed: int, round_id: int, k: int, x, q_lse, q_tok, ws,
               stream=None, q_norm=None) -> None:
    """dspark_draft_pick: position k's token, q_lse and q_tok from d[:, k-1]."""
    B, K, V = d.shape
    dev, f32, i32 = d.device, torch.float32, torch.int32
    args = (
        _ptr(d, "d", None, (B, K, V), dev), _ptr(last_tok, "last_tok", i32, (B,), dev),
        _ptr(temp, "temp", f32, (B,), dev), B, K, V, _dtype_code(d), seed, round_id, int(k),
        _ptr(x, "x", i32, (B, K), dev), _ptr(q_lse, "q_lse", f32, (B, K), dev),
        _ptr(q_tok, "q_tok", f32, (B, K), dev), _ptr(q_norm, "q_norm", f32, (B, K, 2), dev),
        _ptr(ws, "ws", None, None, dev), ws.numel() * ws.element_size())
    _call("dspark_draft_pick", dev, args, stream)


def draft_sample_static(base, U, W, bias_scale, last_tok, temp, seed: int, round_id: int,
                        x, d, q_lse, q_tok, status_out=None, stream=None) -> None:
    """dspark_draft_sample_static: dspark_draft_sample with the library's fixed
    scratch instead of a workspace (for callers that cannot allocate)."""
    B, K, V = base.shape
    r = U.shape[1]
    dt = _dtype_code(base)
    dev, f32, i32 = base.device, torch.float32, torch.int32
    args = (
        _ptr(base, "base", None, (B, K, V), dev), _ptr(U, "U", base.dtype, (V, r), dev),
        _ptr(W, "W", base.dtype, (r, V), dev), _ptr(bias_scale, "bias_scale", f32, (B,), dev),
        _ptr(last_tok, "last_tok", i32, (B,), dev), _ptr(temp, "temp", f32, (B,), dev),
        B, K, V, r, dt, seed, round_id,
        _ptr(x, "x", i32, (B, K), dev), _ptr(d, "d", base.dtype, (B, K, V), dev),
        _ptr(q_lse, "q_lse", f32, (B, K), dev), _ptr(q_tok, "q_tok", f32, (B, K), dev),
        _ptr(status_out, "status_out", i32, (2,), dev))
    _call("dspark_draft_sample_static", dev, args, stream)


def prefix_schedule(conf_logit, pos_temp, step_cost, fixed_cost: float, mode: int,
                    threshold: float, cut, survival, ws, stream=None) -> None:
    """dspark_prefix_schedule: conf_logit [B,K], pos_temp [K], step_cost [B(K+1)] -> cut, survival."""
    B, K = conf_logit.shape
    dev, f32 = conf_logit.device, torch.float32
    args = (
        _ptr(conf_logit, "conf_logit", f32, (B, K), dev), _ptr(pos_temp, "pos_temp", f32, (K,), dev),
        _ptr(step_cost, "step_cost", f32, (B * (K + 1),), dev), float(fixed_cost), B, K, mode,
        float(threshold), _ptr(cut, "cut", torch.int32, (B,), dev),
        _ptr(survival, "survival", f32, (B, K), dev), _ptr(ws, "ws", None, None, dev),
        ws.numel() * ws.element_size())
    _call("dspark_prefix_schedule", dev, args, stream)


def _verify_args(target, d, x, q_tok, cut, temp, seed, round_id, accepted, out, n_emit, ws,
                 q_norm):
    B, K1, V = target.shape
    K = K1 - 1
    dt = _dtype_code(target)
    dev, f32, i32 = target.device, torch.float32, torch.int32
    args = (
        _ptr(target, "target", None, (B, K1, V), dev), _ptr(d, "d", target.dtype, (B, K, V), dev),
        _ptr(x, "x", i32, (B, K), dev), _ptr(q_tok, "q_tok", f32, (B, K), dev),
        _ptr(q_norm, "q_norm", f32, (B, K, 2), dev), _ptr(cut, "cut", i32, (B,), dev),
        _ptr(temp, "temp", f32, (B,), dev), B, K, V, dt, seed, round_id,
        _ptr(accepted, "accepted", i32, (B,), dev), _ptr(out, "out", i32, (B, K1), dev),
        _ptr(n_emit, "n_emit", i32, (B,), dev), _ptr(ws, "ws", None, None, dev),
        ws.numel() * ws.element_size())
    return dev, args


def verify(target, d, x, q_tok, cut, temp, seed: int, round_id: int, accepted, out, n_emit,
           ws, stream=None, q_norm=None) -> None:
    """dspark_verify: target [B,K+1,V], d [B,K,V], x, q_tok [B,K], cut [B] -> accepted, out, n_emit."""
    dev, args = _verify_args(target, d, x, q_tok, cut, temp, seed, round_id, accepted, out, n_emit,
                             ws, q_norm)
    _call("dspark_verify", dev, args, stream)


def verify_target_stats(target, cut, temp, ws, stream=None) -> None:
    """dspark_verify_target_stats: softmax partials of target rows 0..cut[b] into ws."""
    B, K1, V = target.shape
    dev = target.device
    args = (_ptr(target, "target", None, (B, K1, V), dev),
            _ptr(cut, "cut", torch.int32, (B,), dev), _ptr(temp, "temp", torch.float32, (B,), dev),
            B, K1 - 1, V, _dtype_code(target), _ptr(ws, "ws", None, None, dev),
            ws.numel() * ws.element_size())
    _call("dspark_verify_target_stats", dev, args, stream)


def verify_from_stats(target, d, x, q_tok, cut, temp, seed: int, round_id: int, accepted, out,
                      n_emit, ws, stream=None, q_norm=None) -> None:
    """dspark_verify_from_stats: dspark_verify after dspark_verify_target_stats."""
    dev, args = _verify_args(target, d, x, q_tok, cut, temp, seed, round_id, accepted, out, n_emit,
                             ws, q_norm)
    _call("dspark_verify_from_stats", dev, args, stream)


def sts_fit(conf_logit, survived, T_out, index_out, ece_before, ece_after, ws, stream=None) -> None:
    """dspark_sts_fit: conf_logit [N,K] f32, survived [N,K] u8 -> T [K], index [K], ECE [K] x 2."""
    N, K = conf_logit.shape
    dev, f32 = conf_logit.device, torch.float32
    args = (
        _ptr(conf_logit, "conf_logit", f32, (N, K), dev),
        _ptr(survived, "survived", torch.uint8, (N, K), dev), N, K,
        _ptr(T_out, "T_out", f32, (K,), dev), _ptr(index_out, "index_out", torch.int32, (K,), dev),
        _ptr(ece_before, "ece_before", f32, (K,), dev), _ptr(ece_after, "ece_after", f32, (K,), dev),
        _ptr(ws, "ws", None, None, dev), ws.numel() * ws.element_size())
    _call("dspark_sts_fit", dev, args, stream)


def selftest_waits(result, ws, stream=None) -> None:
    """dspark_selftest_waits: an mbarrier wait and a grid-barrier wait that must give
    up after the kernels' 2 s limit; result [2] int32 gets 1 for each that gave up."""
    dev = ws.device
    args = (_ptr(result, "result", torch.int32, (2,), dev), _ptr(ws, "ws", None, None, dev),
            ws.numel() * ws.element_size())
    _call("dspark_selftest_waits", dev, args, stream)


def read_status(ws, stream=None) -> Tuple[int, int]:
    """(status bits, first offending request or -1); synchronises and clears."""
    code = ctypes.c_uint32(0)
    first = ctypes.c_int32(-1)
    p = _ptr(ws, "ws")
    dev = ws.device
    s = _stream(stream, dev)
    with torch.cuda.device(dev):
        rc = lib().dspark_read_status(p, s, ctypes.byref(code), ctypes.byref(first))
    _check(rc, "dspark_read_status")
    return int(code.value), int(first.value)


def clear_status(ws, stream=None) -> None:
    p = _ptr(ws, "ws")
    dev = ws.device
    s = _stream(stream, dev)
    with torch.cuda.device(dev):
        _check(lib().dspark_clear_status(p, s), "dspark_clear_status")
