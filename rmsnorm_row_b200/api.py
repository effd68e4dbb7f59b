"""Tensor-level entry points over the C ABI (argument marshalling only).

Mirrors the pages' two ops (sglang PR #36349 "[AMD][Diffusion] Migrate FlyDSL
fused norm kernels to the v0.3.0 stable API", section "Microbenchmark"):

    fused_residual_norm_scale_shift(residual, x, gate, weight, bias, scale, shift,
                                    norm_type, eps) -> (y, r)
    norm_scale_shift(x, weight, bias, scale, shift, norm_type, eps) -> y

PyTorch only provides device memory and the stream; each call resolves operand
shapes to (pointer, strides) and makes one fused_norm_launch. Inputs must be bf16
CUDA tensors with a contiguous channel dimension; anything else raises (there is no
fallback path).

weight and bias are (D,) vectors, bf16 or fp32 (both the same dtype when both are given);
fp32 values are used at full precision.

Calls are asynchronous on `stream` (default: the current stream of the inputs' device)
and run on the inputs' device whichever device is current, like any PyTorch kernel: when `stream` is not the stream the tensors were produced on, the
caller orders the two streams and keeps the tensors alive (e.g. Tensor.record_stream).

Accepted operand shapes for gate / scale / shift against x of shape (B, L, D):
    (D,), (1, D), (1, 1, D)      broadcast
    (B, L, D)                    per token
    (B, 1, D) or (B, D)          per batch
    (B or 1, F, 1, D)            per frame: token l uses frame l // (L / F)
"""
from __future__ import annotations

import threading
from typing import Dict, Optional, Tuple

import torch

from . import _abi

_handles: Dict[Tuple, int] = {}
_handles_lock = threading.Lock()


def _handle(D: int, is_rms: bool, has_gate: bool, has_weight: bool, has_bias: bool,
            norm_only: bool, eps: float, affine_fp32: bool = False) -> int:
    key = (D, is_rms, has_gate, has_weight, has_bias, norm_only, float(eps), affine_fp32)
    with _handles_lock:
        h = _handles.get(key)
        if h is None:
            cfg = _abi.fn_config(D=D, is_rms=int(is_rms), has_gate=int(has_gate),
                                 has_weight=int(has_weight), has_bias=int(has_bias),
                                 norm_only=int(norm_only), affine_fp32=int(affine_fp32),
                                 eps=float(eps))
            st, h = _abi.fused_norm_create(cfg)
            if st != _abi.FN_OK:
                raise _abi.FusedNormError(st, "fused_norm_create", _abi.fused_norm_status_string(st))
            _handles[key] = h
        return h


def _check_tensor(t: torch.Tensor, name: str, device: torch.device) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dim() >= 1 and t.shape[-1] > 1 and t.stride(-1) != 1:
        raise ValueError(f"{name} needs a contiguous channel dimension")


def _operand(t: Optional[torch.Tensor], name: str, B: int, L: int, D: int, device):
    """(fn_operand, frames) for a gate/scale/shift tensor; frames is 0 without a frame axis."""
    if t is None:
        return _abi.fn_operand(None, 0, 0, 0), 0
    _check_tensor(t, name, device)
    if t.shape[-1] != D:
        raise ValueError(f"{name} has {t.shape[-1]} channels, expected {D}")
    s = t.stride()
    sh = tuple(t.shape)
    if t.dim() == 1:
        return _abi.fn_operand(t.data_ptr(), 0, 0, 0), 0
    if t.dim() == 2:
        n = sh[0]
        if n == 1:
            return _abi.fn_operand(t.data_ptr(), 0, 0, 0), 0
        if n == B:
            return _abi.fn_operand(t.data_ptr(), s[0], 0, 0), 0
        raise ValueError(f"{name} of shape {sh} does not broadcast against ({B}, {L}, {D})")
    if t.dim() == 3:
        nb, nl = sh[0], sh[1]
        if nb not in (1, B) or nl not in (1, L):
            raise ValueError(f"{name} of shape {sh} does not broadcast against ({B}, {L}, {D})")
        return _abi.fn_operand(t.data_ptr(), s[0] if nb > 1 else 0, 0, s[1] if nl > 1 else 0), 0
    if t.dim() == 4:
        nb, F, one = sh[0], sh[1], sh[2]
        if nb not in (1, B) or one != 1 or F < 1 or L % F != 0:
            raise ValueError(f"{name} of shape {sh} is not a (B, F, 1, D) frame operand for L={L}")
        return _abi.fn_operand(t.data_ptr(), s[0] if nb > 1 else 0, s[1] if F > 1 else 0, 0), F
    raise ValueError(f"{name} has unsupported rank {t.dim()}")


def _vector(t: Optional[torch.Tensor], name: str, D: int, device):
    if t is None:
        return None
    if t.dtype == torch.float32:       # fp32 affine parameters are used as given
        if t.device != device:
            raise ValueError(f"{name} is on {t.device}, expected {device}")
        if t.numel() != D or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous ({D},) vector")
        return t.data_ptr()
    _check_tensor(t, name, device)
    if t.numel() != D or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous ({D},) vector")
    return t.data_ptr()


def _norm_flag(norm_type: str) -> bool:
    if norm_type in ("layer", "ln", "layernorm"):
        return False
    if norm_type in ("rms", "rmsnorm"):
        return True
    raise ValueError(f"norm_type must be 'layer' or 'rms', got {norm_type!r}")


def _affine_fp32(weight, bias) -> bool:
    dts = {t.dtype for t in (weight, bias) if t is not None}
    if len(dts) > 1:
        raise TypeError("weight and bias must have the same dtype")
    if dts and dts.pop() not in (torch.bfloat16, torch.float32):
        raise TypeError("weight and bias must be bfloat16 or float32")
    return any(t is not None and t.dtype == torch.float32 for t in (weight, bias))


def _launch(h: int, args: _abi.fn_args, device: torch.device, stream) -> None:
    # The library launches on the calling thread's current device: make it the tensors'
    # device for the call (the caller's current device is restored afterwards).
    with torch.cuda.device(device):
        if stream is None:
            stream = torch.cuda.current_stream(device)
        st = _abi.fused_norm_launch(h, args, int(stream.cuda_stream))
    if st != _abi.FN_OK:
        detail = _abi.fused_norm_status_string(st)
        if st == _abi.FN_ERR_CUDA:
            detail += f" (cudaError {_abi.fused_norm_last_cuda_error()})"
        raise _abi.FusedNormError(st, "fused_norm_launch", detail)


def build_args(x: torch.Tensor, residual: Optional[torch.Tensor], gate, weight, bias, scale, shift,
               y: torch.Tensor, r: Optional[torch.Tensor]) -> _abi.fn_args:
    """fn_args for 3-D (B, L, D) x / residual / y / r tensors and any accepted operand shapes."""
    device = x.device
    _check_tensor(x, "x", device)
    if x.dim() != 3:
        raise ValueError("x must be (B, L, D)")
    B, L, D = x.shape
    xs = x.stride()
    frames = set()
    ops = {}
    for name, t in (("gate", gate), ("scale", scale), ("shift", shift)):
        ops[name], F = _operand(t, name, B, L, D, device)
        if F:
            frames.add(F)
    if len(frames) > 1:
        raise ValueError(f"operands disagree on the frame count: {sorted(frames)}")
    tpf = L // frames.pop() if frames else 0
    a = _abi.fn_args()
    a.B, a.L, a.tokens_per_frame = B, L, tpf
    a.x = _abi.fn_operand(x.data_ptr(), xs[0] if B > 1 else 0, 0, xs[1] if L > 1 else 0)
    if residual is not None:
        _check_tensor(residual, "residual", device)
        if tuple(residual.shape) != (B, L, D):
            raise ValueError("residual must match x")
        rs = residual.stride()
        a.residual = _abi.fn_operand(residual.data_ptr(), rs[0] if B > 1 else 0, 0,
                                     rs[1] if L > 1 else 0)
    a.gate, a.scale, a.shift = ops["gate"], ops["scale"], ops["shift"]
    a.weight = _vector(weight, "weight", D, device)
    a.bias = _vector(bias, "bias", D, device)
    for name, t in (("y", y), ("r", r)):
        if t is None:
            continue
        _check_tensor(t, name, device)
        if tuple(t.shape) != (B, L, D):
            raise ValueError(f"{name} must be ({B}, {L}, {D})")
    ys = y.stride()
    a.y, a.y_stride_b, a.y_stride_l = y.data_ptr(), ys[0], ys[1]
    if r is not None:
        rs_ = r.stride()
        a.r, a.r_stride_b, a.r_stride_l = r.data_ptr(), rs_[0], rs_[1]
    return a


def fused_residual_norm_scale_shift(residual: torch.Tensor, x: torch.Tensor,
                                    gate: Optional[torch.Tensor], weight: Optional[torch.Tensor],
                                    bias: Optional[torch.Tensor], scale: torch.Tensor,
                                    shift: torch.Tensor, norm_type: str = "layer",
                                    eps: float = 1e-6, *, out: Optional[torch.Tensor] = None,
                                    residual_out: Optional[torch.Tensor] = None,
                                    stream: Optional[torch.cuda.Stream] = None):
    """y = norm(residual + gate * x) (* weight + bias) * (1 + scale) + shift; returns (y, r).

    `residual_out` may be `residual` itself (in-place residual update).
    """
    if x.dim() != 3:
        raise ValueError("x must be (B, L, D)")
    y = out if out is not None else torch.empty_like(x, memory_format=torch.contiguous_format)
    r = residual_out if residual_out is not None else torch.empty_like(x, memory_format=torch.contiguous_format)
    args = build_args(x, residual, gate, weight, bias, scale, shift, y, r)
    h = _handle(x.shape[-1], _norm_flag(norm_type), gate is not None, weight is not None,
                bias is not None, False, eps, _affine_fp32(weight, bias))
    _launch(h, args, x.device, stream)
    return y, r


def norm_scale_shift(x: torch.Tensor, weight: Optional[torch.Tensor], bias: Optional[torch.Tensor],
                     scale: torch.Tensor, shift: torch.Tensor, norm_type: str = "layer",
                     eps: float = 1e-6, *, out: Optional[torch.Tensor] = None,
                     stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """y = norm(x) (* weight + bias) * (1 + scale) + shift (no residual)."""
    if x.dim() != 3:
        raise ValueError("x must be (B, L, D)")
    y = out if out is not None else torch.empty_like(x, memory_format=torch.contiguous_format)
    args = build_args(x, None, None, weight, bias, scale, shift, y, None)
    h = _handle(x.shape[-1], _norm_flag(norm_type), False, weight is not None, bias is not None,
                True, eps, _affine_fp32(weight, bias))
    _launch(h, args, x.device, stream)
    return y
