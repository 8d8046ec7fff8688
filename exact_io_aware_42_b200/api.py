"""Python binding over the C ABI (argument marshalling only).

torch provides device memory and the current CUDA stream; every step of the
computation runs in the library's kernels.  Functions mirror include/fa.h:

* ``fwd(q, k, v, causal, scale)``            -> (o, lse)
  (k, v may have fewer heads than q: grouped K/V heads, H a multiple of H_kv;
  ``window=w`` with causal=True: key j visible to query i iff i - w <= j <= i;
  ``alibi=slopes``: a CUDA fp32 tensor of H slopes, bias -slope_h |i - j|)
* ``bwd(q, k, v, o, do, lse, causal, scale, deterministic=False)`` -> (dq, dk, dv)
* ``quant_fp8(x, signs=None)``               -> (x8 as uint8, block scales)
* ``fwd_fp8(q8, k8, v8, sq, sk, sv, causal, scale)`` -> (o, lse)
"""
from __future__ import annotations

import math
from typing import Optional

import torch

from ._lib import (TUNE_BWD_CAUSAL_GROUP, TUNE_BWD_PAIR, TUNE_BWD_POLY_GROUPS, TUNE_DQ_POLY_PAIRS, TUNE_FP8_POLY_PAIRS,
                   TUNE_FWD_CAUSAL_GROUP, TUNE_FWD_PERSISTENT, TUNE_FWD_Q1, TUNE_FWD_POLY_DEGREE, TUNE_FWD_POLY_PAIRS,
                   check, lib)

__all__ = ["fwd", "bwd", "bwd_workspace_size", "bwd_noalloc", "quant_fp8", "fwd_fp8", "get_status",
           "clear_status", "n_blocks", "set_tuning", "get_tuning", "TUNING_KNOBS"]


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _kv_shape(name: str, q_shape, kv: torch.Tensor):
    """[B, H_kv, N, d] with H_kv dividing H; returns H_kv."""
    B, H, N, d = q_shape
    if kv.dim() != 4 or kv.shape[0] != B or kv.shape[2] != N or kv.shape[3] != d:
        raise ValueError(f"{name} has shape {tuple(kv.shape)}, expected [B, H_kv, N, d] = [{B}, H_kv, {N}, {d}]")
    h_kv = kv.shape[1]
    if h_kv < 1 or H % h_kv != 0:
        raise ValueError(f"{name} has {h_kv} heads, which does not divide H = {H}")
    return h_kv


def _window(window: Optional[int], causal: bool) -> int:
    if window is None:
        return -1
    if window < 0 or not causal:
        raise ValueError("window must be >= 0 and needs causal=True")
    return int(window)


def _alibi(alibi: Optional[torch.Tensor], H: int):
    if alibi is None:
        return None
    if not alibi.is_cuda or alibi.dtype != torch.float32 or alibi.numel() != H or not alibi.is_contiguous():
        raise ValueError("alibi must be a contiguous CUDA fp32 tensor of H slopes")
    return alibi


def _check_bhnd(name: str, t: torch.Tensor, dtype, shape=None) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != 4 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous [B, H, N, d] tensor")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def n_blocks(N: int) -> int:
    """Number of 128-row quantisation blocks of a length-N sequence."""
    return (N + 127) // 128


def fwd(q, k, v, causal: bool = False, scale: Optional[float] = None, out=None, lse=None,
        window: Optional[int] = None, alibi: Optional[torch.Tensor] = None):
    """Exact attention forward (bf16).  Returns (o bf16 [B,H,N,d], lse fp32 [B,H,N])."""
    wl = _window(window, causal)
    _check_bhnd("q", q, torch.bfloat16)
    B, H, N, d = q.shape
    h_kv = _kv_shape("k", q.shape, k)
    _check_bhnd("k", k, torch.bfloat16, (B, h_kv, N, d))
    _check_bhnd("v", v, torch.bfloat16, (B, h_kv, N, d))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = torch.empty_like(q) if out is None else out
    lse_t = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    al = _alibi(alibi, H)
    if h_kv == H and wl < 0 and al is None:
        code = lib().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse_t), B, H, N, d, float(scale),
                            int(bool(causal)), _stream())
        check("fa_fwd", code)
    else:
        code = lib().fa_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse_t), B, H, h_kv, N, d,
                               float(scale), int(bool(causal)), wl, _ptr(al), _stream())
        check("fa_fwd_ex", code)
    return o, lse_t


def _check_bwd_args(q, k, v, o, do, lse, dq=None, dk=None, dv=None):
    """Shapes, dtypes and layout of the backward's tensors; returns (B, H, N, d, H_kv)."""
    _check_bhnd("q", q, torch.bfloat16)
    B, H, N, d = q.shape
    h_kv = _kv_shape("k", q.shape, k)
    for name, t in (("k", k), ("v", v), ("dk", dk), ("dv", dv)):
        if t is not None:
            _check_bhnd(name, t, torch.bfloat16, (B, h_kv, N, d))
    for name, t in (("o", o), ("do", do), ("dq", dq)):
        if t is not None:
            _check_bhnd(name, t, torch.bfloat16, q.shape)
    if (not lse.is_cuda or lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N)
            or not lse.is_contiguous()):
        raise ValueError("lse must be a contiguous CUDA fp32 [B, H, N] tensor")
    return B, H, N, d, h_kv


def bwd_workspace_size(B: int, H: int, N: int, d: int, deterministic: bool = False,
                       H_kv: Optional[int] = None) -> int:
    if H_kv is not None and H_kv != H:
        return int(lib().fa_bwd_ex_workspace_size(B, H, H_kv, N, d, int(bool(deterministic))))
    if deterministic:
        return int(lib().fa_bwd_deterministic_workspace_size(B, H, N, d))
    return int(lib().fa_bwd_workspace_size(B, H, N, d))


def bwd(q, k, v, o, do, lse, causal: bool = False, scale: Optional[float] = None,
        workspace: Optional[torch.Tensor] = None, dq=None, dk=None, dv=None,
        deterministic: bool = False, window: Optional[int] = None,
        alibi: Optional[torch.Tensor] = None):
    """Attention backward (bf16).  Returns (dq, dk, dv).

    ``deterministic=True`` calls fa_bwd_deterministic: bitwise reproducible
    gradients (dQ by a separate query-block-major kernel).  ``window``, ``alibi`` as in fwd."""
    wl = _window(window, causal)
    B, H, N, d, h_kv = _check_bwd_args(q, k, v, o, do, lse)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    ws_bytes = bwd_workspace_size(B, H, N, d, deterministic, h_kv)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    al = _alibi(alibi, H)
    if h_kv == H and wl < 0 and al is None:
        name = "fa_bwd_deterministic" if deterministic else "fa_bwd"
        code = getattr(lib(), name)(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq),
                                    _ptr(dk), _ptr(dv), B, H, N, d, float(scale), int(bool(causal)),
                                    _ptr(workspace), workspace.numel(), _stream())
    else:
        name = "fa_bwd_ex"
        code = lib().fa_bwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq),
                               _ptr(dk), _ptr(dv), B, H, h_kv, N, d, float(scale), int(bool(causal)), wl,
                               _ptr(al), int(bool(deterministic)), _ptr(workspace), workspace.numel(),
                               _stream())
    check(name, code)
    return dq, dk, dv


def quant_fp8(x, signs: Optional[torch.Tensor] = None, out=None, scales=None):
    """Per-128-row E4M3 quantisation.  Returns (codes uint8 [B,H,N,d], scales fp32 [B,H,nblk])."""
    _check_bhnd("x", x, torch.bfloat16)
    B, H, N, d = x.shape
    if signs is not None:
        if signs.dtype != torch.float32 or signs.numel() != d or not signs.is_cuda:
            raise ValueError("signs must be a CUDA fp32 tensor of d elements")
        signs = signs.contiguous()
    x8 = torch.empty((B, H, N, d), dtype=torch.uint8, device=x.device) if out is None else out
    sc = torch.empty((B, H, n_blocks(N)), dtype=torch.float32, device=x.device) if scales is None else scales
    code = lib().fa_quant_fp8(_ptr(x), _ptr(x8), _ptr(sc), B, H, N, d, _ptr(signs), _stream())
    check("fa_quant_fp8", code)
    return x8, sc


def fwd_fp8(q8, k8, v8, sq, sk, sv, causal: bool = False, scale: Optional[float] = None,
            out=None, lse=None, window: Optional[int] = None, alibi: Optional[torch.Tensor] = None):
    """FP8 attention forward on quantised inputs.  Returns (o bf16, lse fp32)."""
    wl = _window(window, causal)
    _check_bhnd("q8", q8, torch.uint8)
    B, H, N, d = q8.shape
    h_kv = _kv_shape("k8", q8.shape, k8)
    _check_bhnd("k8", k8, torch.uint8, (B, h_kv, N, d))
    _check_bhnd("v8", v8, torch.uint8, (B, h_kv, N, d))
    for name, s, h in (("sq", sq, H), ("sk", sk, h_kv), ("sv", sv, h_kv)):
        if s.dtype != torch.float32 or tuple(s.shape) != (B, h, n_blocks(N)) or not s.is_contiguous():
            raise ValueError(f"{name} must be a contiguous fp32 [B, {h}, ceil(N/128)] tensor")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q8.device) if out is None else out
    lse_t = torch.empty((B, H, N), dtype=torch.float32, device=q8.device) if lse is None else lse
    code = lib().fa_fwd_fp8_ex(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(sq), _ptr(sk), _ptr(sv), _ptr(o),
                               _ptr(lse_t), B, H, h_kv, N, d, float(scale), int(bool(causal)), wl,
                               _ptr(_alibi(alibi, H)), _stream())
    check("fa_fwd_fp8_ex", code)
    return o, lse_t


def get_status() -> int:
    return int(lib().fa_get_status())


def clear_status() -> None:
    lib().fa_clear_status()


def bwd_noalloc(q, k, v, o, do, lse, causal: bool = False, scale: Optional[float] = None,
                dq=None, dk=None, dv=None):
    """Backward with the library's built-in scratch instead of a workspace
    (for callers that cannot allocate device memory; see fa_bwd_noalloc).
    Every tensor is checked as in ``bwd``; K/V heads must equal H here."""
    B, H, N, d, h_kv = _check_bwd_args(q, k, v, o, do, lse, dq, dk, dv)
    if h_kv != H:
        raise ValueError("bwd_noalloc takes K/V with H heads (no grouped K/V heads)")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    code = lib().fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq),
                                _ptr(dk), _ptr(dv), B, H, N, d, float(scale), int(bool(causal)),
                                _stream())
    check("fa_bwd_noalloc", code)
    return dq, dk, dv


TUNING_KNOBS = {"fwd_poly_pairs": TUNE_FWD_POLY_PAIRS, "fwd_poly_degree": TUNE_FWD_POLY_DEGREE,
                "bwd_poly_groups": TUNE_BWD_POLY_GROUPS, "dq_poly_pairs": TUNE_DQ_POLY_PAIRS,
                "fp8_poly_pairs": TUNE_FP8_POLY_PAIRS, "bwd_pair": TUNE_BWD_PAIR,
                "fwd_persistent": TUNE_FWD_PERSISTENT,
                "fwd_causal_group": TUNE_FWD_CAUSAL_GROUP, "fwd_q1": TUNE_FWD_Q1,
                "bwd_causal_group": TUNE_BWD_CAUSAL_GROUP}


def set_tuning(knob: str, value: int) -> None:
    """Measurement control (fa_set_tuning): the share of the softmax exp2 on
    the FMA-pipe polynomial, or its degree; -1 restores the default."""
    check("fa_set_tuning", lib().fa_set_tuning(TUNING_KNOBS[knob], int(value)))


def get_tuning(knob: str, d: int = 128) -> int:
    """The value of a measurement control that a call with head dim d uses now."""
    return int(lib().fa_get_tuning(TUNING_KNOBS[knob], int(d)))
