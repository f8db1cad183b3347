"""B200 (sm_100a) Kimi Delta Attention prefill -- Python binding of ``libkda.so``.

This module only marshals arguments: it checks torch tensors, allocates
outputs with torch (device memory), and calls the C ABI declared in
``include/kda.h`` on the current CUDA stream. Every step of the computation
runs in the library's CUDA kernels; there is no fallback. Importing the
module fails loudly if ``libkda.so`` has not been built.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

__all__ = ["kda_fwd", "kda_fwd_fused", "kda_decode", "kda_bwd", "library_path", "wait_timeouts", "device_status", "set_slice_columns", "set_path",
           "set_time_split", "set_schedule", "describe", "KDAError", "HEAD_DIM"]

HEAD_DIM = 128
_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libkda.so")

if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"{_LIB_PATH} is missing: build the CUDA library first "
        "(python kimi_delta_attention_26_b200/build.py or __graft_entry__.build())")

_lib = ctypes.CDLL(_LIB_PATH)

KDA_BF16, KDA_F32, KDA_I32 = 1, 2, 3
_DTYPE = {torch.bfloat16: KDA_BF16, torch.float32: KDA_F32, torch.int32: KDA_I32}


class TensorDesc(ctypes.Structure):
    """``kda_tensor_t``: data pointer, ndim, dtype, shape[4], stride[4] (elements)."""
    _fields_ = [("data", ctypes.c_void_p), ("ndim", ctypes.c_int32), ("dtype", ctypes.c_int),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


def describe(t: Optional[torch.Tensor]):
    """A ``kda_tensor_t`` for a torch tensor (None -> NULL)."""
    if t is None:
        return None
    if t.dim() > 4:
        raise ValueError("at most 4 dimensions")
    d = TensorDesc()
    d.data = t.data_ptr() if t.numel() else None
    d.ndim = t.dim()
    d.dtype = _DTYPE.get(t.dtype, 0)
    for i, (n, st) in enumerate(zip(t.shape, t.stride())):
        d.shape[i] = n
        d.stride[i] = st
    return ctypes.byref(d), d  # keep d alive with the reference


_P = ctypes.c_void_p
_T = ctypes.POINTER(TensorDesc)
_FWD_ARGS = [_T, _T, _T, _T, _T, ctypes.c_float, _P, ctypes.c_int32, _T, _T, _T, _P]
_lib.kda_fwd.argtypes = _FWD_ARGS
_lib.kda_fwd.restype = ctypes.c_int
_lib.kda_fwd_noalloc.argtypes = _FWD_ARGS
_lib.kda_fwd_noalloc.restype = ctypes.c_int
_lib.kda_status_string.argtypes = [ctypes.c_int]
_lib.kda_status_string.restype = ctypes.c_char_p
_lib.kda_last_cuda_error.argtypes = []
_lib.kda_last_cuda_error.restype = ctypes.c_char_p
_lib.kda_abi_version.argtypes = []
_lib.kda_abi_version.restype = ctypes.c_int32
_lib.kda_wait_timeouts.argtypes = [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int32]
_lib.kda_wait_timeouts.restype = ctypes.c_int
_lib.kda_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int32]
_lib.kda_device_status.restype = ctypes.c_int
_lib.kda_set_slice_columns.argtypes = [ctypes.c_int32]
_lib.kda_set_slice_columns.restype = ctypes.c_int
_lib.kda_set_path.argtypes = [ctypes.c_int32]
_lib.kda_set_path.restype = ctypes.c_int
_lib.kda_set_time_split.argtypes = [ctypes.c_int32]
_lib.kda_set_time_split.restype = ctypes.c_int
_lib.kda_set_schedule.argtypes = [ctypes.c_int32, ctypes.c_int32]
_lib.kda_set_schedule.restype = ctypes.c_int
_lib.kda_fwd_fused.argtypes = [_T, _T, _T, _T, _T, ctypes.c_float, ctypes.c_float, _P, ctypes.c_int32, _T, _T, _T, _P]
_lib.kda_fwd_fused.restype = ctypes.c_int
_lib.kda_bwd.argtypes = [_T, _T, _T, _T, _T, ctypes.c_float, _P, ctypes.c_int32, _T, _T, _T, _T, _T, _T, _T, _T, _T, _P]
_lib.kda_bwd.restype = ctypes.c_int
_lib.kda_decode.argtypes = [_T, _T, _T, _T, _T, ctypes.c_float, _T, _P, _T, _P]
_lib.kda_decode.restype = ctypes.c_int


class KDAError(RuntimeError):
    def __init__(self, code: int):
        msg = _lib.kda_status_string(code).decode()
        cuda = _lib.kda_last_cuda_error().decode()
        super().__init__(f"KDA call failed ({code}): {msg}" + (f" [{cuda}]" if cuda else ""))
        self.code = code


def library_path() -> str:
    return _LIB_PATH


def wait_timeouts(reset: bool = True) -> int:
    """Bounded in-kernel waits that ran out of budget on the current device
    since the last reset (0 for a healthy run); synchronises with the device."""
    n = ctypes.c_uint32(0)
    rc = _lib.kda_wait_timeouts(ctypes.byref(n), 1 if reset else 0)
    if rc != 0:
        raise KDAError(rc)
    return int(n.value)


def set_slice_columns(columns: int) -> None:
    """Value columns per CTA of the 16-token path for later calls: 0 chooses per
    call (default), 16 or 32 forces that variant. Process-wide."""
    rc = _lib.kda_set_slice_columns(int(columns))
    if rc != 0:
        raise KDAError(rc)


def set_path(path: int) -> None:
    """Kernel for later calls: 16 (16-token chunks on mma.sync), 64 (64-token
    chunks on tcgen05) or 0 (the library's default). Process-wide."""
    rc = _lib.kda_set_path(int(path))
    if rc != 0:
        raise KDAError(rc)


def set_time_split(mode: int) -> None:
    """Time-split prefill of one long sequence (16-token path): 0 automatic
    (default), 1 never, 2 whenever possible. Process-wide."""
    rc = _lib.kda_set_time_split(int(mode))
    if rc != 0:
        raise KDAError(rc)


def set_schedule(mode: int, clusters: int = 0) -> None:
    """Mapping of (sequence, head) pairs onto clusters (16-token path): 0
    automatic (default), 1 one cluster per pair, 2 persistent clusters taking
    the pairs round robin (at most `clusters` of them when > 0). Process-wide;
    results are bitwise the same."""
    rc = _lib.kda_set_schedule(int(mode), int(clusters))
    if rc != 0:
        raise KDAError(rc)


def device_status(reset: bool = True) -> int:
    """The device status word (bit 0: a bad cu_seqlens was seen, bit 1: a
    bounded in-kernel wait ran out, bit 2: kda_decode met a state index out of
    range); synchronises with the device."""
    n = ctypes.c_uint32(0)
    rc = _lib.kda_device_status(ctypes.byref(n), 1 if reset else 0)
    if rc not in (0, 9):
        raise KDAError(rc)
    return int(n.value)


def _check(t: torch.Tensor, name: str, dtype: torch.dtype, shape: Tuple[int, ...], device,
           contiguous: bool = False) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def kda_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor, beta: torch.Tensor,
            scale: Optional[float] = None, cu_seqlens: Optional[torch.Tensor] = None,
            initial_state: Optional[torch.Tensor] = None, output_final_state: bool = True,
            out: Optional[torch.Tensor] = None, final_state: Optional[torch.Tensor] = None,
            stream: Optional[torch.cuda.Stream] = None, noalloc: bool = False,
            fused_lower_bound: Optional[float] = None):
    """Chunked KDA forward on packed sequences (see ``include/kda.h``).

    q, k, v: bf16 [T, H, 128]; g: fp32 [T, H, 128] (log decay, in [-5, 0]);
    beta: fp32 [T, H]; cu_seqlens: int32 [N + 1] on the device (None: one
    sequence); initial_state: fp32 [N, H, 128, 128] or None.
    Returns ``(out, final_state)``; ``final_state`` is None unless requested.
    With ``fused_lower_bound`` set, calls ``kda_fwd_fused``: q and k are raw
    projections, g and beta are logits (see ``kda_fwd_fused``).
    """
    if q.dim() != 3:
        raise ValueError("q must be [T, H, 128]")
    T, H, d = q.shape
    if d != HEAD_DIM:
        raise ValueError(f"head dimension must be {HEAD_DIM}")
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("kda_fwd runs on CUDA tensors only")
    N = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    _check(q, "q", torch.bfloat16, (T, H, d), dev)
    _check(k, "k", torch.bfloat16, (T, H, d), dev)
    _check(v, "v", torch.bfloat16, (T, H, d), dev)
    _check(g, "g", torch.float32, (T, H, d), dev)
    _check(beta, "beta", torch.float32, (T, H), dev)
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", torch.int32, (N + 1,), dev, contiguous=True)
    if initial_state is not None:
        _check(initial_state, "initial_state", torch.float32, (N, H, d, d), dev, contiguous=True)
    if out is None:
        out = torch.empty((T, H, d), dtype=torch.bfloat16, device=dev)
    _check(out, "out", torch.bfloat16, (T, H, d), dev)
    if final_state is None and output_final_state:
        final_state = torch.empty((N, H, d, d), dtype=torch.float32, device=dev)
    if final_state is not None:
        _check(final_state, "final_state", torch.float32, (N, H, d, d), dev, contiguous=True)
    if scale is None:
        scale = d ** -0.5
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    descs = [describe(t) for t in (q, k, v, g, beta, initial_state, out, final_state)]
    ref = [None if d is None else d[0] for d in descs]
    with torch.cuda.device(dev):
        if fused_lower_bound is not None:
            if noalloc:
                raise ValueError("the fused preprocessing has no allocation-free entry point")
            rc = _lib.kda_fwd_fused(ref[0], ref[1], ref[2], ref[3], ref[4], ctypes.c_float(scale),
                                    ctypes.c_float(fused_lower_bound), _ptr(cu_seqlens), N, ref[5], ref[6], ref[7],
                                    ctypes.c_void_p(stream.cuda_stream))
        else:
            fn = _lib.kda_fwd_noalloc if noalloc else _lib.kda_fwd
            rc = fn(ref[0], ref[1], ref[2], ref[3], ref[4], ctypes.c_float(scale), _ptr(cu_seqlens), N,
                    ref[5], ref[6], ref[7], ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise KDAError(rc)
    return out, final_state


def kda_fwd_fused(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g_logit: torch.Tensor,
                  beta_logit: torch.Tensor, scale: Optional[float] = None, lower_bound: float = -5.0, **kw):
    """``kda_fwd`` with the gate preprocessing fused (see ``include/kda.h``):
    q, k raw bf16 projections (L2-normalised in the kernel), g_logit fp32
    gate logits (decay max(log sigmoid(x), lower_bound)), beta_logit fp32
    (write strength sigmoid(b)). Other arguments as for ``kda_fwd``."""
    return kda_fwd(q, k, v, g_logit, beta_logit, scale, fused_lower_bound=float(lower_bound), **kw)


def kda_decode(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor, beta: torch.Tensor,
               state: torch.Tensor, scale: Optional[float] = None, state_indices: Optional[torch.Tensor] = None,
               out: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """One decode step for B requests (see ``include/kda.h``): advances each
    request's state by its token, in place, and returns the outputs.

    q, k, v: bf16 [B, H, 128]; g: fp32 [B, H, 128] (log decay, in [-5, 0]);
    beta: fp32 [B, H]; state: fp32 [P, H, 128, 128], updated in place;
    state_indices: int32 [B] on the device (distinct slots), or None for slot b.
    """
    if q.dim() != 3:
        raise ValueError("q must be [B, H, 128]")
    B, H, d = q.shape
    if d != HEAD_DIM:
        raise ValueError(f"head dimension must be {HEAD_DIM}")
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("kda_decode runs on CUDA tensors only")
    _check(q, "q", torch.bfloat16, (B, H, d), dev)
    _check(k, "k", torch.bfloat16, (B, H, d), dev)
    _check(v, "v", torch.bfloat16, (B, H, d), dev)
    _check(g, "g", torch.float32, (B, H, d), dev)
    _check(beta, "beta", torch.float32, (B, H), dev)
    if state.dim() != 4:
        raise ValueError("state must be [P, H, 128, 128]")
    _check(state, "state", torch.float32, (state.shape[0], H, d, d), dev, contiguous=True)
    if state_indices is not None:
        _check(state_indices, "state_indices", torch.int32, (B,), dev, contiguous=True)
    if out is None:
        out = torch.empty((B, H, d), dtype=torch.bfloat16, device=dev)
    _check(out, "out", torch.bfloat16, (B, H, d), dev)
    if scale is None:
        scale = d ** -0.5
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    descs = [describe(t) for t in (q, k, v, g, beta, state, out)]
    ref = [x[0] for x in descs]
    with torch.cuda.device(dev):
        rc = _lib.kda_decode(ref[0], ref[1], ref[2], ref[3], ref[4], ctypes.c_float(scale), ref[5],
                             _ptr(state_indices), ref[6], ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise KDAError(rc)
    return out


def kda_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor, beta: torch.Tensor,
            dout: torch.Tensor, scale: Optional[float] = None, cu_seqlens: Optional[torch.Tensor] = None,
            initial_state: Optional[torch.Tensor] = None, dfinal_state: Optional[torch.Tensor] = None,
            stream: Optional[torch.cuda.Stream] = None):
    """Gradients of the prefill (see ``include/kda.h``): returns a dict of fp32
    tensors ``dq, dk, dv, dg`` [T, H, 128], ``dbeta`` [T, H] and
    ``dinitial_state`` [N, H, 128, 128], for the output gradient ``dout``
    (bf16 [T, H, 128]) and the final-state gradient ``dfinal_state``
    (fp32 [N, H, 128, 128] or None)."""
    if q.dim() != 3:
        raise ValueError("q must be [T, H, 128]")
    T, H, d = q.shape
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("kda_bwd runs on CUDA tensors only")
    N = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    _check(dout, "dout", torch.bfloat16, (T, H, d), dev)
    if cu_seqlens is not None:
        _check(cu_seqlens, "cu_seqlens", torch.int32, (N + 1,), dev, contiguous=True)
    if initial_state is not None:
        _check(initial_state, "initial_state", torch.float32, (N, H, d, d), dev, contiguous=True)
    if dfinal_state is not None:
        _check(dfinal_state, "dfinal_state", torch.float32, (N, H, d, d), dev, contiguous=True)
    grads = {n: torch.empty((T, H, d), dtype=torch.float32, device=dev) for n in ("dq", "dk", "dv", "dg")}
    grads["dbeta"] = torch.empty((T, H), dtype=torch.float32, device=dev)
    grads["dinitial_state"] = torch.empty((N, H, d, d), dtype=torch.float32, device=dev)
    if scale is None:
        scale = d ** -0.5
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    ts = (q, k, v, g, beta, initial_state, dout, dfinal_state, grads["dq"], grads["dk"], grads["dv"], grads["dg"],
          grads["dbeta"], grads["dinitial_state"])
    descs = [describe(t) for t in ts]
    r = [None if x is None else x[0] for x in descs]
    with torch.cuda.device(dev):
        rc = _lib.kda_bwd(r[0], r[1], r[2], r[3], r[4], ctypes.c_float(scale), _ptr(cu_seqlens), N, r[5], r[6], r[7],
                          r[8], r[9], r[10], r[11], r[12], r[13], ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise KDAError(rc)
    return grads
