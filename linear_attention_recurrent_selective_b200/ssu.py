"""Thin Python binding of libssu.so (the C ABI declared in include/ssu.h).

Argument marshalling only: every function here checks that tensors are CUDA tensors of
the expected dtype and layout, reads their sizes, and passes raw device pointers and
the current CUDA stream to the C entry point of the same name. All arithmetic runs in
the library's kernels; there is no other implementation to fall back to, and a missing
library raises ``SSULibraryMissing``.

Semantics (Selective State Update page of the TensorRT-Edge-LLM C++ API):
  ssu_decode   new_state = state * exp(A*dt) + B*dt*x ; out = sum(new_state*C) + D*x,
               times silu(z) when z is given (invokeSelectiveStateUpdate)
  ssu_prefill  the same over [batch, T] tokens in one launch, optional replay stash
               (invokeSelectiveStateUpdatePrefill)
  ssu_replay   re-apply the first acceptedLengths[b] stashed tokens (MambaReplayLayerInfo)
  pool_clear_slot / pool_copy_slot  slot maintenance (invokeMambaStateClear;
               Recurrent State Manager clearSlot / copySlotFrom)
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libssu.so")

SSU_F32, SSU_F16, SSU_BF16 = 0, 1, 2
DTYPE_CODE = {torch.float32: SSU_F32, torch.float16: SSU_F16, torch.bfloat16: SSU_BF16}

FLAG_INDEX_RANGE = 1
FLAG_ACCEPTED_RANGE = 2
FLAG_CONTEXT_RANGE = 4
FLAG_NEGATIVE_LENGTH = 8
FLAG_TIMEOUT = 16

# Every C entry point declared in include/ssu.h, in declaration order.
ENTRY_POINTS = ("ssu_decode", "ssu_prefill", "ssu_replay", "pool_clear_slot",
                "pool_copy_slot", "ssu_status_string")


class SSULibraryMissing(RuntimeError):
    """libssu.so is not built (or cannot be loaded); there is no fallback path."""


class SSUError(RuntimeError):
    """A libssu entry point returned a non-zero ssu_status."""

    def __init__(self, fn: str, status: int, text: str):
        super().__init__(f"{fn} failed with status {status}: {text}")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library with argument types declared (loads it on first use)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise SSULibraryMissing(
            f"{LIB_PATH} is missing: build it with "
            "`python -m linear_attention_recurrent_selective_b200.build`")
    try:
        L = ctypes.CDLL(LIB_PATH)
    except OSError as e:
        raise SSULibraryMissing(f"cannot load {LIB_PATH}: {e}") from e
    vp, i32, i64, ci = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_int
    L.ssu_decode.argtypes = [vp, ci, vp, vp, vp, ci, vp, vp, vp, vp, vp, ci, i64, i32, vp, vp,
                             i32, i32, i32, i32, i32, i32, ci, vp, vp]
    L.ssu_prefill.argtypes = [vp, ci, vp, vp, vp, ci, vp, vp, vp, vp, vp, ci, i64, i32, vp, vp,
                              vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, ci, vp, vp]
    L.ssu_replay.argtypes = [vp, ci, i64, i32, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                             i32, i32, vp, vp]
    L.pool_clear_slot.argtypes = [vp, i64, i32, i32, vp]
    L.pool_copy_slot.argtypes = [vp, i32, i32, vp, i32, i32, i64, vp]
    for f in ENTRY_POINTS[:-1]:
        getattr(L, f).restype = ci
    L.ssu_status_string.argtypes = [ci]
    L.ssu_status_string.restype = ctypes.c_char_p
    _lib = L
    return L


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise SSUError(fn, status, lib().ssu_status_string(status).decode())


def _ptr(t: Optional[torch.Tensor], name: str, dtype=None) -> Optional[ctypes.c_void_p]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _pool_geometry(state: torch.Tensor, slot_stride, P, slot_elems):
    """(slot_stride, P) of a pool given as [P, H, Dm, N] (stride(0) may be padded) or as
    flat storage with an explicit slot_stride."""
    if not state.is_cuda:
        raise ValueError("state must be a CUDA tensor")
    if state.dim() == 4:
        inner = state[0] if state.shape[0] > 0 else state.new_empty(state.shape[1:])
        if not inner.is_contiguous():
            raise ValueError("state [P, H, Dm, N] must be contiguous inside a slot")
        stride = state.stride(0) if slot_stride is None else slot_stride
        return stride, state.shape[0] if P is None else P
    if slot_stride is None:
        slot_stride = slot_elems
    if not state.is_contiguous():
        raise ValueError("flat state storage must be contiguous")
    return slot_stride, state.numel() // slot_stride if P is None else P


def _dt(t: torch.Tensor, name: str) -> int:
    try:
        return DTYPE_CODE[t.dtype]
    except KeyError:
        raise ValueError(f"{name} dtype {t.dtype} is not fp32, fp16 or bf16") from None


def ssu_decode(x, A, B, C, dt, state, out, *, dt_bias=None, D=None, z=None,
               state_indices=None, active_batch=None, dt_softplus=True, err_flags=None,
               slot_stride=None, P=None, stream=None):
    """One decode token. x/z/out [batch,H,Dm]; B/C [batch,G,N]; dt [batch,H]; A, dt_bias,
    D [H] fp32; state pool [P,H,Dm,N] (or flat with slot_stride) updated in place."""
    batch, H, Dm = x.shape
    G, N = B.shape[1], B.shape[2]
    active = batch if active_batch is None else active_batch
    stride, P = _pool_geometry(state, slot_stride, P, H * Dm * N)
    if z is not None and z.dtype != x.dtype:
        raise ValueError("z must have x's dtype")
    if out.dtype != x.dtype or out.shape != x.shape:
        raise ValueError("out must match x in shape and dtype")
    rc = lib().ssu_decode(
        _ptr(x, "x"), _dt(x, "x"), _ptr(A, "A", torch.float32), _ptr(B, "B"), _ptr(C, "C", B.dtype),
        _dt(B, "B"), _ptr(dt, "dt", torch.float32), _ptr(dt_bias, "dt_bias", torch.float32),
        _ptr(D, "D", torch.float32), _ptr(z, "z"), ctypes.c_void_p(state.data_ptr()),
        _dt(state, "state"), stride, P, _ptr(out, "out"),
        _ptr(state_indices, "state_indices", torch.int32), batch, active, H, G, Dm, N,
        int(bool(dt_softplus)), _ptr(err_flags, "err_flags", torch.int32), _stream(stream))
    _check("ssu_decode", rc)
    return out


def ssu_prefill(x, A, B, C, dt, state, out, *, dt_bias=None, D=None, z=None,
                state_indices=None, context_lengths=None, stash=None, active_batch=None,
                dt_softplus=True, err_flags=None, slot_stride=None, P=None, stream=None):
    """All T tokens in one launch. x/z/out [batch,T,H,Dm]; B/C [batch,T,G,N];
    dt [batch,T,H]; ``stash`` None or (dA [b,T,H], U [b,T,H,Dm], B [b,T,G,N],
    dt [b,T,H]) fp32 tensors written in place (the pool then stays read-only)."""
    batch, T, H, Dm = x.shape
    G, N = B.shape[2], B.shape[3]
    active = batch if active_batch is None else active_batch
    stride, P = _pool_geometry(state, slot_stride, P, H * Dm * N)
    if z is not None and z.dtype != x.dtype:
        raise ValueError("z must have x's dtype")
    if out.dtype != x.dtype or out.shape != x.shape:
        raise ValueError("out must match x in shape and dtype")
    f32 = torch.float32
    sdA, sU, sB, sdt = stash if stash is not None else (None, None, None, None)
    rc = lib().ssu_prefill(
        _ptr(x, "x"), _dt(x, "x"), _ptr(A, "A", f32), _ptr(B, "B"), _ptr(C, "C", B.dtype),
        _dt(B, "B"), _ptr(dt, "dt", f32), _ptr(dt_bias, "dt_bias", f32), _ptr(D, "D", f32),
        _ptr(z, "z"), ctypes.c_void_p(state.data_ptr()), _dt(state, "state"), stride, P,
        _ptr(out, "out"), _ptr(state_indices, "state_indices", torch.int32),
        _ptr(context_lengths, "context_lengths", torch.int32),
        _ptr(sdA, "stash dA", f32), _ptr(sU, "stash U", f32), _ptr(sB, "stash B", f32),
        _ptr(sdt, "stash dt", f32), batch, active, T, H, G, Dm, N, int(bool(dt_softplus)),
        _ptr(err_flags, "err_flags", torch.int32), _stream(stream))
    _check("ssu_prefill", rc)
    return out


def ssu_replay(state, stash, accepted_lengths, *, state_indices=None, active_batch=None,
               err_flags=None, slot_stride=None, P=None, stream=None):
    """Re-apply the first accepted_lengths[b] stashed tokens to the pool, in place."""
    sdA, sU, sB, sdt = stash
    batch, T, H, Dm = sU.shape
    G, N = sB.shape[2], sB.shape[3]
    active = batch if active_batch is None else active_batch
    stride, P = _pool_geometry(state, slot_stride, P, H * Dm * N)
    f32 = torch.float32
    rc = lib().ssu_replay(
        ctypes.c_void_p(state.data_ptr()), _dt(state, "state"), stride, P,
        _ptr(sdA, "stash dA", f32), _ptr(sU, "stash U", f32), _ptr(sB, "stash B", f32),
        _ptr(sdt, "stash dt", f32), _ptr(accepted_lengths, "accepted_lengths", torch.int32),
        _ptr(state_indices, "state_indices", torch.int32), batch, active, T, H, G, Dm, N,
        _ptr(err_flags, "err_flags", torch.int32), _stream(stream))
    _check("ssu_replay", rc)


def pool_clear_slot(pool, slot, *, slot_bytes=None, P=None, stream=None):
    """Zero slot ``slot`` of the pool, or every slot when slot == -1. A [P, ...] pool gives
    its own slot size; flat storage needs ``slot_bytes`` and ``P``."""
    if not pool.is_cuda:
        raise ValueError("pool must be a CUDA tensor")
    if slot_bytes is None:
        slot_bytes = pool.stride(0) * pool.element_size()
        P = pool.shape[0]
    rc = lib().pool_clear_slot(ctypes.c_void_p(pool.data_ptr()), slot_bytes, P, slot,
                               _stream(stream))
    _check("pool_clear_slot", rc)


def pool_copy_slot(dst_pool, dst_slot, src_pool, src_slot, *, slot_bytes=None, dst_P=None,
                   src_P=None, stream=None):
    """Copy one slot between pools of the same per-slot geometry (slot counts may differ)."""
    if not (dst_pool.is_cuda and src_pool.is_cuda):
        raise ValueError("pools must be CUDA tensors")
    if slot_bytes is None:
        slot_bytes = dst_pool.stride(0) * dst_pool.element_size()
        if src_pool.stride(0) * src_pool.element_size() != slot_bytes:
            raise ValueError("pools differ in per-slot geometry")
        dst_P, src_P = dst_pool.shape[0], src_pool.shape[0]
    rc = lib().pool_copy_slot(ctypes.c_void_p(dst_pool.data_ptr()), dst_P, dst_slot,
                              ctypes.c_void_p(src_pool.data_ptr()), src_P, src_slot,
                              slot_bytes, _stream(stream))
    _check("pool_copy_slot", rc)
