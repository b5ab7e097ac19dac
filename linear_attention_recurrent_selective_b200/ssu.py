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
  ssu_conv_decode  causal conv1d update of the raw xBC channels fused with the decode
               (convState beside the recurrent state; FlashInfer conv update)
  gdn_decode   gated delta-rule decode core over a paged fp32 pool (FlashInfer GDN page)
  ssu_ddtree   tree verify: every node of a draft tree from the committed state along its
               ancestor path, stash per node (invokeSelectiveStateUpdateDDTree)
  ssu_replay   re-apply the first acceptedLengths[b] stashed tokens, or the accepted
               tree nodes acceptedNodeIds[b][:acceptedLengths[b]] (MambaReplayLayerInfo)
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
FLAG_LAYER = 32
FLAG_TREE = 64
FLAG_DUPLICATE_INDEX = 128

# Every C entry point declared in include/ssu.h, in declaration order.
ENTRY_POINTS = ("ssu_decode", "ssu_prefill", "ssu_replay", "ssu_replay_layers",
                "ssu_conv_decode", "gdn_decode", "ssu_ddtree", "pool_clear_slot",
                "pool_copy_slot", "pool_clear_slot_layers", "pool_gather", "pool_scatter",
                "ssu_check_state_indices", "ssu_status_string")

# Byte layouts of the per-layer pointer records of include/ssu.h (packed pointers).
REPLAY_LAYER_FIELDS = 5     # state, st_dA, st_U, st_B, st_dt
LAYER_STATES_FIELDS = 2     # recurrent_state, conv_state


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
    if _lib is None:
        _lib = load(LIB_PATH)
    return _lib


def load(path: str) -> ctypes.CDLL:
    """Load a build of the library (libssu.so, or the test suite's libssu_waittest.so,
    which exports the same entry points) and declare the entry points' argument types."""
    if not os.path.exists(path):
        raise SSULibraryMissing(
            f"{path} is missing: build it with "
            "`python -m linear_attention_recurrent_selective_b200.build`")
    try:
        L = ctypes.CDLL(path)
    except OSError as e:
        raise SSULibraryMissing(f"cannot load {path}: {e}") from e
    vp, i32, i64, ci = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_int
    L.ssu_decode.argtypes = [vp, ci, vp, vp, vp, ci, vp, vp, vp, vp, vp, ci, i64, i32, vp, vp,
                             i32, i32, i32, i32, i32, i32, ci, vp, vp]
    L.ssu_prefill.argtypes = [vp, ci, vp, vp, vp, ci, vp, vp, vp, vp, vp, ci, i64, i32, vp, vp,
                              vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, ci, vp, vp]
    L.ssu_replay.argtypes = [vp, ci, i64, i32, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                             i32, i32, vp, i32, vp, vp]
    L.ssu_replay_layers.argtypes = [vp, i32, ci, i64, i32, vp, vp, i32, i32, i32, i32, i32,
                                    i32, i32, vp, i32, vp, vp]
    L.ssu_conv_decode.argtypes = [vp, ci, vp, vp, vp, i64, i64, i64, i32, ci, vp, vp, vp, vp,
                                  vp, vp, ci, i64, i32, vp, vp, i32, i32, i32, i32, i32, i32,
                                  ci, vp, vp]
    L.gdn_decode.argtypes = [vp, vp, vp, ci, vp, vp, vp, vp, ctypes.c_float, ci, vp, i64, i32,
                             vp, vp, i32, i32, i32, i32, i32, i32, vp, vp]
    L.ssu_ddtree.argtypes = [vp, ci, vp, vp, vp, ci, vp, vp, vp, vp, ci, i64, i32, vp, vp, vp,
                             vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, ci, vp, vp]
    L.pool_clear_slot.argtypes = [vp, i64, i32, i32, vp]
    L.pool_copy_slot.argtypes = [vp, i32, i32, vp, i32, i32, i64, vp]
    L.pool_clear_slot_layers.argtypes = [vp, i32, i32, i32, i64, i64, vp]
    L.pool_gather.argtypes = [vp, i64, i32, vp, vp, i32, i32, vp, vp]
    L.pool_scatter.argtypes = [vp, vp, i64, i32, vp, i32, i32, vp, vp]
    L.ssu_check_state_indices.argtypes = [vp, i32, i32, i32, vp, vp]
    for f in ENTRY_POINTS[:-1]:
        getattr(L, f).restype = ci
    L.ssu_status_string.argtypes = [ci]
    L.ssu_status_string.restype = ctypes.c_char_p
    return L


# Debug mode: when on, every call that takes state_indices first checks them with
# check_state_indices (which synchronises, so it cannot run under CUDA-graph capture).
_debug_checks = os.environ.get("SSU_DEBUG_CHECKS", "") not in ("", "0")


def set_debug_checks(enabled: bool) -> bool:
    """Turn the debug check of state_indices before every call on or off (also set by the
    environment variable SSU_DEBUG_CHECKS=1). Returns the previous setting."""
    global _debug_checks
    before, _debug_checks = _debug_checks, bool(enabled)
    return before


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


def ssu_check_state_indices(state_indices, P, err_flags, *, active_batch=None, stream=None):
    """Enqueue the library's check of a row-to-slot map: ORs FLAG_DUPLICATE_INDEX into
    err_flags when two active rows name the same slot (>= 0), FLAG_INDEX_RANGE when one
    names a slot >= P. Asynchronous, like every entry point."""
    batch = state_indices.shape[0]
    active = batch if active_batch is None else active_batch
    rc = lib().ssu_check_state_indices(
        _ptr(state_indices, "state_indices", torch.int32), batch, active, P,
        _ptr(err_flags, "err_flags", torch.int32), _stream(stream))
    _check("ssu_check_state_indices", rc)


def check_state_indices(state_indices, P, *, active_batch=None, stream=None) -> None:
    """Debug helper: run the library's check on ``stream``, wait for it and raise
    ValueError when the active rows' indices repeat a slot or leave the pool. It
    synchronises the stream, so it is not for use under CUDA-graph capture."""
    if state_indices is None:
        return
    flags = torch.zeros(1, dtype=torch.int32, device=state_indices.device)
    ssu_check_state_indices(state_indices, P, flags, active_batch=active_batch, stream=stream)
    s = torch.cuda.current_stream(state_indices.device) if stream is None else stream
    s.synchronize()
    f = int(flags.item())
    problems = []
    if f & FLAG_DUPLICATE_INDEX:
        problems.append("two active rows share a pool slot")
    if f & FLAG_INDEX_RANGE:
        problems.append(f"an active row's slot is >= P ({P})")
    if problems:
        raise ValueError("state_indices: " + "; ".join(problems))


def _debug_indices(state_indices, P, active, stream):
    if _debug_checks and state_indices is not None:
        check_state_indices(state_indices, P, active_batch=active, stream=stream)


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
    _debug_indices(state_indices, P, active, stream)
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
    _debug_indices(state_indices, P, active, stream)
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


def _node_ids(accepted_node_ids):
    if accepted_node_ids is None:
        return None, 0
    if accepted_node_ids.dim() != 2:
        raise ValueError("accepted_node_ids must be [batch, maxAcceptLen]")
    return _ptr(accepted_node_ids, "accepted_node_ids", torch.int32), accepted_node_ids.shape[1]


def ssu_replay(state, stash, accepted_lengths, *, state_indices=None, active_batch=None,
               err_flags=None, slot_stride=None, P=None, accepted_node_ids=None, stream=None):
    """Re-apply the first accepted_lengths[b] stashed tokens to the pool, in place; with
    ``accepted_node_ids`` [batch, maxAcceptLen] token t of row b is stash entry
    accepted_node_ids[b, t] (an accepted path of a tree verify)."""
    sdA, sU, sB, sdt = stash
    batch, T, H, Dm = sU.shape
    G, N = sB.shape[2], sB.shape[3]
    active = batch if active_batch is None else active_batch
    stride, P = _pool_geometry(state, slot_stride, P, H * Dm * N)
    f32 = torch.float32
    _debug_indices(state_indices, P, active, stream)
    rc = lib().ssu_replay(
        ctypes.c_void_p(state.data_ptr()), _dt(state, "state"), stride, P,
        _ptr(sdA, "stash dA", f32), _ptr(sU, "stash U", f32), _ptr(sB, "stash B", f32),
        _ptr(sdt, "stash dt", f32), _ptr(accepted_lengths, "accepted_lengths", torch.int32),
        _ptr(state_indices, "state_indices", torch.int32), batch, active, T, H, G, Dm, N,
        *_node_ids(accepted_node_ids), _ptr(err_flags, "err_flags", torch.int32),
        _stream(stream))
    _check("ssu_replay", rc)


def ssu_conv_decode(xbc, conv_weight, conv_state, A, dt, state, out, *, width, conv_strides,
                    nheads, ngroups, dim, conv_bias=None, conv_silu=True, dt_bias=None,
                    D=None, z=None, state_indices=None, active_batch=None, dt_softplus=True,
                    err_flags=None, slot_stride=None, P=None, stream=None):
    """Causal conv1d update of the raw channels xbc [batch, H*Dm + 2*G*N] (x, B, C order)
    fused with one decode token. conv_state: the conv pool (any layout), with
    conv_strides = (slot, channel, tap) element strides; both pools updated in place."""
    batch = xbc.shape[0]
    H, G, Dm = nheads, ngroups, dim
    N = (xbc.shape[1] - H * Dm) // (2 * G)
    active = batch if active_batch is None else active_batch
    stride, P = _pool_geometry(state, slot_stride, P, H * Dm * N)
    if out.dtype != xbc.dtype or tuple(out.shape) != (batch, H, Dm):
        raise ValueError("out must be [batch, H, Dm] in xbc's dtype")
    for t, name in ((conv_weight, "conv_weight"), (conv_bias, "conv_bias"), (z, "z")):
        if t is not None and t.dtype != xbc.dtype:
            raise ValueError(f"{name} must have xbc's dtype")
    if conv_state is not None and conv_state.dtype != xbc.dtype:
        raise ValueError("conv_state must have xbc's dtype")
    cs, cc, ck = conv_strides
    f32 = torch.float32
    _debug_indices(state_indices, P, active, stream)
    rc = lib().ssu_conv_decode(
        _ptr(xbc, "xbc"), _dt(xbc, "xbc"), _ptr(conv_weight, "conv_weight"),
        _ptr(conv_bias, "conv_bias"),
        None if conv_state is None else ctypes.c_void_p(conv_state.data_ptr()), cs, cc, ck,
        width, int(bool(conv_silu)), _ptr(A, "A", f32), _ptr(dt, "dt", f32),
        _ptr(dt_bias, "dt_bias", f32), _ptr(D, "D", f32), _ptr(z, "z"),
        ctypes.c_void_p(state.data_ptr()), _dt(state, "state"), stride, P, _ptr(out, "out"),
        _ptr(state_indices, "state_indices", torch.int32), batch, active, H, G, Dm, N,
        int(bool(dt_softplus)), _ptr(err_flags, "err_flags", torch.int32), _stream(stream))
    _check("ssu_conv_decode", rc)
    return out


def gdn_decode(q, k, v, a, b, A_log, state, out, *, dt_bias=None, scale=None,
               use_qk_l2norm=True, state_indices=None, active_batch=None, err_flags=None,
               slot_stride=None, P=None, stream=None):
    """Gated delta-rule decode token. q, k [batch, HK, K]; v, out [batch, HV, V]; a, b
    [batch, HV] (same dtype); A_log, dt_bias [HV] fp32; state: fp32 pool [P, HV, V, K]
    (or flat with slot_stride), updated in place. scale None/0: 1/sqrt(K)."""
    batch, HK, K = q.shape
    HV, V = v.shape[1], v.shape[2]
    active = batch if active_batch is None else active_batch
    if state.dtype != torch.float32:
        raise ValueError("the GDN state pool is fp32")
    stride, P = _pool_geometry(state, slot_stride, P, HV * V * K)
    for t, name in ((k, "k"), (v, "v"), (a, "a"), (b, "b"), (out, "out")):
        if t.dtype != q.dtype:
            raise ValueError(f"{name} must have q's dtype")
    if tuple(out.shape) != (batch, HV, V):
        raise ValueError("out must be [batch, HV, V]")
    f32 = torch.float32
    _debug_indices(state_indices, P, active, stream)
    rc = lib().gdn_decode(
        _ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _dt(q, "q"), _ptr(a, "a"), _ptr(b, "b"),
        _ptr(A_log, "A_log", f32), _ptr(dt_bias, "dt_bias", f32), float(scale or 0.0),
        int(bool(use_qk_l2norm)), ctypes.c_void_p(state.data_ptr()), stride, P,
        _ptr(out, "out"), _ptr(state_indices, "state_indices", torch.int32), batch, active,
        HK, HV, K, V, _ptr(err_flags, "err_flags", torch.int32), _stream(stream))
    _check("gdn_decode", rc)
    return out


def ssu_ddtree(x, A, B, C, dt, state, out, parent_ids, depths, stash, *, dt_bias=None,
               D=None, state_indices=None, active_batch=None, dt_softplus=True,
               err_flags=None, slot_stride=None, P=None, stream=None):
    """Tree verify of one draft tree of T <= 128 nodes per row. x/out [batch,T,H,Dm];
    B/C [batch,T,G,N]; dt [batch,T,H]; parent_ids/depths [batch,T] int32; ``stash`` =
    (dA [b,T,H], U [b,T,H,Dm], B [b,T,G,N], dt [b,T,H]) fp32, written for every node.
    The pool is only read."""
    batch, T, H, Dm = x.shape
    G, N = B.shape[2], B.shape[3]
    active = batch if active_batch is None else active_batch
    stride, P = _pool_geometry(state, slot_stride, P, H * Dm * N)
    if out.dtype != x.dtype or out.shape != x.shape:
        raise ValueError("out must match x in shape and dtype")
    f32, i32 = torch.float32, torch.int32
    sdA, sU, sB, sdt = stash
    _debug_indices(state_indices, P, active, stream)
    rc = lib().ssu_ddtree(
        _ptr(x, "x"), _dt(x, "x"), _ptr(A, "A", f32), _ptr(B, "B"), _ptr(C, "C", B.dtype),
        _dt(B, "B"), _ptr(dt, "dt", f32), _ptr(dt_bias, "dt_bias", f32), _ptr(D, "D", f32),
        ctypes.c_void_p(state.data_ptr()), _dt(state, "state"), stride, P, _ptr(out, "out"),
        _ptr(parent_ids, "parent_ids", i32), _ptr(depths, "depths", i32),
        _ptr(state_indices, "state_indices", i32), _ptr(sdA, "stash dA", f32),
        _ptr(sU, "stash U", f32), _ptr(sB, "stash B", f32), _ptr(sdt, "stash dt", f32),
        batch, active, T, H, G, Dm, N, int(bool(dt_softplus)),
        _ptr(err_flags, "err_flags", i32), _stream(stream))
    _check("ssu_ddtree", rc)
    return out


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


def replay_layer_table(layers, device=None):
    """Device array of ssu_replay_layer records for ``ssu_replay_layers``: ``layers`` is a
    list of (state, (dA, U, B, dt)) CUDA tensors. Keep the returned tensor alive until
    the launch that uses it has run."""
    ptrs = []
    for state, (sdA, sU, sB, sdt) in layers:
        ptrs += [t.data_ptr() for t in (state, sdA, sU, sB, sdt)]
    dev = device if device is not None else layers[0][0].device
    return torch.tensor(ptrs, dtype=torch.int64, device=dev)


def layer_states_table(layers, device=None):
    """Device array of ssu_layer_states records for ``pool_clear_slot_layers``: ``layers``
    is a list of (recurrent_state, conv_state or None) CUDA tensors."""
    ptrs = []
    for rec, conv in layers:
        ptrs += [rec.data_ptr(), 0 if conv is None else conv.data_ptr()]
    dev = device if device is not None else layers[0][0].device
    return torch.tensor(ptrs, dtype=torch.int64, device=dev)


def ssu_replay_layers(table, num_layers, like_state, like_stash, accepted_lengths, *,
                      state_indices=None, active_batch=None, err_flags=None, slot_stride=None,
                      P=None, accepted_node_ids=None, stream=None):
    """ssu_replay over ``num_layers`` layers in one launch. ``table`` comes from
    ``replay_layer_table``; ``like_state`` / ``like_stash`` are any one layer's pool and
    stash, which give the (shared) geometry and dtypes."""
    sdA, sU, sB, sdt = like_stash
    batch, T, H, Dm = sU.shape
    G, N = sB.shape[2], sB.shape[3]
    active = batch if active_batch is None else active_batch
    stride, P = _pool_geometry(like_state, slot_stride, P, H * Dm * N)
    _debug_indices(state_indices, P, active, stream)
    rc = lib().ssu_replay_layers(
        _ptr(table, "layer table", torch.int64), num_layers, _dt(like_state, "state"), stride,
        P, _ptr(accepted_lengths, "accepted_lengths", torch.int32),
        _ptr(state_indices, "state_indices", torch.int32), batch, active, T, H, G, Dm, N,
        *_node_ids(accepted_node_ids), _ptr(err_flags, "err_flags", torch.int32),
        _stream(stream))
    _check("ssu_replay_layers", rc)


def pool_clear_slot_layers(table, num_layers, P, slot, recurrent_slot_bytes,
                           conv_slot_bytes=0, *, stream=None):
    """Zero one slot (or all, slot == -1) of every layer's recurrent and conv pools."""
    rc = lib().pool_clear_slot_layers(_ptr(table, "layer table", torch.int64), num_layers, P,
                                      slot, recurrent_slot_bytes, conv_slot_bytes,
                                      _stream(stream))
    _check("pool_clear_slot_layers", rc)


def pool_gather(pool, dense, *, state_indices=None, active_batch=None, err_flags=None,
                slot_bytes=None, P=None, stream=None):
    """dense[b] = pool[state_indices[b]] for the active rows (padding rows get zeros)."""
    batch = dense.shape[0]
    active = batch if active_batch is None else active_batch
    if slot_bytes is None:
        slot_bytes = pool.stride(0) * pool.element_size()
        P = pool.shape[0]
    if not (pool.is_cuda and dense.is_cuda and dense.is_contiguous()):
        raise ValueError("pool and dense must be CUDA tensors, dense contiguous")
    _debug_indices(state_indices, P, active, stream)
    rc = lib().pool_gather(ctypes.c_void_p(pool.data_ptr()), slot_bytes, P,
                           ctypes.c_void_p(dense.data_ptr()),
                           _ptr(state_indices, "state_indices", torch.int32), batch, active,
                           _ptr(err_flags, "err_flags", torch.int32), _stream(stream))
    _check("pool_gather", rc)


def pool_scatter(dense, pool, *, state_indices=None, active_batch=None, err_flags=None,
                 slot_bytes=None, P=None, stream=None):
    """pool[state_indices[b]] = dense[b] for the active rows (padding rows are skipped)."""
    batch = dense.shape[0]
    active = batch if active_batch is None else active_batch
    if slot_bytes is None:
        slot_bytes = pool.stride(0) * pool.element_size()
        P = pool.shape[0]
    if not (pool.is_cuda and dense.is_cuda and dense.is_contiguous()):
        raise ValueError("pool and dense must be CUDA tensors, dense contiguous")
    _debug_indices(state_indices, P, active, stream)
    rc = lib().pool_scatter(ctypes.c_void_p(dense.data_ptr()), ctypes.c_void_p(pool.data_ptr()),
                            slot_bytes, P, _ptr(state_indices, "state_indices", torch.int32),
                            batch, active, _ptr(err_flags, "err_flags", torch.int32),
                            _stream(stream))
    _check("pool_scatter", rc)
