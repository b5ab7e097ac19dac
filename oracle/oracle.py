"""Python access to the float64 CPU oracle (``ssu_oracle.c``).

TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg import this module. It never touches the CUDA library.

The functions take CPU torch tensors (used here only as typed host buffers) and return
float64 outputs. The pool is updated in place in its own storage type, exactly as the
Selective State Update page (TensorRT-Edge-LLM C++ API) describes for
``invokeSelectiveStateUpdate``, ``invokeSelectiveStateUpdatePrefill``, the tree verify
``invokeSelectiveStateUpdateDDTree`` and the replay.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ssu_oracle.c")
LIB = os.path.join(HERE, "libssu_oracle.so")

_CODES = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2, torch.float64: 3}


def build(force: bool = False) -> str:
    """Compile the oracle with gcc into ``oracle/libssu_oracle.so``."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + ".tmp"
        subprocess.run(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-Wall", "-Wextra", "-fopenmp",
             "-fno-fast-math", "-ffp-contract=off", "-o", tmp, SRC, "-lm"],
            check=True,
        )
        os.replace(tmp, LIB)
    return LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB)
        vp, i32, i64, i = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_int
        L.oracle_decode.argtypes = [vp, i, vp, vp, vp, i, vp, vp, vp, vp, vp, i, i64, i32,
                                    vp, vp, i32, i32, i32, i32, i32, i32, i, vp]
        L.oracle_prefill.argtypes = [vp, i, vp, vp, vp, i, vp, vp, vp, vp, vp, i, i64, i32,
                                     vp, vp, vp, vp, vp, vp, vp,
                                     i32, i32, i32, i32, i32, i32, i32, i, vp]
        L.oracle_replay.argtypes = [vp, i, i64, i32, vp, vp, vp, vp, vp, vp,
                                    i32, i32, i32, i32, i32, i32, i32, vp, i32, vp]
        L.oracle_conv_decode.argtypes = [vp, i, vp, vp, vp, i64, i64, i64, i32, i, vp, vp, vp,
                                         vp, vp, vp, i, i64, i32, vp, vp, i32, i32, i32, i32,
                                         i32, i32, i, vp]
        L.oracle_gdn_decode.argtypes = [vp, vp, vp, i, vp, vp, vp, vp, ctypes.c_double, i, vp,
                                        i64, i32, vp, vp, i32, i32, i32, i32, i32, i32, vp]
        L.oracle_ddtree.argtypes = [vp, i, vp, vp, vp, i, vp, vp, vp, vp, i, i64, i32,
                                    vp, vp, vp, vp, vp, vp, vp, vp,
                                    i32, i32, i32, i32, i32, i32, i32, i, vp]
        L.oracle_clear_slot.argtypes = [vp, i64, i32, i32]
        L.oracle_replay_layers.argtypes = [vp, vp, vp, vp, vp, i32, i, i64, i32, vp, vp, i32,
                                           i32, i32, i32, i32, i32, i32, vp, i32, vp]
        L.oracle_clear_slot_layers.argtypes = [vp, vp, i32, i32, i32, i64, i64]
        L.oracle_gather_scatter.argtypes = [vp, i64, i32, vp, vp, i32, i32, i, vp]
        L.oracle_copy_slot.argtypes = [vp, i32, i32, vp, i32, i32, i64]
        L.oracle_f16_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_f16_to_double.restype = ctypes.c_double
        L.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_double.restype = ctypes.c_double
        L.oracle_double_to_f16.argtypes = [ctypes.c_double]
        L.oracle_double_to_f16.restype = ctypes.c_uint16
        L.oracle_double_to_bf16.argtypes = [ctypes.c_double]
        L.oracle_double_to_bf16.restype = ctypes.c_uint16
        L.oracle_set_threads.argtypes = [i]
        L.oracle_set_threads.restype = None
        L.oracle_max_threads.restype = ctypes.c_int
        L.oracle_host_cores.restype = ctypes.c_int
        for f in ("oracle_decode", "oracle_prefill", "oracle_replay",
                  "oracle_clear_slot", "oracle_copy_slot", "oracle_replay_layers",
                  "oracle_clear_slot_layers", "oracle_gather_scatter", "oracle_ddtree",
                  "oracle_conv_decode", "oracle_gdn_decode"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def set_threads(n: int) -> int:
    """Run the oracle's independent (row, head) units on n OpenMP threads (n <= 0: every
    host core). Results do not depend on n. Returns the thread count now in effect."""
    lib().oracle_set_threads(int(n))
    return lib().oracle_max_threads()


def threads() -> int:
    return lib().oracle_max_threads()


def host_cores() -> int:
    return lib().oracle_host_cores()


def _p(t):
    if t is None:
        return None
    assert t.device.type == "cpu" and t.is_contiguous(), "oracle takes contiguous CPU tensors"
    return ctypes.c_void_p(t.data_ptr())


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"{what}: oracle rejected the arguments (code {rc})")


def decode(x, A, B, C, dt, pool, *, dt_bias=None, D=None, z=None, state_indices=None,
           batch, active=None, H, G, Dm, N, slot_stride=None, P=None, dt_softplus=True,
           out=None):
    """One decode token; ``pool`` (flat, storage dtype) is updated in place.

    Returns (out float64 [batch,H,Dm], err_flags). Rows not visited keep ``out``'s
    initial contents (NaN unless ``out`` is given).
    """
    active = batch if active is None else active
    slot_stride = H * Dm * N if slot_stride is None else slot_stride
    P = pool.numel() // slot_stride if P is None else P
    if out is None:
        out = torch.full((batch, H, Dm), float("nan"), dtype=torch.float64)
    err = ctypes.c_int32(0)
    rc = lib().oracle_decode(
        _p(x), _CODES[x.dtype], _p(A), _p(B), _p(C), _CODES[B.dtype], _p(dt), _p(dt_bias),
        _p(D), _p(z), _p(pool), _CODES[pool.dtype], slot_stride, P, _p(out),
        _p(state_indices), batch, active, H, G, Dm, N, int(dt_softplus),
        ctypes.byref(err))
    _check(rc, "oracle_decode")
    return out, err.value


def prefill(x, A, B, C, dt, pool, *, dt_bias=None, D=None, z=None, state_indices=None,
            context_lengths=None, stash=None, batch, active=None, T, H, G, Dm, N,
            slot_stride=None, P=None, dt_softplus=True, out=None):
    """All T tokens in one call. ``stash`` is None or a tuple (DA, U, Bst, DT) of fp32
    CPU tensors written in place. Returns (out float64 [batch,T,H,Dm], err_flags)."""
    active = batch if active is None else active
    slot_stride = H * Dm * N if slot_stride is None else slot_stride
    P = pool.numel() // slot_stride if P is None else P
    if out is None:
        out = torch.full((batch, T, H, Dm), float("nan"), dtype=torch.float64)
    DA, U, Bst, DT = stash if stash is not None else (None, None, None, None)
    err = ctypes.c_int32(0)
    rc = lib().oracle_prefill(
        _p(x), _CODES[x.dtype], _p(A), _p(B), _p(C), _CODES[B.dtype], _p(dt), _p(dt_bias),
        _p(D), _p(z), _p(pool), _CODES[pool.dtype], slot_stride, P, _p(out),
        _p(state_indices), _p(context_lengths), _p(DA), _p(U), _p(Bst), _p(DT),
        batch, active, T, H, G, Dm, N, int(dt_softplus), ctypes.byref(err))
    _check(rc, "oracle_prefill")
    return out, err.value


def new_stash(batch, T, H, G, Dm, N, fill=float("nan")):
    """Fresh fp32 stash buffers (DA, U, Bst, DT) filled with ``fill``."""
    return (torch.full((batch, T, H), fill, dtype=torch.float32),
            torch.full((batch, T, H, Dm), fill, dtype=torch.float32),
            torch.full((batch, T, G, N), fill, dtype=torch.float32),
            torch.full((batch, T, H), fill, dtype=torch.float32))


def replay(pool, stash, accepted_lengths, *, state_indices=None, batch, active=None, T,
           H, G, Dm, N, slot_stride=None, P=None, node_ids=None):
    """Re-apply the first acceptedLengths[b] stashed tokens in place; with ``node_ids``
    ([batch, maxAcceptLen] int32) token t of row b is stash entry node_ids[b, t].
    Returns err_flags."""
    active = batch if active is None else active
    slot_stride = H * Dm * N if slot_stride is None else slot_stride
    P = pool.numel() // slot_stride if P is None else P
    DA, U, Bst, DT = stash
    err = ctypes.c_int32(0)
    rc = lib().oracle_replay(
        _p(pool), _CODES[pool.dtype], slot_stride, P, _p(DA), _p(U), _p(Bst), _p(DT),
        _p(accepted_lengths), _p(state_indices), batch, active, T, H, G, Dm, N,
        _p(node_ids), 0 if node_ids is None else node_ids.shape[1], ctypes.byref(err))
    _check(rc, "oracle_replay")
    return err.value


def ddtree(x, A, B, C, dt, pool, parent_ids, depths, *, dt_bias=None, D=None,
           state_indices=None, batch, active=None, T, H, G, Dm, N, slot_stride=None,
           P=None, dt_softplus=True, out=None, stash=None):
    """Tree verify: every node's output from the committed state along its ancestor path
    (the pool is only read). Returns (out float64 [batch,T,H,Dm], stash, err_flags)."""
    active = batch if active is None else active
    slot_stride = H * Dm * N if slot_stride is None else slot_stride
    P = pool.numel() // slot_stride if P is None else P
    if out is None:
        out = torch.full((batch, T, H, Dm), float("nan"), dtype=torch.float64)
    if stash is None:
        stash = new_stash(batch, T, H, G, Dm, N)
    DA, U, Bst, DT = stash
    err = ctypes.c_int32(0)
    rc = lib().oracle_ddtree(
        _p(x), _CODES[x.dtype], _p(A), _p(B), _p(C), _CODES[B.dtype], _p(dt), _p(dt_bias),
        _p(D), _p(pool), _CODES[pool.dtype], slot_stride, P, _p(out), _p(parent_ids),
        _p(depths), _p(state_indices), _p(DA), _p(U), _p(Bst), _p(DT), batch, active, T, H,
        G, Dm, N, int(dt_softplus), ctypes.byref(err))
    _check(rc, "oracle_ddtree")
    return out, stash, err.value


def conv_decode(xbc, conv_w, conv_b, conv_state, width, A, dt, pool, *, conv_strides,
                dt_bias=None, D=None, z=None, state_indices=None, batch, active=None, H, G,
                Dm, N, slot_stride=None, P=None, dt_softplus=True, conv_silu=True, out=None):
    """Causal conv1d update of the raw xBC channels followed by one decode token; both
    pools are updated in place. conv_strides = (slot, channel, tap) element strides of the
    conv pool. Returns (out float64 [batch,H,Dm], err_flags)."""
    active = batch if active is None else active
    slot_stride = H * Dm * N if slot_stride is None else slot_stride
    P = pool.numel() // slot_stride if P is None else P
    if out is None:
        out = torch.full((batch, H, Dm), float("nan"), dtype=torch.float64)
    err = ctypes.c_int32(0)
    cs, cc, ck = conv_strides
    rc = lib().oracle_conv_decode(
        _p(xbc), _CODES[xbc.dtype], _p(conv_w), _p(conv_b), _p(conv_state), cs, cc, ck, width,
        int(conv_silu), _p(A), _p(dt), _p(dt_bias), _p(D), _p(z), _p(pool), _CODES[pool.dtype],
        slot_stride, P, _p(out), _p(state_indices), batch, active, H, G, Dm, N,
        int(dt_softplus), ctypes.byref(err))
    _check(rc, "oracle_conv_decode")
    return out, err.value


def gdn_decode(q, k, v, a, b, A_log, pool, *, dt_bias=None, scale=None, use_l2norm=True,
               state_indices=None, batch, active=None, HK, HV, K, V, slot_stride=None, P=None,
               out=None):
    """Gated delta-rule decode token; the fp32 pool [P, HV, V, K] is updated in place.
    Returns (out float64 [batch, HV, V], err_flags)."""
    active = batch if active is None else active
    slot_stride = HV * V * K if slot_stride is None else slot_stride
    P = pool.numel() // slot_stride if P is None else P
    scale = K ** -0.5 if not scale else scale
    if out is None:
        out = torch.full((batch, HV, V), float("nan"), dtype=torch.float64)
    err = ctypes.c_int32(0)
    rc = lib().oracle_gdn_decode(
        _p(q), _p(k), _p(v), _CODES[q.dtype], _p(a), _p(b), _p(A_log), _p(dt_bias), scale,
        int(use_l2norm), _p(pool), slot_stride, P, _p(out), _p(state_indices), batch, active,
        HK, HV, K, V, ctypes.byref(err))
    _check(rc, "oracle_gdn_decode")
    return out, err.value


def clear_slot(pool, slot_bytes, P, slot):
    _check(lib().oracle_clear_slot(_p(pool), slot_bytes, P, slot), "oracle_clear_slot")


def copy_slot(dst_pool, dst_P, dst_slot, src_pool, src_P, src_slot, slot_bytes):
    _check(lib().oracle_copy_slot(_p(dst_pool), dst_P, dst_slot, _p(src_pool), src_P,
                                  src_slot, slot_bytes), "oracle_copy_slot")


def _ptr_array(tensors):
    arr = (ctypes.c_void_p * len(tensors))(*[None if t is None else t.data_ptr()
                                             for t in tensors])
    return arr


def replay_layers(pools, stashes, accepted_lengths, *, state_indices=None, batch, active=None,
                  T, H, G, Dm, N, slot_stride=None, P=None, node_ids=None):
    """Replay every layer l: pools[l] (in place) with stashes[l] = (DA, U, Bst, DT)."""
    active = batch if active is None else active
    slot_stride = H * Dm * N if slot_stride is None else slot_stride
    P = pools[0].numel() // slot_stride if P is None else P
    for t in list(pools) + [x for st in stashes for x in st]:
        assert t.device.type == "cpu" and t.is_contiguous()
    err = ctypes.c_int32(0)
    rc = lib().oracle_replay_layers(
        _ptr_array(pools), _ptr_array([s[0] for s in stashes]), _ptr_array([s[1] for s in stashes]),
        _ptr_array([s[2] for s in stashes]), _ptr_array([s[3] for s in stashes]), len(pools),
        _CODES[pools[0].dtype], slot_stride, P, _p(accepted_lengths), _p(state_indices), batch,
        active, T, H, G, Dm, N, _p(node_ids), 0 if node_ids is None else node_ids.shape[1],
        ctypes.byref(err))
    _check(rc, "oracle_replay_layers")
    return err.value


def clear_slot_layers(recurrent, conv, P, slot, recurrent_slot_bytes, conv_slot_bytes):
    """Zero slot ``slot`` (or all, -1) of every layer's recurrent and conv buffers."""
    rc = lib().oracle_clear_slot_layers(_ptr_array(recurrent),
                                        _ptr_array(conv) if conv is not None else None,
                                        len(recurrent), P, slot, recurrent_slot_bytes,
                                        conv_slot_bytes)
    _check(rc, "oracle_clear_slot_layers")


def gather(pool, dense, slot_bytes, P, *, state_indices=None, batch, active=None):
    """dense[b] = pool[slot(b)] (zeros for padding rows). Returns err_flags."""
    active = batch if active is None else active
    err = ctypes.c_int32(0)
    _check(lib().oracle_gather_scatter(_p(pool), slot_bytes, P, _p(dense), _p(state_indices),
                                       batch, active, 0, ctypes.byref(err)), "oracle gather")
    return err.value


def scatter(dense, pool, slot_bytes, P, *, state_indices=None, batch, active=None):
    """pool[slot(b)] = dense[b] (padding rows skipped). Returns err_flags."""
    active = batch if active is None else active
    err = ctypes.c_int32(0)
    _check(lib().oracle_gather_scatter(_p(pool), slot_bytes, P, _p(dense), _p(state_indices),
                                       batch, active, 1, ctypes.byref(err)), "oracle scatter")
    return err.value


# --- convenience wrappers over a workloads.SSUCase (inputs only; no arithmetic) ---

def decode_case(case, pool=None):
    """Run the oracle decode on a case; returns (out, pool_after, err)."""
    pool = case.pool.clone() if pool is None else pool
    out, err = decode(case.x, case.A, case.B, case.C, case.dt, pool, dt_bias=case.dt_bias,
                      D=case.D, z=case.z, state_indices=case.state_indices,
                      batch=case.batch, active=case.active, H=case.H, G=case.G,
                      Dm=case.Dm, N=case.N, slot_stride=case.slot_stride, P=case.P,
                      dt_softplus=case.dt_softplus)
    return out, pool, err


def prefill_case(case, pool=None, stash=False):
    """Run the oracle prefill on a case; returns (out, pool_after, stash or None, err)."""
    pool = case.pool.clone() if pool is None else pool
    st = new_stash(case.batch, case.T, case.H, case.G, case.Dm, case.N) if stash else None
    out, err = prefill(case.x, case.A, case.B, case.C, case.dt, pool, dt_bias=case.dt_bias,
                       D=case.D, z=case.z, state_indices=case.state_indices,
                       context_lengths=case.context_lengths, stash=st, batch=case.batch,
                       active=case.active, T=case.T, H=case.H, G=case.G, Dm=case.Dm,
                       N=case.N, slot_stride=case.slot_stride, P=case.P,
                       dt_softplus=case.dt_softplus)
    return out, pool, st, err


def ddtree_case(case):
    """Run the oracle tree verify on a tree case; returns (out, stash, err)."""
    return ddtree(case.x, case.A, case.B, case.C, case.dt, case.pool, case.parent_ids,
                  case.depths, dt_bias=case.dt_bias, D=case.D,
                  state_indices=case.state_indices, batch=case.batch, active=case.active,
                  T=case.T, H=case.H, G=case.G, Dm=case.Dm, N=case.N,
                  slot_stride=case.slot_stride, P=case.P, dt_softplus=case.dt_softplus)


def conv_decode_case(case, pool=None, conv_state=None):
    """Fused conv1d + decode on a conv case; returns (out, pool_after, conv_after, err)."""
    pool = case.pool.clone() if pool is None else pool
    conv = case.conv_state.clone() if conv_state is None else conv_state
    out, err = conv_decode(case.xbc, case.conv_w, case.conv_b, conv, case.width, case.A,
                           case.dt, pool, conv_strides=case.conv_strides, dt_bias=case.dt_bias,
                           D=case.D, z=case.z, state_indices=case.state_indices,
                           batch=case.batch, active=case.active, H=case.H, G=case.G,
                           Dm=case.Dm, N=case.N, slot_stride=case.slot_stride, P=case.P,
                           dt_softplus=case.dt_softplus, conv_silu=case.conv_silu)
    return out, pool, conv, err


def gdn_case(case, pool=None):
    """Gated delta-rule decode of a workloads.GDNCase; returns (out, pool_after, err)."""
    pool = case.pool.clone() if pool is None else pool
    out, err = gdn_decode(case.q, case.k, case.v, case.a, case.b, case.A_log, pool,
                          dt_bias=case.dt_bias, scale=case.scale, use_l2norm=case.use_l2norm,
                          state_indices=case.state_indices, batch=case.batch,
                          active=case.active, HK=case.HK, HV=case.HV, K=case.K, V=case.V,
                          slot_stride=case.slot_stride, P=case.P)
    return out, pool, err
