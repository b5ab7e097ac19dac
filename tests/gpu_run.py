"""Run a workloads.SSUCase through the CUDA library (via the C-ABI binding) and return
host copies of what it wrote. Outputs and stash buffers start as NaN so that positions
the kernels must not write stay recognisable."""

import torch

from linear_attention_recurrent_selective_b200 import ssu

NAN = float("nan")


def dev(case):
    return case.to("cuda")


def decode(case, pool=None, err=True, out=None, stream=None):
    d = dev(case)
    pool = d.pool.clone() if pool is None else pool
    out = torch.full_like(d.x, NAN) if out is None else out
    e = torch.zeros(1, dtype=torch.int32, device="cuda") if err else None
    ssu.ssu_decode(d.x, d.A, d.B, d.C, d.dt, pool, out, dt_bias=d.dt_bias, D=d.D, z=d.z,
                   state_indices=d.state_indices, active_batch=case.active,
                   dt_softplus=case.dt_softplus, err_flags=e, slot_stride=case.slot_stride,
                   P=case.P, stream=stream)
    torch.cuda.synchronize()
    return out.cpu(), pool.cpu(), (int(e.item()) if err else None)


def new_stash(case, fill=NAN):
    b, T, H, G, Dm, N = case.batch, case.T, case.H, case.G, case.Dm, case.N
    f = dict(dtype=torch.float32, device="cuda")
    return (torch.full((b, T, H), fill, **f), torch.full((b, T, H, Dm), fill, **f),
            torch.full((b, T, G, N), fill, **f), torch.full((b, T, H), fill, **f))


def prefill(case, pool=None, stash=False, err=True):
    d = dev(case)
    pool = d.pool.clone() if pool is None else pool
    out = torch.full_like(d.x, NAN)
    st = new_stash(case) if stash else None
    e = torch.zeros(1, dtype=torch.int32, device="cuda") if err else None
    ssu.ssu_prefill(d.x, d.A, d.B, d.C, d.dt, pool, out, dt_bias=d.dt_bias, D=d.D, z=d.z,
                    state_indices=d.state_indices, context_lengths=d.context_lengths,
                    stash=st, active_batch=case.active, dt_softplus=case.dt_softplus,
                    err_flags=e, slot_stride=case.slot_stride, P=case.P)
    torch.cuda.synchronize()
    st_cpu = tuple(t.cpu() for t in st) if st is not None else None
    return out.cpu(), pool.cpu(), st_cpu, (int(e.item()) if err else None)


def replay(case, stash, accepted, pool=None, err=True, node_ids=None):
    d = dev(case)
    pool = d.pool.clone() if pool is None else pool
    st = tuple(t.cuda() for t in stash)
    e = torch.zeros(1, dtype=torch.int32, device="cuda") if err else None
    ssu.ssu_replay(pool, st, accepted.cuda(), state_indices=d.state_indices,
                   active_batch=case.active, err_flags=e, slot_stride=case.slot_stride,
                   P=case.P, accepted_node_ids=None if node_ids is None else node_ids.cuda())
    torch.cuda.synchronize()
    return pool.cpu(), (int(e.item()) if err else None)


def ddtree(case, pool=None, err=True):
    """Tree verify of a tree case; returns (out, pool after, stash, err) on the host."""
    d = dev(case)
    pool = d.pool.clone() if pool is None else pool
    out = torch.full_like(d.x, NAN)
    st = new_stash(case)
    e = torch.zeros(1, dtype=torch.int32, device="cuda") if err else None
    ssu.ssu_ddtree(d.x, d.A, d.B, d.C, d.dt, pool, out, d.parent_ids, d.depths, st,
                   dt_bias=d.dt_bias, D=d.D, state_indices=d.state_indices,
                   active_batch=case.active, dt_softplus=case.dt_softplus, err_flags=e,
                   slot_stride=case.slot_stride, P=case.P)
    torch.cuda.synchronize()
    return out.cpu(), pool.cpu(), tuple(t.cpu() for t in st), (int(e.item()) if err else None)


def conv_decode(case, pool=None, conv=None, err=True, stream=None):
    """Fused conv1d + decode of a conv case; returns (out, pool, conv pool, err) on the host."""
    d = dev(case)
    pool = d.pool.clone() if pool is None else pool
    conv = d.conv_state.clone() if conv is None else conv
    out = torch.full((case.batch, case.H, case.Dm), NAN, dtype=case.xbc.dtype, device="cuda")
    e = torch.zeros(1, dtype=torch.int32, device="cuda") if err else None
    ssu.ssu_conv_decode(d.xbc, d.conv_w, conv, d.A, d.dt, pool, out, width=case.width,
                        conv_strides=case.conv_strides, nheads=case.H, ngroups=case.G,
                        dim=case.Dm, conv_bias=d.conv_b, conv_silu=case.conv_silu,
                        dt_bias=d.dt_bias, D=d.D, z=d.z, state_indices=d.state_indices,
                        active_batch=case.active, dt_softplus=case.dt_softplus, err_flags=e,
                        slot_stride=case.slot_stride, P=case.P, stream=stream)
    torch.cuda.synchronize()
    return out.cpu(), pool.cpu(), conv.cpu(), (int(e.item()) if err else None)


def gdn(case, pool=None, err=True):
    """Gated delta-rule decode of a GDNCase; returns (out, pool, err) on the host."""
    d = case.to("cuda")
    pool = d.pool.clone() if pool is None else pool
    out = torch.full((case.batch, case.HV, case.V), NAN, dtype=case.q.dtype, device="cuda")
    e = torch.zeros(1, dtype=torch.int32, device="cuda") if err else None
    ssu.gdn_decode(d.q, d.k, d.v, d.a, d.b, d.A_log, pool, out, dt_bias=d.dt_bias,
                   scale=case.scale, use_qk_l2norm=case.use_l2norm,
                   state_indices=d.state_indices, active_batch=case.active, err_flags=e,
                   slot_stride=case.slot_stride, P=case.P)
    torch.cuda.synchronize()
    return out.cpu(), pool.cpu(), (int(e.item()) if err else None)
