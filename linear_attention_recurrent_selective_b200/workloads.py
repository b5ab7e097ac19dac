"""Seeded synthetic inputs for the selective state update (decode, prefill, replay, tree).

This module only draws random numbers and lays them out in the shapes the
Selective State Update page (TensorRT-Edge-LLM C++ API, ``invokeSelectiveStateUpdate``,
``invokeSelectiveStateUpdatePrefill``, ``invokeSelectiveStateUpdateDDTree`` and
``MambaReplayLayerInfo``) gives for each argument. It holds no part of the recurrence: both the CUDA path and the CPU oracle
receive the same tensors from here and do all of the arithmetic themselves.

Value laws (one set for every workload):
  x, z, B, C, pool state ~ N(0, 1); dt ~ N(0, 1); dt_bias ~ N(0, 0.1);
  A = -exp(U(0, 2)); D ~ N(0, 1).
  The "slow decay" variant draws A = -exp(U(-2, 0)) and sets dt_bias = -4, so that the
  state remembers many tokens.
Every tensor is drawn in fp32 from one ``torch.Generator`` in a fixed order
(pool, x, B, C, dt, z, A, dt_bias, D, stateIndices, padding positions, lengths, tree,
conv inputs)
and then cast to its storage dtype, so both sides see the same (already rounded) values.

Draft trees (tree verify): node 0 is a root; every later node i picks its parent
uniformly among nodes 0..i-1 (a random recursive tree, expected depth about ln T), or
i-1 ("chain"); "forest" turns each later node into another root with probability 1/8;
"shuffled" relabels the nodes by a random permutation so that parents need not precede
their children. An accepted path is the root-to-node path of a uniformly drawn node,
with acceptedLengths ~ U{0..path length}.
"""

from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import torch

F32, F16, BF16 = torch.float32, torch.float16, torch.bfloat16


@dataclasses.dataclass
class SSUCase:
    """One seeded workload: shapes, flags and CPU tensors.

    Shapes (batch-major, contiguous):
      decode:  x, z [batch, H, Dm]; B, C [batch, G, N]; dt [batch, H]
      prefill / replay inputs: x, z [batch, T, H, Dm]; B, C [batch, T, G, N]; dt [batch, T, H]
      pool [P, H, Dm, N] (slot stride H*Dm*N elements unless ``slot_stride`` says more)
      A, dt_bias, D [H] fp32; state_indices [batch] int32 (None = row b uses slot b)
      context_lengths / accepted_lengths [batch] int32 (None = all T tokens)
      tree verify: parent_ids, depths [batch, T] int32 (T = tree nodes);
      accepted_node_ids [batch, T] int32 (an accepted root-to-node path, -1 beyond it)
      fused conv1d decode: xbc [batch, conv_dim] raw channels (x, B, C order; conv_dim =
      H*Dm + 2*G*N), conv_w [conv_dim, width], conv_b [conv_dim], conv_state flat pool
      with element (s, c, k) at the conv_strides (slot, channel, tap) offsets
    """

    name: str
    batch: int
    P: int
    H: int
    G: int
    Dm: int
    N: int
    T: Optional[int]          # None for the single-token decode form
    active: int
    slot_stride: int
    x: torch.Tensor
    B: torch.Tensor
    C: torch.Tensor
    dt: torch.Tensor
    A: torch.Tensor
    pool: torch.Tensor        # flat storage of P * slot_stride elements
    z: Optional[torch.Tensor] = None
    dt_bias: Optional[torch.Tensor] = None
    D: Optional[torch.Tensor] = None
    state_indices: Optional[torch.Tensor] = None
    context_lengths: Optional[torch.Tensor] = None
    accepted_lengths: Optional[torch.Tensor] = None
    dt_softplus: bool = True
    parent_ids: Optional[torch.Tensor] = None
    depths: Optional[torch.Tensor] = None
    accepted_node_ids: Optional[torch.Tensor] = None
    xbc: Optional[torch.Tensor] = None
    conv_w: Optional[torch.Tensor] = None
    conv_b: Optional[torch.Tensor] = None
    conv_state: Optional[torch.Tensor] = None
    conv_strides: Optional[tuple] = None
    width: int = 0
    conv_silu: bool = True

    @property
    def x_dtype(self):
        return self.x.dtype

    @property
    def bc_dtype(self):
        return self.B.dtype

    @property
    def state_dtype(self):
        return self.pool.dtype

    def to(self, device) -> "SSUCase":
        """Copy of the case with every tensor moved to ``device``."""
        fields = {}
        for f in dataclasses.fields(self):
            v = getattr(self, f.name)
            fields[f.name] = v.to(device) if isinstance(v, torch.Tensor) else v
        return SSUCase(**fields)


def make_case(
    name: str = "case",
    *,
    seed: int,
    batch: int,
    P: Optional[int] = None,
    H: int,
    G: int,
    Dm: int,
    N: int,
    T: Optional[int] = None,
    active: Optional[int] = None,
    x_dtype=F32,
    bc_dtype=F32,
    state_dtype=F32,
    z: bool = False,
    dt_bias: bool = True,
    D: bool = True,
    dt_softplus: bool = True,
    indices: str | Sequence[int] = "perm",
    n_pad: int = 0,
    lengths: Optional[str] = None,
    slot_pad: int = 0,
    slow_decay: bool = False,
    tree: Optional[str] = None,
    conv: int = 0,
    conv_layout: str = "ds",
    conv_pad: int = 0,
) -> SSUCase:
    """Draw one workload.

    indices: "perm" (distinct slots from a random permutation of [0, P)), "none"
      (no stateIndices: row b is slot b) or an explicit list.
    n_pad: how many of the first ``active`` rows get stateIndices = -1 (random rows).
    lengths: None, "context" (contextLengths ~ U{1..T}) or "accepted"
      (acceptedLengths ~ U{0..T}).
    slot_pad: extra elements per pool slot beyond H*Dm*N (a padded slot stride).
    tree: None, "random", "chain", "forest" or "shuffled" (draft trees of T nodes, with
      an accepted path and acceptedLengths along it).
    conv: conv1d width (0: no conv inputs); conv_layout "ds" (channel-major windows,
      [P, conv_dim, width-1]) or "sd" (tap-major, [P, width-1, conv_dim]); conv_pad: extra
      elements per conv slot.
    """
    if P is None:
        P = batch
    if active is None:
        active = batch
    g = torch.Generator().manual_seed(seed)
    slot = H * Dm * N
    stride = slot + slot_pad

    def randn(*shape):
        return torch.randn(*shape, generator=g, dtype=F32)

    pool = randn(P * stride).to(state_dtype)
    lead = (batch,) if T is None else (batch, T)
    x = randn(*lead, H, Dm).to(x_dtype)
    B = randn(*lead, G, N).to(bc_dtype)
    C = randn(*lead, G, N).to(bc_dtype)
    dt = randn(*lead, H)
    zt = randn(*lead, H, Dm).to(x_dtype) if z else None
    if slow_decay:
        A = -torch.exp(torch.rand(H, generator=g, dtype=F32) * 2.0 - 2.0)
    else:
        A = -torch.exp(torch.rand(H, generator=g, dtype=F32) * 2.0)
    if slow_decay:
        bias = torch.full((H,), -4.0, dtype=F32)
    else:
        bias = randn(H) * 0.1 if dt_bias else None
    Dv = randn(H) if D else None

    if isinstance(indices, str):
        if indices == "perm":
            si = torch.randperm(P, generator=g)[:batch].to(torch.int32)
        elif indices == "none":
            si = None
        else:
            raise ValueError(f"unknown indices mode {indices!r}")
    else:
        si = torch.tensor(list(indices), dtype=torch.int32)
    if n_pad:
        if si is None:
            raise ValueError("padding rows need stateIndices")
        rows = torch.randperm(active, generator=g)[:n_pad]
        si = si.clone()
        si[rows] = -1

    ctx = acc = None
    if lengths == "context":
        ctx = torch.randint(1, T + 1, (batch,), generator=g, dtype=torch.int32)
    elif lengths == "accepted":
        acc = torch.randint(0, T + 1, (batch,), generator=g, dtype=torch.int32)
    elif lengths is not None:
        raise ValueError(f"unknown lengths mode {lengths!r}")

    par = dep = nodes = None
    if tree is not None:
        par, dep = draw_trees(g, batch, T, tree)
        nodes, acc = draw_accepted_paths(g, par, dep)

    xbc = cw = cb = cst = strides = None
    if conv:
        cd = H * Dm + 2 * G * N
        taps = conv - 1
        cslot = cd * taps + conv_pad
        xbc = randn(batch, cd).to(x_dtype)
        cw = (randn(cd, conv) * 0.5).to(x_dtype)
        cb = (randn(cd) * 0.1).to(x_dtype)
        cst = randn(max(P * cslot, 1)).to(x_dtype)
        strides = (cslot, taps, 1) if conv_layout == "ds" else (cslot, 1, cd)
        if conv_layout not in ("ds", "sd"):
            raise ValueError(f"unknown conv layout {conv_layout!r}")

    return SSUCase(
        name=name, batch=batch, P=P, H=H, G=G, Dm=Dm, N=N, T=T, active=active,
        slot_stride=stride, x=x, B=B, C=C, dt=dt, A=A, pool=pool, z=zt,
        dt_bias=bias, D=Dv, state_indices=si, context_lengths=ctx,
        accepted_lengths=acc, dt_softplus=dt_softplus, parent_ids=par, depths=dep,
        accepted_node_ids=nodes, xbc=xbc, conv_w=cw, conv_b=cb, conv_state=cst,
        conv_strides=strides, width=conv,
    )


def tree_depths(parents: torch.Tensor) -> torch.Tensor:
    """Number of tree ancestors of every node (parents [batch, T], -1 = root)."""
    batch, T = parents.shape
    dep = torch.zeros(batch, T, dtype=torch.int32)
    for b in range(batch):
        row = parents[b].tolist()
        for i in range(T):
            k, v = 0, row[i]
            while v != -1:
                k, v = k + 1, row[v]
            dep[b, i] = k
    return dep


def draw_trees(g: torch.Generator, batch: int, T: int, mode: str):
    """Parents and depths [batch, T] int32 of one draft tree per row (see module doc)."""
    par = torch.full((batch, T), -1, dtype=torch.int32)
    for i in range(1, T):
        if mode == "chain":
            par[:, i] = i - 1
        else:
            par[:, i] = torch.randint(0, i, (batch,), generator=g, dtype=torch.int32)
    if mode == "forest":
        roots = torch.rand(batch, T, generator=g) < 0.125
        roots[:, 0] = True
        par[roots] = -1
    elif mode == "shuffled":
        for b in range(batch):
            perm = torch.randperm(T, generator=g)
            new = torch.full((T,), -1, dtype=torch.int32)
            for i in range(T):
                p = int(par[b, i])
                new[perm[i]] = -1 if p < 0 else int(perm[p])
            par[b] = new
    elif mode not in ("random", "chain"):
        raise ValueError(f"unknown tree mode {mode!r}")
    return par, tree_depths(par)


def draw_accepted_paths(g: torch.Generator, par: torch.Tensor, dep: torch.Tensor):
    """Accepted root-to-node paths [batch, T] (-1 beyond each path) and their lengths."""
    batch, T = par.shape
    nodes = torch.full((batch, T), -1, dtype=torch.int32)
    acc = torch.zeros(batch, dtype=torch.int32)
    for b in range(batch):
        v = int(torch.randint(0, T, (1,), generator=g))
        path = []
        while v != -1:
            path.append(v)
            v = int(par[b, v])
        path.reverse()
        nodes[b, :len(path)] = torch.tensor(path, dtype=torch.int32)
        acc[b] = int(torch.randint(0, len(path) + 1, (1,), generator=g))
    return nodes, acc


# The named workloads. Seeds: 0 for the tiny decode, then 1..6 in order.
CONFIGS = {
    # batch 2, pool of 4 slots, H 4, Dm 16, N 16, fp32 everything, stateIndices [2, 0]
    "tiny_decode": dict(seed=0, batch=2, P=4, H=4, G=1, Dm=16, N=16,
                        x_dtype=F32, bc_dtype=F32, state_dtype=F32, z=False,
                        indices=[2, 0]),
    # Mamba2-2.7B-like decode: batch 256 over a 512-slot pool, H 80, Dm 64, N 128
    "mamba2_decode_b256": dict(seed=1, batch=256, P=512, H=80, G=1, Dm=64, N=128,
                               x_dtype=BF16, bc_dtype=BF16, state_dtype=F32, z=True),
    # CUDA-graph decode captured at batch 128 with 96 live rows, 24 of them padding
    "padded_graph_decode": dict(seed=2, batch=128, active=96, n_pad=24, P=256, H=64,
                                G=8, Dm=64, N=128, x_dtype=F16, bc_dtype=F16,
                                state_dtype=F16, z=True),
    # multi-token prefill, contextLengths ~ U{1..512}, pool of 32 slots
    "prefill_b16_t512": dict(seed=3, batch=16, P=32, T=512, H=80, G=1, Dm=64, N=128,
                             x_dtype=BF16, bc_dtype=BF16, state_dtype=F32, z=True,
                             lengths="context"),
    # speculative replay of up to 5 drafted tokens, acceptedLengths ~ U{0..5}
    "spec_replay_b64_t5": dict(seed=4, batch=64, P=128, T=5, H=80, G=1, Dm=64, N=128,
                               x_dtype=BF16, bc_dtype=BF16, state_dtype=F32, z=True,
                               lengths="accepted"),
    # the batch-256 decode with the causal conv1d (width 4) of its xBC channels fused in
    "mamba2_conv_decode_b256": dict(seed=6, batch=256, P=512, H=80, G=1, Dm=64, N=128,
                                    x_dtype=BF16, bc_dtype=BF16, state_dtype=F32, z=True,
                                    conv=4),
    # tree verify of one 128-node draft tree per row (the verify budget), no gate
    "ddtree_b16_n128": dict(seed=5, batch=16, P=32, T=128, H=80, G=1, Dm=64, N=128,
                            x_dtype=BF16, bc_dtype=BF16, state_dtype=F32, z=False,
                            tree="random"),
}


def make_config(name: str, **overrides) -> SSUCase:
    """Draw one of the named workloads (``CONFIGS``), optionally with overrides."""
    kw = dict(CONFIGS[name])
    kw.update(overrides)
    return make_case(name, **kw)


@dataclasses.dataclass
class GDNCase:
    """One seeded gated delta-rule decode workload (FlashInfer page
    flashinfer.gdn_fused_decode_step, its recurrent core).

    q, k [batch, HK, K]; v [batch, HV, V]; a (decay input), b (beta input) [batch, HV];
    A_log, dt_bias [HV] fp32; pool: flat fp32 storage of P slots of slot_stride elements,
    a slot being [HV, V, K] (V-major, K-last); state_indices [batch] int32 (None: slot b).
    """

    name: str
    batch: int
    P: int
    HK: int
    HV: int
    K: int
    V: int
    active: int
    slot_stride: int
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    a: torch.Tensor
    b: torch.Tensor
    A_log: torch.Tensor
    dt_bias: Optional[torch.Tensor]
    pool: torch.Tensor
    state_indices: Optional[torch.Tensor]
    scale: float = 0.0            # 0: the default 1/sqrt(K)
    use_l2norm: bool = True

    def to(self, device) -> "GDNCase":
        fields = {}
        for f in dataclasses.fields(self):
            v = getattr(self, f.name)
            fields[f.name] = v.to(device) if isinstance(v, torch.Tensor) else v
        return GDNCase(**fields)


def make_gdn_case(name: str = "gdn", *, seed: int, batch: int, P: Optional[int] = None,
                  HK: int, HV: int, K: int, V: int, active: Optional[int] = None,
                  x_dtype=BF16, indices: str | Sequence[int] = "perm", n_pad: int = 0,
                  slot_pad: int = 0, dt_bias: bool = True) -> GDNCase:
    """Draw a GDN decode workload. Laws: pool ~ N(0, 0.1^2); q, k, v, a, b ~ N(0, 1);
    A_log = log(U(1, 16)); dt_bias ~ N(0, 0.5^2). Draw order: pool, q, k, v, a, b, A_log,
    dt_bias, stateIndices, padding positions."""
    P = batch if P is None else P
    active = batch if active is None else active
    g = torch.Generator().manual_seed(seed)
    stride = HV * V * K + slot_pad

    def randn(*shape):
        return torch.randn(*shape, generator=g, dtype=F32)

    pool = randn(P * stride) * 0.1
    q = randn(batch, HK, K).to(x_dtype)
    k = randn(batch, HK, K).to(x_dtype)
    v = randn(batch, HV, V).to(x_dtype)
    a = randn(batch, HV).to(x_dtype)
    b = randn(batch, HV).to(x_dtype)
    A_log = torch.log(1.0 + 15.0 * torch.rand(HV, generator=g, dtype=F32))
    bias = randn(HV) * 0.5 if dt_bias else None
    if isinstance(indices, str):
        if indices == "perm":
            si = torch.randperm(P, generator=g)[:batch].to(torch.int32)
        elif indices == "none":
            si = None
        else:
            raise ValueError(f"unknown indices mode {indices!r}")
    else:
        si = torch.tensor(list(indices), dtype=torch.int32)
    if n_pad:
        rows = torch.randperm(active, generator=g)[:n_pad]
        si = si.clone()
        si[rows] = -1
    return GDNCase(name=name, batch=batch, P=P, HK=HK, HV=HV, K=K, V=V, active=active,
                   slot_stride=stride, q=q, k=k, v=v, a=a, b=b, A_log=A_log, dt_bias=bias,
                   pool=pool, state_indices=si)


# Gated delta-rule decode at a Qwen3-Next-like geometry: 16 key heads, 32 value heads,
# 128 x 128 fp32 state per value head (2 MiB per slot), batch 256 over a 512-slot pool.
GDN_CONFIGS = {
    "gdn_decode_b256": dict(seed=7, batch=256, P=512, HK=16, HV=32, K=128, V=128,
                            x_dtype=BF16),
}


def make_gdn_config(name: str, **overrides) -> GDNCase:
    kw = dict(GDN_CONFIGS[name])
    kw.update(overrides)
    return make_gdn_case(name, **kw)
