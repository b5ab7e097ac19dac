"""GPU tests of the debug check of the row-to-slot map (ssu_check_state_indices).

FlashInfer page flashinfer.gdn_fused_decode_step, state_indices: every batch row reads and
writes its own slot and a negative index is padding, so the active rows' non-negative
indices must be distinct. The expected flags are computed here by brute force over all
pairs of rows, the definition itself."""

import pytest
import torch

from linear_attention_recurrent_selective_b200 import ssu
from linear_attention_recurrent_selective_b200.workloads import make_case

pytestmark = pytest.mark.gpu


def flags_of(idx, P, active=None):
    e = torch.zeros(1, dtype=torch.int32, device="cuda")
    ssu.ssu_check_state_indices(idx.cuda(), P, e, active_batch=active)
    torch.cuda.synchronize()
    return int(e.item())


def brute_force(idx, P, active):
    v = idx[:active].tolist()
    f = ssu.FLAG_INDEX_RANGE if any(s >= P for s in v) else 0
    live = [s for s in v if s >= 0]
    if len(set(live)) != len(live):
        f |= ssu.FLAG_DUPLICATE_INDEX
    return f


I32 = dict(dtype=torch.int32)


@pytest.mark.parametrize("idx,P,active,want", [
    ([3, -1, 0, -1, 2, -1], 4, None, 0),                      # padding may repeat
    ([3, 1, 0, 1], 4, None, ssu.FLAG_DUPLICATE_INDEX),
    ([0, 5, 1], 4, None, ssu.FLAG_INDEX_RANGE),
    ([2, 2, 7, -1], 4, None, ssu.FLAG_DUPLICATE_INDEX | ssu.FLAG_INDEX_RANGE),
    ([0, 1, 2, 0, 9], 4, 3, 0),                                # rows >= active are not looked at
    ([7], 8, None, 0),
])
def test_small_maps(idx, P, active, want):
    t = torch.tensor(idx, **I32)
    assert flags_of(t, P, active) == want == brute_force(t, P, len(idx) if active is None else active)


@pytest.mark.parametrize("n,active,plant", [(5000, 5000, True), (5000, 4321, False),
                                            (257, 257, True), (1, 1, False)])
def test_large_maps_against_brute_force(n, active, plant):
    g = torch.Generator().manual_seed(n + active)
    P = 3 * n
    idx = torch.randperm(P, generator=g)[:n].to(torch.int32)
    idx[torch.randperm(n, generator=g)[: n // 5]] = -1
    if plant and n > 1:                  # one duplicate between two far-apart live rows
        live = (idx[:active] >= 0).nonzero().flatten()
        idx[live[-1]] = idx[live[0]]
    assert flags_of(idx, P, active) == brute_force(idx, P, active)
    if plant and n > 1:
        assert flags_of(idx, P, active) == ssu.FLAG_DUPLICATE_INDEX


def test_debug_mode_rejects_duplicates_before_launching():
    case = make_case(seed=995, batch=4, P=6, H=2, G=1, Dm=16, N=32)
    d = case.to("cuda")
    idx = d.state_indices.clone()
    idx[3] = idx[1]
    pool = d.pool.clone()
    out = torch.zeros_like(d.x)
    before = ssu.set_debug_checks(True)
    try:
        with pytest.raises(ValueError, match="share a pool slot"):
            ssu.ssu_decode(d.x, d.A, d.B, d.C, d.dt, pool, out, dt_bias=d.dt_bias, D=d.D,
                           state_indices=idx, slot_stride=case.slot_stride, P=case.P)
        torch.cuda.synchronize()
        assert torch.equal(pool, d.pool)          # nothing was launched
        ssu.ssu_decode(d.x, d.A, d.B, d.C, d.dt, pool, out, dt_bias=d.dt_bias, D=d.D,
                       state_indices=d.state_indices, slot_stride=case.slot_stride, P=case.P)
    finally:
        ssu.set_debug_checks(before)
