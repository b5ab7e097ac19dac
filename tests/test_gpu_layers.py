"""GPU parity of the multi-layer launches and of gather/scatter against the oracle.

Selective State Update page (TensorRT-Edge-LLM C++ API): invokeMambaReplayReconstructBatched
over MambaReplayLayerInfo arrays, invokeMambaStateClear over MambaStateLayerInfo arrays,
invokeMambaStateGather / invokeMambaStateScatter. Stashes come from the oracle's prefill."""

import pytest
import torch

from linear_attention_recurrent_selective_b200 import ssu
from linear_attention_recurrent_selective_b200.workloads import make_case
from parity import check_state, same_bits

pytestmark = pytest.mark.gpu

F32, F16 = torch.float32, torch.float16


def layered(orc, n_layers, sdt=F32, **shape):
    """n_layers pools and oracle stashes sharing one batch's indices and accepted lengths."""
    base = make_case(seed=500, lengths="accepted", state_dtype=sdt, **shape)
    pools, stashes = [], []
    for layer in range(n_layers):
        c = make_case(seed=501 + layer, state_dtype=sdt, **shape)
        c.state_indices = base.state_indices
        _, _, st, _ = orc.prefill_case(c, stash=True)
        pools.append(c.pool.clone())
        stashes.append(st)
    return base, pools, stashes


@pytest.mark.parametrize("sdt", [F32, F16])
def test_replay_layers_matches_oracle(orc, sdt):
    shape = dict(batch=6, P=12, T=5, H=4, G=2, Dm=64, N=128, active=5, n_pad=1)
    base, pools, stashes = layered(orc, 3, sdt, **shape)
    acc = base.accepted_lengths.clone()
    acc[0], acc[2] = 5, 0
    want = [p.clone() for p in pools]
    orc.replay_layers(want, stashes, acc, state_indices=base.state_indices, batch=6, active=5,
                      T=5, H=4, G=2, Dm=64, N=128)
    dev_pools = [p.cuda() for p in pools]
    dev_st = [tuple(t.cuda() for t in st) for st in stashes]
    table = ssu.replay_layer_table(list(zip(dev_pools, dev_st)))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ssu.ssu_replay_layers(table, 3, dev_pools[0], dev_st[0], acc.cuda(),
                          state_indices=base.state_indices.cuda(), active_batch=5,
                          err_flags=err, slot_stride=base.slot_stride, P=base.P)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for g, w, p0 in zip(dev_pools, want, pools):
        check_state(g.cpu(), w, sdt)
        changed = (g.cpu().view(base.P, -1) != p0.view(base.P, -1)).any(1)
        assert torch.equal(changed, (w.view(base.P, -1) != p0.view(base.P, -1)).any(1))


def test_replay_layers_equal_single_replays_bitwise(orc):
    shape = dict(batch=4, P=8, T=5, H=2, G=1, Dm=64, N=128)
    base, pools, stashes = layered(orc, 2, **shape)
    single = [p.cuda() for p in pools]
    for p, st in zip(single, stashes):
        ssu.ssu_replay(p, tuple(t.cuda() for t in st), base.accepted_lengths.cuda(),
                       state_indices=base.state_indices.cuda(), slot_stride=base.slot_stride,
                       P=base.P)
    batched = [p.cuda() for p in pools]
    dev_st = [tuple(t.cuda() for t in st) for st in stashes]
    table = ssu.replay_layer_table(list(zip(batched, dev_st)))
    ssu.ssu_replay_layers(table, 2, batched[0], dev_st[0], base.accepted_lengths.cuda(),
                          state_indices=base.state_indices.cuda(),
                          slot_stride=base.slot_stride, P=base.P)
    torch.cuda.synchronize()
    for a, b in zip(single, batched):
        assert same_bits(a.cpu(), b.cpu())


def test_replay_layers_skips_and_flags_a_misaligned_layer(orc):
    shape = dict(batch=3, P=6, T=4, H=2, G=1, Dm=32, N=64)
    base, pools, stashes = layered(orc, 2, **shape)
    acc = torch.full((3,), 2, dtype=torch.int32)
    good = pools[0].cuda()
    slab = torch.zeros(pools[1].numel() + 4, dtype=torch.float32, device="cuda")
    bad = slab[1: 1 + pools[1].numel()]             # 4-byte offset: not 16-byte aligned
    bad.copy_(pools[1].cuda())
    dev_st = [tuple(t.cuda() for t in st) for st in stashes]
    table = ssu.replay_layer_table([(good, dev_st[0]), (bad, dev_st[1])])
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ssu.ssu_replay_layers(table, 2, good, dev_st[0], acc.cuda(),
                          state_indices=base.state_indices.cuda(), err_flags=err,
                          slot_stride=base.slot_stride, P=base.P)
    torch.cuda.synchronize()
    assert int(err.item()) & ssu.FLAG_LAYER
    assert same_bits(bad.cpu(), pools[1])           # skipped: untouched
    want = pools[0].clone()
    orc.replay(want, stashes[0], acc, state_indices=base.state_indices, batch=3, T=4, H=2,
               G=1, Dm=32, N=64)
    check_state(good.cpu(), want, F32)


def test_clear_slot_layers_matches_oracle(orc):
    g = torch.Generator().manual_seed(510)
    rec = [torch.randn(6, 2, 16, 32, generator=g) for _ in range(4)]
    conv = [torch.randn(6, 40, 3, generator=g).half(), None, torch.randn(6, 40, 3, generator=g).half(),
            torch.randn(6, 40, 3, generator=g).half()]
    for slot in (4, -1):
        want_r = [r.clone() for r in rec]
        want_c = [None if c is None else c.clone() for c in conv]
        orc.clear_slot_layers(want_r, want_c, 6, slot, 2 * 16 * 32 * 4, 40 * 3 * 2)
        dr = [r.cuda() for r in rec]
        dc = [None if c is None else c.cuda() for c in conv]
        table = ssu.layer_states_table(list(zip(dr, dc)))
        ssu.pool_clear_slot_layers(table, 4, 6, slot, 2 * 16 * 32 * 4, 40 * 3 * 2)
        torch.cuda.synchronize()
        for a, b in zip(dr, want_r):
            assert same_bits(a.cpu(), b)
        for a, b in zip(dc, want_c):
            assert (a is None and b is None) or same_bits(a.cpu(), b)


@pytest.mark.parametrize("slot_bytes_extra", [0, 6])
def test_gather_scatter_match_oracle(orc, slot_bytes_extra):
    # a slot of 2*16*32 halves plus a ragged byte tail in the second case
    g = torch.Generator().manual_seed(520)
    sb = 2 * 16 * 32 * 2 + slot_bytes_extra
    pool = torch.randint(0, 255, (9, sb), dtype=torch.uint8, generator=g)
    idx = torch.tensor([3, -1, 8, 0, 5, 7], dtype=torch.int32)
    dense_o = torch.full((6, sb), 7, dtype=torch.uint8)
    orc.gather(pool, dense_o, sb, 9, state_indices=idx, batch=6, active=5)
    dense_g = torch.full((6, sb), 7, dtype=torch.uint8, device="cuda")
    dpool = pool.cuda()
    ssu.pool_gather(dpool, dense_g, state_indices=idx.cuda(), active_batch=5)
    torch.cuda.synchronize()
    assert same_bits(dense_g.cpu(), dense_o)
    upd = torch.randint(0, 255, (6, sb), dtype=torch.uint8, generator=g)
    pool_o = pool.clone()
    orc.scatter(upd, pool_o, sb, 9, state_indices=idx, batch=6, active=5)
    ssu.pool_scatter(upd.cuda(), dpool, state_indices=idx.cuda(), active_batch=5)
    torch.cuda.synchronize()
    assert same_bits(dpool.cpu(), pool_o)


def test_gather_flags_out_of_range():
    pool = torch.zeros(4, 64, device="cuda")
    dense = torch.full((2, 64), 3.0, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ssu.pool_gather(pool, dense, state_indices=torch.tensor([1, 4], dtype=torch.int32,
                                                            device="cuda"), err_flags=err)
    torch.cuda.synchronize()
    assert int(err.item()) == ssu.FLAG_INDEX_RANGE
    assert (dense[0] == 0).all() and (dense[1] == 3).all()


def test_indexed_decode_equals_gather_dense_scatter_on_gpu():
    """Running the decode through stateIndices equals gathering the rows, running a dense
    batch (row b is slot b) and scattering back, bit for bit."""
    case = make_case(seed=530, batch=6, P=10, H=4, G=2, Dm=64, N=128, z=True,
                     x_dtype=torch.bfloat16, bc_dtype=torch.bfloat16)
    d = case.to("cuda")
    pool_a = d.pool.clone()
    out_a = torch.empty_like(d.x)
    ssu.ssu_decode(d.x, d.A, d.B, d.C, d.dt, pool_a, out_a, dt_bias=d.dt_bias, D=d.D, z=d.z,
                   state_indices=d.state_indices, slot_stride=case.slot_stride, P=case.P)
    pool_b = d.pool.clone().view(case.P, case.slot_stride)
    dense = torch.empty(case.batch, case.slot_stride, device="cuda")
    ssu.pool_gather(pool_b, dense, state_indices=d.state_indices)
    out_b = torch.empty_like(d.x)
    ssu.ssu_decode(d.x, d.A, d.B, d.C, d.dt, dense.view(-1), out_b, dt_bias=d.dt_bias, D=d.D,
                   z=d.z, slot_stride=case.slot_stride, P=case.batch)
    ssu.pool_scatter(dense, pool_b, state_indices=d.state_indices)
    torch.cuda.synchronize()
    assert same_bits(out_a.cpu(), out_b.cpu())
    assert same_bits(pool_a.cpu(), pool_b.reshape(-1).cpu())
