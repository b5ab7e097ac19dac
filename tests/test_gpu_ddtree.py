"""GPU parity of the tree verify (ssu_ddtree) and of the accepted-node replay.

Selective State Update page (TensorRT-Edge-LLM C++ API): invokeSelectiveStateUpdateDDTree
(every node of a draft tree from the committed state along its ancestor path, the stash
per node) and the acceptedNodeIds / maxAcceptLen form of
invokeMambaReplayReconstructBatched."""

import dataclasses

import pytest
import torch

import gpu_run
from linear_attention_recurrent_selective_b200 import ssu
from linear_attention_recurrent_selective_b200.workloads import make_case, make_config
from parity import changed_slots, check_fp32, check_out, check_state, same_bits

pytestmark = pytest.mark.gpu

F32, F16, BF16 = torch.float32, torch.float16, torch.bfloat16


def compare_ddtree(orc, case):
    out_o, st_o, err_o = orc.ddtree_case(case)
    out_g, pool_g, st_g, err_g = gpu_run.ddtree(case)
    assert err_g == err_o
    check_out(out_g, out_o, case.x_dtype)
    assert same_bits(pool_g, case.pool)              # the committed state is only read
    dA_g, U_g, B_g, dt_g = st_g
    dA_o, U_o, B_o, dt_o = st_o
    assert same_bits(U_g, U_o) and same_bits(B_g, B_o)
    check_fp32(dA_g, dA_o)
    check_fp32(dt_g, dt_o)
    return out_g, st_g


SHAPES = [
    # (N, state dtype, Dm, H, G, T, x dtype, tree)
    (8, F32, 9, 4, 2, 20, F32, "random"),
    (16, F16, 16, 2, 1, 17, F16, "shuffled"),
    (32, BF16, 33, 4, 4, 5, BF16, "forest"),
    (64, F32, 70, 3, 1, 40, BF16, "random"),
    (128, F32, 64, 4, 1, 33, BF16, "shuffled"),
    (128, F16, 40, 4, 2, 16, F16, "chain"),
    (128, F32, 130, 2, 1, 128, F32, "random"),
    (256, F32, 36, 2, 1, 18, F32, "forest"),
]


@pytest.mark.parametrize("N,sdt,Dm,H,G,T,xdt,tree", SHAPES)
def test_ddtree_shapes(orc, N, sdt, Dm, H, G, T, xdt, tree):
    case = make_case(seed=600 + N + T, batch=5, P=9, T=T, H=H, G=G, Dm=Dm, N=N,
                     x_dtype=xdt, bc_dtype=xdt, state_dtype=sdt, active=4, n_pad=1,
                     slot_pad=4 if sdt == F32 else 8, tree=tree)
    compare_ddtree(orc, case)


# bf16 B/C with dstate 64 or 128 take the tensor-core form (the state split into bf16
# pieces: three for fp32, two for fp16, one for bf16); every state and x type of it, with
# ragged dim tiles and rows whose x/out are not 16-byte aligned (Dm 33 in 16-bit types)
TC_SHAPES = [
    # (N, state dtype, Dm, H, G, T, x dtype, tree)
    (128, F32, 64, 4, 1, 57, F32, "random"),
    (64, F16, 40, 4, 2, 23, F16, "forest"),
    (128, BF16, 70, 2, 1, 128, BF16, "random"),
    (64, F32, 130, 2, 2, 128, F16, "shuffled"),
    (128, F32, 33, 3, 1, 19, BF16, "chain"),
    (64, BF16, 8, 2, 1, 9, F32, "random"),
]


@pytest.mark.parametrize("N,sdt,Dm,H,G,T,xdt,tree", TC_SHAPES)
def test_ddtree_tensor_core_types(orc, N, sdt, Dm, H, G, T, xdt, tree):
    case = make_case(seed=650 + N + T + Dm, batch=4, P=7, T=T, H=H, G=G, Dm=Dm, N=N,
                     x_dtype=xdt, bc_dtype=BF16, state_dtype=sdt, active=3, n_pad=1,
                     slot_pad=4 if sdt == F32 else 8, tree=tree)
    compare_ddtree(orc, case)


def _shifted(t):
    """A copy of t whose data starts one element past a 16-byte boundary."""
    buf = torch.empty(t.numel() + 1, dtype=t.dtype, device=t.device)
    v = buf[1:].view(t.shape)
    v.copy_(t)
    return v


# The tensor-core form moves the x tiles in and the outputs out by tensor copies when
# their rows allow it (16-byte aligned, 128 bytes of dims or more), and by plain loads and
# stores otherwise; each side decides for itself. Here one side is shifted off the
# 16-byte boundary, so the launch mixes the two ways.
@pytest.mark.parametrize("shift_x,shift_out", [(True, False), (False, True)])
def test_ddtree_tensor_core_mixed_copy_paths(orc, shift_x, shift_out):
    case = make_case(seed=656, batch=3, P=5, T=40, H=4, G=1, Dm=64, N=128, x_dtype=BF16,
                     bc_dtype=BF16, tree="random")
    out_o, st_o, err_o = orc.ddtree_case(case)
    d = gpu_run.dev(case)
    x = _shifted(d.x) if shift_x else d.x
    out = torch.full_like(d.x, float("nan"))
    if shift_out:
        out = _shifted(out)
    st = gpu_run.new_stash(case)
    e = torch.zeros(1, dtype=torch.int32, device="cuda")
    pool = d.pool.clone()
    ssu.ssu_ddtree(x, d.A, d.B, d.C, d.dt, pool, out, d.parent_ids, d.depths, st,
                   dt_bias=d.dt_bias, D=d.D, state_indices=d.state_indices,
                   active_batch=case.active, dt_softplus=case.dt_softplus, err_flags=e,
                   slot_stride=case.slot_stride, P=case.P)
    torch.cuda.synchronize()
    assert int(e.item()) == err_o
    check_out(out.cpu(), out_o, BF16)
    assert same_bits(pool.cpu(), case.pool)
    assert same_bits(st[1].cpu(), st_o[1]) and same_bits(st[2].cpu(), st_o[2])


def test_ddtree_tensor_core_single_x_buffer(orc):
    # fp32 x at 128 nodes leaves room for one x tile only: the next item's tile is then
    # fetched after the item's closing barrier, behind its output store
    case = make_case(seed=657, batch=3, P=5, T=128, H=3, G=1, Dm=64, N=128, x_dtype=F32,
                     bc_dtype=BF16, tree="random")
    compare_ddtree(orc, case)


@pytest.mark.parametrize("H,G,Dm", [(2, 1, 16), (4, 2, 80), (3, 3, 64)])
def test_ddtree_more_rows_than_ctas(orc, H, G, Dm):
    """160 rows over at most 148 CTAs: contiguous item ranges that cross rows, so a CTA
    builds several rows' tables and a row's heads (and their B stash shares, by group and
    over several dim tiles) are split between CTAs; some rows are padding."""
    case = make_case(seed=660 + H + Dm, batch=160, P=170, T=6, H=H, G=G, Dm=Dm, N=64,
                     x_dtype=BF16, bc_dtype=BF16, tree="random", n_pad=3)
    compare_ddtree(orc, case)


@pytest.mark.parametrize("T", [1, 2, 31, 128])
def test_ddtree_node_counts(orc, T):
    case = make_case(seed=610 + T, batch=3, P=4, T=T, H=2, G=1, Dm=64, N=128,
                     x_dtype=BF16, bc_dtype=BF16, tree="random", slow_decay=True)
    compare_ddtree(orc, case)


@pytest.mark.parametrize("bcdt,N", [(F32, 32), (BF16, 64)])   # CUDA-core and tensor-core forms
def test_ddtree_options_off(orc, bcdt, N):
    case = make_case(seed=620, batch=3, P=5, T=12, H=2, G=2, Dm=24, N=N, dt_bias=False,
                     D=False, dt_softplus=False, tree="random", indices="none",
                     x_dtype=bcdt, bc_dtype=bcdt)
    case.dt = case.dt.abs()                          # softplus off: keep dt_eff >= 0
    compare_ddtree(orc, case)


@pytest.mark.parametrize("bcdt", [F32, BF16])     # bf16 B/C: the tensor-core form, fp32 out
def test_ddtree_chain_matches_prefill_with_stash(bcdt):
    """A chain tree evaluates the prefill's token sequence: same stash bits, outputs
    within the fp32 output tolerance of each other (different summation orders)."""
    case = make_case(seed=630, batch=4, P=6, T=24, H=4, G=1, Dm=64, N=128, tree="chain",
                     bc_dtype=bcdt)
    out_t, _, st_t, err = gpu_run.ddtree(case)
    out_p, _, st_p, _ = gpu_run.prefill(case, stash=True)
    assert err == 0
    for a, b in zip(st_t, st_p):
        assert same_bits(a, b)
    check_fp32(out_t, out_p.double(), tol=2e-5)


@pytest.mark.parametrize("bcdt", [F32, BF16])     # the CUDA-core and tensor-core forms
def test_ddtree_malformed_nodes_and_bad_index(orc, bcdt):
    case = make_case(seed=640, batch=4, P=6, T=10, H=2, G=1, Dm=16, N=64, tree="random",
                     x_dtype=bcdt, bc_dtype=bcdt)
    case.depths[0, 3] += 1                           # walk runs past the root
    case.parent_ids[1, 5] = 10                       # parent outside [0, T)
    case.parent_ids[1, 7] = 7                        # self loop
    case.depths[1, 7] = 4
    case.state_indices[2] = case.P                   # index out of range: row skipped
    out_g, _, _, err_g = gpu_run.ddtree(case)
    out_o, _, err_o = orc.ddtree_case(case)
    assert err_g == err_o == ssu.FLAG_TREE | ssu.FLAG_INDEX_RANGE
    check_out(out_g, out_o, case.x_dtype)
    assert torch.isnan(out_g[2]).all()               # skipped row: nothing written
    assert (out_g[0, 3] == 0).all() and (out_g[1, 5] == 0).all()


def test_ddtree_headline_workload_every_row(orc):
    """The 16 x 128-node workload in its benchmarked launch, every row compared with the
    oracle: every node's outputs and the whole stash; the pool is only read. Then the
    accepted root-to-node paths replayed from each side's stash."""
    case = make_config("ddtree_b16_n128")
    out_g, pool_g, st_g, err_g = gpu_run.ddtree(case)
    out_o, st_o, err_o = orc.ddtree_case(case)
    assert err_g == err_o == 0
    assert same_bits(pool_g, case.pool)
    check_out(out_g, out_o, case.x_dtype)
    assert same_bits(st_g[1], st_o[1]) and same_bits(st_g[2], st_o[2])   # U, B widened
    check_fp32(st_g[0], st_o[0])
    check_fp32(st_g[3], st_o[3])
    want = case.pool.clone()
    err_o = orc.replay(want, st_o, case.accepted_lengths, state_indices=case.state_indices,
                       batch=case.batch, active=case.active, T=case.T, H=case.H, G=case.G,
                       Dm=case.Dm, N=case.N, slot_stride=case.slot_stride, P=case.P,
                       node_ids=case.accepted_node_ids)
    pool_r, err_r = gpu_run.replay(case, st_g, case.accepted_lengths,
                                   node_ids=case.accepted_node_ids)
    assert err_r == err_o == 0
    check_state(pool_r, want, case.state_dtype)
    assert changed_slots(case.pool, pool_r, case) == changed_slots(case.pool, want, case)


# ---------------------------------------------------------------- accepted-node replay

@pytest.mark.parametrize("sdt", [F32, BF16])
def test_replay_accepted_nodes_matches_oracle(orc, sdt):
    case = make_case(seed=650, batch=6, P=10, T=40, H=4, G=2, Dm=64, N=128, state_dtype=sdt,
                     active=5, n_pad=1, tree="shuffled")
    _, st_o, _ = orc.ddtree_case(case)
    want = case.pool.clone()
    err_o = orc.replay(want, st_o, case.accepted_lengths, state_indices=case.state_indices,
                       batch=6, active=5, T=40, H=4, G=2, Dm=64, N=128,
                       node_ids=case.accepted_node_ids)
    _, _, st_g, _ = gpu_run.ddtree(case)
    pool_g, err_g = gpu_run.replay(case, st_g, case.accepted_lengths,
                                   node_ids=case.accepted_node_ids)
    assert err_g == err_o == 0
    check_state(pool_g, want, sdt)
    changed = (pool_g.view(case.P, -1) != case.pool.view(case.P, -1)).any(1)
    assert torch.equal(changed, (want.view(case.P, -1) != case.pool.view(case.P, -1)).any(1))


def test_replay_accepted_path_equals_decodes_along_it():
    """fp32 pool: replaying the accepted path from the tree stash gives the state of one
    decode step per accepted node, bit for bit (same factors, same association)."""
    case = make_case(seed=660, batch=4, P=6, T=30, H=2, G=1, Dm=64, N=128, tree="random")
    case.accepted_lengths = torch.tensor([3, 1, 0, 5], dtype=torch.int32)
    for r in range(4):                               # paths long enough for the counts
        par, node, path = case.parent_ids[r].tolist(), 29, []
        while node != -1:
            path.append(node)
            node = par[node]
        path = path[::-1][:5]
        case.accepted_lengths[r] = min(int(case.accepted_lengths[r]), len(path))
        case.accepted_node_ids[r] = -1
        case.accepted_node_ids[r, :len(path)] = torch.tensor(path, dtype=torch.int32)
    _, _, st_g, _ = gpu_run.ddtree(case)
    pool_r, err = gpu_run.replay(case, st_g, case.accepted_lengths,
                                 node_ids=case.accepted_node_ids)
    assert err == 0
    pool_d = case.pool.clone().cuda()
    d = case.to("cuda")
    for r in range(4):
        for t in range(int(case.accepted_lengths[r])):
            j = int(case.accepted_node_ids[r, t])
            out = torch.empty(1, 2, 64, device="cuda")
            ssu.ssu_decode(d.x[r:r + 1, j].contiguous(), d.A, d.B[r:r + 1, j].contiguous(),
                           d.C[r:r + 1, j].contiguous(), d.dt[r:r + 1, j].contiguous(), pool_d,
                           out, dt_bias=d.dt_bias, D=d.D,
                           state_indices=d.state_indices[r:r + 1].contiguous(),
                           slot_stride=case.slot_stride, P=case.P)
    torch.cuda.synchronize()
    assert same_bits(pool_r, pool_d.cpu())


def test_replay_node_id_flags(orc):
    case = make_case(seed=670, batch=3, P=3, T=9, H=2, G=1, Dm=32, N=64, tree="random",
                     indices="none")
    _, _, st_g, _ = gpu_run.ddtree(case)
    _, st_o, _ = orc.ddtree_case(case)
    ids = torch.tensor([[0, 1, 99, 99], [0, 3, 9, 2], [0, 1, 2, 5]], dtype=torch.int32)
    acc = torch.tensor([2, 3, 7], dtype=torch.int32)    # 7 > maxAcceptLen 4: clamped
    pool_g, err_g = gpu_run.replay(case, st_g, acc, node_ids=ids)
    want = case.pool.clone()
    err_o = orc.replay(want, st_o, acc, batch=3, T=9, H=2, G=1, Dm=32, N=64, node_ids=ids)
    assert err_g == err_o == ssu.FLAG_ACCEPTED_RANGE | ssu.FLAG_TREE
    check_state(pool_g, want, F32)
    assert same_bits(pool_g.view(3, -1)[1], case.pool.view(3, -1)[1])   # id 9 >= T


def test_replay_layers_with_accepted_nodes(orc):
    case = make_case(seed=680, batch=3, P=5, T=12, H=2, G=1, Dm=32, N=64, tree="random")
    pools, stashes_g, stashes_o = [], [], []
    for layer in range(2):
        c = dataclasses.replace(case, pool=make_case(seed=681 + layer, batch=3, P=5, H=2, G=1,
                                                     Dm=32, N=64).pool)
        _, _, st, _ = gpu_run.ddtree(c)
        pools.append(c.pool.clone())
        stashes_g.append(st)
        stashes_o.append(orc.ddtree_case(c)[1])
    want = [p.clone() for p in pools]
    orc.replay_layers(want, stashes_o, case.accepted_lengths, state_indices=case.state_indices,
                      batch=3, T=12, H=2, G=1, Dm=32, N=64, node_ids=case.accepted_node_ids)
    dev_pools = [p.cuda() for p in pools]
    dev_st = [tuple(t.cuda() for t in st) for st in stashes_g]
    table = ssu.replay_layer_table(list(zip(dev_pools, dev_st)))
    ssu.ssu_replay_layers(table, 2, dev_pools[0], dev_st[0], case.accepted_lengths.cuda(),
                          state_indices=case.state_indices.cuda(), slot_stride=case.slot_stride,
                          P=case.P, accepted_node_ids=case.accepted_node_ids.cuda())
    torch.cuda.synchronize()
    for g, w in zip(dev_pools, want):
        check_state(g.cpu(), w, F32)


def test_ddtree_limits():
    case = make_case(seed=690, batch=1, P=1, T=128, H=1, G=1, Dm=8, N=256, tree="random")
    with pytest.raises(ssu.SSUError) as e:
        gpu_run.ddtree(case)
    assert e.value.status == 4                       # tables exceed shared memory
    empty = make_case(seed=691, batch=2, P=2, T=4, H=1, G=1, Dm=8, N=16, tree="chain",
                      active=0)
    out, _, _, err = gpu_run.ddtree(empty)
    assert err == 0 and torch.isnan(out).all()
