"""GPU parity of ssu_replay (commit of accepted speculative tokens) against the oracle.

Selective State Update page (TensorRT-Edge-LLM C++ API), struct MambaReplayLayerInfo and
invokeMambaReplayReconstructBatched. The stash comes from the oracle's prefill in stash
mode, never from the CUDA path."""

import pytest
import torch

import gpu_run
from linear_attention_recurrent_selective_b200 import ssu
from linear_attention_recurrent_selective_b200.workloads import make_case, make_config
from parity import changed_slots, check_state, same_bits

pytestmark = pytest.mark.gpu

F32, F16, BF16 = torch.float32, torch.float16, torch.bfloat16


def compare_replay(orc, case, acc):
    _, _, st, _ = orc.prefill_case(case, stash=True)
    pool_o = case.pool.clone()
    err_o = orc.replay(pool_o, st, acc, state_indices=case.state_indices, batch=case.batch,
                       active=case.active, T=case.T, H=case.H, G=case.G, Dm=case.Dm,
                       N=case.N, slot_stride=case.slot_stride, P=case.P)
    pool_g, err_g = gpu_run.replay(case, st, acc)
    assert err_g == err_o
    check_state(pool_g, pool_o, case.state_dtype)
    assert changed_slots(case.pool, pool_g, case) == changed_slots(case.pool, pool_o, case)
    si = case.state_indices
    want = {int(si[b]) if si is not None else b for b in range(case.active)
            if (si is None or si[b] >= 0) and min(int(acc[b]), case.T) > 0}
    assert changed_slots(case.pool, pool_g, case) == want
    return pool_g


def test_spec_replay_b64_t5(orc):
    case = make_config("spec_replay_b64_t5")
    assert (case.accepted_lengths == 0).any()
    compare_replay(orc, case, case.accepted_lengths)


@pytest.mark.parametrize("N,sdt,Dm,H,G", [
    (8, F32, 7, 2, 1), (16, F16, 40, 4, 2), (32, BF16, 64, 2, 2), (64, F32, 33, 3, 1),
    (128, F16, 64, 4, 4), (128, F32, 100, 2, 1), (256, F32, 24, 2, 1),
])
def test_replay_shapes(orc, N, sdt, Dm, H, G):
    case = make_case(seed=300 + N + Dm, batch=6, P=10, T=4, H=H, G=G, Dm=Dm, N=N,
                     x_dtype=BF16, bc_dtype=BF16, state_dtype=sdt, z=True, active=5,
                     n_pad=1, lengths="accepted", slot_pad=4 if sdt == F32 else 8)
    acc = case.accepted_lengths.clone()
    acc[0], acc[1] = 4, 0
    compare_replay(orc, case, acc)


def test_replay_flags(orc):
    case = make_case(seed=310, batch=4, P=6, T=3, H=2, G=1, Dm=16, N=32)
    acc = torch.tensor([7, -1, 2, 3], dtype=torch.int32)
    compare_replay(orc, case, acc)
    _, _, st, _ = orc.prefill_case(case, stash=True)
    _, err = gpu_run.replay(case, st, acc)
    assert err == ssu.FLAG_ACCEPTED_RANGE | ssu.FLAG_NEGATIVE_LENGTH


def test_replay_zero_accepted_is_a_no_op(orc):
    case = make_config("spec_replay_b64_t5", batch=8, P=16)
    _, _, st, _ = orc.prefill_case(case, stash=True)
    pool_g, err = gpu_run.replay(case, st, torch.zeros(8, dtype=torch.int32))
    assert err == 0 and same_bits(pool_g, case.pool)


def test_prefill_stash_then_replay_equals_k_decodes_on_gpu():
    """GPU against GPU, fp32 state: prefill with the stash, then replay(k) gives the state
    of k decode steps bit for bit (the stash holds exactly the factors decode uses)."""
    case = make_case(seed=320, batch=6, P=12, T=5, H=4, G=2, Dm=64, N=128, x_dtype=BF16,
                     bc_dtype=BF16, z=True, slow_decay=True)
    _, pool_s, st, _ = gpu_run.prefill(case, stash=True)
    acc = torch.tensor([0, 1, 2, 3, 4, 5], dtype=torch.int32)
    pool_r, _ = gpu_run.replay(case, st, acc)
    d = case.to("cuda")
    for b in range(case.batch):
        pool = d.pool.clone()
        row = slice(b, b + 1)
        for t in range(int(acc[b])):
            out = torch.empty(d.x[row, t].shape, dtype=d.x.dtype, device="cuda")
            ssu.ssu_decode(d.x[row, t].contiguous(), d.A, d.B[row, t].contiguous(),
                           d.C[row, t].contiguous(), d.dt[row, t].contiguous(), pool, out,
                           dt_bias=d.dt_bias, D=d.D, z=d.z[row, t].contiguous(),
                           state_indices=d.state_indices[row].contiguous(),
                           slot_stride=case.slot_stride, P=case.P)
        s = int(case.state_indices[b])
        sl = slice(s * case.slot_stride, (s + 1) * case.slot_stride)
        assert same_bits(pool[sl].cpu(), pool_r[sl])
