"""GPU parity of ssu_decode (single-token selective state update) against the oracle.

Selective State Update page (TensorRT-Edge-LLM C++ API), invokeSelectiveStateUpdate;
padding contract of flashinfer.gdn_fused_decode_step (state_indices)."""

import pytest
import torch

import gpu_run
from linear_attention_recurrent_selective_b200 import ssu
from linear_attention_recurrent_selective_b200.workloads import make_case, make_config
from parity import (changed_slots, check_out, check_state, expected_decode_slots,
                    same_bits)

pytestmark = pytest.mark.gpu

F32, F16, BF16 = torch.float32, torch.float16, torch.bfloat16


def run_and_compare(orc, case):
    out_o, pool_o, err_o = orc.decode_case(case)
    out_g, pool_g, err_g = gpu_run.decode(case)
    assert err_g == err_o
    check_state(pool_g, pool_o, case.state_dtype)
    check_out(out_g, out_o, case.x_dtype)
    assert changed_slots(case.pool, pool_g, case) == changed_slots(case.pool, pool_o, case)
    assert changed_slots(case.pool, pool_g, case) <= expected_decode_slots(case)
    return out_g, pool_g


def test_tiny_decode(orc):
    case = make_config("tiny_decode")
    out, pool = run_and_compare(orc, case)
    assert changed_slots(case.pool, pool, case) == {0, 2}


def test_mamba2_decode_b256(orc):
    case = make_config("mamba2_decode_b256")
    run_and_compare(orc, case)


def test_mamba2_decode_b256_fp32_output(orc):
    # x and z widened exactly to fp32 (same values), so the output is fp32 and is checked
    # at the fp32 tolerance; B and C stay bf16.
    case = make_config("mamba2_decode_b256", batch=64, P=128)
    case.x, case.z = case.x.float(), case.z.float()
    run_and_compare(orc, case)


SHAPES = [
    # (N, state dtype, Dm, H, G, x dtype, bc dtype)
    (8, F32, 7, 4, 2, F32, F32),
    (8, F16, 33, 2, 1, F16, F16),
    (16, F32, 16, 4, 1, F32, F32),
    (16, BF16, 50, 6, 3, BF16, BF16),
    (32, F32, 70, 4, 4, BF16, F32),
    (32, F16, 5, 8, 2, F16, BF16),
    (64, F32, 65, 3, 1, F16, F16),
    (64, BF16, 128, 4, 2, BF16, BF16),
    (128, F32, 64, 8, 1, BF16, BF16),
    (128, F32, 100, 4, 2, F32, F32),
    (128, F16, 64, 8, 8, F16, F16),
    (128, BF16, 1, 4, 1, BF16, BF16),
    (256, F32, 40, 4, 2, F32, BF16),
    (256, F16, 96, 2, 1, F16, F16),
]


@pytest.mark.parametrize("N,sdt,Dm,H,G,xdt,bcdt", SHAPES)
@pytest.mark.parametrize("variant", ["full", "bare"])
def test_decode_shapes(orc, N, sdt, Dm, H, G, xdt, bcdt, variant):
    full = variant == "full"
    case = make_case(seed=100 + N + Dm, batch=6, P=11, H=H, G=G, Dm=Dm, N=N,
                     x_dtype=xdt, bc_dtype=bcdt, state_dtype=sdt, z=full, dt_bias=full,
                     D=full, dt_softplus=full, active=5, n_pad=1 if full else 0,
                     slot_pad=8 if full else 0, indices="perm" if full else "none")
    if not full:
        case.P = 6
        case.pool = case.pool[: 6 * case.slot_stride].clone()
        case.dt = case.dt.abs()      # without softplus the caller passes a positive step
    run_and_compare(orc, case)


def test_slow_decay_decode(orc):
    case = make_case(seed=5, batch=16, P=32, H=8, G=2, Dm=64, N=128, x_dtype=BF16,
                     bc_dtype=BF16, z=True, slow_decay=True)
    run_and_compare(orc, case)


def test_padded_graph_decode_under_cuda_graph(orc):
    """Captured at batch 128 with 96 live rows (24 of them padding); the graph is then
    replayed with a different set of indices written into the captured buffer."""
    case = make_config("padded_graph_decode")
    d = case.to("cuda")
    pool = d.pool.clone()
    out = torch.full_like(d.x, float("nan"))
    idx = d.state_indices.clone()

    def step():
        ssu.ssu_decode(d.x, d.A, d.B, d.C, d.dt, pool, out, dt_bias=d.dt_bias, D=d.D,
                       z=d.z, state_indices=idx, active_batch=case.active)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()                                   # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()

    for trial in range(2):
        if trial == 1:                           # new live set, new padding rows
            gen = torch.Generator().manual_seed(99)
            new = torch.randperm(case.P, generator=gen)[: case.batch].to(torch.int32)
            new[torch.randperm(case.active, generator=gen)[:24]] = -1
            case.state_indices = new
            idx.copy_(new.cuda())
        pool.copy_(d.pool)
        out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        out_o, pool_o, _ = orc.decode_case(case)
        check_state(pool.cpu(), pool_o, case.state_dtype)
        check_out(out.cpu(), out_o, case.x_dtype)
        si = case.state_indices
        for b in range(case.active):
            if si[b] < 0:
                assert torch.all(out[b].cpu() == 0)
        assert torch.isnan(out[case.active:].float()).all()
        live = {int(si[b]) for b in range(case.active) if si[b] >= 0}
        assert len(live) == 72
        assert changed_slots(case.pool, pool.cpu(), case) == live
    del g


def test_index_out_of_range_flags_and_skips(orc):
    case = make_case(seed=31, batch=4, P=6, H=4, G=1, Dm=32, N=64, indices=[1, 6, 100, 3])
    out_o, pool_o, err_o = orc.decode_case(case)
    out_g, pool_g, err_g = gpu_run.decode(case)
    assert err_g == err_o == ssu.FLAG_INDEX_RANGE
    assert torch.isnan(out_g[1:3].float()).all()
    assert changed_slots(case.pool, pool_g, case) == {1, 3}
    check_state(pool_g, pool_o, case.state_dtype)


def test_empty_batches_launch_nothing(orc):
    case = make_case(seed=32, batch=4, P=4, H=2, G=1, Dm=16, N=32, active=0)
    out_g, pool_g, err = gpu_run.decode(case)
    assert err == 0 and same_bits(pool_g, case.pool) and torch.isnan(out_g).all()
    case0 = make_case(seed=33, batch=0, P=4, H=2, G=1, Dm=16, N=32, indices="none")
    out0, pool0, _ = gpu_run.decode(case0)
    assert out0.numel() == 0 and same_bits(pool0, case0.pool)


def test_unsupported_dstate_raises():
    case = make_case(seed=34, batch=2, P=2, H=2, G=1, Dm=4, N=48).to("cuda")
    with pytest.raises(ssu.SSUError) as ei:
        ssu.ssu_decode(case.x, case.A, case.B, case.C, case.dt, case.pool,
                       torch.empty_like(case.x), slot_stride=case.slot_stride, P=case.P)
    assert ei.value.status == 4


def test_pool_view_as_4d_tensor(orc):
    # a [P, H, Dm, N] view of a padded slab: stride(0) gives the slot stride
    case = make_case(seed=35, batch=3, P=5, H=2, G=1, Dm=8, N=16, slot_pad=16, z=True)
    d = case.to("cuda")
    pool4 = d.pool.view(case.P, case.slot_stride)[:, : case.H * case.Dm * case.N]
    pool4 = pool4.view(case.P, case.H, case.Dm, case.N)
    out = torch.full_like(d.x, float("nan"))
    ssu.ssu_decode(d.x, d.A, d.B, d.C, d.dt, pool4, out, dt_bias=d.dt_bias, D=d.D, z=d.z,
                   state_indices=d.state_indices)
    out_o, pool_o, _ = orc.decode_case(case)
    check_state(d.pool.cpu(), pool_o, case.state_dtype)
    check_out(out.cpu(), out_o, case.x_dtype)
