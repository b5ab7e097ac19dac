"""GPU parity of ssu_prefill (multi-token scan, optional replay stash) against the oracle.

Selective State Update page (TensorRT-Edge-LLM C++ API),
invokeSelectiveStateUpdatePrefill."""

import pytest
import torch

import gpu_run
from linear_attention_recurrent_selective_b200 import ssu
from linear_attention_recurrent_selective_b200.workloads import make_case, make_config
from parity import changed_slots, check_fp32, check_out, check_state, same_bits

pytestmark = pytest.mark.gpu

F32, F16, BF16 = torch.float32, torch.float16, torch.bfloat16


def compare_prefill(orc, case, stash):
    out_o, pool_o, st_o, err_o = orc.prefill_case(case, stash=stash)
    out_g, pool_g, st_g, err_g = gpu_run.prefill(case, stash=stash)
    assert err_g == err_o
    check_out(out_g, out_o, case.x_dtype)
    check_state(pool_g, pool_o, case.state_dtype)
    assert changed_slots(case.pool, pool_g, case) == changed_slots(case.pool, pool_o, case)
    if stash:
        assert same_bits(pool_g, case.pool)          # committed state read only
        dA_g, U_g, B_g, dt_g = st_g
        dA_o, U_o, B_o, dt_o = st_o
        assert same_bits(U_g, U_o) and same_bits(B_g, B_o)   # exact widening, same spots
        check_fp32(dA_g, dA_o)
        check_fp32(dt_g, dt_o)
    return out_g, pool_g, st_g


SHAPES = [
    # (N, state dtype, Dm, H, G, T, x dtype)
    (8, F32, 9, 4, 2, 20, F32),
    (16, F16, 16, 2, 1, 17, F16),
    (32, BF16, 33, 4, 4, 5, BF16),
    (64, F32, 70, 3, 1, 40, BF16),
    (128, F32, 64, 4, 1, 33, BF16),
    (128, F16, 40, 4, 2, 16, F16),
    (256, F32, 36, 2, 1, 18, F32),
]


@pytest.mark.parametrize("N,sdt,Dm,H,G,T,xdt", SHAPES)
@pytest.mark.parametrize("stash", [False, True])
def test_prefill_shapes(orc, N, sdt, Dm, H, G, T, xdt, stash):
    case = make_case(seed=200 + N + T, batch=5, P=9, T=T, H=H, G=G, Dm=Dm, N=N, x_dtype=xdt,
                     bc_dtype=xdt, state_dtype=sdt, z=True, active=4, n_pad=1,
                     lengths="context", slot_pad=4 if sdt == F32 else 8)
    case.context_lengths[0] = T
    compare_prefill(orc, case, stash)


def test_prefill_without_lengths_or_options(orc):
    case = make_case(seed=210, batch=3, P=3, T=24, H=4, G=2, Dm=20, N=64, indices="none",
                     z=False, dt_bias=False, D=False, dt_softplus=False)
    case.dt = case.dt.abs()          # without softplus the caller passes a positive step
    compare_prefill(orc, case, stash=False)


def test_prefill_length_edge_cases(orc):
    case = make_case(seed=211, batch=5, P=8, T=6, H=2, G=1, Dm=16, N=32, z=True,
                     lengths="context")
    case.context_lengths = torch.tensor([0, 6, 9, -3, 1], dtype=torch.int32)
    out_o, pool_o, _, err_o = orc.prefill_case(case)
    out_g, pool_g, _, err_g = gpu_run.prefill(case)
    assert err_g == err_o == ssu.FLAG_CONTEXT_RANGE | ssu.FLAG_NEGATIVE_LENGTH
    check_out(out_g, out_o, case.x_dtype)
    check_state(pool_g, pool_o, case.state_dtype)
    assert torch.isnan(out_g[0].float()).all() and torch.isnan(out_g[3].float()).all()


def test_prefill_b16_t512_every_row(orc):
    """The full multi-token prefill workload in the benchmarked launch, every row compared
    with the oracle element by element: with the replay stash the outputs, the whole
    stash and the untouched committed state; without it the outputs and every pool slot
    (the live rows' final states, all other slots byte-identical)."""
    case = make_config("prefill_b16_t512")
    assert int(case.context_lengths.min()) < case.T    # ragged lengths
    out_s, _, _ = compare_prefill(orc, case, stash=True)
    out_n, pool_n, _ = compare_prefill(orc, case, stash=False)
    assert same_bits(out_s, out_n)                  # the stash changes nothing in the outputs
    touched = {int(case.state_indices[b]) for b in range(case.batch)}
    assert changed_slots(case.pool, pool_n, case) == touched


# The chunked tensor-core form (bf16 x/z/B/C, dstate 128, dim a multiple of 8): several
# chunks of 128 tokens with ragged ends, 16-bit pools, ragged dim tiles, groups, options.
TC_SHAPES = [
    # (T, state dtype, Dm, H, G, z, stash, slow decay)
    (300, F32, 64, 3, 1, True, False, True),
    (300, F32, 64, 3, 1, True, True, True),
    (257, F16, 72, 2, 2, True, False, False),
    (129, BF16, 136, 2, 1, False, False, True),
    (128, F32, 8, 4, 4, True, True, False),
    (40, F32, 64, 4, 2, True, False, True),
]


@pytest.mark.parametrize("T,sdt,Dm,H,G,z,stash,slow", TC_SHAPES)
def test_prefill_tensor_core_form(orc, T, sdt, Dm, H, G, z, stash, slow):
    case = make_case(seed=230 + T + Dm, batch=5, P=9, T=T, H=H, G=G, Dm=Dm, N=128,
                     x_dtype=BF16, bc_dtype=BF16, state_dtype=sdt, z=z, active=4, n_pad=1,
                     lengths="context", slot_pad=4 if sdt == F32 else 8, slow_decay=slow)
    case.context_lengths[0] = T                    # one full-length row
    case.context_lengths[2] = min(T, 128)          # one that ends on a chunk boundary
    compare_prefill(orc, case, stash)


def test_prefill_tensor_core_form_options_off(orc):
    case = make_case(seed=240, batch=3, P=3, T=150, H=4, G=2, Dm=64, N=128, indices="none",
                     x_dtype=BF16, bc_dtype=BF16, z=False, dt_bias=False, D=False,
                     dt_softplus=False)
    case.dt = case.dt.abs()          # without softplus the caller passes a positive step
    compare_prefill(orc, case, stash=False)


def test_prefill_tensor_core_form_length_edge_cases(orc):
    case = make_case(seed=241, batch=6, P=8, T=140, H=2, G=1, Dm=64, N=128, x_dtype=BF16,
                     bc_dtype=BF16, z=True, lengths="context")
    case.context_lengths = torch.tensor([0, 140, 170, -3, 1, 129], dtype=torch.int32)
    out_o, pool_o, _, err_o = orc.prefill_case(case)
    out_g, pool_g, _, err_g = gpu_run.prefill(case)
    assert err_g == err_o == ssu.FLAG_CONTEXT_RANGE | ssu.FLAG_NEGATIVE_LENGTH
    check_out(out_g, out_o, case.x_dtype)
    check_state(pool_g, pool_o, case.state_dtype)
    assert torch.isnan(out_g[0].float()).all() and torch.isnan(out_g[3].float()).all()


def test_T_decodes_equal_one_prefill_on_gpu():
    """GPU against GPU: T decode steps leave the same fp32 state as one T-token prefill,
    and the same outputs up to the order of the dstate reduction. On the sequential
    (CUDA-core) form of the prefill (fp32 B and C) the state agrees bit for bit, since every
    element is computed as fma(s, dA, B * (dt * x)) in both; the chunked tensor-core form
    (bf16 B and C) sums the same terms in another order, so there it agrees within the
    fp32 tolerance."""
    for bc, exact in ((F32, True), (BF16, False)):
        case = make_case(seed=212, batch=4, P=8, T=7, H=4, G=2, Dm=64, N=128, x_dtype=BF16,
                         bc_dtype=bc, z=True, slow_decay=True)
        _decodes_equal_prefill(case, exact)


def _decodes_equal_prefill(case, exact):
    out_p, pool_p, _, _ = gpu_run.prefill(case)
    d = case.to("cuda")
    pool = d.pool.clone()
    for t in range(case.T):
        out = torch.empty(d.x[:, t].shape, dtype=d.x.dtype, device="cuda")
        ssu.ssu_decode(d.x[:, t].contiguous(), d.A, d.B[:, t].contiguous(),
                       d.C[:, t].contiguous(), d.dt[:, t].contiguous(), pool, out,
                       dt_bias=d.dt_bias, D=d.D, z=d.z[:, t].contiguous(),
                       state_indices=d.state_indices, slot_stride=case.slot_stride, P=case.P)
        o = out_p[:, t].double()
        assert ((out.cpu().double() - o).abs() <= (2.0 ** -7) * o.abs() + 1e-5).all()
    torch.cuda.synchronize()
    if exact:
        assert same_bits(pool.cpu(), pool_p)
    else:
        check_state(pool.cpu(), pool_p, torch.float32)
