"""Pins for the float64 CPU oracle, against things other than itself.

Each test ties the oracle to a fact the pages or the mathematics fix: the decode
formula of the Selective State Update page (TensorRT-Edge-LLM C++ API,
invokeSelectiveStateUpdate), the prefill/stash and replay contracts on the same page,
the tree verify (invokeSelectiveStateUpdateDDTree) and the accepted-node replay on the
same page, the causal conv1d update and the gated delta-rule core of flashinfer.gdn_fused_decode_step,
the padding contract of flashinfer.gdn_fused_decode_step (state_indices),
closed forms, independent vectorised formulations and the IEEE storage formats.
"""

import math

import numpy as np
import pytest
import torch

from einsum_ref import (ancestor_path, causal_conv_step, ddtree_dual, decode_dense, f64,
                        gdn_dense, prefill_dense)
from linear_attention_recurrent_selective_b200.workloads import make_case, make_config, make_gdn_case

F64 = torch.float64


def dense_state(case, pool=None):
    pool = case.pool if pool is None else pool
    P = case.P
    full = pool.view(P, case.slot_stride)[:, : case.H * case.Dm * case.N]
    return full.reshape(P, case.H, case.Dm, case.N)


def same_bits(a, b):
    """Byte identity (NaN-aware) of two tensors of one dtype."""
    return a.dtype == b.dtype and a.shape == b.shape and torch.equal(
        a.contiguous().view(torch.uint8), b.contiguous().view(torch.uint8))


def softplus(v):
    return v + math.log1p(math.exp(-v)) if v > 0 else math.log1p(math.exp(v))


# ---------------------------------------------------------------- storage formats

def test_f16_decode_all_bit_patterns(orc):
    L = orc.lib()
    bits = np.arange(65536, dtype=np.uint16)
    want = bits.view(np.float16).astype(np.float64)
    got = np.array([L.oracle_f16_to_double(int(b)) for b in bits])
    same = (got == want) | (np.isnan(got) & np.isnan(want))
    assert same.all()


def test_bf16_decode_all_bit_patterns(orc):
    L = orc.lib()
    bits = torch.arange(65536, dtype=torch.int32).to(torch.int16)
    want = bits.view(torch.bfloat16).double().numpy()
    got = np.array([L.oracle_bf16_to_double(int(b) & 0xFFFF) for b in bits])
    same = (got == want) | (np.isnan(got) & np.isnan(want))
    assert same.all()


def test_f16_encode_round_to_nearest_even(orc):
    L = orc.lib()
    rng = np.random.default_rng(0)
    vals = np.concatenate([
        rng.standard_normal(4000) * 10.0 ** rng.uniform(-9, 5, 4000),
        [0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e6, -1e6, 2.0 ** -24, 2.0 ** -25,
         3 * 2.0 ** -26, 2.0 ** -14, 1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11,
         2.0 ** -14 - 2.0 ** -25],
    ])
    with np.errstate(over="ignore"):
        want = vals.astype(np.float16).view(np.uint16)   # numpy rounds from double directly
    got = np.array([L.oracle_double_to_f16(float(v)) for v in vals], dtype=np.uint16)
    assert (got == want).all()
    # ties go to the even neighbour
    assert L.oracle_double_to_f16(1 + 2.0 ** -11) == 0x3C00
    assert L.oracle_double_to_f16(1 + 3 * 2.0 ** -11) == 0x3C02


def test_bf16_encode_round_to_nearest_even(orc):
    L = orc.lib()
    g = torch.Generator().manual_seed(1)
    v = torch.randn(4000, generator=g) * torch.exp(torch.rand(4000, generator=g) * 60 - 30)
    v = torch.cat([v, torch.tensor([0.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 3e38, 1e-40])])
    want = v.to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    got = np.array([L.oracle_double_to_bf16(float(x)) for x in v.double()], dtype=np.uint16)
    assert (got == want).all()


# ---------------------------------------------------------------- decode

@pytest.mark.parametrize("shape", [
    dict(batch=2, P=4, H=4, G=1, Dm=16, N=16),
    dict(batch=3, P=7, H=6, G=3, Dm=5, N=8),
    dict(batch=4, P=4, H=2, G=2, Dm=3, N=7),
])
@pytest.mark.parametrize("z", [False, True])
@pytest.mark.parametrize("softplus", [False, True])
def test_decode_matches_einsum(orc, shape, z, softplus):
    case = make_case(seed=11, state_dtype=F64, z=z, dt_softplus=softplus, **shape)
    idx = case.state_indices.long()
    s0 = dense_state(case)[idx].double().numpy()
    new, y = decode_dense(s0, f64(case.x), f64(case.A), f64(case.B), f64(case.C),
                          f64(case.dt), f64(case.dt_bias), f64(case.D), f64(case.z),
                          case.G, softplus)
    out, pool, err = orc.decode_case(case)
    assert err == 0
    np.testing.assert_allclose(out.numpy(), y, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dense_state(case, pool)[idx].numpy(), new, rtol=1e-12,
                               atol=1e-12)


def test_tiny_decode_config_matches_einsum(orc):
    case = make_config("tiny_decode")
    idx = case.state_indices.long()
    s0 = dense_state(case)[idx].double().numpy()
    new, y = decode_dense(s0, f64(case.x), f64(case.A), f64(case.B), f64(case.C),
                          f64(case.dt), f64(case.dt_bias), f64(case.D), None, case.G, True)
    out, pool, err = orc.decode_case(case)
    np.testing.assert_allclose(out.numpy(), y, rtol=1e-12, atol=1e-12)
    # fp32 pool: the stored state is the float64 result rounded once to fp32
    got = dense_state(case, pool)[idx]
    assert torch.equal(got, torch.from_numpy(new).float())
    # slots 1 and 3 are not indexed: byte-identical
    for s in (1, 3):
        assert torch.equal(dense_state(case, pool)[s], dense_state(case)[s])


def test_zero_dt_leaves_state_bit_identical(orc):
    # softplus off, no bias, dt = 0: decay exp(0) = 1 and the input term vanishes
    case = make_case(seed=3, batch=3, P=5, H=4, G=2, Dm=8, N=16, dt_bias=False,
                     dt_softplus=False, z=False)
    case.dt.zero_()
    out, pool, _ = orc.decode_case(case)
    assert torch.equal(pool, case.pool)
    idx = case.state_indices.long()
    S = dense_state(case)[idx].double()
    grp = torch.arange(case.H) // (case.H // case.G)
    y = torch.einsum("bhdn,bhn->bhd", S, case.C.double()[:, grp])
    y += case.D.double()[None, :, None] * case.x.double()
    np.testing.assert_allclose(out.numpy(), y.numpy(), rtol=1e-13, atol=1e-13)


def test_scalar_worked_example(orc):
    # H = Dm = N = G = 1, softplus off: dt = 0.5, A = -2 -> decay e^-1;
    # state 2, B 3, x 4, C 0.5, D 0.25, z 1:
    #   new state = 2 e^-1 + 3 * 0.5 * 4 = 6 + 2/e
    #   out = ((6 + 2/e) * 0.5 + 0.25 * 4) * silu(1),  silu(1) = 1 / (1 + e^-1)
    f = lambda v: torch.tensor(v, dtype=torch.float32)
    pool = torch.tensor([2.0], dtype=F64)
    out, err = orc.decode(f([[[4.0]]]), f([-2.0]), f([[[3.0]]]), f([[[0.5]]]), f([[0.5]]),
                          pool, D=f([0.25]), z=f([[[1.0]]]), batch=1, H=1, G=1, Dm=1, N=1,
                          dt_softplus=False)
    e = math.e
    assert pool.item() == pytest.approx(6 + 2 / e, rel=1e-15)
    assert out.item() == pytest.approx((3 + 1 / e + 1) / (1 + 1 / e), rel=1e-15)


def test_group_map_contiguous_blocks(orc):
    # H = 4, G = 2: heads 0,1 read group 0 and heads 2,3 read group 1. With B of group 1
    # zero, heads 2,3 see pure decay while heads 0,1 still get input.
    case = make_case(seed=5, batch=2, P=2, H=4, G=2, Dm=3, N=4, indices="none",
                     state_dtype=F64)
    case.B[:, 1].zero_()
    out, pool, _ = orc.decode_case(case)
    S0, S1 = dense_state(case), dense_state(case, pool)
    v = case.dt.double() + case.dt_bias.double()
    dte = torch.nn.functional.softplus(v)
    decay = torch.exp(case.A.double()[None] * dte)
    for h in (2, 3):
        np.testing.assert_allclose(S1[:, h], S0[:, h] * decay[:, h, None, None], rtol=1e-14)
    for h in (0, 1):
        assert not torch.allclose(S1[:, h], S0[:, h] * decay[:, h, None, None])


def test_padding_rows_and_inactive_rows(orc):
    # 10 rows captured, 7 active, 2 of the active rows are padding (index -1)
    case = make_case(seed=7, batch=10, P=16, H=4, G=2, Dm=8, N=16, active=7, n_pad=2,
                     z=True, x_dtype=torch.float16, bc_dtype=torch.float16,
                     state_dtype=torch.float16)
    out, pool, err = orc.decode_case(case)
    assert err == 0
    si = case.state_indices
    pad = [b for b in range(7) if si[b] < 0]
    assert len(pad) == 2
    for b in pad:
        assert torch.all(out[b] == 0)
    assert torch.isnan(out[7:]).all()               # rows >= active not written
    live = {int(si[b]) for b in range(7) if si[b] >= 0}
    for s in range(case.P):
        same = torch.equal(dense_state(case, pool)[s], dense_state(case)[s])
        assert same == (s not in live), s            # exactly the live slots change


def test_index_out_of_range_sets_flag_and_skips(orc):
    case = make_case(seed=8, batch=3, P=4, H=2, G=1, Dm=4, N=8, indices=[1, 4, 7])
    out, pool, err = orc.decode_case(case)
    assert err == 1
    assert torch.isnan(out[1:]).all()
    changed = [s for s in range(4)
               if not torch.equal(dense_state(case, pool)[s], dense_state(case)[s])]
    assert changed == [1]


def test_padded_slot_stride_untouched(orc):
    case = make_case(seed=9, batch=2, P=3, H=2, G=1, Dm=4, N=8, slot_pad=5)
    _, pool, _ = orc.decode_case(case)
    tail = lambda p: p.view(case.P, case.slot_stride)[:, case.H * case.Dm * case.N:]
    assert torch.equal(tail(pool), tail(case.pool))


def test_linearity_without_gate(orc):
    # with z absent, (state, x) -> (state', y) is linear for fixed A, B, C, dt, D
    c1 = make_case(seed=10, batch=2, H=3, G=1, Dm=4, N=6, indices="none", state_dtype=F64,
                   x_dtype=F64)
    c2 = make_case(seed=20, batch=2, H=3, G=1, Dm=4, N=6, indices="none", state_dtype=F64,
                   x_dtype=F64)
    al, be = 0.7, -1.3

    def run(pool, x):
        pool = pool.clone()
        out, _ = orc.decode(x, c1.A, c1.B, c1.C, c1.dt, pool, dt_bias=c1.dt_bias, D=c1.D,
                            batch=2, H=3, G=1, Dm=4, N=6)
        return pool, out

    p1, y1 = run(c1.pool, c1.x)
    p2, y2 = run(c2.pool, c2.x)
    p3, y3 = run(al * c1.pool + be * c2.pool, al * c1.x + be * c2.x)
    np.testing.assert_allclose(p3, al * p1 + be * p2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(y3, al * y1 + be * y2, rtol=1e-12, atol=1e-12)


def test_indices_equal_gather_run_scatter(orc):
    # Selective State Update page, invokeMambaStateGather / Scatter: running through
    # stateIndices equals gathering the rows to a dense batch, running with identity
    # indices and scattering back.
    case = make_case(seed=12, batch=5, P=9, H=4, G=2, Dm=4, N=8, z=True)
    out_idx, pool_idx, _ = orc.decode_case(case)
    idx = case.state_indices.long()
    slot = case.slot_stride
    dense = case.pool.view(case.P, slot)[idx].clone().reshape(-1)
    out_dense, _ = orc.decode(case.x, case.A, case.B, case.C, case.dt, dense,
                              dt_bias=case.dt_bias, D=case.D, z=case.z, batch=5, H=4, G=2,
                              Dm=4, N=8)
    scattered = case.pool.clone().view(case.P, slot)
    scattered[idx] = dense.view(5, slot)
    assert torch.equal(out_idx, out_dense)
    assert torch.equal(scattered.reshape(-1), pool_idx)


def test_16bit_pool_store_is_round_of_exact(orc):
    for sdt in (torch.float16, torch.bfloat16):
        case = make_case(seed=13, batch=3, P=3, H=2, G=1, Dm=8, N=16, state_dtype=sdt,
                         indices="none")
        _, pool16, _ = orc.decode_case(case)
        exact = case.pool.double()
        _, pool64 = orc.decode_case(case, pool=exact)[:2]
        assert torch.equal(pool16, pool64.to(sdt))


# ---------------------------------------------------------------- prefill

def test_prefill_matches_einsum_with_lengths(orc):
    case = make_case(seed=14, batch=4, P=6, T=7, H=4, G=2, Dm=3, N=8, z=True,
                     state_dtype=F64, lengths="context")
    case.context_lengths[0] = 7
    idx = case.state_indices.long()
    s0 = dense_state(case)[idx].numpy().copy()
    L = case.context_lengths.numpy()
    sT, y = prefill_dense(s0, f64(case.x), f64(case.A), f64(case.B), f64(case.C),
                          f64(case.dt), f64(case.dt_bias), f64(case.D), f64(case.z),
                          case.G, True, lengths=L)
    out, pool, _, err = orc.prefill_case(case)
    assert err == 0
    np.testing.assert_allclose(out.numpy(), y, rtol=1e-12, atol=1e-12)   # NaN where t >= L
    np.testing.assert_allclose(dense_state(case, pool)[idx].numpy(), sT, rtol=1e-12,
                               atol=1e-12)


def test_T_decodes_equal_one_prefill(orc):
    case = make_case(seed=15, batch=3, P=5, T=6, H=4, G=1, Dm=4, N=8, z=True,
                     state_dtype=F64, slow_decay=True)
    out_p, pool_p, _, _ = orc.prefill_case(case)
    pool_d = case.pool.clone()
    for t in range(case.T):
        out_t, _ = orc.decode(case.x[:, t].contiguous(), case.A, case.B[:, t].contiguous(),
                              case.C[:, t].contiguous(), case.dt[:, t].contiguous(), pool_d,
                              dt_bias=case.dt_bias, D=case.D, z=case.z[:, t].contiguous(),
                              state_indices=case.state_indices, batch=3, H=4, G=1, Dm=4,
                              N=8)
        assert same_bits(out_t, out_p[:, t].contiguous())
    assert torch.equal(pool_d, pool_p)


def test_pure_decay_closed_form(orc):
    # B = 0: S_T = S_0 * exp(A * sum_t dt_eff_t)
    case = make_case(seed=16, batch=2, P=2, T=9, H=3, G=1, Dm=2, N=4, indices="none",
                     state_dtype=F64, slow_decay=True)
    case.B.zero_()
    _, pool, _, _ = orc.prefill_case(case)
    for b in range(2):
        for h in range(3):
            tot = sum(softplus(float(case.dt[b, t, h]) + float(case.dt_bias[h]))
                      for t in range(case.T))
            want = dense_state(case)[b, h] * math.exp(float(case.A[h]) * tot)
            np.testing.assert_allclose(dense_state(case, pool)[b, h], want, rtol=1e-12)


def test_pure_accumulation_closed_form(orc):
    # A = 0: S_T = S_0 + sum_t B_t * dt_eff_t * x_t
    case = make_case(seed=17, batch=2, P=2, T=5, H=2, G=1, Dm=3, N=4, indices="none",
                     state_dtype=F64)
    case.A.zero_()
    _, pool, _, _ = orc.prefill_case(case)
    S0, S1 = dense_state(case), dense_state(case, pool)
    for b in range(2):
        for h in range(2):
            acc = S0[b, h].clone()
            for t in range(case.T):
                dte = softplus(float(case.dt[b, t, h]) + float(case.dt_bias[h]))
                acc += dte * torch.outer(case.x[b, t, h].double(), case.B[b, t, 0].double())
            np.testing.assert_allclose(S1[b, h], acc, rtol=1e-12, atol=1e-12)


def test_scalar_recurrence_closed_form(orc):
    # H = Dm = N = G = 1: s_t = a_t s_{t-1} + b_t, so
    # s_T = (prod_t a_t) s_0 + sum_t b_t prod_{u>t} a_u, and y_t = s_t C_t + D x_t, gated.
    case = make_case(seed=18, batch=1, P=1, T=8, H=1, G=1, Dm=1, N=1, indices="none",
                     state_dtype=F64, z=True, slow_decay=True)
    out, pool, _, _ = orc.prefill_case(case)
    A, bias, D = float(case.A[0]), float(case.dt_bias[0]), float(case.D[0])
    a, bb = [], []
    for t in range(case.T):
        dte = softplus(float(case.dt[0, t, 0]) + bias)
        a.append(math.exp(A * dte))
        bb.append(float(case.B[0, t, 0, 0]) * dte * float(case.x[0, t, 0, 0]))
    s0 = float(case.pool[0])
    sT = math.prod(a) * s0 + sum(bb[t] * math.prod(a[t + 1:]) for t in range(case.T))
    assert float(pool[0]) == pytest.approx(sT, rel=1e-13, abs=1e-14)
    s = s0
    for t in range(case.T):
        s = a[t] * s + bb[t]
        zt = float(case.z[0, t, 0, 0])
        y = (s * float(case.C[0, t, 0, 0]) + D * float(case.x[0, t, 0, 0])) * zt / (1 + math.exp(-zt))
        assert float(out[0, t, 0, 0]) == pytest.approx(y, rel=1e-13, abs=1e-14)


def test_prefill_stash_leaves_pool_and_matches_no_stash(orc):
    case = make_case(seed=19, batch=4, P=8, T=5, H=4, G=2, Dm=4, N=8, z=True,
                     x_dtype=torch.bfloat16, bc_dtype=torch.bfloat16, lengths="context")
    out_s, pool_s, st, _ = orc.prefill_case(case, stash=True)
    out_n, _, _, _ = orc.prefill_case(case)
    assert torch.equal(pool_s, case.pool)             # committed state read only
    assert same_bits(out_s, out_n)
    DA, U, Bst, DT = st
    for b in range(case.batch):
        L = int(case.context_lengths[b])
        # U and B are the inputs widened exactly; positions >= L are untouched
        assert torch.equal(U[b, :L], case.x[b, :L].float())
        assert torch.equal(Bst[b, :L], case.B[b, :L].float())
        assert torch.isnan(U[b, L:]).all() and torch.isnan(DA[b, L:]).all()
        dte = torch.nn.functional.softplus(case.dt[b, :L].double() + case.dt_bias.double())
        np.testing.assert_allclose(DT[b, :L], dte, rtol=1e-7)
        np.testing.assert_allclose(DA[b, :L], torch.exp(case.A.double() * dte), rtol=1e-7)


@pytest.mark.parametrize("k", [0, 1, 3, 5])
def test_replay_k_equals_k_decodes(orc, k):
    case = make_case(seed=21, batch=3, P=6, T=5, H=4, G=2, Dm=4, N=8, z=True,
                     state_dtype=F64)
    _, _, st, _ = orc.prefill_case(case, stash=True)
    acc = torch.full((3,), k, dtype=torch.int32)
    pool_r = case.pool.clone()
    assert orc.replay(pool_r, st, acc, state_indices=case.state_indices, batch=3, T=5, H=4,
                      G=2, Dm=4, N=8) == 0
    pool_d = case.pool.clone()
    for t in range(k):
        orc.decode(case.x[:, t].contiguous(), case.A, case.B[:, t].contiguous(),
                   case.C[:, t].contiguous(), case.dt[:, t].contiguous(), pool_d,
                   dt_bias=case.dt_bias, D=case.D, state_indices=case.state_indices,
                   batch=3, H=4, G=2, Dm=4, N=8)
    if k == 0:
        assert torch.equal(pool_r, case.pool)
    # the stash carries fp32 decay/dt: agreement to fp32 rounding of those factors
    np.testing.assert_allclose(pool_r, pool_d, rtol=1e-6, atol=1e-6)


def test_replay_rows_and_flags(orc):
    case = make_case(seed=22, batch=6, P=10, T=4, H=2, G=1, Dm=4, N=8, active=5, n_pad=1,
                     lengths="accepted")
    _, _, st, _ = orc.prefill_case(case, stash=True)
    acc = torch.tensor([4, 2, 0, 9, -1, 3], dtype=torch.int32)
    pool = case.pool.clone()
    err = orc.replay(pool, st, acc, state_indices=case.state_indices, batch=6, active=5,
                     T=4, H=2, G=1, Dm=4, N=8)
    assert err == 2 | 8
    si = case.state_indices
    touched = {int(si[b]) for b in range(5) if si[b] >= 0 and int(acc[b]) > 0}
    for s in range(case.P):
        same = torch.equal(dense_state(case, pool)[s], dense_state(case)[s])
        assert same == (s not in touched)


def test_prefill_length_flags(orc):
    case = make_case(seed=23, batch=3, P=3, T=4, H=2, G=1, Dm=2, N=4, indices="none")
    case.context_lengths = torch.tensor([9, -2, 0], dtype=torch.int32)
    out, pool, _, err = orc.prefill_case(case)
    assert err == 4 | 8
    assert not torch.isnan(out[0]).any()           # clamped to T
    assert torch.isnan(out[1:]).all()              # length <= 0: row untouched
    assert torch.equal(dense_state(case, pool)[1:], dense_state(case)[1:])


def test_clear_and_copy_slot(orc):
    pool = torch.arange(1, 4 * 6 + 1, dtype=torch.float32)
    orc.clear_slot(pool, 6 * 4, 4, 2)
    assert (pool.view(4, 6)[2] == 0).all() and (pool.view(4, 6)[[0, 1, 3]] != 0).all()
    orc.clear_slot(pool, 6 * 4, 4, -1)
    assert (pool == 0).all()
    src = torch.arange(3 * 6, dtype=torch.float32)
    dst = torch.zeros(5 * 6)
    orc.copy_slot(dst, 5, 4, src, 3, 1, 6 * 4)
    assert torch.equal(dst.view(5, 6)[4], src.view(3, 6)[1])
    assert (dst.view(5, 6)[:4] == 0).all()


def test_golden_tiny_decode_snapshot(orc):
    # Snapshot written by tests/golden/make_golden.py; changing the oracle's arithmetic
    # must regenerate it on purpose.
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_decode.txt")
    sec, vals = None, {"out": [], "state": []}
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line in vals:
            sec = line
            continue
        vals[sec].append(float(line))
    case = make_config("tiny_decode")
    out, pool, _ = orc.decode_case(case)
    assert out.reshape(-1).tolist() == vals["out"]
    assert pool.view(4, -1)[[2, 0]].reshape(-1).tolist() == vals["state"]


# ---------------------------------------------------------------- multi-layer, gather/scatter

def test_replay_layers_is_every_layer_replayed(orc):
    # Selective State Update page, invokeMambaReplayReconstructBatched: each layer replays
    # its own stash into its own pool with the shared accepted lengths and indices.
    base = make_case(seed=40, batch=4, P=7, T=3, H=2, G=1, Dm=4, N=8, lengths="accepted")
    pools, stashes = [], []
    for layer in range(3):
        c = make_case(seed=41 + layer, batch=4, P=7, T=3, H=2, G=1, Dm=4, N=8)
        c.state_indices = base.state_indices
        _, _, st, _ = orc.prefill_case(c, stash=True)
        pools.append(c.pool.clone())
        stashes.append(st)
    want = [p.clone() for p in pools]
    for p, st in zip(want, stashes):
        orc.replay(p, st, base.accepted_lengths, state_indices=base.state_indices, batch=4,
                   T=3, H=2, G=1, Dm=4, N=8)
    got = [p.clone() for p in pools]
    orc.replay_layers(got, stashes, base.accepted_lengths, state_indices=base.state_indices,
                      batch=4, T=3, H=2, G=1, Dm=4, N=8)
    for g, w in zip(got, want):
        assert same_bits(g, w)


def test_gather_and_scatter_against_indexing(orc):
    g = torch.Generator().manual_seed(42)
    pool = torch.randn(9, 6, generator=g)
    idx = torch.tensor([4, -1, 0, 8, 3], dtype=torch.int32)
    dense = torch.full((5, 6), float("nan"))
    err = orc.gather(pool, dense, 6 * 4, 9, state_indices=idx, batch=5, active=4)
    assert err == 0
    assert torch.equal(dense[0], pool[4]) and torch.equal(dense[2], pool[0])
    assert torch.equal(dense[3], pool[8])
    assert (dense[1] == 0).all()                    # padding row: zeros
    assert torch.isnan(dense[4]).all()              # row >= active untouched
    upd = torch.randn(5, 6, generator=g)
    pool2 = pool.clone()
    err = orc.scatter(upd, pool2, 6 * 4, 9, state_indices=idx, batch=5, active=4)
    want = pool.clone()
    for b in (0, 2, 3):
        want[int(idx[b])] = upd[b]
    assert err == 0 and torch.equal(pool2, want)
    bad = torch.tensor([1, 9], dtype=torch.int32)
    assert orc.gather(pool, torch.zeros(2, 6), 24, 9, state_indices=bad, batch=2) == 1


def test_indexed_decode_equals_oracle_gather_run_scatter(orc):
    case = make_case(seed=43, batch=5, P=9, H=4, G=2, Dm=4, N=8, z=True, active=4, n_pad=1)
    out_idx, pool_idx, _ = orc.decode_case(case)
    slot = case.slot_stride
    dense = torch.zeros(case.batch, slot)
    orc.gather(case.pool, dense, slot * 4, case.P, state_indices=case.state_indices,
               batch=case.batch, active=case.active)
    dense = dense.reshape(-1)
    out_d, _ = orc.decode(case.x, case.A, case.B, case.C, case.dt, dense, dt_bias=case.dt_bias,
                          D=case.D, z=case.z, batch=case.batch, active=case.active, H=4, G=2,
                          Dm=4, N=8)
    pool = case.pool.clone()
    orc.scatter(dense, pool, slot * 4, case.P, state_indices=case.state_indices,
                batch=case.batch, active=case.active)
    assert same_bits(pool, pool_idx)
    live = case.state_indices[: case.active] >= 0
    assert same_bits(out_d[: case.active][live], out_idx[: case.active][live])


def test_clear_slot_layers(orc):
    g = torch.Generator().manual_seed(44)
    rec = [torch.randn(5, 8, generator=g) + 3 for _ in range(3)]
    conv = [torch.randn(5, 2, generator=g) + 3, None, torch.randn(5, 2, generator=g) + 3]
    r2, c2 = [r.clone() for r in rec], [None if c is None else c.clone() for c in conv]
    orc.clear_slot_layers(r2, c2, 5, 3, 8 * 4, 2 * 4)
    for r, r0 in zip(r2, rec):
        assert (r[3] == 0).all() and torch.equal(r[[0, 1, 2, 4]], r0[[0, 1, 2, 4]])
    for c, c0 in zip(c2, conv):
        if c is not None:
            assert (c[3] == 0).all() and torch.equal(c[[0, 1, 2, 4]], c0[[0, 1, 2, 4]])
    orc.clear_slot_layers(r2, c2, 5, -1, 8 * 4, 2 * 4)
    assert all((r == 0).all() for r in r2) and all(c is None or (c == 0).all() for c in c2)


# ---------------------------------------------------------------- tree verify (DDTree)

def tree_case(seed, mode, **kw):
    shape = dict(batch=3, P=6, T=9, H=4, G=2, Dm=3, N=8)
    shape.update(kw)
    return make_case(seed=seed, tree=mode, **shape)


def test_ddtree_chain_equals_prefill_with_stash(orc):
    """A chain tree's path to node i is tokens 0..i: the prefill over the same inputs."""
    case = tree_case(40, "chain", x_dtype=torch.bfloat16, bc_dtype=torch.bfloat16)
    out_t, st_t, err = orc.ddtree_case(case)
    out_p, pool_p, st_p, _ = orc.prefill_case(case, stash=True)
    assert err == 0
    assert torch.equal(pool_p, case.pool)
    for a, b in zip(st_t, st_p):
        assert same_bits(a, b)
    np.testing.assert_allclose(out_t.numpy(), out_p.numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mode", ["random", "forest", "shuffled"])
def test_ddtree_matches_decodes_along_each_path(orc, mode):
    case = tree_case(41, mode, state_dtype=F64)
    out, _, err = orc.ddtree_case(case)
    assert err == 0
    idx = case.state_indices.long()
    s0 = dense_state(case)[idx].numpy()
    x, B, C, dt = f64(case.x), f64(case.B), f64(case.C), f64(case.dt)
    for r in range(case.batch):
        parents = case.parent_ids[r].tolist()
        for i in range(case.T):
            s = s0[r:r + 1].copy()
            for j in ancestor_path(parents, i):
                s, y = decode_dense(s, x[r:r + 1, j], f64(case.A), B[r:r + 1, j],
                                    C[r:r + 1, j], dt[r:r + 1, j], f64(case.dt_bias),
                                    f64(case.D), None, case.G, True)
            np.testing.assert_allclose(out[r, i].numpy(), y[0], rtol=1e-12, atol=1e-12)


def test_ddtree_matches_closed_form(orc):
    case = tree_case(42, "shuffled", T=12, slow_decay=True, state_dtype=F64)
    out, _, _ = orc.ddtree_case(case)
    idx = case.state_indices.long()
    want = ddtree_dual(dense_state(case)[idx].numpy(), f64(case.x), f64(case.A),
                       f64(case.B), f64(case.C), f64(case.dt), f64(case.dt_bias),
                       f64(case.D), case.G, True,
                       [case.parent_ids[r].tolist() for r in range(case.batch)])
    np.testing.assert_allclose(out.numpy(), want, rtol=1e-11, atol=1e-11)


def test_ddtree_leaves_pool_and_handles_padding(orc):
    case = tree_case(43, "random", batch=5, P=8, active=4, n_pad=1)
    case.state_indices[3] = 8                         # out of range: skipped, flag 1
    pool0 = case.pool.clone()
    out, st, err = orc.ddtree_case(case)
    assert err == 1
    assert torch.equal(case.pool, pool0)
    for b in range(case.batch):
        si = int(case.state_indices[b])
        if b >= case.active or si >= case.P:
            assert torch.isnan(out[b]).all() and torch.isnan(st[1][b]).all()
        elif si < 0:
            assert (out[b] == 0).all() and torch.isnan(st[1][b]).all()
        else:
            assert not torch.isnan(out[b]).any()
            assert torch.equal(st[1][b], case.x[b].float())
            assert torch.equal(st[2][b], case.B[b].float())


def test_ddtree_malformed_nodes_flagged_and_zeroed(orc):
    case = tree_case(44, "random", batch=1, T=8, indices="none", P=1)
    par = torch.tensor([[-1, 0, 1, 2, 1, 4, 5, 0]], dtype=torch.int32)
    case.parent_ids = par.clone()
    case.depths = torch.tensor([[0, 1, 2, 3, 2, 3, 4, 1]], dtype=torch.int32)
    good, _, err = orc.ddtree_case(case)
    assert err == 0
    case.depths[0, 3] = 2                             # walk does not end at the root
    case.parent_ids[0, 6] = 6                         # self-loop: 5 -> 6 -> 6 ...
    case.depths[0, 6] = 9
    case.parent_ids[0, 7] = 12                        # parent outside [0, T)
    out, _, err = orc.ddtree_case(case)
    assert err == 64
    bad = [3, 6, 7]
    assert (out[0, bad] == 0).all()
    keep = [0, 1, 2, 4, 5]
    assert same_bits(out[0, keep].contiguous(), good[0, keep].contiguous())


@pytest.mark.parametrize("mode", ["random", "shuffled"])
def test_replay_accepted_nodes_equals_decodes_along_path(orc, mode):
    case = tree_case(45, mode, state_dtype=F64)
    _, st, _ = orc.ddtree_case(case)
    pool = case.pool.clone()
    assert orc.replay(pool, st, case.accepted_lengths, state_indices=case.state_indices,
                      batch=case.batch, T=case.T, H=4, G=2, Dm=3, N=8,
                      node_ids=case.accepted_node_ids) == 0
    idx = case.state_indices.long()
    x, B, C, dt = f64(case.x), f64(case.B), f64(case.C), f64(case.dt)
    for r in range(case.batch):
        s = dense_state(case)[idx[r:r + 1]].numpy().copy()
        k = int(case.accepted_lengths[r])
        for j in case.accepted_node_ids[r, :k].tolist():
            s, _ = decode_dense(s, x[r:r + 1, j], f64(case.A), B[r:r + 1, j], C[r:r + 1, j],
                                dt[r:r + 1, j], f64(case.dt_bias), f64(case.D), None,
                                case.G, True)
        # the stash carries fp32 decay/dt factors
        np.testing.assert_allclose(dense_state(case, pool)[idx[r]].numpy(), s[0],
                                   rtol=1e-6, atol=1e-6)


def test_replay_identity_node_ids_equal_plain_replay(orc):
    case = make_case(seed=46, batch=4, P=6, T=5, H=2, G=1, Dm=4, N=8, lengths="accepted")
    _, _, st, _ = orc.prefill_case(case, stash=True)
    plain = case.pool.clone()
    orc.replay(plain, st, case.accepted_lengths, state_indices=case.state_indices, batch=4,
               T=5, H=2, G=1, Dm=4, N=8)
    ids = torch.arange(5, dtype=torch.int32).repeat(4, 1)
    by_ids = case.pool.clone()
    orc.replay(by_ids, st, case.accepted_lengths, state_indices=case.state_indices, batch=4,
               T=5, H=2, G=1, Dm=4, N=8, node_ids=ids)
    assert same_bits(plain, by_ids)


def test_replay_node_id_flags(orc):
    case = tree_case(47, "random", batch=3, P=3, indices="none")
    _, st, _ = orc.ddtree_case(case)
    ids = case.accepted_node_ids[:, :4].contiguous()  # maxAcceptLen 4
    ids[1] = torch.tensor([0, 3, 9, 2])               # 9 >= T
    ids[2] = torch.tensor([0, 1, 2, 5])
    acc = torch.tensor([2, 3, 7], dtype=torch.int32)  # 7 > maxAcceptLen: clamped to 4
    ids[0] = torch.tensor([0, 1, 99, 99])             # beyond acc: never read
    pool = case.pool.clone()
    err = orc.replay(pool, st, acc, batch=3, T=9, H=4, G=2, Dm=3, N=8, node_ids=ids)
    assert err == 2 | 64
    assert torch.equal(dense_state(case, pool)[1], dense_state(case)[1])
    assert not torch.equal(dense_state(case, pool)[0], dense_state(case)[0])
    assert not torch.equal(dense_state(case, pool)[2], dense_state(case)[2])


# ---------------------------------------------------------------- fused conv1d + decode

def conv_view(case, conv=None):
    """The conv pool as [P, conv_dim, width-1] (a strided view for either layout)."""
    conv = case.conv_state if conv is None else conv
    cd = case.H * case.Dm + 2 * case.G * case.N
    cs, cc, ck = case.conv_strides
    return conv.as_strided((case.P, cd, case.width - 1), (cs, cc, ck))


def split_xbc(case, v):
    hd, gn = case.H * case.Dm, case.G * case.N
    b = v.shape[0]
    return (v[:, :hd].reshape(b, case.H, case.Dm), v[:, hd:hd + gn].reshape(b, case.G, case.N),
            v[:, hd + gn:].reshape(b, case.G, case.N))


def test_conv_width1_identity_is_plain_decode(orc):
    case = make_case(seed=70, batch=3, P=5, H=4, G=2, Dm=3, N=8, z=True, conv=1,
                     state_dtype=F64)
    case.conv_w = torch.ones_like(case.conv_w)
    case.conv_b = None
    case.conv_silu = False
    out_c, pool_c, _, err = orc.conv_decode_case(case)
    x, B, C = split_xbc(case, case.xbc)
    out_d, err_d = orc.decode(x.contiguous(), case.A, B.contiguous(), C.contiguous(), case.dt,
                              pool_d := case.pool.clone(), dt_bias=case.dt_bias, D=case.D,
                              z=case.z, state_indices=case.state_indices, batch=3, H=4, G=2,
                              Dm=3, N=8)
    assert err == err_d == 0
    assert same_bits(out_c, out_d) and torch.equal(pool_c, pool_d)


@pytest.mark.parametrize("layout", ["ds", "sd"])
def test_conv_decode_matches_conv_then_einsum(orc, layout):
    case = make_case(seed=71, batch=4, P=6, H=4, G=2, Dm=3, N=8, z=True, conv=4,
                     conv_layout=layout, conv_pad=3, state_dtype=F64, n_pad=1)
    out, pool, conv, err = orc.conv_decode_case(case)
    assert err == 0
    idx = case.state_indices.long()
    live = idx >= 0
    st0 = conv_view(case)[idx[live]].double().numpy()
    v, shifted = causal_conv_step(st0, f64(case.xbc)[live.numpy()], f64(case.conv_w),
                                  f64(case.conv_b), True)
    x, B, C = split_xbc(case, torch.from_numpy(v))
    s_new, y = decode_dense(dense_state(case)[idx[live]].numpy(), x.numpy(), f64(case.A),
                            B.numpy(), C.numpy(), f64(case.dt)[live.numpy()], f64(case.dt_bias),
                            f64(case.D), f64(case.z)[live.numpy()], case.G, True)
    np.testing.assert_allclose(out[live].numpy(), y, rtol=1e-12, atol=1e-12)
    assert (out[~live] == 0).all()
    np.testing.assert_allclose(dense_state(case, pool)[idx[live]].numpy(), s_new, rtol=1e-12,
                               atol=1e-12)
    # the window shift is exact: new taps = old taps 1.. and the raw input
    assert torch.equal(conv_view(case, conv)[idx[live]],
                       torch.from_numpy(shifted).to(case.conv_state.dtype))
    # padding rows and unindexed slots: both pools untouched, padding of the conv slots too
    used = set(idx[live].tolist())
    for s_ in range(case.P):
        if s_ not in used:
            assert torch.equal(dense_state(case, pool)[s_], dense_state(case)[s_])
            assert torch.equal(conv_view(case, conv)[s_], conv_view(case)[s_])
    cs = case.conv_strides[0]
    pad = conv.view(case.P, cs)[:, cs - 3:]
    assert torch.equal(pad, case.conv_state.view(case.P, cs)[:, cs - 3:])


def test_conv_layouts_agree(orc):
    a = make_case(seed=72, batch=3, P=4, H=2, G=1, Dm=4, N=8, conv=3, conv_layout="ds")
    b = make_case(seed=72, batch=3, P=4, H=2, G=1, Dm=4, N=8, conv=3, conv_layout="sd")
    cd = 2 * 4 + 2 * 8
    b.conv_state = a.conv_state.view(4, cd, 2).transpose(1, 2).contiguous().view(-1)
    out_a, pool_a, conv_a, _ = orc.conv_decode_case(a)
    out_b, pool_b, conv_b, _ = orc.conv_decode_case(b)
    assert same_bits(out_a, out_b) and same_bits(pool_a, pool_b)
    assert torch.equal(conv_a.view(4, cd, 2), conv_b.view(4, 2, cd).transpose(1, 2))


def test_T_conv_decodes_equal_sequence_conv_then_prefill(orc):
    """T fused steps equal a causal conv over the whole raw sequence (from the initial
    window) followed by one T-token prefill over the conv outputs."""
    T = 5
    case = make_case(seed=73, batch=2, P=3, H=2, G=1, Dm=4, N=8, z=True, conv=4,
                     state_dtype=F64, slow_decay=True)
    g = torch.Generator().manual_seed(74)
    seq = torch.randn(2, T, case.xbc.shape[1], generator=g).to(case.xbc.dtype)
    zs = torch.randn(2, T, 2, 4, generator=g)
    dts = torch.randn(2, T, 2, generator=g)
    pool, conv = case.pool.clone(), case.conv_state.clone()
    outs = []
    for t in range(T):
        out, _ = orc.conv_decode(seq[:, t].contiguous(), case.conv_w, case.conv_b, conv,
                                 case.width, case.A, dts[:, t].contiguous(), pool,
                                 conv_strides=case.conv_strides, dt_bias=case.dt_bias,
                                 D=case.D, z=zs[:, t].contiguous(),
                                 state_indices=case.state_indices, batch=2, H=2, G=1, Dm=4,
                                 N=8)
        outs.append(out)
    idx = case.state_indices.long()
    st = conv_view(case)[idx].double().numpy()
    full = np.concatenate([st, f64(seq).transpose(0, 2, 1)], axis=2)   # [b, C, W-1+T]
    w = f64(case.conv_w)
    v = np.stack([np.einsum("bck,ck->bc", full[:, :, t:t + 4], w) for t in range(T)], 1)
    v = v + f64(case.conv_b)[None, None, :]
    v = v / (1.0 + np.exp(-v))
    hd, gn = 8, 8
    x = torch.from_numpy(v[:, :, :hd].reshape(2, T, 2, 4).copy())
    B = torch.from_numpy(v[:, :, hd:hd + gn].reshape(2, T, 1, 8).copy())
    C = torch.from_numpy(v[:, :, hd + gn:].reshape(2, T, 1, 8).copy())
    pool_p = case.pool.clone()
    out_p, _ = orc.prefill(x, case.A, B, C, dts, pool_p, dt_bias=case.dt_bias, D=case.D,
                           z=zs.double(), state_indices=case.state_indices, batch=2, T=T, H=2,
                           G=1, Dm=4, N=8)
    for t in range(T):
        np.testing.assert_allclose(outs[t].numpy(), out_p[:, t].numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(pool.numpy(), pool_p.numpy(), rtol=1e-10, atol=1e-12)
    # after T steps the window holds the last width-1 raw inputs
    assert torch.equal(conv_view(case, conv)[idx], seq[:, T - 3:].transpose(1, 2))


def test_conv_decode_index_flag(orc):
    case = make_case(seed=75, batch=2, P=2, H=2, G=1, Dm=4, N=8, conv=2, indices=[1, 2])
    out, pool, conv, err = orc.conv_decode_case(case)
    assert err == 1
    assert torch.isnan(out[1]).all()
    assert torch.equal(conv_view(case, conv)[0], conv_view(case)[0])


# ---------------------------------------------------------------- gated delta rule (GDN)

def gdn_slots(case, pool=None):
    pool = case.pool if pool is None else pool
    return pool.view(case.P, case.slot_stride)[:, :case.HV * case.V * case.K].reshape(
        case.P, case.HV, case.V, case.K)


@pytest.mark.parametrize("l2norm", [True, False])
def test_gdn_matches_einsum(orc, l2norm):
    case = make_gdn_case(seed=80, batch=4, P=6, HK=2, HV=4, K=8, V=5, n_pad=1, slot_pad=3)
    case.use_l2norm = l2norm
    case.scale = 0.3 if not l2norm else 0.0
    out, pool, err = orc.gdn_case(case)
    assert err == 0
    idx = case.state_indices.long()
    live = idx >= 0
    S0 = gdn_slots(case)[idx[live]].double().numpy()
    Sn, y = gdn_dense(S0, f64(case.q)[live.numpy()], f64(case.k)[live.numpy()],
                      f64(case.v)[live.numpy()], f64(case.a)[live.numpy()],
                      f64(case.b)[live.numpy()], f64(case.A_log), f64(case.dt_bias),
                      case.scale or case.K ** -0.5, l2norm, case.HK)
    np.testing.assert_allclose(out[live].numpy(), y, rtol=1e-12, atol=1e-12)
    assert (out[~live] == 0).all()
    np.testing.assert_allclose(gdn_slots(case, pool)[idx[live]].double().numpy(), Sn,
                               rtol=2e-7, atol=1e-12)      # one fp32 rounding of the state
    untouched = set(range(case.P)) - set(idx[live].tolist())
    for s_ in untouched:
        assert torch.equal(gdn_slots(case, pool)[s_], gdn_slots(case)[s_])
    pad = pool.view(case.P, case.slot_stride)[:, -3:]
    assert torch.equal(pad, case.pool.view(case.P, case.slot_stride)[:, -3:])


def test_gdn_delta_rule_stores_value_under_unit_key(orc):
    """No decay (alpha = 1) and beta = 1 with a one-hot key e_j: the update writes v into
    column j exactly (S k = v afterwards), leaves the other columns alone, and a query
    e_j reads v back."""
    case = make_gdn_case(seed=81, batch=2, P=2, HK=1, HV=2, K=8, V=6, indices="none",
                         x_dtype=torch.float32, dt_bias=False)
    case.use_l2norm = False
    case.scale = 1.0
    case.A_log = torch.full((2,), -100.0)
    case.b = torch.full((2, 2), 40.0)
    j = 3
    case.k = torch.zeros(2, 1, 8)
    case.k[:, :, j] = 1.0
    case.q = case.k.clone()
    out, pool, _ = orc.gdn_case(case)
    np.testing.assert_allclose(out.numpy(), case.v.double().numpy(), rtol=0, atol=1e-15)
    after, before = gdn_slots(case, pool), gdn_slots(case)
    assert torch.equal(after[..., j], case.v.float())
    others = [c for c in range(8) if c != j]
    assert torch.equal(after[..., others], before[..., others])


def test_gdn_beta_zero_is_pure_decay(orc):
    case = make_gdn_case(seed=82, batch=3, P=3, HK=2, HV=2, K=16, V=4, indices="none")
    case.b = torch.full((3, 2), -60.0).to(case.b.dtype)   # sigmoid(-60) ~ 9e-27
    out, pool, _ = orc.gdn_case(case)
    e = case.a.double() + case.dt_bias.double()
    alpha = torch.exp(-torch.exp(case.A_log.double()) * torch.nn.functional.softplus(e))
    S0 = gdn_slots(case).double()
    np.testing.assert_allclose(gdn_slots(case, pool).double().numpy(),
                               (S0 * alpha[:, :, None, None]).numpy(), rtol=1e-7, atol=1e-30)
    kq = case.q.double()
    qn = kq / torch.sqrt((kq * kq).sum(-1, keepdim=True) + 1e-6) * 16 ** -0.5
    want = torch.einsum("bhvk,bhk->bhv", S0 * alpha[:, :, None, None], qn)
    np.testing.assert_allclose(out.numpy(), want.numpy(), rtol=1e-6, atol=1e-12)


def test_gdn_value_heads_share_their_key_head(orc):
    """HV = 2 HK: value heads 2j and 2j+1 read key head j; giving them the same state,
    value and gates gives them the same output."""
    case = make_gdn_case(seed=83, batch=2, P=2, HK=2, HV=4, K=8, V=4, indices="none")
    sl = gdn_slots(case)
    sl[:, 1] = sl[:, 0]
    sl[:, 3] = sl[:, 2]
    for t in (case.v, case.a, case.b):
        t[:, 1] = t[:, 0]
        t[:, 3] = t[:, 2]
    case.A_log[1], case.A_log[3] = case.A_log[0], case.A_log[2]
    case.dt_bias[1], case.dt_bias[3] = case.dt_bias[0], case.dt_bias[2]
    out, _, _ = orc.gdn_case(case)
    assert torch.equal(out[:, 0], out[:, 1]) and torch.equal(out[:, 2], out[:, 3])
    assert not torch.equal(out[:, 0], out[:, 2])


def test_gdn_index_flag(orc):
    case = make_gdn_case(seed=84, batch=2, P=2, HK=1, HV=1, K=8, V=4, indices=[1, 2])
    out, pool, err = orc.gdn_case(case)
    assert err == 1 and torch.isnan(out[1]).all()
    assert torch.equal(gdn_slots(case, pool)[0], gdn_slots(case)[0])


# ---------------------------------------------------------------- thread count

def _run_all_forms(orc):
    """Every parallel oracle routine on a small case with padding, lengths, a padded slot
    stride, several groups, trees and out-of-range lengths; returns everything written."""
    outs = []
    c = make_case(seed=901, batch=6, P=9, T=5, H=4, G=2, Dm=12, N=16, z=True, active=5,
                  n_pad=1, lengths="context", slot_pad=4)
    c.context_lengths[1] = 9                      # clamped, flagged
    outs += list(orc.decode_case(dataclass_t0(c)))
    o, p, st, e = orc.prefill_case(c, stash=True)
    outs += [o, p, *st, e]
    o, p, _, e = orc.prefill_case(c, stash=False)
    outs += [o, p, e]
    acc = torch.tensor([3, 0, 5, 7, 1, 2], dtype=torch.int32)
    pool = c.pool.clone()
    outs += [orc.replay(pool, st, acc, state_indices=c.state_indices, batch=c.batch,
                        active=c.active, T=c.T, H=c.H, G=c.G, Dm=c.Dm, N=c.N,
                        slot_stride=c.slot_stride, P=c.P), pool]
    t = make_case(seed=902, batch=4, P=6, T=9, H=4, G=2, Dm=8, N=16, tree="forest", active=4,
                  n_pad=1)
    t.parent_ids[2, 3] = 7                        # one malformed walk
    o, st, e = orc.ddtree_case(t)
    outs += [o, *st, e]
    k = make_case(seed=903, batch=5, P=7, H=4, G=2, Dm=8, N=16, z=True, conv=4, n_pad=1)
    outs += list(orc.conv_decode_case(k))
    gd = make_gdn_case(seed=904, batch=5, P=7, HK=2, HV=4, K=16, V=8, n_pad=1)
    outs += list(orc.gdn_case(gd))
    return outs


def dataclass_t0(case):
    """Token 0 of a prefill case as a decode case (x/B/C/dt/z without the token axis)."""
    import dataclasses
    one = {f: getattr(case, f)[:, 0].contiguous() for f in ("x", "B", "C", "dt", "z")}
    return dataclasses.replace(case, T=1, **one)


def test_results_do_not_depend_on_thread_count(orc):
    """The (row, head) units run on OpenMP threads; each unit's arithmetic is sequential,
    so one thread and every host core give the same bytes."""
    before = orc.threads()
    try:
        orc.set_threads(1)
        one = _run_all_forms(orc)
        orc.set_threads(max(4, orc.host_cores()))
        many = _run_all_forms(orc)
    finally:
        orc.set_threads(before)
    assert len(one) == len(many)
    for a, b in zip(one, many):
        if isinstance(a, torch.Tensor):
            assert same_bits(a, b)
        else:
            assert a == b
