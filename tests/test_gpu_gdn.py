"""GPU parity of gdn_decode (gated delta-rule decode core over a paged fp32 pool).

FlashInfer page flashinfer.gdn_fused_decode_step: the recurrent core with qk L2 norm,
the A_log / dt_bias decay gate, the sigmoid beta gate and the state_indices padding
contract."""

import dataclasses

import pytest
import torch

import gpu_run
from linear_attention_recurrent_selective_b200 import ssu
from linear_attention_recurrent_selective_b200.workloads import make_gdn_case, make_gdn_config
from parity import check_out, check_state, same_bits

pytestmark = pytest.mark.gpu

F32, F16, BF16 = torch.float32, torch.float16, torch.bfloat16


def slots(case, pool):
    return pool.view(case.P, case.slot_stride)


def compare_gdn(orc, case):
    out_o, pool_o, err_o = orc.gdn_case(case)
    out_g, pool_g, err_g = gpu_run.gdn(case)
    assert err_g == err_o
    check_out(out_g, out_o, case.q.dtype)
    check_state(pool_g, pool_o, F32)
    changed_g = (slots(case, pool_g) != slots(case, case.pool)).any(1)
    changed_o = (slots(case, pool_o) != slots(case, case.pool)).any(1)
    assert torch.equal(changed_g, changed_o)
    return out_g, pool_g


SHAPES = [
    # (K, V, HK, HV, x dtype)
    (8, 9, 1, 2, F32),
    (16, 16, 2, 2, F16),
    (32, 33, 2, 4, BF16),
    (64, 70, 1, 3, BF16),
    (128, 128, 2, 4, BF16),
    (128, 40, 4, 4, F16),
    (256, 36, 1, 2, F32),
]


@pytest.mark.parametrize("K,V,HK,HV,xdt", SHAPES)
def test_gdn_shapes(orc, K, V, HK, HV, xdt):
    case = make_gdn_case(seed=800 + K + V, batch=6, P=10, HK=HK, HV=HV, K=K, V=V, x_dtype=xdt,
                         active=5, n_pad=1, slot_pad=4)
    compare_gdn(orc, case)


def test_gdn_options(orc):
    case = make_gdn_case(seed=820, batch=3, P=4, HK=2, HV=4, K=64, V=32, indices="none",
                         dt_bias=False)
    case.use_l2norm = False
    case.scale = 0.25
    compare_gdn(orc, case)


def test_gdn_index_flag_and_padding(orc):
    case = make_gdn_case(seed=830, batch=4, P=5, HK=1, HV=2, K=128, V=64,
                         indices=[3, -1, 5, 0])
    out_g, pool_g, err = gpu_run.gdn(case)
    out_o, pool_o, err_o = orc.gdn_case(case)
    assert err == err_o == ssu.FLAG_INDEX_RANGE
    check_out(out_g, out_o, case.q.dtype)
    assert (out_g[1] == 0).all() and torch.isnan(out_g[2]).all()


def test_gdn_headline_workload_every_row(orc):
    """The batch-256 GDN workload in its benchmarked launch, every row and value head
    compared with the oracle: outputs and the whole pool."""
    case = make_gdn_config("gdn_decode_b256")
    out_g, pool_g, err = gpu_run.gdn(case)
    out_o, pool_o, err_o = orc.gdn_case(case)
    assert err == err_o == 0
    check_out(out_g, out_o, case.q.dtype)
    check_state(pool_g, pool_o, F32)
    live = {int(s) for s in case.state_indices.tolist()}
    for s in range(case.P):
        if s not in live:
            assert same_bits(slots(case, pool_g)[s], slots(case, case.pool)[s])


def test_gdn_two_steps_compose(orc):
    """Two GPU steps on one pool equal the oracle's two steps."""
    case = make_gdn_case(seed=840, batch=3, P=4, HK=1, HV=2, K=128, V=64)
    step2 = make_gdn_case(seed=841, batch=3, P=4, HK=1, HV=2, K=128, V=64)
    _, pool_g, _ = gpu_run.gdn(case)
    step2.pool = pool_g
    step2.state_indices = case.state_indices
    out_g, pool_g2, _ = gpu_run.gdn(step2)
    _, pool_o, _ = orc.gdn_case(case)
    s2 = dataclasses.replace(step2, pool=pool_o)
    out_o, pool_o2, _ = orc.gdn_case(s2)
    check_out(out_g, out_o, case.q.dtype)
    check_state(pool_g2, pool_o2, F32)
