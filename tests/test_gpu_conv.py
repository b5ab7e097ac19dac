"""GPU parity of ssu_conv_decode (causal conv1d window update fused with the decode).

Selective State Update page (TensorRT-Edge-LLM C++ API): MambaStateLayerInfo (convState
beside recurrentState) and invokeSelectiveStateUpdate; the causal conv1d update of the
FlashInfer page flashinfer.gdn_fused_decode_step."""

import pytest
import torch

import gpu_run
from linear_attention_recurrent_selective_b200 import ssu
from linear_attention_recurrent_selective_b200.workloads import make_case, make_config
from parity import changed_slots, check_out, check_state, expected_decode_slots, same_bits

pytestmark = pytest.mark.gpu

F32, F16, BF16 = torch.float32, torch.float16, torch.bfloat16


def compare_conv(orc, case):
    out_o, pool_o, conv_o, err_o = orc.conv_decode_case(case)
    out_g, pool_g, conv_g, err_g = gpu_run.conv_decode(case)
    assert err_g == err_o
    check_out(out_g, out_o, case.x_dtype)
    check_state(pool_g, pool_o, case.state_dtype)
    assert changed_slots(case.pool, pool_g, case) == changed_slots(case.pool, pool_o, case)
    assert same_bits(conv_g, conv_o)             # the window shift is a copy
    return out_g, pool_g, conv_g


SHAPES = [
    # (N, state dtype, Dm, H, G, x dtype, width, layout)
    (8, F32, 9, 4, 2, F32, 4, "ds"),
    (16, F16, 16, 2, 1, F16, 2, "sd"),
    (32, BF16, 33, 4, 4, BF16, 3, "ds"),
    (64, F32, 70, 3, 1, BF16, 4, "sd"),
    (128, F32, 64, 4, 1, BF16, 4, "ds"),
    (128, F16, 40, 4, 2, F16, 1, "ds"),
    (256, F32, 36, 2, 1, F32, 4, "sd"),
    (64, F32, 32, 2, 1, BF16, 16, "sd"),     # the widest window the ABI takes
    (128, BF16, 64, 2, 2, F32, 8, "ds"),
]


@pytest.mark.parametrize("N,sdt,Dm,H,G,xdt,width,layout", SHAPES)
def test_conv_decode_shapes(orc, N, sdt, Dm, H, G, xdt, width, layout):
    case = make_case(seed=700 + N + width, batch=6, P=10, H=H, G=G, Dm=Dm, N=N, x_dtype=xdt,
                     bc_dtype=xdt, state_dtype=sdt, z=True, active=5, n_pad=1,
                     slot_pad=4 if sdt == F32 else 8, conv=width, conv_layout=layout,
                     conv_pad=5)
    compare_conv(orc, case)


def test_conv_decode_options_off(orc):
    case = make_case(seed=720, batch=3, P=4, H=2, G=2, Dm=24, N=32, dt_bias=False, D=False,
                     dt_softplus=False, indices="none", conv=4)
    case.dt = case.dt.abs()
    case.conv_b = None
    case.conv_silu = False
    compare_conv(orc, case)


def test_conv_decode_index_flag_and_padding(orc):
    case = make_case(seed=730, batch=4, P=5, H=2, G=1, Dm=32, N=64, conv=4, z=True,
                     indices=[3, -1, 5, 0])
    out_g, pool_g, conv_g, err = gpu_run.conv_decode(case)
    out_o, pool_o, conv_o, err_o = orc.conv_decode_case(case)
    assert err == err_o == ssu.FLAG_INDEX_RANGE
    check_out(out_g, out_o, case.x_dtype)
    assert (out_g[1] == 0).all() and torch.isnan(out_g[2]).all()
    assert same_bits(conv_g, conv_o)


def test_conv_decode_headline_workload_every_row(orc):
    """The batch-256 workload in its benchmarked launches, every row compared with the
    oracle: outputs, the whole recurrent pool and the whole conv pool (raw taps, so
    byte for byte)."""
    case = make_config("mamba2_conv_decode_b256")
    out_g, pool_g, conv_g, err = gpu_run.conv_decode(case)
    out_o, pool_o, conv_o, err_o = orc.conv_decode_case(case)
    assert err == err_o == 0
    check_out(out_g, out_o, case.x_dtype)
    check_state(pool_g, pool_o, case.state_dtype)
    assert same_bits(conv_g, conv_o)
    assert changed_slots(case.pool, pool_g, case) == expected_decode_slots(case)


def test_conv_decode_in_cuda_graph_equals_direct():
    case = make_case(seed=740, batch=8, P=12, H=4, G=2, Dm=64, N=128, z=True, conv=4,
                     x_dtype=BF16, bc_dtype=BF16, active=6, n_pad=2)
    out_a, pool_a, conv_a, _ = gpu_run.conv_decode(case)
    d = case.to("cuda")
    pool, conv = d.pool.clone(), d.conv_state.clone()
    out = torch.full((8, 4, 64), float("nan"), dtype=BF16, device="cuda")
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            ssu.ssu_conv_decode(d.xbc, d.conv_w, conv, d.A, d.dt, pool, out, width=4,
                                conv_strides=case.conv_strides, nheads=4, ngroups=2, dim=64,
                                conv_bias=d.conv_b, dt_bias=d.dt_bias, D=d.D, z=d.z,
                                state_indices=d.state_indices, active_batch=6,
                                slot_stride=case.slot_stride, P=case.P, stream=s)
    g.replay()
    torch.cuda.synchronize()
    assert same_bits(out.cpu(), out_a) and same_bits(pool.cpu(), pool_a)
    assert same_bits(conv.cpu(), conv_a)
