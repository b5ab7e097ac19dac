"""The bounded-wait exits, exercised on the GPU without a fault.

Every wait of the kernels on their own asynchronous copies (and the tree verify's wait on
its MMAs) gives up after a time limit, sets SSU_FLAG_TIMEOUT, waits once more for what it
still has in flight, and returns, so that a protocol error can never hang the GPU. These
tests run the test library libssu_waittest.so (the same sources built with SSU_WAIT_TEST,
include/ssu_wait_test.h): the limit is cut to 20 ms and one chosen barrier is armed for 16
bytes more than its copies bring, so the copies land but that wait cannot complete. Each
test checks that the launch returns, that the flag is set, that everything outside the
affected unit of work matches the oracle, that the affected unit stopped where it should
(tile, chunk or item granular), and that the context still runs the product library.
The shapes are chosen so that the kernels' mapping of work to CTAs and warps is known:
one decode CTA of 8 warps, warp w taking head w % 4 of row w // 4; one prefill CTA per
(row, head); one tree-verify item per CTA.
"""

import ctypes
import math

import pytest
import torch

import gpu_run
from linear_attention_recurrent_selective_b200 import build, ssu
from linear_attention_recurrent_selective_b200.workloads import make_case
from parity import check_fp32, check_out, check_state, same_bits

pytestmark = pytest.mark.gpu

BF16, F32 = torch.bfloat16, torch.float32
STREAM, PREFILL, TREE_STATE, TREE_X, TREE_MMA = 1, 2, 3, 4, 5
LIMIT_NS = 20_000_000                    # 20 ms instead of 2 s
PRODUCT_LIMIT_NS = 2_000_000_000


@pytest.fixture
def waitlib():
    """Route the binding to libssu_waittest.so for one test; disarm and restore after."""
    L = ssu.load(build.build(waittest=True))
    L.ssu_test_wait_fault.argtypes = [ctypes.c_int] * 4 + [ctypes.c_ulonglong]
    L.ssu_test_wait_fault.restype = ctypes.c_int
    saved = ssu._lib
    ssu._lib = L
    try:
        yield L
    finally:
        torch.cuda.synchronize()
        assert L.ssu_test_wait_fault(0, -1, -1, -1, PRODUCT_LIMIT_NS) == 0
        ssu._lib = saved


def arm(L, site, block, warp, index):
    assert L.ssu_test_wait_fault(site, block, warp, index, LIMIT_NS) == 0


def product_still_runs(orc):
    """A decode through the product library after the give-up matches the oracle."""
    assert ssu._lib is None or not hasattr(ssu._lib, "ssu_test_wait_fault")
    case = make_case(seed=999, batch=3, P=5, H=4, G=2, Dm=64, N=128, x_dtype=BF16,
                     bc_dtype=BF16, z=True)
    out_g, pool_g, err = gpu_run.decode(case)
    out_o, pool_o, _ = orc.decode_case(case)
    assert err == 0
    check_out(out_g, out_o, BF16)
    check_state(pool_g, pool_o, F32)


def head_rows(pool, case, slot, h):
    """[Dm, N] state block of (slot, head h) of a flat pool."""
    s = pool.view(case.P, case.slot_stride)[slot, : case.H * case.Dm * case.N]
    return s.view(case.H, case.Dm, case.N)[h]


def without_head(pool, case, slot, h):
    """The pool's bytes with (slot, head h) cut out."""
    p = pool.view(case.P, case.slot_stride).clone()
    blk = p[slot, : case.H * case.Dm * case.N].view(case.H, case.Dm, case.N)
    blk[h] = 0
    return p


def test_decode_tile_wait_runs_out(orc, waitlib):
    # 2 rows x 4 heads = 8 units of one head (64 rows, 8 tiles of 8 rows) on one CTA of 8
    # warps; warp 3 (row 0, head 3) waits in vain for its third tile (rows 16 .. 23)
    case = make_case(seed=990, batch=2, P=4, H=4, G=1, Dm=64, N=128, x_dtype=BF16,
                     bc_dtype=BF16, z=True)
    arm(waitlib, STREAM, 0, 3, 2)
    out_g, pool_g, err = gpu_run.decode(case)
    assert err == ssu.FLAG_TIMEOUT
    out_o, pool_o, _ = orc.decode_case(case)
    s0 = int(case.state_indices[0])
    assert torch.isnan(out_g[0, 3].float()).all()          # the unit never got to its outputs
    keep = torch.ones(2, 4, dtype=torch.bool)
    keep[0, 3] = False
    check_out(out_g[keep], out_o[keep], BF16)
    check_state(without_head(pool_g, case, s0, 3), without_head(pool_o, case, s0, 3), F32)
    g, o, before = (head_rows(p, case, s0, 3) for p in (pool_g, pool_o, case.pool))
    check_state(g[:16], o[:16], F32)                       # the two tiles it finished
    assert same_bits(g[16:], before[16:])                 # the rest untouched
    ssu._lib = None
    product_still_runs(orc)


def test_replay_tile_wait_runs_out(orc, waitlib):
    # replay units are 4 tiles (32 rows): 2 rows x 2 heads x 2 units = 8 units (both rows
    # live) on one CTA of 8 warps; warp 1 (unit 1: row 0, head 0, rows 32 .. 63) loses its
    # first tile
    case = make_case(seed=991, batch=2, P=4, T=3, H=2, G=1, Dm=64, N=128, x_dtype=BF16,
                     bc_dtype=BF16, lengths="accepted")
    case.accepted_lengths = torch.tensor([3, 2], dtype=torch.int32)
    _, _, st, _ = orc.prefill_case(case, stash=True)
    arm(waitlib, STREAM, 0, 1, 0)
    pool_g, err = gpu_run.replay(case, st, case.accepted_lengths)
    assert err == ssu.FLAG_TIMEOUT
    want = case.pool.clone()
    orc.replay(want, st, case.accepted_lengths, state_indices=case.state_indices, batch=2,
               T=3, H=2, G=1, Dm=64, N=128)
    s0 = int(case.state_indices[0])
    g, o, before = (head_rows(p, case, s0, 0) for p in (pool_g, want, case.pool))
    assert same_bits(g[32:], before[32:])                 # the unit that gave up
    check_state(g[:32], o[:32], F32)
    check_state(without_head(pool_g, case, s0, 0), without_head(want, case, s0, 0), F32)
    ssu._lib = None
    product_still_runs(orc)


def test_prefill_chunk_wait_runs_out(orc, waitlib):
    # the CUDA-core form (fp32 B and C): 2 rows x 2 heads, one CTA each (rows ranked by
    # length: equal lengths keep index order, so CTA 1 is row 0, head 1); its second
    # 16-token chunk of staged inputs never completes
    case = make_case(seed=992, batch=2, P=4, T=40, H=2, G=1, Dm=64, N=128, x_dtype=BF16,
                     bc_dtype=F32, z=True)
    assert case.context_lengths is None
    arm(waitlib, PREFILL, 1, -1, 1)
    out_g, pool_g, _, err = gpu_run.prefill(case)
    assert err == ssu.FLAG_TIMEOUT
    out_o, pool_o, _, _ = orc.prefill_case(case)
    s0 = int(case.state_indices[0])
    check_out(out_g[0, :16, 1], out_o[0, :16, 1], BF16)    # the chunk it finished
    assert torch.isnan(out_g[0, 16:, 1].float()).all()
    keep = torch.ones(2, 40, 2, dtype=torch.bool)
    keep[0, :, 1] = False
    check_out(out_g[keep], out_o[keep], BF16)
    # its final state is never stored; every other head's is
    assert same_bits(head_rows(pool_g, case, s0, 1), head_rows(case.pool, case, s0, 1))
    check_state(without_head(pool_g, case, s0, 1), without_head(pool_o, case, s0, 1), F32)
    ssu._lib = None
    product_still_runs(orc)


def test_prefill_tensor_core_mma_wait_runs_out(orc, waitlib):
    # the chunked tensor-core form (bf16 x, B, C): 2 rows x 2 heads, one CTA each; CTA 1
    # (row 0, head 1) does not issue the first products of its second 128-token chunk,
    # so that chunk's wait runs out: its first chunk's outputs are written, the rest not,
    # and its final state is never stored
    case = make_case(seed=996, batch=2, P=4, T=200, H=2, G=1, Dm=64, N=128, x_dtype=BF16,
                     bc_dtype=BF16, z=True)
    assert case.context_lengths is None
    arm(waitlib, PREFILL, 1, -1, 1)
    out_g, pool_g, _, err = gpu_run.prefill(case)
    assert err == ssu.FLAG_TIMEOUT
    out_o, pool_o, _, _ = orc.prefill_case(case)
    s0 = int(case.state_indices[0])
    check_out(out_g[0, :128, 1], out_o[0, :128, 1], BF16)
    assert torch.isnan(out_g[0, 128:, 1].float()).all()
    keep = torch.ones(2, 200, 2, dtype=torch.bool)
    keep[0, :, 1] = False
    check_out(out_g[keep], out_o[keep], BF16)
    assert same_bits(head_rows(pool_g, case, s0, 1), head_rows(case.pool, case, s0, 1))
    check_state(without_head(pool_g, case, s0, 1), without_head(pool_o, case, s0, 1), F32)
    ssu._lib = None
    product_still_runs(orc)


@pytest.mark.parametrize("site,block", [(TREE_STATE, 5), (TREE_X, 2), (TREE_MMA, 6)])
def test_tree_verify_wait_runs_out(orc, waitlib, site, block):
    # tensor-core form (bf16 B and C, dstate 128): 2 rows x 4 heads = 8 items on 8 CTAs,
    # CTA k taking item k = (row k // 4, head k % 4); its first (only) item's wait runs out
    case = make_case(seed=993, batch=2, P=4, T=20, H=4, G=1, Dm=64, N=128, x_dtype=BF16,
                     bc_dtype=BF16, tree="random")
    b, h = block // 4, block % 4
    arm(waitlib, site, block, -1, 0)
    out_g, pool_g, st_g, err = gpu_run.ddtree(case)
    assert err == ssu.FLAG_TIMEOUT
    out_o, st_o, _ = orc.ddtree_case(case)
    assert same_bits(pool_g, case.pool)
    assert torch.isnan(out_g[b, :, h].float()).all()       # no output of the item
    keep = torch.ones(2, 20, 4, dtype=torch.bool)
    keep[b, :, h] = False
    check_out(out_g[keep], out_o[keep], BF16)
    assert same_bits(st_g[2], st_o[2])                    # B: staged before the waits
    dA_g, U_g, _, dt_g = st_g
    dA_o, U_o, _, dt_o = st_o
    if site == TREE_MMA:                                  # stash written before the MMA wait
        check_fp32(dA_g, dA_o)
        check_fp32(dt_g, dt_o)
        assert same_bits(U_g, U_o)
    else:                                                 # the item stopped before its stash
        assert torch.isnan(dA_g[b, :, h]).all() and torch.isnan(U_g[b, :, h]).all()
        check_fp32(dA_g[keep], dA_o[keep])
        check_fp32(dt_g[keep], dt_o[keep])
        assert same_bits(U_g[keep], U_o[keep])
    ssu._lib = None
    product_still_runs(orc)


def test_disarmed_test_library_matches_oracle(orc, waitlib):
    """With nothing armed the test library computes what the product library does."""
    assert waitlib.ssu_test_wait_fault(0, -1, -1, -1, LIMIT_NS) == 0
    case = make_case(seed=994, batch=3, P=5, T=20, H=4, G=1, Dm=64, N=128, x_dtype=BF16,
                     bc_dtype=BF16, tree="random")
    out_g, _, _, err = gpu_run.ddtree(case)
    out_o, _, _ = orc.ddtree_case(case)
    assert err == 0
    check_out(out_g, out_o, BF16)
    assert not math.isnan(float(out_g.float().sum()))
