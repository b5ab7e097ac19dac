"""GPU checks of pool_clear_slot and pool_copy_slot against the oracle's byte operations.

Selective State Update page (TensorRT-Edge-LLM C++ API), invokeMambaStateClear;
Recurrent State Manager page, clearSlot / clear / copySlotFrom."""

import pytest
import torch

from linear_attention_recurrent_selective_b200 import ssu
from parity import same_bits

pytestmark = pytest.mark.gpu


def test_clear_one_slot_and_all(orc):
    g = torch.Generator().manual_seed(400)
    host = torch.randn(7, 4, 16, 32, generator=g)
    pool = host.cuda()
    ssu.pool_clear_slot(pool, 3)
    want = host.clone()
    orc.clear_slot(want, 4 * 16 * 32 * 4, 7, 3)
    torch.cuda.synchronize()
    assert same_bits(pool.cpu(), want)
    ssu.pool_clear_slot(pool, -1)
    torch.cuda.synchronize()
    assert (pool == 0).all()


def test_clear_padded_flat_pool_with_odd_sizes(orc):
    # slot stride of 1000 bytes: neither 16-byte aligned slots nor whole vectors
    host = torch.randint(1, 255, (5 * 1000,), dtype=torch.uint8)
    pool = host.cuda()
    ssu.pool_clear_slot(pool, 2, slot_bytes=1000, P=5)
    want = host.clone()
    orc.clear_slot(want, 1000, 5, 2)
    torch.cuda.synchronize()
    assert same_bits(pool.cpu(), want)


def test_copy_slot_between_pools_of_different_counts(orc):
    g = torch.Generator().manual_seed(401)
    src_h = torch.randn(3, 2, 8, 16, generator=g).half()
    dst_h = torch.randn(9, 2, 8, 16, generator=g).half()
    src, dst = src_h.cuda(), dst_h.cuda()
    ssu.pool_copy_slot(dst, 7, src, 1)
    orc.copy_slot(dst_h, 9, 7, src_h, 3, 1, 2 * 8 * 16 * 2)
    torch.cuda.synchronize()
    assert same_bits(dst.cpu(), dst_h)
    assert same_bits(src.cpu(), src_h)


def test_pool_bad_slot_raises():
    pool = torch.zeros(4, 8, device="cuda")
    with pytest.raises(ssu.SSUError):
        ssu.pool_clear_slot(pool, 4)
    with pytest.raises(ssu.SSUError):
        ssu.pool_copy_slot(pool, 0, pool, 9)
