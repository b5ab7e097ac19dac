"""Tolerances and comparisons shared by the parity tests.

The bar (derived from the fp32 arithmetic of the kernels):
  state, fp32 pool      |g - o| <= 1e-5 + 1e-5 |o|
  state, fp16/bf16 pool |g - o| <= max(2e-3 + 2e-3 |o|, ulp(o)): both sides round once to
                        the pool format, and when the exact value sits near a rounding
                        midpoint the two roundings may differ by one unit, which for bf16
                        (2^-7 relative) is more than 2e-3
  out, fp32             |g - o| <= 1e-5 + 1e-5 |o|     (o = unrounded float64 oracle)
  out, fp16/bf16        |g - o| <= ulp(o) + 1e-5, one unit in the last place of the
                        output format at |o|: the kernel rounds its fp32 result once, so
                        it lands within half an ulp of its own value, which is itself
                        within fp32 rounding of o.
  stash U and B         bit-exact (exact widening of the inputs)
  stash dA, dt          fp32 tolerance
Written rows are compared byte for byte where nothing may change.
"""

import math

import torch

STATE_TOL = {torch.float32: 1e-5, torch.float16: 2e-3, torch.bfloat16: 2e-3}
OUT_ATOL = 1e-5
_MANT = {torch.float16: 10, torch.bfloat16: 7}
_EMIN = {torch.float16: -14, torch.bfloat16: -126}


def same_bits(a, b):
    a, b = a.detach().cpu().contiguous(), b.detach().cpu().contiguous()
    return a.dtype == b.dtype and a.shape == b.shape and torch.equal(
        a.view(torch.uint8), b.view(torch.uint8))


def _report(bad, g, o, lim, what):
    idx = bad.nonzero()[:5].tolist()
    worst = ((g - o).abs() - lim).masked_fill(~bad, -math.inf).max().item()
    return f"{what}: {int(bad.sum())} elements out of tolerance (first {idx}, worst excess {worst:.3g})"


def check_state(g, o, dtype):
    """g: pool elements from the GPU, o: the oracle's pool, both in ``dtype``."""
    tol = STATE_TOL[dtype]
    g, o = g.detach().cpu().double(), o.detach().cpu().double()
    same = (g == o) | (torch.isnan(g) & torch.isnan(o))     # includes equal infinities
    lim = tol + tol * o.abs()
    if dtype != torch.float32:
        lim = torch.maximum(lim, ulp(o, dtype))
    bad = ~(((g - o).abs() <= lim) | same)
    assert not bad.any(), _report(bad, g, o, lim, f"state ({dtype})")


def ulp(o, dtype):
    a = o.abs().clamp_min(2.0 ** _EMIN[dtype])
    e = torch.floor(torch.log2(a))
    return torch.pow(2.0, e - _MANT[dtype])


def check_out(g, o, dtype):
    """g: GPU output in ``dtype``; o: the oracle's float64 output (NaN = not written)."""
    g, o = g.detach().cpu().double(), o.detach().cpu().double()
    if dtype == torch.float32:
        lim = STATE_TOL[torch.float32] * (1 + o.abs())
    else:
        lim = ulp(o, dtype) + OUT_ATOL
    same = (g == o) | (torch.isnan(g) & torch.isnan(o))
    bad = ~(((g - o).abs() <= lim) | same)
    assert not bad.any(), _report(bad, g, o, lim, f"out ({dtype})")


def check_fp32(g, o, tol=1e-5):
    g, o = g.detach().cpu().double(), o.detach().cpu().double()
    lim = tol + tol * o.abs()
    same = (g == o) | (torch.isnan(g) & torch.isnan(o))
    bad = ~(((g - o).abs() <= lim) | same)
    assert not bad.any(), _report(bad, g, o, lim, "fp32 values")


def slots(pool, case):
    """[P, slot_stride] view of a flat pool."""
    return pool.view(case.P, case.slot_stride)


def changed_slots(before, after, case):
    a, b = slots(before, case).cpu(), slots(after, case).cpu()
    return {s for s in range(case.P)
            if not torch.equal(a[s].view(torch.uint8) if a.dtype != torch.uint8 else a[s],
                               b[s].view(torch.uint8) if b.dtype != torch.uint8 else b[s])}


def expected_decode_slots(case):
    if case.state_indices is None:
        return set(range(case.active))
    return {int(s) for s in case.state_indices[: case.active].tolist() if 0 <= s < case.P}
