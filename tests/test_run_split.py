"""The decode schedule's run arithmetic (csrc/paged_merge.cuh, RunSplit).

The global chunk order of NC chunks is split evenly over W warps: warp w runs
chunks [floor(w*NC/W), floor((w+1)*NC/W)), and the warp holding chunk g is
ceil((g+1)*W/NC) - 1.  The kernel evaluates both without 64-bit division:
floor(w*NC/W) as w*q + floor(w*r/W) with NC = q*W + r, and the owner warp as
a single-precision estimate of that quotient corrected by one step against the
run bounds.  These checks restate that arithmetic in float32 (numpy) and hold
it against the exact integer definitions, including chunk totals up to 2^40
and grids with more warps than chunks.
"""
import math
import random

import numpy as np


def exact_begin(w, nc, warps):
    return w * nc // warps


def exact_owner(g, nc, warps):
    return ((g + 1) * warps + nc - 1) // nc - 1


def split_begin(w, nc, warps):
    q, r = divmod(nc, warps)
    assert w * r < 2**32  # the 32-bit product of the device code
    return w * q + (w * r) // warps


def split_owner(g, nc, warps):
    f32 = np.float32
    x = f32(f32(g + 1) * f32(warps)) / f32(nc)  # IEEE single precision, as on the device
    w = int(math.ceil(float(x))) - 1
    w = max(0, min(warps - 1, w))
    if split_begin(w, nc, warps) > g:
        w -= 1
    elif w + 1 < warps and split_begin(w + 1, nc, warps) <= g:
        w += 1
    return w


def _cases(rng):
    totals = (1, 2, 3, 7, 31, 32, 33, 100, 1183, 1184, 1185, 65536, 10**6, 536870912, 2**40 + 12345)
    grids = (1, 2, 7, 32, 148, 888, 1184, 1600)
    cases = [(nc, w) for nc in totals for w in grids]
    cases += [(rng.randrange(1, 2**41), rng.randrange(1, 1601)) for _ in range(150)]
    return cases


def test_run_bounds_equal_the_exact_split():
    rng = random.Random(7)
    for nc, warps in _cases(rng):
        probes = set(range(min(warps + 1, 40))) | {warps - 1, warps} | {rng.randrange(0, warps + 1) for _ in range(40)}
        for w in probes:
            assert split_begin(w, nc, warps) == exact_begin(w, nc, warps), (nc, warps, w)
        assert split_begin(warps, nc, warps) == nc


def test_owner_warp_equals_the_exact_formula():
    rng = random.Random(11)
    n = 0
    for nc, warps in _cases(rng):
        chunks = {0, nc - 1, nc // 2} | {rng.randrange(0, nc) for _ in range(60)}
        for w in [rng.randrange(0, warps) for _ in range(30)] + [0, warps - 1]:
            b = exact_begin(w, nc, warps)
            chunks |= {c for c in (b - 1, b, b + 1) if 0 <= c < nc}  # run boundaries: where rounding bites
        for g in chunks:
            owner = split_owner(g, nc, warps)
            assert owner == exact_owner(g, nc, warps), (nc, warps, g)
            # and the owner's run holds the chunk
            assert exact_begin(owner, nc, warps) <= g < exact_begin(owner + 1, nc, warps)
            n += 1
    assert n > 10000
