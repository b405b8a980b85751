"""Host-side logic checked on the CPU: the decode kernel's split-K work
decomposition (restated from kvpop_internal.cuh) covers every tile exactly
once and never gives a unit more partials than the scratch holds."""
import random

import pytest

K_MAX_SEG = 64


def seg_lo(w, total, nw):
    return (w * total) // nw


def warp_of_tile(x, total, nw):
    return ((x + 1) * nw - 1) // total


def active_warps(total, tpu, launched):
    nw = min(launched, total)
    min_tiles = max(1, (tpu + K_MAX_SEG - 2) // (K_MAX_SEG - 1))
    cap = max(1, total // min_tiles)
    return min(nw, cap)


def _check(units, tpu, launched):
    total = units * tpu
    nw = active_warps(total, tpu, launched)
    assert 1 <= nw <= launched
    owner = []
    for w in range(nw):
        lo, hi = seg_lo(w, total, nw), seg_lo(w + 1, total, nw)
        assert hi > lo, "every active warp gets at least one tile"
        owner += [w] * (hi - lo)
    assert len(owner) == total
    for x in (0, total - 1, total // 2, random.randrange(total)):
        assert warp_of_tile(x, total, nw) == owner[x]
    for u in range(units):
        first, last = owner[u * tpu], owner[u * tpu + tpu - 1]
        assert warp_of_tile(u * tpu, total, nw) == first
        assert warp_of_tile(u * tpu + tpu - 1, total, nw) == last
        assert last - first + 1 <= K_MAX_SEG


@pytest.mark.parametrize("units", [1, 2, 3, 8, 16, 64, 128, 512])
@pytest.mark.parametrize("tpu", [1, 2, 5, 63, 64, 65, 127, 128, 129, 257, 512])
def test_decode_work_split(units, tpu):
    random.seed(units * 1000 + tpu)
    for launched in (8, 9 * 8, 148 * 8, 1184):
        _check(units, tpu, launched)
