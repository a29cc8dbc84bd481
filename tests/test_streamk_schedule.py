"""The stream-K partition of the tensor-core path, restated on the host.

The prefill kernel cuts a GEMM's (tile, 256-column block) units, tile-major,
into gridDim.x contiguous ranges: CTA c takes units [U*c/G, U*(c+1)/G).  Its
correctness rests on three properties of that arithmetic, checked here for the
layer shapes and ragged ones over several grid sizes:
  * every unit is covered exactly once;
  * only a CTA's first segment can start inside a tile (so one partial-tile
    slot per CTA suffices) and only its last can stop inside one (so the CTA
    that finishes a tile has no later work to hold up);
  * the finisher's rule — the CTAs after it whose ranges start before the
    tile's end — names exactly the CTAs whose first segments hold the tile's
    later blocks, in order.
"""
import pytest


def segments(units, nblk, grid, c):
    lo, hi = units * c // grid, units * (c + 1) // grid
    out, u = [], lo
    while u < hi:
        tile, b0 = divmod(u, nblk)
        b1 = min(nblk, b0 + (hi - u))
        out.append((tile, b0, b1))
        u += b1 - b0
    return out


def finisher_contributors(units, nblk, grid, c, tile):
    end = c + 1
    while end < grid and units * end // grid < (tile + 1) * nblk:
        end += 1
    return list(range(c + 1, end))


SHAPES = [(832, 4096), (1024, 832), (2048, 4096), (4096, 2048), (3200, 14336), (4096, 3200), (4736, 4096),
          (14336, 4736), (6400, 14336), (2400, 2368), (100, 64), (129, 1664)]


@pytest.mark.parametrize("M,K", SHAPES)
@pytest.mark.parametrize("batch", [129, 300, 2048, 4096])
@pytest.mark.parametrize("grid", [148, 132, 160, 7])
def test_partition_properties(M, K, batch, grid):
    tiles = -(-M // 128) * -(-batch // 256)
    nblk = (K // 64 + 3) // 4
    units = tiles * nblk
    if units < grid:
        pytest.skip("the planner takes stream-K only with at least one unit per CTA")
    covered = {}
    first_parts = {}
    for c in range(grid):
        segs = segments(units, nblk, grid, c)
        assert segs, "every CTA has work"
        for i, (tile, b0, b1) in enumerate(segs):
            for b in range(b0, b1):
                covered[(tile, b)] = covered.get((tile, b), 0) + 1
            if b0 > 0:
                assert i == 0, "only the first segment starts inside a tile"
                first_parts.setdefault(tile, []).append(c)
            if b1 < nblk:
                assert i == len(segs) - 1, "only the last segment stops inside a tile"
    assert len(covered) == units and set(covered.values()) == {1}
    for c in range(grid):
        tile, b0, b1 = segments(units, nblk, grid, c)[-1]
        if b0 == 0 and b1 < nblk:
            assert finisher_contributors(units, nblk, grid, c, tile) == first_parts.get(tile, [])
