"""Pins for the oracle's Hilbert-curve token order (DFSAttn's Hilbert curve-based
token reordering, read as the 3-D Hilbert curve over the enclosing
power-of-two cube, axes (t, y, x), grid points in curve order).

What makes a curve a Hilbert curve is checked directly, not by re-typing the
oracle:
- on a full cube it is a bijection that starts at the origin and moves to a
  face-adjacent cell at every step (continuity);
- every aligned sub-cube of side 2^k is one contiguous run of 8^k positions
  (the recursive nesting that defines the curve);
- at order 1 the eight corners are visited in Gray-code order (one axis
  changes per step);
- a grid that is not a power-of-two cube takes the enclosing cube's order
  with the points outside the grid skipped.
"""
import numpy as np
import pytest

import oracle


def _coords(perm, T, Hs, Ws):
    t = perm // (Hs * Ws)
    y = (perm // Ws) % Hs
    x = perm % Ws
    return np.stack([t, y, x], axis=1)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_full_cube_is_continuous_bijection_from_origin(bits):
    side = 1 << bits
    perm = oracle.hilbert_order(side, side, side)
    assert sorted(perm.tolist()) == list(range(side ** 3))
    c = _coords(perm, side, side, side)
    assert c[0].tolist() == [0, 0, 0]
    steps = np.abs(np.diff(c, axis=0)).sum(axis=1)
    assert np.all(steps == 1)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_aligned_subcubes_are_contiguous_runs(bits):
    side = 1 << bits
    c = _coords(oracle.hilbert_order(side, side, side), side, side, side)
    for k in range(1, bits):
        run = 8 ** k
        for start in range(0, side ** 3, run):
            block = c[start:start + run] >> k
            # every point of the run lies in one aligned sub-cube of side 2^k ...
            assert np.all(block == block[0])
            # ... and the run covers that sub-cube exactly once
            local = c[start:start + run] - (block[0] << k)
            assert len({tuple(v) for v in local.tolist()}) == run


def test_order_one_is_gray_code():
    c = _coords(oracle.hilbert_order(2, 2, 2), 2, 2, 2)
    codes = (c[:, 0] << 2) | (c[:, 1] << 1) | c[:, 2]
    assert sorted(codes.tolist()) == list(range(8))
    flips = codes[1:] ^ codes[:-1]
    assert all(f in (1, 2, 4) for f in flips.tolist())


def test_keys_are_a_bijection_on_the_cube():
    bits = 3
    side = 1 << bits
    keys = {oracle.hilbert_key(t, y, x, bits)
            for t in range(side) for y in range(side) for x in range(side)}
    assert keys == set(range(side ** 3))


@pytest.mark.parametrize("grid", [(3, 5, 7), (21, 30, 52), (1, 16, 16), (5, 1, 9)])
def test_non_cube_grid_is_the_cube_order_restricted(grid):
    T, Hs, Ws = grid
    bits = max(1, int(np.ceil(np.log2(max(grid)))))
    side = 1 << bits
    cube = _coords(oracle.hilbert_order(side, side, side), side, side, side)
    inside = (cube[:, 0] < T) & (cube[:, 1] < Hs) & (cube[:, 2] < Ws)
    want = (cube[inside, 0] * Hs + cube[inside, 1]) * Ws + cube[inside, 2]
    got = oracle.hilbert_order(T, Hs, Ws)
    np.testing.assert_array_equal(got, want)
