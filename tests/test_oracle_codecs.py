"""Pins for the oracle's E2M1 and E4M3 codecs.

Pinned against: the E2M1 grid the Four-Over-Six summary prints (section
"문제 제기"), a hand-worked rounding table, an independent per-binade rint
formulation over a dense sweep, torch's float8_e4m3fn cast (a library
routine) over every code, midpoint and a log-uniform sweep, and brute-force
nearest-value enumeration over both grids (E4M3's built from the format's
definition).
"""
import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden


def _grid():
    rows = [ln.split() for ln in read_golden("e2m1_grid.txt")]
    return {int(c): float(v) for c, v in rows}


def test_e2m1_grid_matches_pages():
    grid = _grid()
    assert len(grid) == 8
    for code, mag in grid.items():
        assert oracle.e2m1_value(code) == mag
        assert oracle.e2m1_value(code | 8) == -mag
        assert np.signbit(oracle.e2m1_value(code | 8))
    mags = [grid[c] for c in range(8)]
    steps = np.diff(mags)
    # step 0.5 on [0,2], 1 on [2,4], 2 on [4,6]
    assert list(steps) == [0.5, 0.5, 0.5, 0.5, 1.0, 1.0, 2.0]
    assert mags[-1] == 6.0


def test_e2m1_rounding_table():
    for ln in read_golden("e2m1_rounding.txt"):
        v, code = ln.split()
        assert oracle.e2m1_encode(float(v)) == int(code), v


def _e2m1_rint_reference(v: np.ndarray) -> np.ndarray:
    """Independent formulation: round |v| to a multiple of the binade's step
    with numpy's round-half-even rint, clamp at 6, map value -> code."""
    a = np.abs(v.astype(np.float64))
    step = np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0))
    q = np.minimum(np.rint(a / step) * step, 6.0)
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    code = np.searchsorted(mags, q)
    assert np.all(mags[code] == q)
    return (code + 8 * np.signbit(v)).astype(np.uint8)


def test_e2m1_dense_sweep_vs_rint():
    sweep = np.linspace(-8, 8, 40001, dtype=np.float32)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 2.0, 4.0], np.float32)
    near = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(10))])
    vals = np.concatenate([sweep, near, -near, np.array([0.0, -0.0, 1e-30, -1e-30, 1e30], np.float32)])
    ref = _e2m1_rint_reference(vals)
    got = np.array([oracle.e2m1_encode(float(v)) for v in vals], np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(vals[i]), int(got[i]), int(ref[i])) for i in bad[:10]]


def test_e4m3_decode_properties():
    vals = [oracle.e4m3_value(c) for c in range(0x7F)]
    assert vals[0] == 0.0
    assert vals[1] == 2.0 ** -9            # smallest subnormal
    assert vals[8] == 2.0 ** -6            # smallest normal
    assert vals[0x7E] == 448.0             # largest finite
    assert all(b > a for a, b in zip(vals, vals[1:]))
    assert np.isnan(oracle.e4m3_value(0x7F))
    # agree with torch's decoding of every finite non-negative code
    t = torch.arange(0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    assert np.array_equal(t, np.array(vals, np.float32))


def _torch_e4m3(v: np.ndarray) -> np.ndarray:
    """torch's RNE float32 -> float8_e4m3fn cast (NaN above 480, so only call
    it on values <= 448)."""
    t = torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def test_e4m3_encode_vs_torch_cast():
    codes = np.arange(0x7F, dtype=np.uint8)
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    mids = (vals[:-1] + vals[1:]) / 2
    rng = np.random.default_rng(0)
    logu = np.exp2(rng.uniform(-12, np.log2(448), 20000)).astype(np.float32)
    cand = np.concatenate([vals, mids, np.nextafter(mids, np.float32(0)),
                           np.nextafter(mids, np.float32(1000)), logu,
                           np.array([2.0 ** -10, 2.0 ** -11, 3 * 2.0 ** -11], np.float32)])
    cand = cand[(cand >= 0) & (cand <= 448)].astype(np.float32)
    ref = _torch_e4m3(cand)
    got = np.array([oracle.e4m3_encode(float(v)) for v in cand], np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(cand[i]), int(got[i]), int(ref[i])) for i in bad[:10]]


@pytest.mark.parametrize("v", [448.0, 449.0, 463.9, 464.0, 480.0, 672.0, 1e30])
def test_e4m3_saturates(v):
    assert oracle.e4m3_encode(v) == 0x7E
    assert oracle.e4m3_value(0x7E) == 448.0


def test_e4m3_subnormal_ties():
    # 2^-10 is the midpoint of 0 and 2^-9: the tie goes to the even code 0.
    assert oracle.e4m3_encode(2.0 ** -10) == 0
    # 3 * 2^-10 is the midpoint of codes 1 and 2: even code 2.
    assert oracle.e4m3_encode(3 * 2.0 ** -10) == 2
    assert oracle.e4m3_encode(0.0) == 0


# ------------------------------------------- brute-force nearest value --
# Round-to-nearest-even by enumeration: the nearest grid value wins; of two
# equally near ones, the code with an even mantissa (bit 0 clear) wins; with
# saturation nothing is above the largest finite value.  The grids come from
# the format definitions, not from the oracle or torch.

def _e4m3_grid() -> np.ndarray:
    """All 127 non-negative finite E4M3 values (bias 7, 3 mantissa bits,
    subnormals at exponent field 0, code 0x7F is NaN), by code."""
    vals = []
    for code in range(0x7F):
        e, m = code >> 3, code & 7
        vals.append(m / 8 * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))
    return np.array(vals)


def _nearest_even(v: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Code of the grid value nearest to |v|; ties to the even code.  Above
    the largest value the nearest is that value; clamping first keeps the
    binary64 distances exact (|v| - g for a huge v would round to a tie)."""
    a = np.minimum(np.abs(v.astype(np.float64)), grid[-1])
    d = np.abs(a[:, None] - grid[None, :])
    best = d.min(axis=1, keepdims=True)
    tied = d == best
    even = tied & (np.arange(grid.size)[None, :] % 2 == 0)
    pick_even = even.any(axis=1)
    return np.where(pick_even, even.argmax(axis=1), tied.argmax(axis=1))


def test_e2m1_encode_is_nearest_grid_value_by_enumeration():
    grid = np.array([_grid()[c] for c in range(8)])          # the pages' grid
    rng = np.random.default_rng(1)
    mids = (grid[:-1] + grid[1:]) / 2
    vals = np.concatenate([
        rng.uniform(-7, 7, 20000), np.exp2(rng.uniform(-30, 3, 5000)),
        mids, np.nextafter(mids.astype(np.float32), np.float32(0)),
        np.nextafter(mids.astype(np.float32), np.float32(10)), grid, [6.5, 7.0, 1e20, 0.0]]).astype(np.float32)
    vals = np.concatenate([vals, -vals])
    ref = _nearest_even(vals, grid) + 8 * np.signbit(vals)
    got = np.array([oracle.e2m1_encode(float(v)) for v in vals])
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(vals[i]), int(got[i]), int(ref[i])) for i in bad[:10]]


def test_e4m3_encode_is_nearest_grid_value_by_enumeration():
    grid = _e4m3_grid()
    assert grid[1] == 2.0 ** -9 and grid[8] == 2.0 ** -6 and grid[0x7E] == 448.0
    rng = np.random.default_rng(2)
    mids = (grid[:-1] + grid[1:]) / 2
    m32 = mids.astype(np.float32)
    assert np.array_equal(m32.astype(np.float64), mids)          # midpoints are exact in binary32
    vals = np.concatenate([
        np.exp2(rng.uniform(-14, 10, 30000)), grid, m32, np.nextafter(m32, np.float32(0)),
        np.nextafter(m32, np.float32(1000)), [449.0, 464.0, 480.0, 1e6, 0.0]]).astype(np.float32)
    ref = _nearest_even(vals, grid)                               # saturates at 448 by construction
    got = np.array([oracle.e4m3_encode(float(v)) for v in vals])
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(vals[i]), int(got[i]), int(ref[i])) for i in bad[:10]]
