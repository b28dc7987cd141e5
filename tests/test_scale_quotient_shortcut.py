"""The block step's scale quotient s_raw = fl(b / fl(alpha * Q)) (reading
pinned in test_oracle_readings.py) is computed in the CUDA block step as
fl(b * fl(1 / fl(alpha * Q))), with the exact quotient taken instead whenever
that product lies below E4M3's normal range or within 5 units (of 2^-20 of the
binary32 significand) of an E4M3 rounding midpoint.  The claim is that the
E4M3 code is then always that of the exact quotient ("Four Over Six (4/6)"
technical summary, 적응형 블록 스케일링 알고리즘).  Here the guard is replayed
in binary32 numpy arithmetic on millions of (b, alpha) pairs, random and
placed next to midpoints, and the code compared with that of fl(b / a); the
same replay without the guard gets some codes wrong, so the pairs reach the
cases the guard is for."""
import numpy as np
import pytest
import torch


def _e4m3(v: np.ndarray) -> np.ndarray:
    """E4M3 codes of non-negative binary32 values: nearest, ties to even,
    saturating to 448."""
    return torch.from_numpy(np.minimum(v, np.float32(448.0))).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _needs_exact(q: np.ndarray) -> np.ndarray:
    b = q.view(np.uint32)
    return (b < np.uint32(0x3C800008)) | (((b & np.uint32(0xFFFFF)) - np.uint32(0x7FFFB)) < np.uint32(11))


def _codes(b: np.ndarray, a: np.ndarray, guard: bool) -> np.ndarray:
    inv = np.float32(1.0) / a
    q = b * inv
    if guard:
        q = np.where(_needs_exact(q), b / a, q)
    return _e4m3(q)


def _pairs(n: int, seed: int):
    rng = np.random.default_rng(seed)
    a = (np.exp2(rng.uniform(-20, 20, n)) * rng.uniform(1, 2, n)).astype(np.float32)
    q = np.exp2(rng.uniform(-8, 9.5, n)).astype(np.float32)
    b = (q * a).astype(np.float32)
    return b, a


def _near_midpoints(n: int, seed: int):
    """b with b / a within a few binary32 units of an E4M3 rounding midpoint."""
    rng = np.random.default_rng(seed)
    a = (np.exp2(rng.uniform(-20, 20, n)) * rng.uniform(1, 2, n)).astype(np.float32)
    e = rng.integers(-6, 8, n)
    m = rng.integers(0, 8, n)
    mid = np.ldexp(1.0 + (2 * m + 1) / 16.0, e)        # halfway between two E4M3 values
    mid = np.where(mid > 448.0, 416.0, mid)            # keep below saturation
    b = (mid * a.astype(np.float64)).astype(np.float32)
    steps = rng.integers(-8, 9, n).astype(np.int64)
    b = (b.view(np.int32) + steps.astype(np.int32)).view(np.float32)
    return b, a


@pytest.mark.parametrize("source", ["random", "near_midpoints"])
def test_guarded_reciprocal_gives_the_exact_quotient_s_code(source):
    b, a = (_pairs if source == "random" else _near_midpoints)(2_000_000, 11)
    with np.errstate(over="ignore", under="ignore"):
        exact = _e4m3(b / a)
        got = _codes(b, a, guard=True)
    assert np.array_equal(got, exact)


def test_unguarded_reciprocal_gets_some_codes_wrong():
    b, a = _near_midpoints(2_000_000, 12)
    with np.errstate(over="ignore", under="ignore"):
        wrong = np.count_nonzero(_codes(b, a, guard=False) != _e4m3(b / a))
    assert wrong > 0
