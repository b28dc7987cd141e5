"""The bound the RMS pass takes for a row's largest |bf16(y)| (RMSNorm ahead
of the augmented quantization, ARCQuant page, 방법론, 커널 구현), checked on
the CPU against the element-by-element definition.

y_k = bf16((x_k * r) * gamma_k), two binary32 roundings then one to bf16.
With P = max_k |x_k * gamma_k| (exact for bf16 operands), every |y_k| before
the bf16 rounding lies within a factor (1 +- 2^-24)^2 of |x_k gamma_k| r, so
the row's max lies in [P r (1 - 2^-20), P r (1 + 2^-20)] once both ends are
rounded outward; rounding to bf16 is monotone, so when both ends round to the
same bf16 value that value is the row's max |bf16(y)|.  The pass uses that
only while P r >= 2^-90 and max |gamma| <= 2^20 (the slack then also covers
underflow).  Here the bound's decision is recomputed with exact rationals
(directed roundings spelled out) and compared with the definition on rows of
several shapes; a bound without the slack is shown to fail on some of them,
so the rows are close enough to bf16 rounding boundaries to matter.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import exact_binary32 as xb
import workloads


def _rd32(q: Fraction) -> Fraction:
    """Largest binary32 value <= q (q > 0, in range)."""
    r = xb.rn32(q)
    if r > q:
        r = Fraction(float(np.nextafter(np.float32(float(r)), np.float32(0))))
    return r


def _ru32(q: Fraction) -> Fraction:
    r = xb.rn32(q)
    if r < q:
        r = Fraction(float(np.nextafter(np.float32(float(r)), np.float32(np.inf))))
    return r


def _rows_r(xf: np.ndarray, eps: float) -> np.ndarray:
    """r = 1 / sqrt(pairwise_sum(x^2) / K + eps) per row, binary32 steps (the
    zero-padded pairwise tree)."""
    rows, K = xf.shape
    n = 1 << (K - 1).bit_length()
    a = np.zeros((rows, n), np.float32)
    a[:, :K] = xf * xf
    while a.shape[1] > 1:
        a = a[:, 0::2] + a[:, 1::2]
    return np.float32(1.0) / np.sqrt(a[:, 0] / np.float32(K) + np.float32(eps))


def _decide(P: float, r: float, slack: Fraction):
    """The pass's bound: the bf16 value it returns, or None (rows go one by one)."""
    if not (P > 0 and np.isfinite(P)):
        return None
    pr = Fraction(float(P)) * Fraction(float(r))
    plo, phi = _rd32(pr), _ru32(pr)
    if plo < Fraction(2) ** -90:
        return None
    lo, hi = _rd32(plo * (1 - slack)), _ru32(phi * (1 + slack))
    blo, bhi = xb.bf16_rne(lo), xb.bf16_rne(hi)
    return blo if blo == bhi else None


def _check(x: torch.Tensor, gamma: torch.Tensor, eps: float, slack: Fraction):
    """(rows decided by the bound, rows where its answer is wrong)."""
    xf = x.float().numpy()
    gf = gamma.float().numpy()
    assert np.abs(gf).max() <= 2.0 ** 20
    r = _rows_r(xf, eps)
    y = (xf * r[:, None]) * gf[None, :]  # binary32, in this order
    ymax = torch.from_numpy(np.abs(y)).to(torch.bfloat16).float().numpy().max(axis=1)
    P = np.abs(xf * gf[None, :]).max(axis=1)
    decided = wrong = 0
    for i in range(xf.shape[0]):
        v = _decide(float(P[i]), float(r[i]), slack)
        if v is None:
            continue
        decided += 1
        wrong += v != Fraction(float(ymax[i]))
    return decided, wrong


def _gains(K: int, seed: int, spread: float) -> torch.Tensor:
    g = torch.Generator().manual_seed(seed)
    return ((1.0 + 0.25 * torch.randn(K, generator=g)) * torch.exp2(spread * torch.randn(K, generator=g))).to(
        torch.bfloat16)


@pytest.mark.parametrize("K,rows,spread", [(64, 20000, 0.0), (256, 8000, 4.0), (1024, 2000, 0.0), (5120, 400, 2.0)])
def test_bound_decides_the_row_max_exactly(K, rows, spread):
    x = workloads.small_operand(rows, K, seed=K + rows).make()
    gamma = _gains(K, K, spread)
    decided, wrong = _check(x, gamma, 1e-6, Fraction(1, 2 ** 20))
    assert wrong == 0
    assert decided >= 0.99 * rows  # the bound decides nearly every row


def _bf16_rne_f64(v: np.ndarray) -> np.ndarray:
    """Nearest bf16 value of positive normal float64 values, ties to even (one
    rounding: the 8-bit significand taken from the exact float64 value)."""
    m, e = np.frexp(v)
    return np.ldexp(np.rint(m * 2.0 ** 8), e - 8)


def test_bound_without_slack_is_wrong_on_some_rows():
    """Taking bf16(P r) itself as the row's max is wrong on some rows (where
    P r and the twice-rounded max straddle a bf16 rounding boundary); on those
    rows the bound with its slack either gives the right value or leaves the
    row to the element-by-element path."""
    rows, K = 400000, 16
    x = workloads.small_operand(rows, K, seed=77).make()
    gamma = _gains(K, 16, 0.0)
    xf, gf = x.float().numpy(), gamma.float().numpy()
    r = _rows_r(xf, 1e-6)
    y = (xf * r[:, None]) * gf[None, :]
    ymax = torch.from_numpy(np.abs(y)).to(torch.bfloat16).float().numpy().max(axis=1).astype(np.float64)
    P = np.abs(xf * gf[None, :]).max(axis=1).astype(np.float64)
    # the helper agrees with torch's bf16 rounding where both apply (binary32 inputs)
    v = ymax[:1000] * 1.37
    v32 = v.astype(np.float32).astype(np.float64)
    assert np.array_equal(_bf16_rne_f64(v32), torch.from_numpy(v32.astype(np.float32)).to(torch.bfloat16).double().numpy())
    naive = _bf16_rne_f64(P * r.astype(np.float64))  # exact product, one rounding to bf16
    bad = np.nonzero(naive != ymax)[0]
    assert bad.size > 0
    for i in bad:
        v = _decide(float(P[i]), float(r[i]), Fraction(1, 2 ** 20))
        assert v is None or v == Fraction(float(ymax[i]))


def test_tiny_rows_are_left_to_the_element_by_element_path():
    x = (workloads.small_operand(64, 256, seed=3).make().float() * 2.0 ** -120).to(torch.bfloat16)
    gamma = _gains(256, 5, 0.0)
    decided, wrong = _check(x, gamma, 1e-6, Fraction(1, 2 ** 20))
    assert decided == 0 and wrong == 0
