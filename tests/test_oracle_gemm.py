"""Pins for the oracle's dequantization and binary64 GEMM reference.

The W4A4 GEMM (ARCQuant summary, gist.science/ko/paper/2601.07475, "방법론"
section: one uniform NVFP4 contraction over K) is defined here as
Y = A_hat @ B_hat^T with A_hat = val(code) * val(E4M3 scale) * alpha.
Pinned against exact rational arithmetic, brute-force Python loops on tiny
shapes, a closed form and one-hot K blocks.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads

MAGS = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3), Fraction(4), Fraction(6)]


def _frac_e2m1(c):
    v = MAGS[c & 7]
    return -v if c & 8 else v


def _frac_e4m3(c):
    e, m = (c >> 3) & 15, c & 7
    if e == 0:
        return Fraction(m, 2 ** 9)
    return (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)


def _random_operand(rows, K, rng):
    codes = rng.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)
    scales = rng.integers(0, 0x7F, size=(rows, K // 16), dtype=np.uint8)  # finite, non-negative
    return codes, scales


def test_dequantize_exact():
    rng = np.random.default_rng(0)
    codes, scales = _random_operand(3, 64, rng)
    alpha = float(np.float32(0.0123))
    got = oracle.dequantize(codes, scales, alpha)
    fa = Fraction(alpha)
    for r in range(3):
        for k in range(64):
            byte = int(codes[r, k // 2])
            c = (byte >> 4) if k % 2 else (byte & 15)
            want = _frac_e2m1(c) * _frac_e4m3(int(scales[r, k // 16])) * fa
            assert Fraction(got[r, k]) == want


@pytest.mark.parametrize("M,N,K", [(1, 1, 64), (3, 5, 128), (7, 3, 512)])
def test_gemm_brute_force(M, N, K):
    rng = np.random.default_rng(M * 100 + N * 10 + K)
    ac, as_ = _random_operand(M, K, rng)
    bc, bs = _random_operand(N, K, rng)
    aa, ba = float(np.float32(0.37)), float(np.float32(1.9e-3))
    y, guard = oracle.gemm_reference(ac, as_, aa, bc, bs, ba)
    for m in range(M):
        for n in range(N):
            acc = Fraction(0)
            mag = Fraction(0)
            for k in range(K):
                ca = (int(ac[m, k // 2]) >> 4) if k % 2 else (int(ac[m, k // 2]) & 15)
                cb = (int(bc[n, k // 2]) >> 4) if k % 2 else (int(bc[n, k // 2]) & 15)
                a = _frac_e2m1(ca) * _frac_e4m3(int(as_[m, k // 16])) * Fraction(aa)
                b = _frac_e2m1(cb) * _frac_e4m3(int(bs[n, k // 16])) * Fraction(ba)
                acc += a * b
                mag += abs(a * b)
            assert y[m, n] == pytest.approx(float(acc), rel=1e-12, abs=1e-300)
            assert guard[m, n] == pytest.approx(float(mag), rel=1e-12, abs=1e-300)


def test_gemm_closed_form():
    """Every A and B element code +1 (value 0.5) with scales s_A, s_B: every
    output is K * 0.25 * s_A * s_B * alpha_A * alpha_B."""
    M, N, K = 4, 6, 256
    s_a, s_b = 0x38, 0x41   # E4M3 1.0 and 2.25
    ac = np.full((M, K // 2), 0x11, np.uint8)
    bc = np.full((N, K // 2), 0x11, np.uint8)
    as_ = np.full((M, K // 16), s_a, np.uint8)
    bs = np.full((N, K // 16), s_b, np.uint8)
    y, _ = oracle.gemm_reference(ac, as_, 0.5, bc, bs, 0.25)
    assert np.all(y == K * 0.25 * 1.0 * 2.25 * 0.5 * 0.25)


@pytest.mark.parametrize("kb", [0, 3, 7])
def test_gemm_one_hot_block(kb):
    """Only K block kb nonzero: Y = alpha_A alpha_B sA[m,kb] sB[n,kb] sum q q."""
    M, N, K = 5, 4, 128
    rng = np.random.default_rng(kb)
    ac, as_ = _random_operand(M, K, rng)
    bc, bs = _random_operand(N, K, rng)
    mask = np.zeros((1, K // 2), np.uint8)
    mask[0, kb * 8:(kb + 1) * 8] = 0xFF
    ac &= mask
    bc &= mask
    y, _ = oracle.gemm_reference(ac, as_, 1.0, bc, bs, 1.0)
    for m in range(M):
        for n in range(N):
            qq = 0.0
            for k in range(kb * 16, kb * 16 + 16):
                ca = (int(ac[m, k // 2]) >> 4) if k % 2 else (int(ac[m, k // 2]) & 15)
                cb = (int(bc[n, k // 2]) >> 4) if k % 2 else (int(bc[n, k // 2]) & 15)
                qq += float(_frac_e2m1(ca) * _frac_e2m1(cb))
            want = float(_frac_e4m3(int(as_[m, kb]))) * float(_frac_e4m3(int(bs[n, kb]))) * qq
            assert y[m, n] == want


def test_pr1_end_to_end_is_close_to_bf16_product():
    """Sanity of the whole oracle chain on PR1: the W4A4 product tracks the
    unquantized product (NVFP4 keeps ~1-2 significant bits per element, so
    only a loose relative-norm bound holds)."""
    wl = workloads.WORKLOADS["pr1"]
    x, w = wl.x.make(), wl.w.make()
    for mode, rule, F in ((oracle.MODE_SIX, oracle.RULE_MAX, 448.0),
                          (oracle.MODE_FOUR_OVER_SIX, oracle.RULE_MSE, 256.0)):
        xc, xs, xa = oracle.quantize(x, mode, rule, F)
        wc, ws, wa = oracle.quantize(w, mode, rule, F)
        y, _ = oracle.gemm_reference(xc, xs, xa, wc, ws, wa)
        ref = x.double().numpy() @ w.double().numpy().T
        rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
        assert rel < 0.2, rel
    # 4/6 should not be worse than scale-6 on this input (the pages' claim, loosely)
    x6 = oracle.dequantize(*oracle.quantize(x, oracle.MODE_SIX, oracle.RULE_MAX, 448.0))
    x46 = oracle.dequantize(*oracle.quantize(x, oracle.MODE_FOUR_OVER_SIX, oracle.RULE_MSE, 256.0))
    xf = x.double().numpy()
    assert np.sum((x46 - xf) ** 2) < np.sum((x6 - xf) ** 2)
