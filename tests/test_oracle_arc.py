"""Pins for the oracle's ARCQuant augmented quantization (ARCQuant page,
기술 요약 / 방법론): a hand-worked residual example, reduction to the plain
quantizer when S = 0, duplicated channels for weights, and the error
reduction the residual stage exists for."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from conftest import read_golden


def _nibbles(codes_row, block):
    b = codes_row[block * 8: block * 8 + 8]
    out = []
    for v in b:
        out += [int(v) & 15, int(v) >> 4]
    return out


def test_worked_example():
    g = {k: v for k, *v in (line.split() for line in read_golden("arc_residual.txt"))}
    x = torch.zeros(1, 64)
    x[0, 0] = 2.625
    x[0, 16:20] = torch.tensor([1.5, 0.6875, -0.3125, 1.125])
    x = x.to(torch.bfloat16)
    codes, scales, alpha = oracle.quantize_arc(x, np.arange(64), 64, oracle.AUG_RESIDUAL,
                                               oracle.MODE_SIX, oracle.RULE_MAX, 448.0)
    assert alpha == float(g["alpha"][0])
    assert [int(v) for v in scales[0]] == [int(h, 16) for h in g["scales"]]
    assert _nibbles(codes[0], 1)[:4] == [int(h, 16) for h in g["codes_block1"]]
    assert _nibbles(codes[0], 5)[:4] == [int(h, 16) for h in g["codes_block5"]]
    assert all(n == 0 for n in _nibbles(codes[0], 5)[4:])


@pytest.mark.parametrize("mode,rule,F", [(oracle.MODE_SIX, oracle.RULE_MAX, 448.0),
                                         (oracle.MODE_FOUR_OVER_SIX, oracle.RULE_MSE, 256.0)])
def test_no_augment_is_plain_quantize_of_reordered(mode, rule, F):
    x = workloads.small_operand(37, 128, seed=3).make()
    perm = torch.randperm(128, generator=torch.Generator().manual_seed(1)).numpy()
    c, s, a = oracle.quantize_arc(x, perm, 0, oracle.AUG_RESIDUAL, mode, rule, F)
    c0, s0, a0 = oracle.quantize(x[:, torch.from_numpy(perm)], mode, rule, F)
    assert a == a0 and np.array_equal(c, c0) and np.array_equal(s, s0)


def test_duplicate_augment_copies_the_first_channels():
    x = workloads.small_operand(20, 192, seed=4).make()
    perm = torch.randperm(192, generator=torch.Generator().manual_seed(2)).numpy()
    c, s, a = oracle.quantize_arc(x, perm, 64, oracle.AUG_DUPLICATE, oracle.MODE_FOUR_OVER_SIX,
                                  oracle.RULE_MAE, 256.0)
    assert np.array_equal(c[:, 96:], c[:, :32]) and np.array_equal(s[:, 12:], s[:, :4])
    c0, s0, _ = oracle.quantize(x[:, torch.from_numpy(perm)], oracle.MODE_FOUR_OVER_SIX,
                                oracle.RULE_MAE, 256.0)
    assert np.array_equal(c[:, :96], c0) and np.array_equal(s[:, :12], s0)


def test_residual_reduces_the_error_of_the_outlier_channels():
    """x ~ primary + residual: on the S augmented channels the two-stage
    reconstruction is far closer to x than the primary stage alone."""
    x = workloads.small_operand(64, 256, seed=5).make()
    xf = x.float().numpy().astype(np.float64)
    amax_col = np.abs(xf).max(axis=0)
    perm = np.argsort(-amax_col, kind="stable")
    S = 64
    c, s, a = oracle.quantize_arc(x, perm, S, oracle.AUG_RESIDUAL, oracle.MODE_SIX, oracle.RULE_MAX, 448.0)
    deq = oracle.dequantize(c, s, a)  # [64, 256 + 64]
    xp = xf[:, perm]
    err1 = np.abs(xp[:, :S] - deq[:, :S]).sum()
    err2 = np.abs(xp[:, :S] - (deq[:, :S] + deq[:, 256:])).sum()
    assert err2 < 0.25 * err1
