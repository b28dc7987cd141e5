"""The seeded input generators match the recipes they state: the same seed
gives the same bytes, the outlier counts are exact, and the value
distributions have the moments of their definitions (CPU only)."""
import dataclasses

import numpy as np
import pytest
import torch

import workloads


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).numpy()


def test_same_seed_same_bytes_other_seed_other_bytes():
    op = workloads.WORKLOADS["pr1"].x
    assert np.array_equal(_bits(op.make()), _bits(op.make()))
    other = dataclasses.replace(op, seed=op.seed + 1)
    assert not np.array_equal(_bits(op.make()), _bits(other.make()))


def test_pr1_has_exactly_one_percent_outlier_entries():
    op = workloads.WORKLOADS["pr1"].x
    base = dataclasses.replace(op, outliers="", out_frac=0.0, out_mult=1.0).make().float()
    x = op.make().float()
    changed = (x != base)
    n = round(0.01 * op.numel)
    # every chosen entry is multiplied by 20 (a zero base entry would not show, N(0,1) has none)
    assert int(changed.sum()) == n
    ratio = x[changed] / base[changed]
    assert torch.allclose(ratio, torch.full_like(ratio, 20.0), rtol=2 ** -7)


@pytest.mark.parametrize("name,frac,mult", [("mlp8b", 0.005, 50.0), ("prefill", 0.002, 100.0)])
def test_outlier_channels_are_whole_columns(name, frac, mult):
    full = workloads.WORKLOADS[name].x
    op = dataclasses.replace(full, rows=64)           # same recipe, few rows
    base = dataclasses.replace(op, outliers="", out_frac=0.0, out_mult=1.0).make().float()
    x = op.make().float()
    cols = (x != base).any(dim=0)
    assert int(cols.sum()) == max(1, round(frac * op.K))
    # the chosen columns are scaled in every row, the others untouched
    assert torch.allclose(x[:, cols], base[:, cols] * mult, rtol=2 ** -7)
    assert torch.equal(x[:, ~cols], base[:, ~cols])


def test_normal_moments():
    x = workloads.normal(512, 1024, 0.02, seed=3)
    assert abs(float(x.mean())) < 3 * 0.02 / np.sqrt(x.numel())
    assert float(x.std()) == pytest.approx(0.02, rel=0.01)


def test_student_t_moments():
    # t with nu = 4 (scale 1) has variance nu / (nu - 2) = 2
    x = workloads.student_t(512, 1024, 4, 1.0, seed=4)
    assert float(x.var()) == pytest.approx(2.0, rel=0.1)
    assert abs(float(x.mean())) < 0.02
    # heavier tails than the normal: P(|t_4| > 4) is about 1.6 %, P(|z| > 4) about 6e-5
    tail = float((x.abs() > 4).float().mean())
    assert 0.01 < tail < 0.025


def test_sampled_rows_include_both_ends():
    idx = workloads.sample_rows(32768, 64, 1)
    assert idx[0] == 0 and idx[-1] == 32767
    assert torch.all(idx[1:] > idx[:-1])
    assert 60 <= idx.numel() <= 64
