"""Parity of the CUDA quantizer (nvfp4_quantize through the C ABI) with the CPU
oracle: codes, swizzled scales (padding bytes included) and alpha must be
bit-identical, in both modes and all three Four-Over-Six rules."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import w4a4_gemm_nvfp4_b200 as nv
from gpu_util import MODE, RULE, alpha_of, assert_quant_equal, gpu_quantize, to_np

pytestmark = pytest.mark.gpu

RECIPES = [("six", "max", 448.0), ("four_over_six", "max", 256.0), ("four_over_six", "mae", 256.0),
           ("four_over_six", "mse", 256.0), ("six", "max", 256.0), ("four_over_six", "mse", 448.0)]
SHAPES = [(1, 64), (64, 512), (129, 128), (300, 192), (257, 1024), (1000, 320), (128, 64)]


@pytest.mark.parametrize("recipe", RECIPES, ids=lambda r: "-".join(map(str, r)))
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"{s[0]}x{s[1]}")
@pytest.mark.parametrize("kind", ["t", "normal"])
def test_quantize_matches_oracle(shape, recipe, kind):
    x = workloads.small_operand(*shape, seed=shape[0] * 7 + shape[1], kind=kind).make()
    q, status = gpu_quantize(x, *recipe)
    assert status == nv.OK
    assert_quant_equal(q, x, *recipe)


@pytest.mark.parametrize("recipe", RECIPES[:4], ids=lambda r: "-".join(map(str, r)))
def test_pr1_operands(recipe):
    wl = workloads.WORKLOADS["pr1"]
    for op in (wl.x, wl.w):
        x = op.make()
        q, status = gpu_quantize(x, *recipe)
        assert status == nv.OK
        assert_quant_equal(q, x, *recipe)


@pytest.mark.parametrize("ldx_pad", [64, 8])  # 8: rows not 32-byte aligned (two 16-byte loads per block)
def test_strided_rows(ldx_pad):
    x = workloads.small_operand(200, 256, seed=9).make()
    for recipe in (("four_over_six", "mse", 256.0), ("six", "max", 448.0)):
        q, status = gpu_quantize(x, *recipe, ldx_pad=ldx_pad)
        assert status == nv.OK
        assert_quant_equal(q, x, *recipe)


def test_zero_tensor():
    x = torch.zeros(130, 128, dtype=torch.bfloat16)
    x[5, 7] = -0.0
    q, status = gpu_quantize(x, "four_over_six", "mae", 256.0)
    assert status == nv.OK and alpha_of(q) == 1.0
    assert_quant_equal(q, x, "four_over_six", "mae", 256.0)


def test_tiny_values_reciprocal_overflow():
    """Block maxima near 2^-130: 1/d overflows and the block encodes as +-0."""
    x = (workloads.small_operand(64, 128, seed=4).make().float() * 2.0 ** -133).to(torch.bfloat16)
    for recipe in RECIPES[:4]:
        q, status = gpu_quantize(x, *recipe)
        assert status == nv.OK
        assert_quant_equal(q, x, *recipe)


def test_mixed_magnitudes_and_signed_zeros():
    """Rows with wildly different scales (E4M3 subnormal and saturated block
    scales) and explicit negative zeros / tiny negatives."""
    g = torch.Generator().manual_seed(5)
    x = torch.randn(256, 256, generator=g)
    x *= torch.logspace(-30, 30, 256, base=2.0).unsqueeze(1)
    x[:, ::17] = -0.0
    x[::3, 5] = -1e-30
    x = x.to(torch.bfloat16)
    for recipe in RECIPES:
        q, status = gpu_quantize(x, *recipe)
        assert status == nv.OK
        assert_quant_equal(q, x, *recipe)


@pytest.mark.parametrize("bad", [float("inf"), float("nan")])
def test_nonfinite_reports_status(bad):
    x = workloads.small_operand(64, 128, seed=1).make()
    x[10, 3] = bad
    q, status = gpu_quantize(x, "six", "max", 448.0)
    assert status == nv.ERR_NONFINITE
    assert np.isnan(alpha_of(q))
    # codes untouched (still the canary)
    assert (to_np(q.codes) == 0xA5).all()


def test_workspace_reuse_and_repeat_is_deterministic():
    x = workloads.small_operand(512, 512, seed=8).make()
    q1, _ = gpu_quantize(x, "four_over_six", "mse", 256.0)
    q2 = nv.quantize(x.cuda(), "four_over_six", "mse", 256.0)
    q2 = nv.quantize(x.cuda(), "four_over_six", "mse", 256.0, out=q2)
    assert torch.equal(q1.codes, q2.codes) and torch.equal(q1.scales, q2.scales)
    assert torch.equal(q1.global_scale, q2.global_scale)


# ------------------------------------------------ full sizes, sampled rows --

_FULL = {}


def _full_tensor(key, make):
    if key not in _FULL:
        _FULL.clear()
        _FULL[key] = make()
    return _FULL[key]


def _check_sampled(x, recipe, nsample=48, seed=0):
    mode, rule, F = recipe
    rows, K = x.shape
    q, status = gpu_quantize(x, mode, rule, F, canary=0)
    assert status == nv.OK
    amax, bad = oracle.amax(x)
    assert not bad
    alpha = oracle.global_scale(amax, F)
    assert np.float32(alpha_of(q)) == np.float32(alpha)
    idx = workloads.sample_rows(rows, nsample, seed).numpy()
    oc, os_ = oracle.quantize_rows(x[idx], alpha, MODE[mode], RULE[rule])
    gc = to_np(q.codes[torch.from_numpy(idx).cuda()])
    assert np.array_equal(gc, oc)
    gs = oracle.unswizzle_scales(to_np(q.scales), rows, K)[idx]
    assert np.array_equal(gs, os_)
    # padding rows of the last scale row block are zero
    pad = oracle.unswizzle_scales(to_np(q.scales), -(-rows // 128) * 128, K)[rows:]
    assert not pad.any()


@pytest.mark.slow
@pytest.mark.parametrize("shape", workloads.SWEEP_SHAPES, ids=lambda s: f"{s[0]}x{s[1]}")
def test_sweep_full_size_sampled(shape):
    x = _full_tensor(("sweep",) + shape, lambda: workloads.sweep_operand(*shape).make())
    for recipe in workloads.SWEEP_RECIPES:
        _check_sampled(x, recipe)


@pytest.mark.slow
@pytest.mark.parametrize("name", ["mlp8b", "attn27b", "prefill"])
def test_config_operands_full_size_sampled(name):
    wl = workloads.WORKLOADS[name]
    x = _full_tensor((name, "x"), wl.x.make)
    for recipe in wl.x_recipes:
        _check_sampled(x, recipe)
    w = _full_tensor((name, "w"), wl.w.make)
    _check_sampled(w, wl.w_recipe)


def _reading_pin_cases():
    import test_oracle_readings as tr
    return tr.CASES


@pytest.mark.parametrize("case", _reading_pin_cases(), ids=lambda c: c["name"])
def test_reading_pins(case):
    """The blocks that pin the quotient order, the reciprocal-multiply scaling
    and the pairwise error sum (tests/golden/reading_pins.txt, derived in
    exact arithmetic): every quantizer kernel gives the stored bits."""
    import test_oracle_readings as tr

    x = tr._tensor(case)
    recipe = (case["mode"], case["rule"], case["F"])

    def block1(codes_row, scales_swz):
        unpacked = [int(v) for b in codes_row[8:16] for v in (b & 15, b >> 4)]
        return unpacked, int(scales_swz[1])  # row 0, K block 1 of the first atom

    # row-wise kernel (amax pass included)
    q, status = gpu_quantize(x, *recipe)
    assert status == nv.OK
    assert block1(to_np(q.codes)[0], to_np(q.scales)) == (case["codes"], case["scale"])
    assert_quant_equal(q, x, *recipe)
    # static alpha: the quantize kernel alone, at the golden tensor's alpha
    qs = nv.quantize(x.cuda(), case["mode"], case["rule"], global_scale=q.global_scale.clone())
    assert nv.device_status(qs.workspace) == nv.OK
    assert block1(to_np(qs.codes)[0], to_np(qs.scales)) == (case["codes"], case["scale"])
    # column-wise kernel: the golden row as column 0 of a 64 x 8 matrix
    xt = torch.zeros(64, 8, dtype=torch.bfloat16)
    xt[:, 0] = x[0]
    qt = nv.quantize_t(xt.cuda(), *recipe)
    assert nv.device_status(qt.workspace) == nv.OK
    assert block1(to_np(qt.codes)[0], to_np(qt.scales)) == (case["codes"], case["scale"])
    # augmented-channel kernel with the identity order and no extra channels
    perm = torch.arange(64, dtype=torch.int32, device="cuda")
    qa = nv.quantize_arc(x.cuda(), perm, 0, nv.AUG_RESIDUAL, *recipe)
    assert nv.device_status(qa.workspace) == nv.OK
    assert block1(to_np(qa.codes)[0], to_np(qa.scales)) == (case["codes"], case["scale"])
