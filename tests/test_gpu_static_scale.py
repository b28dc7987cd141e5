"""Parity of nvfp4_quantize_with_scale (the tensor scale alpha supplied by the
caller, e.g. calibrated, instead of reduced from the tensor's amax) with the
oracle's row quantizer run at the same alpha: codes and swizzled scales
bit-identical, including alphas small enough to saturate block scales at 448
and codes at 6."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import w4a4_gemm_nvfp4_b200 as nv
from gpu_util import MODE, RULE, gpu_quantize, to_np

pytestmark = pytest.mark.gpu

RECIPES = [("six", "max"), ("four_over_six", "max"), ("four_over_six", "mae"), ("four_over_six", "mse")]


def static_quantize(x_cpu, mode, rule, alpha, ldx_pad=0, canary=0xA5):
    rows, K = x_cpu.shape
    if ldx_pad:
        big = torch.zeros(rows, K + ldx_pad, dtype=torch.bfloat16)
        big[:, :K] = x_cpu
        xd = big.cuda()[:, :K]
    else:
        xd = x_cpu.cuda()
    out = nv.NVFP4Tensor(
        codes=torch.full((rows, K // 2), canary, dtype=torch.uint8, device="cuda"),
        scales=torch.full((nv.nvfp4_scales_bytes(rows, K),), canary, dtype=torch.uint8, device="cuda"),
        global_scale=torch.empty(1, dtype=torch.float32, device="cuda"),
        workspace=torch.full((nv.nvfp4_gemm_workspace_bytes(),), 0xFF, dtype=torch.uint8, device="cuda"),
        rows=rows, K=K)
    a = torch.tensor([alpha], dtype=torch.float32, device="cuda")
    nv.quantize(xd, mode, rule, out=out, global_scale=a)
    return out, nv.device_status(out.workspace)


def assert_matches_rows_oracle(q, x_cpu, mode, rule, alpha):
    rows, K = x_cpu.shape
    oc, os_ = oracle.quantize_rows(x_cpu, alpha, MODE[mode], RULE[rule])
    gc = to_np(q.codes)
    bad = np.argwhere(gc != oc)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first {bad[:5].tolist()}"
    gs = to_np(q.scales)
    swz = oracle.swizzle_scales(os_, rows, K)
    bad = np.nonzero(gs != swz)[0]
    assert bad.size == 0, f"{bad.size} scale bytes differ, first {bad[:5].tolist()}"
    assert float(q.global_scale.cpu()[0]) == np.float32(alpha)


@pytest.mark.parametrize("recipe", RECIPES, ids=lambda r: "-".join(r))
def test_dynamic_alpha_given_back_reproduces_nvfp4_quantize(recipe):
    """Feeding the alpha nvfp4_quantize computed reproduces its output."""
    mode, rule = recipe
    x = workloads.small_operand(300, 320, seed=21, kind="t").make()
    F = nv.DEFAULT_FP8_MAX[mode]
    qd, st = gpu_quantize(x, mode, rule, F)
    assert st == nv.OK
    qs, st = static_quantize(x, mode, rule, float(qd.global_scale.cpu()[0]))
    assert st == nv.OK
    assert torch.equal(qs.codes, qd.codes) and torch.equal(qs.scales, qd.scales)


@pytest.mark.parametrize("recipe", RECIPES, ids=lambda r: "-".join(r))
@pytest.mark.parametrize("factor", [1 / 5.0, 0.37, 1.0, 3.3, 2.0 ** 20])
@pytest.mark.parametrize("shape", [(1, 64), (129, 128), (257, 1024)], ids=lambda s: f"{s[0]}x{s[1]}")
def test_static_alpha_matches_oracle(shape, recipe, factor):
    mode, rule = recipe
    x = workloads.small_operand(*shape, seed=shape[0] + 3 * shape[1], kind="t").make()
    amax, _ = oracle.amax(x)
    alpha = float(np.float32(oracle.global_scale(amax, nv.DEFAULT_FP8_MAX[mode]) * factor))
    q, st = static_quantize(x, mode, rule, alpha)
    assert st == nv.OK
    assert_matches_rows_oracle(q, x, mode, rule, alpha)


def test_static_alpha_strided_rows():
    x = workloads.small_operand(200, 256, seed=5).make()
    q, st = static_quantize(x, "four_over_six", "mse", 0.0021, ldx_pad=64)
    assert st == nv.OK
    assert_matches_rows_oracle(q, x, "four_over_six", "mse", 0.0021)


@pytest.mark.parametrize("alpha", [0.0, -1.0, float("inf"), float("nan"), -0.0])
def test_invalid_alpha_writes_nothing(alpha):
    x = workloads.small_operand(64, 128, seed=2).make()
    q, st = static_quantize(x, "four_over_six", "mse", alpha)
    assert st == nv.ERR_INVALID_ARG
    assert bool((q.codes == 0xA5).all()) and bool((q.scales == 0xA5).all())


@pytest.mark.parametrize("bad", [float("inf"), float("-inf"), float("nan")])
def test_nonfinite_block_is_zeroed_and_reported(bad):
    x = workloads.small_operand(130, 256, seed=8).make()
    x[77, 40] = bad
    alpha = 0.003
    q, st = static_quantize(x, "four_over_six", "mae", alpha)
    assert st == nv.ERR_NONFINITE
    gc, gs = to_np(q.codes), oracle.unswizzle_scales(to_np(q.scales), 130, 256)
    assert (gc[77, 16:24] == 0).all() and gs[77, 2] == 0
    xc = x.clone()
    xc[77, 32:48] = 0.0  # the block the kernel zeroed
    oc, os_ = oracle.quantize_rows(xc, alpha, MODE["four_over_six"], RULE["mae"])
    assert np.array_equal(gc, oc) and np.array_equal(gs, os_)


@pytest.mark.parametrize("recipe", RECIPES, ids=lambda r: "-".join(r))
# the first four make b * fl(1/(6 alpha)) round to another E4M3 scale than
# b / (6 alpha) for some bf16 b (found by search); the last two put quotients
# on or next to E4M3 rounding midpoints
@pytest.mark.parametrize("alpha", [1.220588207244873, 0.6263441443443298, 0.5588235259056091,
                                   0.26644739508628845, 0.0123456789, 1.0 / 6.0])
def test_scale_quotient_near_e4m3_midpoints(recipe, alpha):
    """Blocks whose b / (alpha*Q) lies where a reciprocal-multiply would round
    to a different E4M3 scale than the correctly rounded quotient."""
    from gpu_util import blocks_with_maxima, hard_block_maxima

    mode, rule = recipe
    alpha = float(np.float32(alpha))
    maxima = np.concatenate([hard_block_maxima(alpha, 6.0), hard_block_maxima(alpha, 4.0)])
    if maxima.size == 0:
        pytest.skip("no hard maxima for this alpha")
    x = blocks_with_maxima(maxima, 256, seed=len(maxima))
    q, st = static_quantize(x, mode, rule, alpha)
    assert st == nv.OK
    assert_matches_rows_oracle(q, x, mode, rule, alpha)
