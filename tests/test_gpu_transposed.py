"""Parity of nvfp4_quantize_t (the NVFP4 operand of x^T: 16-element blocks
running down the columns of x) with the oracle applied to the transposed
matrix, and of a GEMM on two such operands (an A^T.B product, as in a
weight-gradient GEMM) with the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import w4a4_gemm_nvfp4_b200 as nv
from gpu_util import MODE, RULE, assert_gemm_close, to_np

pytestmark = pytest.mark.gpu

RECIPES = [("six", "max", 448.0), ("four_over_six", "max", 256.0), ("four_over_six", "mae", 256.0),
           ("four_over_six", "mse", 256.0), ("six", "max", 256.0)]
SHAPES = [(64, 8), (64, 64), (128, 200), (192, 320), (320, 1000), (1024, 136), (256, 1032)]


def gpu_quantize_t(x_cpu, mode, rule, F, ldx_pad=0, canary=0xA5):
    rows, K = x_cpu.shape
    if ldx_pad:
        big = torch.zeros(rows, K + ldx_pad, dtype=torch.bfloat16)
        big[:, :K] = x_cpu
        xd = big.cuda()[:, :K]
    else:
        xd = x_cpu.cuda()
    out = nv.NVFP4Tensor(
        codes=torch.full((K, rows // 2), canary, dtype=torch.uint8, device="cuda"),
        scales=torch.full((nv.nvfp4_scales_bytes(K, rows),), canary, dtype=torch.uint8, device="cuda"),
        global_scale=torch.full((1,), -1.0, dtype=torch.float32, device="cuda"),
        workspace=torch.full((nv.nvfp4_quantize_workspace_bytes(rows, K),), 0xFF, dtype=torch.uint8,
                             device="cuda"),
        rows=K, K=rows)
    nv.quantize_t(xd, mode, rule, F, out=out)
    return out, nv.device_status(out.workspace)


def assert_t_matches_oracle(q, x_cpu, mode, rule, F):
    xt = x_cpu.t().contiguous()
    Kt, Mt = xt.shape  # rows and K of the transposed operand
    oc, os_, oa = oracle.quantize(xt, MODE[mode], RULE[rule], F)
    assert float(q.global_scale.cpu()[0]) == np.float32(oa)
    gc = to_np(q.codes)
    bad = np.argwhere(gc != oc)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first {bad[:5].tolist()}"
    gs = to_np(q.scales)
    swz = oracle.swizzle_scales(os_, Kt, Mt)
    bad = np.nonzero(gs != swz)[0]
    assert bad.size == 0, f"{bad.size} scale bytes differ, first {bad[:5].tolist()}"


@pytest.mark.parametrize("recipe", RECIPES, ids=lambda r: "-".join(map(str, r)))
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"{s[0]}x{s[1]}")
def test_quantize_t_matches_oracle(shape, recipe):
    x = workloads.small_operand(*shape, seed=shape[0] + 5 * shape[1], kind="t").make()
    q, st = gpu_quantize_t(x, *recipe)
    assert st == nv.OK
    assert_t_matches_oracle(q, x, *recipe)


def test_quantize_t_strided_and_outlier_columns():
    x = workloads.small_operand(384, 264, seed=3, kind="t").make()
    x[:, ::37] *= 40
    for pad in (8, 64):
        q, st = gpu_quantize_t(x, "four_over_six", "mse", 256.0, ldx_pad=pad)
        assert st == nv.OK
        assert_t_matches_oracle(q, x, "four_over_six", "mse", 256.0)


def test_quantize_t_nonfinite():
    x = workloads.small_operand(128, 64, seed=1).make()
    x[7, 9] = float("nan")
    q, st = gpu_quantize_t(x, "six", "max", 448.0)
    assert st == nv.ERR_NONFINITE


def test_gemm_on_transposed_operands():
    """Y = A^T . B for A [M, K1], B [M, K2], both quantized along M."""
    M, K1, K2 = 512, 192, 320
    a = workloads.small_operand(M, K1, seed=11, kind="t").make()
    b = workloads.small_operand(M, K2, seed=12, kind="normal").make()
    qa = nv.quantize_t(a.cuda(), "four_over_six", "mse", 256.0)
    qb = nv.quantize_t(b.cuda(), "six", "max", 448.0)
    y = nv.gemm(qa, qb, out_dtype=torch.float32)
    ac, as_, aa = oracle.quantize(a.t().contiguous(), MODE["four_over_six"], RULE["mse"], 256.0)
    bc, bs, ba = oracle.quantize(b.t().contiguous(), MODE["six"], RULE["max"], 448.0)
    ref, guard = oracle.gemm_reference(ac, as_, aa, bc, bs, ba)
    assert_gemm_close(to_np(y), ref, guard)
