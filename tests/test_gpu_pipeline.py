"""The one-call linear layer (nvfp4_quantize_gemm through the C ABI): the
quantize and GEMM kernels start as programmatic dependents of the kernel
before them, and the results must be those of nvfp4_quantize followed by
nvfp4_gemm, bit for bit -- eagerly and replayed from a CUDA graph."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import w4a4_gemm_nvfp4_b200 as nv
from gpu_util import MODE, RULE, assert_gemm_close, to_np

pytestmark = pytest.mark.gpu

CASES = [(64, 512, 256, ("four_over_six", "mse", 256.0), torch.float32),
         (300, 1024, 384, ("six", "max", 448.0), torch.bfloat16),
         (1000, 5120, 640, ("four_over_six", "mae", 256.0), torch.bfloat16),
         (129, 2048, 1000, ("four_over_six", "max", 256.0), torch.float32)]


def _operands(M, K, N, seed):
    x = workloads.small_operand(M, K, seed=seed).make().cuda()
    w = workloads.small_operand(N, K, seed=seed + 1, kind="normal").make().cuda()
    return x, nv.quantize(w, "six", "max", 448.0)


@pytest.mark.parametrize("M,K,N,recipe,dtype", CASES, ids=lambda v: str(v))
def test_quantize_gemm_equals_the_two_calls(M, K, N, recipe, dtype):
    x, qw = _operands(M, K, N, seed=M + K)
    mode, rule, F = recipe
    qx_ref = nv.quantize(x, mode, rule, F)
    y_ref = nv.gemm(qx_ref, qw, out_dtype=dtype)
    ws = torch.zeros(nv.nvfp4_gemm_workspace_bytes(), dtype=torch.uint8, device="cuda")
    qx, y = nv.quantize_gemm(x, qw, mode, rule, F, out_dtype=dtype, workspace=ws)
    torch.cuda.synchronize()
    assert nv.device_status(qx.workspace) == nv.OK and nv.device_status(ws) == nv.OK
    assert torch.equal(qx.codes, qx_ref.codes) and torch.equal(qx.scales, qx_ref.scales)
    assert torch.equal(qx.global_scale, qx_ref.global_scale)
    assert torch.equal(y, y_ref)
    # and the oracle, on the first rows
    xc, xs, xa = oracle.quantize(x.cpu(), MODE[mode], RULE[rule], F)
    assert np.array_equal(to_np(qx.codes), xc)
    wc, ws_, wa = oracle.quantize(workloads.small_operand(N, K, seed=M + K + 1, kind="normal").make(),
                                  MODE["six"], RULE["max"], 448.0)
    ref, guard = oracle.gemm_reference(xc[:32], xs[:32], xa, wc, ws_, wa)
    assert_gemm_close(to_np(y.float())[:32], ref, guard, bf16=dtype == torch.bfloat16)


def test_quantize_gemm_in_a_cuda_graph():
    """Captured once, replayed: the programmatic dependencies survive capture,
    replay equals eager, and new activations written into the captured input
    flow through."""
    M, K, N = 512, 2048, 768
    x, qw = _operands(M, K, N, seed=71)
    ws = torch.zeros(nv.nvfp4_gemm_workspace_bytes(), dtype=torch.uint8, device="cuda")
    qx, y = nv.quantize_gemm(x, qw, "four_over_six", "mse", 256.0, out_dtype=torch.bfloat16, workspace=ws)
    torch.cuda.synchronize()
    y_eager = y.clone()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            nv.quantize_gemm(x, qw, "four_over_six", "mse", 256.0, x_out=qx, out=y, workspace=ws)
    torch.cuda.current_stream().wait_stream(s)
    y.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert nv.device_status(qx.workspace) == nv.OK and nv.device_status(ws) == nv.OK
    assert torch.equal(y, y_eager)
    x.copy_(workloads.small_operand(M, K, seed=72).make().cuda())
    g.replay()
    torch.cuda.synchronize()
    qx_ref = nv.quantize(x, "four_over_six", "mse", 256.0)
    assert torch.equal(y, nv.gemm(qx_ref, qw, out_dtype=torch.bfloat16))
    del g


@pytest.mark.parametrize("M,K,N,S,recipe", [(64, 512, 256, 64, ("four_over_six", "mse", 256.0)),
                                           (300, 1024, 384, 128, ("six", "max", 448.0)),
                                           (1000, 5120, 640, 128, ("four_over_six", "mae", 256.0))],
                         ids=lambda v: str(v))
def test_quantize_arc_gemm_equals_the_two_calls(M, K, N, S, recipe):
    """nvfp4_quantize_arc_gemm: the augmented quantizer and the GEMM over K + S
    in one call give the bytes and the Y of nvfp4_quantize_arc (residual)
    followed by nvfp4_gemm, and the augmented operand is the oracle's."""
    mode, rule, F = recipe
    x = workloads.small_operand(M, K, seed=M + S).make().cuda()
    w = workloads.small_operand(N, K, seed=M + S + 1, kind="normal").make().cuda()
    perm = x.float().abs().amax(dim=0).argsort(descending=True).to(torch.int32)
    qw = nv.quantize_arc(w, perm, S, nv.AUG_DUPLICATE, "six", "max", 448.0)
    qx_ref = nv.quantize_arc(x, perm, S, nv.AUG_RESIDUAL, mode, rule, F)
    y_ref = nv.gemm(qx_ref, qw, out_dtype=torch.bfloat16)
    ws = torch.zeros(nv.nvfp4_gemm_workspace_bytes(), dtype=torch.uint8, device="cuda")
    qx, y = nv.quantize_arc_gemm(x, perm, S, qw, mode, rule, F, out_dtype=torch.bfloat16, workspace=ws)
    torch.cuda.synchronize()
    assert nv.device_status(qx.workspace) == nv.OK and nv.device_status(ws) == nv.OK
    assert torch.equal(qx.codes, qx_ref.codes) and torch.equal(qx.scales, qx_ref.scales)
    assert torch.equal(qx.global_scale, qx_ref.global_scale)
    assert torch.equal(y, y_ref)
    codes, scales, alpha = oracle.quantize_arc(x.cpu(), perm.cpu().numpy(), S, oracle.AUG_RESIDUAL, MODE[mode],
                                               RULE[rule], F)
    assert np.array_equal(to_np(qx.codes), codes)
