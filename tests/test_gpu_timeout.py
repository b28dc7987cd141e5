"""Failure detection in the GEMM without faulting or hanging the GPU: a test
hook keeps the first pipeline stage from ever being filled, so the MMA
issuer's bounded wait runs out.  The kernel must record NVFP4_ERR_TIMEOUT in
the workspace status word, drain its in-flight copies, free TMEM and return;
the CUDA context must stay usable, and the next call with the hook cleared
must produce the right result."""
import time

import numpy as np
import pytest
import torch

import oracle
import workloads
import w4a4_gemm_nvfp4_b200 as nv
from gpu_util import MODE, RULE, assert_gemm_close, to_np, upload_operand

pytestmark = pytest.mark.gpu


def _operands(M, N, K):
    xa = workloads.small_operand(M, K, seed=31).make()
    xb = workloads.small_operand(N, K, seed=32, kind="normal").make()
    ac, as_, aa = oracle.quantize(xa, MODE["four_over_six"], RULE["mse"], 256.0)
    bc, bs, ba = oracle.quantize(xb, MODE["six"], RULE["max"], 448.0)
    return (ac, as_, aa), (bc, bs, ba)


@pytest.mark.parametrize("M,N,K", [(256, 256, 1024), (512, 768, 4096)])
def test_bounded_wait_reports_timeout_and_context_survives(M, N, K):
    (ac, as_, aa), (bc, bs, ba) = _operands(M, N, K)
    A, B = upload_operand(ac, as_, aa), upload_operand(bc, bs, ba)
    ws = torch.zeros(nv.nvfp4_gemm_workspace_bytes(), dtype=torch.uint8, device="cuda")
    y = torch.full((M, N), 7.0, dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    nv.testing_set_gemm_wait(50_000_000, 1)  # 50 ms deadline, first stage never filled
    try:
        t0 = time.perf_counter()
        nv.gemm(A, B, out_dtype=torch.float32, out=y, workspace=ws)
        status = nv.device_status(ws)
        elapsed = time.perf_counter() - t0
    finally:
        nv.testing_set_gemm_wait(0, 0)
    assert status == nv.ERR_TIMEOUT
    assert elapsed < 5.0
    # the context still works: the same call without the hook is correct
    nv.gemm(A, B, out_dtype=torch.float32, out=y, workspace=ws)
    assert nv.device_status(ws) == nv.OK
    ref, guard = oracle.gemm_reference(ac, as_, aa, bc, bs, ba)
    assert_gemm_close(to_np(y), ref, guard)


def test_timeout_bounds_lack_of_progress_not_run_time():
    """Every bounded wait gets the whole timeout from when it starts, so a GEMM
    that runs several times longer than the timeout, with every wait making
    progress, completes with NVFP4_OK and the right result (sampled rows and
    columns against the oracle)."""
    M, N, K = 32768, 8192, 8192          # 4.4 TFLOP: about 0.9 ms on a B200
    timeout_ns = 200_000                  # 0.2 ms per wait
    g = np.random.default_rng(41)
    ac = g.integers(0, 256, (M, K // 2), dtype=np.uint8)
    bc = g.integers(0, 256, (N, K // 2), dtype=np.uint8)
    as_ = g.integers(0x28, 0x48, (M, K // 16), dtype=np.uint8)   # E4M3 scales 2^-2 .. 2^2
    bs = g.integers(0x28, 0x48, (N, K // 16), dtype=np.uint8)
    A, B = upload_operand(ac, as_, 0.75), upload_operand(bc, bs, 1.25)
    ws = torch.zeros(nv.nvfp4_gemm_workspace_bytes(), dtype=torch.uint8, device="cuda")
    y = torch.empty(M, N, dtype=torch.float32, device="cuda")
    nv.gemm(A, B, out_dtype=torch.float32, out=y, workspace=ws)   # warm-up at the default timeout
    assert nv.device_status(ws) == nv.OK
    nv.testing_set_gemm_wait(timeout_ns, 0)
    try:
        y.fill_(7.0)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        nv.gemm(A, B, out_dtype=torch.float32, out=y, workspace=ws)
        e1.record()
        status = nv.device_status(ws)
        ms = e0.elapsed_time(e1)
    finally:
        nv.testing_set_gemm_wait(0, 0)
    assert status == nv.OK
    assert ms * 1e6 > 2 * timeout_ns, f"the GEMM took {ms} ms: too short to show the timeout is per wait"
    rows = g.choice(M, 48, replace=False)
    cols = g.choice(N, 320, replace=False)
    ref, guard = oracle.gemm_reference(ac[rows], as_[rows], 0.75, bc[cols], bs[cols], 1.25)
    assert_gemm_close(to_np(y)[np.ix_(rows, cols)], ref, guard)
