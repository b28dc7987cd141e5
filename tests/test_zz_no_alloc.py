"""nvfp4_quantize_noalloc, the workspace-free quantizer entry point for
callers that cannot allocate device memory where they quantize (an op hook
inside another runtime that owns all device memory, or a service that must
not allocate on its request path).  It is called through the C ABI and must
reproduce nvfp4_quantize bit for bit -- the quantizer's parity tolerance --
on two calls in a row, so stale contents of the shared static scratch from the
first call cannot leak into the second.

This file is collected last on purpose: a run that stops at the first failure
has already run every other test.  It also passes alone in a fresh process
(the first call performs the per-device scratch lookup)."""
import pytest
import torch

import workloads
import w4a4_gemm_nvfp4_b200 as nv

pytestmark = pytest.mark.gpu


def _outputs(rows, K):
    return (torch.full((rows, K // 2), 0x5A, dtype=torch.uint8, device="cuda"),
            torch.full((nv.nvfp4_scales_bytes(rows, K),), 0x5A, dtype=torch.uint8, device="cuda"),
            torch.full((1,), -3.0, dtype=torch.float32, device="cuda"))


def _noalloc(x, mode, rule, fp8_max):
    rows, K = x.shape
    codes, scales, gs = _outputs(rows, K)
    st = nv.nvfp4_quantize_noalloc(x.data_ptr(), rows, K, x.stride(0), nv.MODES[mode], nv.RULES[rule],
                                   fp8_max, codes.data_ptr(), scales.data_ptr(), gs.data_ptr(),
                                   torch.cuda.current_stream().cuda_stream)
    assert st == nv.OK, nv.last_error_message()
    return codes, scales, gs


def test_noalloc_matches_workspace_entry_point_twice():
    cases = [
        (workloads.sweep_operand(1000, 768, seed=21).make(), "four_over_six", "mse", 256.0),
        (workloads.small_operand(333, 2048, seed=22, kind="normal").make(), "six", "max", 448.0),
    ]
    for x_cpu, mode, rule, F in cases:
        x = x_cpu.cuda()
        codes, scales, gs = _noalloc(x, mode, rule, F)
        ref = nv.quantize(x, mode, rule, F)
        torch.cuda.synchronize()
        assert nv.device_status(ref.workspace) == nv.OK
        assert torch.equal(codes, ref.codes)
        assert torch.equal(scales, ref.scales)
        assert torch.equal(gs, ref.global_scale)
