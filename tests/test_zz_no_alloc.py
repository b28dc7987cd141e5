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



_CONTEXT_CHILD = r'''
import ctypes, os, sys
import numpy as np
sys.path.insert(0, os.environ["NVFP4_ROOT"])
import torch  # CPU only: makes the input
import workloads
import w4a4_gemm_nvfp4_b200._lib as L

lib = L.load()
cu = ctypes.CDLL("libcuda.so.1")
P, U64 = ctypes.c_void_p, ctypes.c_uint64

def check(r, what):
    assert r == 0, f"{what}: CUresult {r}"

x = workloads.sweep_operand(300, 512, seed=23).make()
xb = np.ascontiguousarray(x.view(torch.int16).numpy().view(np.uint16))
rows, K = xb.shape

def run_in_current_context():
    """This test allocates its own buffers with the driver API in the current
    context; the entry point under test allocates nothing."""
    sizes = {"x": xb.nbytes, "codes": rows * K // 2, "scales": L.nvfp4_scales_bytes(rows, K), "gs": 4,
             "codes2": rows * K // 2, "scales2": L.nvfp4_scales_bytes(rows, K), "gs2": 4,
             "ws": L.nvfp4_quantize_workspace_bytes(rows, K)}
    bufs = {}
    for k, n in sizes.items():
        p = U64()
        check(cu.cuMemAlloc_v2(ctypes.byref(p), ctypes.c_size_t(n)), "cuMemAlloc")
        bufs[k] = p.value
    check(cu.cuMemcpyHtoD_v2(U64(bufs["x"]), xb.ctypes.data_as(P), ctypes.c_size_t(xb.nbytes)), "HtoD")
    st = lib.nvfp4_quantize_noalloc(bufs["x"], rows, K, K, 1, 2, 256.0, bufs["codes"], bufs["scales"],
                                    bufs["gs"], None)
    assert st == 0, L.last_error_message()
    st = lib.nvfp4_quantize(bufs["x"], rows, K, K, 1, 2, 256.0, bufs["codes2"], bufs["scales2"], bufs["gs2"],
                            bufs["ws"], sizes["ws"], None)
    assert st == 0, L.last_error_message()
    check(cu.cuCtxSynchronize(), "cuCtxSynchronize")
    out = {}
    for k in ("codes", "scales", "gs", "codes2", "scales2", "gs2"):
        h = np.empty(sizes[k], np.uint8)
        check(cu.cuMemcpyDtoH_v2(h.ctypes.data_as(P), U64(bufs[k]), ctypes.c_size_t(sizes[k])), "DtoH")
        out[k] = h
    for p in bufs.values():
        check(cu.cuMemFree_v2(U64(p)), "cuMemFree")
    for k in ("codes", "scales", "gs"):
        assert np.array_equal(out[k], out[k + "2"]), k
    return out

check(cu.cuInit(0), "cuInit")
dev = ctypes.c_int()
check(cu.cuDeviceGet(ctypes.byref(dev), 0), "cuDeviceGet")
primary = P()
check(cu.cuDevicePrimaryCtxRetain(ctypes.byref(primary), dev), "cuDevicePrimaryCtxRetain")
check(cu.cuCtxSetCurrent(primary), "cuCtxSetCurrent")
first = run_in_current_context()
other = P()
check(cu.cuCtxCreate_v2(ctypes.byref(other), 0, dev), "cuCtxCreate")   # current from here on
second = run_in_current_context()
check(cu.cuCtxSetCurrent(primary), "cuCtxSetCurrent")
third = run_in_current_context()
check(cu.cuCtxDestroy_v2(other), "cuCtxDestroy")
check(cu.cuDevicePrimaryCtxRelease_v2(dev), "cuDevicePrimaryCtxRelease")
for out in (second, third):
    for k in ("codes", "scales", "gs"):
        assert np.array_equal(first[k], out[k]), k
print("OK")
'''


def test_noalloc_follows_the_current_context():
    """The static scratch array exists once per CUDA context that loaded the
    library's module, at a different address in each.  A caller that switches
    contexts (here: the primary context, a second context created with the
    driver API, then the primary one again) gets the array of the current
    context on every call, and the result still matches nvfp4_quantize.  Runs
    in a child process that drives the contexts through the CUDA driver API
    (torch only makes the input there, on the CPU), so no CUDA state of this
    process is disturbed."""
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {**os.environ, "NVFP4_ROOT": root}
    r = subprocess.run([sys.executable, "-c", _CONTEXT_CHILD], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0 and r.stdout.strip().endswith("OK"), r.stdout[-2000:] + r.stderr[-2000:]
