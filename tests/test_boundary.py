"""The C-ABI boundary on a machine without a GPU: libnvfp4.so loads, exports
every function include/*.h declares, computes buffer sizes, and rejects bad
arguments on the host before touching any device."""
import ctypes
import os
import re

import pytest

import w4a4_gemm_nvfp4_b200 as nv
from w4a4_gemm_nvfp4_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names |= set(re.findall(r"NVFP4_API\s+[\w\s\*]+?\b(nvfp4_\w+)\s*\(", text))
    return sorted(names)


def test_headers_declare_the_boundary():
    names = _declared_functions()
    for required in ("nvfp4_quantize", "nvfp4_gemm", "nvfp4_get_device_status",
                     "nvfp4_codes_bytes", "nvfp4_scales_bytes", "nvfp4_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = nv.load()
    for name in _declared_functions():
        assert hasattr(lib, name), name
        assert name in _lib._SIGNATURES, f"binding lacks {name}"


def test_sizes():
    assert nv.nvfp4_codes_bytes(64, 512) == 64 * 256
    assert nv.nvfp4_scales_bytes(64, 512) == 128 * 32
    assert nv.nvfp4_scales_bytes(129, 128) == 256 * 8
    assert nv.nvfp4_scales_bytes(32768, 5120) == 32768 * 320
    assert nv.nvfp4_gemm_workspace_bytes() >= 8
    assert nv.nvfp4_quantize_workspace_bytes(1, 64) >= 64
    assert nv.nvfp4_codes_bytes(0, 64) == 0


def test_status_strings():
    assert nv.status_string(nv.OK) == "NVFP4_OK"
    assert nv.status_string(nv.ERR_TIMEOUT) == "NVFP4_ERR_TIMEOUT"
    assert nv.status_string(99) == "NVFP4_ERR_UNKNOWN"


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first


def _q(**kw):
    args = dict(x=FAKE, rows=64, K=512, ldx=512, mode=0, rule=0, fp8_max=448.0, codes=FAKE,
                scales=FAKE, global_scale=FAKE, workspace=FAKE, workspace_bytes=1 << 20, stream=None)
    args.update(kw)
    return nv.nvfp4_quantize(*args.values())


@pytest.mark.parametrize("bad", [
    dict(x=None), dict(codes=None), dict(scales=None), dict(global_scale=None), dict(workspace=None),
    dict(rows=0), dict(K=0), dict(K=48), dict(K=96), dict(ldx=256), dict(ldx=516),
    dict(mode=2), dict(rule=3), dict(rule=-1), dict(fp8_max=300.0), dict(fp8_max=0.0),
    dict(x=FAKE + 8), dict(codes=FAKE + 4), dict(global_scale=FAKE + 2), dict(workspace_bytes=16),
])
def test_quantize_rejects_bad_arguments(bad):
    assert _q(**bad) == nv.ERR_INVALID_ARG
    assert nv.last_error_message()


def _qn(**kw):
    args = dict(x=FAKE, rows=64, K=512, ldx=512, mode=1, rule=2, fp8_max=256.0, codes=FAKE,
                scales=FAKE, global_scale=FAKE, stream=None)
    args.update(kw)
    return nv.nvfp4_quantize_noalloc(*args.values())


@pytest.mark.parametrize("bad", [
    dict(x=None), dict(codes=None), dict(scales=None), dict(global_scale=None), dict(rows=0),
    dict(K=48), dict(ldx=256), dict(ldx=516), dict(mode=2), dict(rule=3), dict(fp8_max=300.0),
    dict(x=FAKE + 8), dict(scales=FAKE + 4), dict(global_scale=FAKE + 2),
    dict(rows=1 << 31, K=1024, ldx=1024),
])
def test_quantize_noalloc_rejects_bad_arguments(bad):
    assert _qn(**bad) == nv.ERR_INVALID_ARG
    assert nv.last_error_message()


@pytest.mark.parametrize("rows,K,ldx", [(1 << 31, 1024, 1024), (1 << 30, 64, 1 << 11), ((1 << 62), 64, 64)])
def test_oversized_tensors_are_rejected(rows, K, ldx):
    """More than 2^40 elements of x (rows * ldx), including products that
    would overflow 64 bits, are an argument error, not a launch."""
    assert _q(rows=rows, K=K, ldx=ldx) == nv.ERR_INVALID_ARG
    assert "too large" in nv.last_error_message()
    assert _qs(rows=rows, K=K, ldx=ldx) == nv.ERR_INVALID_ARG


def _qt(**kw):
    args = dict(x=FAKE, rows=128, K=72, ldx=72, mode=1, rule=2, fp8_max=256.0, codes=FAKE,
                scales=FAKE, global_scale=FAKE, workspace=FAKE, workspace_bytes=1 << 20, stream=None)
    args.update(kw)
    return nv.nvfp4_quantize_t(*args.values())


@pytest.mark.parametrize("bad", [
    dict(x=None), dict(codes=None), dict(rows=0), dict(rows=32), dict(rows=100), dict(K=0), dict(K=12),
    dict(ldx=64), dict(ldx=76), dict(mode=5), dict(rule=7), dict(fp8_max=100.0), dict(x=FAKE + 8),
    dict(workspace_bytes=16),
])
def test_quantize_t_rejects_bad_arguments(bad):
    assert _qt(**bad) == nv.ERR_INVALID_ARG


def _qa(**kw):
    args = dict(x=FAKE, rows=64, K=512, ldx=512, perm=FAKE, S=64, augment=0, mode=1, rule=2, fp8_max=256.0,
                codes=FAKE, scales=FAKE, global_scale=FAKE, workspace=FAKE, workspace_bytes=1 << 20,
                stream=None)
    args.update(kw)
    return nv.nvfp4_quantize_arc(*args.values())


@pytest.mark.parametrize("bad", [
    dict(perm=None), dict(perm=FAKE + 2), dict(S=-64), dict(S=32), dict(S=576), dict(K=16448, ldx=16448),
    dict(augment=2), dict(x=None), dict(K=48), dict(mode=3), dict(fp8_max=1.0),
])
def test_quantize_arc_rejects_bad_arguments(bad):
    assert _qa(**bad) == nv.ERR_INVALID_ARG


def _qs(**kw):
    args = dict(x=FAKE, rows=64, K=512, ldx=512, mode=1, rule=2, global_scale=FAKE, codes=FAKE,
                scales=FAKE, workspace=FAKE, workspace_bytes=64, stream=None)
    args.update(kw)
    return nv.nvfp4_quantize_with_scale(*args.values())


@pytest.mark.parametrize("bad", [
    dict(x=None), dict(codes=None), dict(scales=None), dict(global_scale=None), dict(workspace=None),
    dict(rows=0), dict(K=48), dict(ldx=256), dict(ldx=516), dict(mode=2), dict(rule=3),
    dict(x=FAKE + 8), dict(scales=FAKE + 4), dict(global_scale=FAKE + 2), dict(workspace_bytes=16),
])
def test_quantize_with_scale_rejects_bad_arguments(bad):
    assert _qs(**bad) == nv.ERR_INVALID_ARG
    assert nv.last_error_message()


def _g(**kw):
    args = dict(a_codes=FAKE, a_scales=FAKE, a_global=FAKE, b_codes=FAKE, b_scales=FAKE,
                b_global=FAKE, M=64, N=256, K=512, y=FAKE, ldy=256, out_dtype=0, workspace=FAKE,
                workspace_bytes=64, stream=None)
    args.update(kw)
    return nv.nvfp4_gemm(*args.values())


@pytest.mark.parametrize("bad", [
    dict(a_codes=None), dict(b_scales=None), dict(y=None), dict(workspace=None), dict(M=0),
    dict(N=-1), dict(K=32), dict(K=100), dict(ldy=128), dict(ldy=255), dict(out_dtype=2),
    dict(y=FAKE + 1), dict(a_global=FAKE + 1), dict(workspace_bytes=4),
    dict(M=1 << 31), dict(N=1 << 31, ldy=1 << 31), dict(K=1 << 31), dict(ldy=(1 << 40) + 1), dict(ldy=1 << 62),
])
def test_gemm_rejects_bad_arguments(bad):
    assert _g(**bad) == nv.ERR_INVALID_ARG


def _gq(**kw):
    args = dict(a_codes=FAKE, a_scales=FAKE, a_global=FAKE, b_codes=FAKE, b_scales=FAKE, b_global=FAKE,
                M=64, N=256, K=512, mode=1, rule=2, y_alpha=FAKE, y_codes=FAKE, y_scales=FAKE, workspace=FAKE,
                workspace_bytes=64, stream=None)
    args.update(kw)
    return nv.nvfp4_gemm_quantized(*args.values())


@pytest.mark.parametrize("bad", [
    dict(y_alpha=None), dict(y_codes=None), dict(y_scales=None), dict(N=96), dict(mode=4), dict(rule=9),
    dict(y_codes=FAKE + 8), dict(y_alpha=FAKE + 1), dict(K=100), dict(M=0),
])
def test_gemm_quantized_rejects_bad_arguments(bad):
    assert _gq(**bad) == nv.ERR_INVALID_ARG


def _gs(ends=(256,), nseg=None, **kw):
    import ctypes as C
    arr = (C.c_int64 * max(1, len(ends)))(*ends)
    args = dict(a_codes=FAKE, a_scales=FAKE, a_global=FAKE, b_codes=FAKE, b_scales=FAKE,
                b_globals=FAKE, seg_ends=C.addressof(arr), nseg=len(ends) if nseg is None else nseg,
                M=64, N=256, K=512, y=FAKE, ldy=256, out_dtype=0, workspace=FAKE,
                workspace_bytes=64, stream=None)
    args.update(kw)
    return nv.nvfp4_gemm_segmented(*args.values())


@pytest.mark.parametrize("ends,nseg,kw", [
    ((256,), 0, {}), (tuple(range(64, 64 * 18, 64)), None, dict(N=64 * 17, ldy=64 * 17)), ((128, 100), None, {}),
    ((100, 256), None, {}), ((128, 128, 256), None, {}), ((192, 128), None, {}), ((128,), None, {}),
    ((256,), None, dict(seg_ends=None)), ((256,), None, dict(b_globals=None)),
    ((256,), None, dict(b_globals=FAKE + 2)),
])
def test_gemm_segmented_rejects_bad_arguments(ends, nseg, kw):
    assert _gs(ends, nseg, **kw) == nv.ERR_INVALID_ARG


def test_no_gpu_fails_loudly():
    """Valid arguments without a usable sm_100 device: an error status, never a
    silent fallback."""
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _q() in (nv.ERR_CUDA, nv.ERR_UNSUPPORTED_DEVICE)
    assert _qs() in (nv.ERR_CUDA, nv.ERR_UNSUPPORTED_DEVICE)
    assert _qt() in (nv.ERR_CUDA, nv.ERR_UNSUPPORTED_DEVICE)
    assert _qa() in (nv.ERR_CUDA, nv.ERR_UNSUPPORTED_DEVICE)
    assert _gq() in (nv.ERR_CUDA, nv.ERR_UNSUPPORTED_DEVICE)
    assert _gs((64, 128, 256)) in (nv.ERR_CUDA, nv.ERR_UNSUPPORTED_DEVICE)
    assert _g() in (nv.ERR_CUDA, nv.ERR_UNSUPPORTED_DEVICE)
    assert _g(ldy=1 << 40) in (nv.ERR_CUDA, nv.ERR_UNSUPPORTED_DEVICE)  # the largest legal row pitch
    assert _qn() in (nv.ERR_CUDA, nv.ERR_UNSUPPORTED_DEVICE)


def _qg(**kw):
    args = dict(x=FAKE, M=64, K=512, ldx=512, mode=1, rule=2, fp8_max=256.0, x_codes=FAKE, x_scales=FAKE,
                x_global_scale=FAKE, x_workspace=FAKE, x_workspace_bytes=1 << 20, w_codes=FAKE, w_scales=FAKE,
                w_global=FAKE, N=256, y=FAKE, ldy=256, out_dtype=0, workspace=FAKE, workspace_bytes=64,
                stream=None)
    args.update(kw)
    return nv.nvfp4_quantize_gemm(*args.values())


@pytest.mark.parametrize("bad", [
    # the quantize half
    dict(x=None), dict(x_codes=None), dict(x_global_scale=None), dict(x_workspace=None), dict(M=0), dict(K=96),
    dict(ldx=256), dict(mode=2), dict(rule=5), dict(fp8_max=100.0), dict(x_workspace_bytes=16),
    # the GEMM half
    dict(w_codes=None), dict(w_scales=None), dict(w_global=None), dict(y=None), dict(workspace=None), dict(N=0),
    dict(ldy=128), dict(out_dtype=3), dict(y=FAKE + 1), dict(workspace_bytes=4), dict(w_global=FAKE + 2),
])
def test_quantize_gemm_rejects_bad_arguments(bad):
    assert _qg(**bad) == nv.ERR_INVALID_ARG
    assert nv.last_error_message().startswith("nvfp4_quantize_gemm")


def test_quantize_gemm_without_gpu_fails_loudly():
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _qg() in (nv.ERR_CUDA, nv.ERR_UNSUPPORTED_DEVICE)


def _qag(**kw):
    args = dict(x=FAKE, M=64, K=512, ldx=512, perm=FAKE, S=128, mode=1, rule=2, fp8_max=256.0, x_codes=FAKE,
                x_scales=FAKE, x_global_scale=FAKE, x_workspace=FAKE, x_workspace_bytes=1 << 20, w_codes=FAKE,
                w_scales=FAKE, w_global=FAKE, N=256, y=FAKE, ldy=256, out_dtype=0, workspace=FAKE,
                workspace_bytes=64, stream=None)
    args.update(kw)
    return nv.nvfp4_quantize_arc_gemm(*args.values())


@pytest.mark.parametrize("bad", [
    # the augmented quantize half
    dict(x=None), dict(perm=None), dict(perm=FAKE + 2), dict(S=32), dict(S=576), dict(S=-64), dict(M=0),
    dict(K=96), dict(K=16448, ldx=16448), dict(ldx=256), dict(mode=2), dict(rule=5), dict(fp8_max=100.0),
    dict(x_workspace_bytes=16), dict(x_codes=None),
    # the GEMM half (over K + S)
    dict(w_codes=None), dict(w_global=None), dict(y=None), dict(N=0), dict(ldy=128), dict(out_dtype=3),
    dict(workspace_bytes=4),
])
def test_quantize_arc_gemm_rejects_bad_arguments(bad):
    assert _qag(**bad) == nv.ERR_INVALID_ARG
    assert nv.last_error_message().startswith("nvfp4_quantize_arc_gemm")


def test_quantize_arc_gemm_without_gpu_fails_loudly():
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _qag() in (nv.ERR_CUDA, nv.ERR_UNSUPPORTED_DEVICE)


def _qar(**kw):
    args = dict(x=FAKE, rows=64, K=512, ldx=512, gamma=FAKE, eps=1e-6, perm=FAKE, S=128, mode=1, rule=2,
                fp8_max=256.0, codes=FAKE, scales=FAKE, global_scale=FAKE, workspace=FAKE,
                workspace_bytes=1 << 20, stream=None)
    args.update(kw)
    return nv.nvfp4_quantize_arc_rmsnorm(*args.values())


@pytest.mark.parametrize("bad", [
    dict(gamma=None), dict(gamma=FAKE + 1), dict(gamma=FAKE + 8), dict(eps=0.0), dict(eps=-1e-6), dict(eps=float("inf")),
    dict(eps=float("nan")), dict(x=None), dict(perm=None), dict(S=32), dict(S=576), dict(K=96),
    dict(K=16448, ldx=16448), dict(mode=2), dict(fp8_max=100.0), dict(workspace=None),
    dict(workspace_bytes=16), dict(rows=4096, workspace_bytes=16448 + 4 * 4096 - 1),
])
def test_quantize_arc_rmsnorm_rejects_bad_arguments(bad):
    assert _qar(**bad) == nv.ERR_INVALID_ARG
    assert nv.last_error_message().startswith("nvfp4_quantize_arc_rmsnorm")


def test_quantize_arc_rmsnorm_workspace_holds_a_float_per_row_and_the_gains():
    """The quantize workspace, then a float per row and a bf16 gain per channel,
    each area rounded up to 16 bytes."""
    def up16(n):
        return (n + 15) // 16 * 16
    for rows, K in ((4096, 512), (3, 64), (1, 5120), (77, 16384)):
        assert (nv.nvfp4_quantize_arc_rmsnorm_workspace_bytes(rows, K)
                == nv.nvfp4_quantize_workspace_bytes(rows, K) + up16(4 * rows) + up16(2 * K))


def test_quantize_arc_rmsnorm_without_gpu_fails_loudly():
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _qar() in (nv.ERR_CUDA, nv.ERR_UNSUPPORTED_DEVICE)


def _qarg(**kw):
    args = dict(x=FAKE, M=64, K=512, ldx=512, gamma=FAKE, eps=1e-6, perm=FAKE, S=128, mode=1, rule=2,
                fp8_max=256.0, x_codes=FAKE, x_scales=FAKE, x_global_scale=FAKE, x_workspace=FAKE,
                x_workspace_bytes=1 << 20, w_codes=FAKE, w_scales=FAKE, w_global=FAKE, N=256, y=FAKE, ldy=256,
                out_dtype=0, workspace=FAKE, workspace_bytes=64, stream=None)
    args.update(kw)
    return nv.nvfp4_quantize_arc_rmsnorm_gemm(*args.values())


@pytest.mark.parametrize("bad", [
    dict(gamma=None), dict(gamma=FAKE + 8), dict(eps=0.0), dict(eps=float("nan")), dict(perm=None), dict(S=32),
    dict(K=96), dict(x_workspace_bytes=16448), dict(w_codes=None), dict(N=0), dict(ldy=128), dict(out_dtype=3),
    dict(workspace_bytes=4),
])
def test_quantize_arc_rmsnorm_gemm_rejects_bad_arguments(bad):
    assert _qarg(**bad) == nv.ERR_INVALID_ARG
    assert nv.last_error_message().startswith("nvfp4_quantize_arc_rmsnorm_gemm")


def test_quantize_arc_rmsnorm_gemm_without_gpu_fails_loudly():
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _qarg() in (nv.ERR_CUDA, nv.ERR_UNSUPPORTED_DEVICE)
