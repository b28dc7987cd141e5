"""ctypes binding of libnvfp4.so (argument marshalling only).

The functions named like the C ABI (``nvfp4_quantize``, ``nvfp4_gemm``, ...)
take raw integers (device pointers, sizes, a cudaStream_t handle) and return
the C status.  ``quantize`` / ``gemm`` wrap them for torch CUDA tensors:
they allocate outputs with torch, check every buffer they are given against
the shape, dtype and device the call reads or writes, pass pointers and the
current stream, and raise ``NVFP4Error`` on a non-OK status.  Every step of the computation runs
in the library's kernels; there is no CPU or PyTorch fallback, and importing
this module on a machine without the built library raises at first use.
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnvfp4.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED_DEVICE, ERR_NONFINITE, ERR_TIMEOUT, ERR_CUDA = range(6)
MODES = {"six": 0, "four_over_six": 1}
RULES = {"max": 0, "mae": 1, "mse": 2}
OUT_BF16, OUT_FP32 = 0, 1
DEFAULT_FP8_MAX = {"six": 448.0, "four_over_six": 256.0}

# name -> (restype, argtypes); every function declared in include/nvfp4.h and
# include/nvfp4_testing.h
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_SIGNATURES = {
    "nvfp4_codes_bytes": (ctypes.c_size_t, [_I64, _I64]),
    "nvfp4_scales_bytes": (ctypes.c_size_t, [_I64, _I64]),
    "nvfp4_quantize_workspace_bytes": (ctypes.c_size_t, [_I64, _I64]),
    "nvfp4_gemm_workspace_bytes": (ctypes.c_size_t, []),
    "nvfp4_quantize": (ctypes.c_int, [_P, _I64, _I64, _I64, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_float, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "nvfp4_quantize_noalloc": (ctypes.c_int, [_P, _I64, _I64, _I64, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_float, _P, _P, _P, _P]),
    "nvfp4_quantize_arc": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _I64, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_float, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "nvfp4_quantize_arc_rmsnorm_workspace_bytes": (ctypes.c_size_t, [_I64, _I64]),
    "nvfp4_quantize_arc_rmsnorm": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, ctypes.c_float, _P, _I64, ctypes.c_int,
                                                  ctypes.c_int, ctypes.c_float, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "nvfp4_quantize_t": (ctypes.c_int, [_P, _I64, _I64, _I64, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_float, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "nvfp4_quantize_with_scale": (ctypes.c_int, [_P, _I64, _I64, _I64, ctypes.c_int, ctypes.c_int,
                                                 _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "nvfp4_gemm": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _I64,
                                  ctypes.c_int, _P, ctypes.c_size_t, _P]),
    "nvfp4_gemm_quantized": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, ctypes.c_int, ctypes.c_int,
                                            _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "nvfp4_gemm_segmented": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, ctypes.c_int, _I64, _I64,
                                            _I64, _P, _I64, ctypes.c_int, _P, ctypes.c_size_t, _P]),
    "nvfp4_quantize_gemm": (ctypes.c_int, [_P, _I64, _I64, _I64, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                           _P, _P, _P, _P, ctypes.c_size_t, _P, _P, _P, _I64, _P, _I64,
                                           ctypes.c_int, _P, ctypes.c_size_t, _P]),
    "nvfp4_quantize_arc_gemm": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _I64, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_float, _P, _P, _P, _P, ctypes.c_size_t, _P, _P, _P, _I64,
                                               _P, _I64, ctypes.c_int, _P, ctypes.c_size_t, _P]),
    "nvfp4_quantize_arc_rmsnorm_gemm": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, ctypes.c_float, _P, _I64,
                                                       ctypes.c_int, ctypes.c_int, ctypes.c_float, _P, _P, _P, _P,
                                                       ctypes.c_size_t, _P, _P, _P, _I64, _P, _I64, ctypes.c_int,
                                                       _P, ctypes.c_size_t, _P]),
    "nvfp4_get_device_status": (ctypes.c_int, [_P, _P]),
    "nvfp4_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "nvfp4_last_error_message": (ctypes.c_char_p, []),
    "nvfp4_testing_set_gemm_wait": (None, [ctypes.c_uint64, ctypes.c_int]),
}

_lock = threading.Lock()
_lib = None


class NVFP4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}: {last_error_message()}")


def load() -> ctypes.CDLL:
    """Load libnvfp4.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(
                    f"{LIB_PATH} is missing: build it with `python -m w4a4_gemm_nvfp4_b200.build`")
            lib = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in _SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


# ------------------------------------------------------- raw C functions --

def nvfp4_codes_bytes(rows: int, K: int) -> int:
    return load().nvfp4_codes_bytes(rows, K)


def nvfp4_scales_bytes(rows: int, K: int) -> int:
    return load().nvfp4_scales_bytes(rows, K)


def nvfp4_quantize_workspace_bytes(rows: int, K: int) -> int:
    return load().nvfp4_quantize_workspace_bytes(rows, K)


def nvfp4_gemm_workspace_bytes() -> int:
    return load().nvfp4_gemm_workspace_bytes()


def nvfp4_quantize(x, rows, K, ldx, mode, rule, fp8_max, codes, scales, global_scale, workspace,
                   workspace_bytes, stream) -> int:
    return load().nvfp4_quantize(x, rows, K, ldx, mode, rule, fp8_max, codes, scales, global_scale,
                                 workspace, workspace_bytes, stream)


def nvfp4_quantize_noalloc(x, rows, K, ldx, mode, rule, fp8_max, codes, scales, global_scale,
                           stream) -> int:
    """nvfp4_quantize with its scratch in a static device array inside the
    library: no workspace argument, nothing allocated (see include/nvfp4.h)."""
    return load().nvfp4_quantize_noalloc(x, rows, K, ldx, mode, rule, fp8_max, codes, scales,
                                         global_scale, stream)


def nvfp4_quantize_arc(x, rows, K, ldx, perm, S, augment, mode, rule, fp8_max, codes, scales,
                       global_scale, workspace, workspace_bytes, stream) -> int:
    """Augmented residual-channel quantization (perm: device int32[K])."""
    return load().nvfp4_quantize_arc(x, rows, K, ldx, perm, S, augment, mode, rule, fp8_max, codes,
                                     scales, global_scale, workspace, workspace_bytes, stream)


def nvfp4_quantize_t(x, rows, K, ldx, mode, rule, fp8_max, codes, scales, global_scale, workspace,
                     workspace_bytes, stream) -> int:
    """The NVFP4 operand of x^T (blocks along the rows of x)."""
    return load().nvfp4_quantize_t(x, rows, K, ldx, mode, rule, fp8_max, codes, scales, global_scale,
                                   workspace, workspace_bytes, stream)


def nvfp4_quantize_with_scale(x, rows, K, ldx, mode, rule, global_scale, codes, scales, workspace,
                              workspace_bytes, stream) -> int:
    """nvfp4_quantize against a caller-supplied tensor scale read from the
    device float at ``global_scale`` (no amax pass)."""
    return load().nvfp4_quantize_with_scale(x, rows, K, ldx, mode, rule, global_scale, codes,
                                            scales, workspace, workspace_bytes, stream)


def nvfp4_gemm(a_codes, a_scales, a_global, b_codes, b_scales, b_global, M, N, K, y, ldy,
               out_dtype, workspace, workspace_bytes, stream) -> int:
    return load().nvfp4_gemm(a_codes, a_scales, a_global, b_codes, b_scales, b_global, M, N, K, y,
                             ldy, out_dtype, workspace, workspace_bytes, stream)


def nvfp4_gemm_quantized(a_codes, a_scales, a_global, b_codes, b_scales, b_global, M, N, K, mode, rule,
                         y_alpha, y_codes, y_scales, workspace, workspace_bytes, stream) -> int:
    """nvfp4_gemm with Y written as an NVFP4 operand (static alpha)."""
    return load().nvfp4_gemm_quantized(a_codes, a_scales, a_global, b_codes, b_scales, b_global, M, N, K,
                                       mode, rule, y_alpha, y_codes, y_scales, workspace, workspace_bytes,
                                       stream)


def nvfp4_gemm_segmented(a_codes, a_scales, a_global, b_codes, b_scales, b_globals, seg_ends, nseg,
                         M, N, K, y, ldy, out_dtype, workspace, workspace_bytes, stream) -> int:
    """nvfp4_gemm with one B global scale per output-column segment;
    ``seg_ends`` is a host pointer to nseg int64 exclusive end columns."""
    return load().nvfp4_gemm_segmented(a_codes, a_scales, a_global, b_codes, b_scales, b_globals,
                                       seg_ends, nseg, M, N, K, y, ldy, out_dtype, workspace,
                                       workspace_bytes, stream)


def nvfp4_quantize_arc_rmsnorm_workspace_bytes(rows, K):
    return load().nvfp4_quantize_arc_rmsnorm_workspace_bytes(rows, K)


def nvfp4_quantize_arc_rmsnorm(x, rows, K, ldx, gamma, eps, perm, S, mode, rule, fp8_max, codes, scales,
                               global_scale, workspace, workspace_bytes, stream=None):
    return load().nvfp4_quantize_arc_rmsnorm(x, rows, K, ldx, gamma, eps, perm, S, mode, rule, fp8_max, codes,
                                             scales, global_scale, workspace, workspace_bytes, stream)


def nvfp4_quantize_gemm(x, M, K, ldx, mode, rule, fp8_max, x_codes, x_scales, x_global_scale, x_workspace,
                        x_workspace_bytes, w_codes, w_scales, w_global, N, y, ldy, out_dtype, workspace,
                        workspace_bytes, stream) -> int:
    return load().nvfp4_quantize_gemm(x, M, K, ldx, mode, rule, fp8_max, x_codes, x_scales, x_global_scale,
                                      x_workspace, x_workspace_bytes, w_codes, w_scales, w_global, N, y, ldy,
                                      out_dtype, workspace, workspace_bytes, stream)


def nvfp4_quantize_arc_rmsnorm_gemm(x, M, K, ldx, gamma, eps, perm, S, mode, rule, fp8_max, x_codes, x_scales,
                                    x_global_scale, x_workspace, x_workspace_bytes, w_codes, w_scales, w_global, N,
                                    y, ldy, out_dtype, workspace, workspace_bytes, stream=None):
    return load().nvfp4_quantize_arc_rmsnorm_gemm(x, M, K, ldx, gamma, eps, perm, S, mode, rule, fp8_max, x_codes,
                                                  x_scales, x_global_scale, x_workspace, x_workspace_bytes,
                                                  w_codes, w_scales, w_global, N, y, ldy, out_dtype, workspace,
                                                  workspace_bytes, stream)


def nvfp4_quantize_arc_gemm(x, M, K, ldx, perm, S, mode, rule, fp8_max, x_codes, x_scales, x_global_scale,
                            x_workspace, x_workspace_bytes, w_codes, w_scales, w_global, N, y, ldy, out_dtype,
                            workspace, workspace_bytes, stream=None):
    return load().nvfp4_quantize_arc_gemm(x, M, K, ldx, perm, S, mode, rule, fp8_max, x_codes, x_scales,
                                          x_global_scale, x_workspace, x_workspace_bytes, w_codes, w_scales,
                                          w_global, N, y, ldy, out_dtype, workspace, workspace_bytes, stream)


def nvfp4_get_device_status(workspace, stream) -> int:
    return load().nvfp4_get_device_status(workspace, stream)


def status_string(status: int) -> str:
    return load().nvfp4_status_string(status).decode()


def last_error_message() -> str:
    return load().nvfp4_last_error_message().decode()


def testing_set_gemm_wait(timeout_ns: int = 0, debug_flags: int = 0) -> None:
    load().nvfp4_testing_set_gemm_wait(timeout_ns, debug_flags)


# --------------------------------------------------- torch-level helpers --

@dataclass
class NVFP4Tensor:
    """A quantized [rows, K] operand as the C ABI lays it out."""
    codes: "torch.Tensor"         # uint8 [rows, K/2]
    scales: "torch.Tensor"        # uint8 [nvfp4_scales_bytes(rows, K)], swizzled
    global_scale: "torch.Tensor"  # float32 [1]
    workspace: "torch.Tensor"     # uint8, holds the status word of the call
    rows: int
    K: int


def _stream_handle(stream) -> int:
    import torch

    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _check(status: int, what: str) -> None:
    if status != OK:
        raise NVFP4Error(status, what)


# The C ABI takes raw pointers and cannot see buffer sizes, so the wrappers
# check every torch buffer they pass against the shape the call will read or
# write: a buffer that is too small, of another dtype or on another device is
# rejected here instead of being overrun on the GPU.

def _require(t, name: str, dtype, min_numel: int, device, contiguous: bool = True) -> None:
    import torch

    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, not {t.dtype}")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.numel() < min_numel:
        raise ValueError(f"{name} holds {t.numel()} elements, the call needs {min_numel}")


def _check_operand(q: "NVFP4Tensor", name: str, rows: int, K: int, device, global_scale: bool = True,
                   workspace: bool = False) -> None:
    """q's buffers hold (or will hold) a [rows, K] NVFP4 operand on `device`."""
    import torch

    if (q.rows, q.K) != (rows, K):
        raise ValueError(f"{name} describes a [{q.rows}, {q.K}] operand, the call needs [{rows}, {K}]")
    _require(q.codes, f"{name}.codes", torch.uint8, rows * (K // 2), device)
    _require(q.scales, f"{name}.scales", torch.uint8, nvfp4_scales_bytes(rows, K), device)
    if global_scale:
        _require(q.global_scale, f"{name}.global_scale", torch.float32, 1, device, contiguous=False)
    if workspace:
        _require(q.workspace, f"{name}.workspace", torch.uint8, 0, device)


def _check_output(y, M: int, N: int, dtype, device) -> None:
    """y is an [M, N] matrix of `dtype` on `device` with unit column stride
    (rows may be padded: the row pitch is passed as ldy)."""
    import torch

    if not isinstance(y, torch.Tensor):
        raise TypeError("out must be a torch.Tensor")
    if y.dtype != dtype:
        raise ValueError(f"out must be {dtype}, not {y.dtype}")
    if y.device != device:
        raise ValueError(f"out is on {y.device}, expected {device}")
    if y.dim() != 2 or tuple(y.shape) != (M, N):
        raise ValueError(f"out must have shape ({M}, {N}), not {tuple(y.shape)}")
    if y.stride(1) != 1 or _row_pitch(y) < N:
        raise ValueError("out must have unit stride along N and a row pitch of at least N")


def _row_pitch(x) -> int:
    """Row pitch of a 2-D tensor in elements.  A single row has no pitch to
    speak of (torch may report any stride for a size-1 dimension), so its
    row length stands in."""
    return x.shape[1] if x.shape[0] == 1 else x.stride(0)


def _out_code(out_dtype, out):
    """The C output code for out_dtype (default: out's dtype, else bf16)."""
    import torch

    if out_dtype is None:
        out_dtype = out.dtype if out is not None else torch.bfloat16
    codes = {torch.bfloat16: OUT_BF16, torch.float32: OUT_FP32}
    if out_dtype not in codes:
        raise ValueError(f"out_dtype must be torch.bfloat16 or torch.float32, not {out_dtype}")
    return out_dtype, codes[out_dtype]


def quantize(x, mode: str = "six", rule: str = "max", fp8_max: float | None = None,
             out: NVFP4Tensor | None = None, stream=None, global_scale=None) -> NVFP4Tensor:
    """NVFP4-quantize a CUDA bf16 matrix [rows, K] (K % 64 == 0).

    With ``global_scale`` (a float32 CUDA tensor of one element, e.g. a
    calibrated alpha) the tensor scale is taken from it instead of the
    tensor's amax; ``fp8_max`` is then unused.  A new result refers to that
    tensor as its ``global_scale`` (no copy); into an existing ``out`` it is
    copied unless it already is ``out.global_scale``.
    """
    import torch

    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise ValueError("x must be a 2-D bfloat16 CUDA tensor")
    if x.stride(1) != 1:
        raise ValueError("x must have unit stride along K")
    if global_scale is not None and (global_scale.dtype != torch.float32 or global_scale.numel() != 1
                                     or global_scale.device != x.device):
        raise ValueError("global_scale must be a one-element float32 tensor on x's device")
    rows, K = x.shape
    F = DEFAULT_FP8_MAX[mode] if fp8_max is None else float(fp8_max)
    if out is None:
        dev = x.device
        out = NVFP4Tensor(
            codes=torch.empty(rows, K // 2, dtype=torch.uint8, device=dev),
            scales=torch.empty(max(1, nvfp4_scales_bytes(rows, K)), dtype=torch.uint8, device=dev),
            global_scale=(torch.empty(1, dtype=torch.float32, device=dev) if global_scale is None
                          else global_scale.reshape(1)),
            workspace=torch.empty(nvfp4_quantize_workspace_bytes(rows, K), dtype=torch.uint8, device=dev),
            rows=rows, K=K)
    _check_operand(out, "out", rows, K, x.device, workspace=True)
    if global_scale is not None:
        if out.global_scale.data_ptr() != global_scale.data_ptr():
            out.global_scale.copy_(global_scale.reshape(1))
        st = nvfp4_quantize_with_scale(x.data_ptr(), rows, K, _row_pitch(x), MODES[mode], RULES[rule],
                                       out.global_scale.data_ptr(), out.codes.data_ptr(),
                                       out.scales.data_ptr(), out.workspace.data_ptr(),
                                       out.workspace.numel(), _stream_handle(stream))
        _check(st, "nvfp4_quantize_with_scale")
        return out
    st = nvfp4_quantize(x.data_ptr(), rows, K, _row_pitch(x), MODES[mode], RULES[rule], F,
                        out.codes.data_ptr(), out.scales.data_ptr(), out.global_scale.data_ptr(),
                        out.workspace.data_ptr(), out.workspace.numel(), _stream_handle(stream))
    _check(st, "nvfp4_quantize")
    return out


AUG_RESIDUAL = 0
AUG_DUPLICATE = 1


def quantize_arc(x, perm, S: int, augment: int = AUG_RESIDUAL, mode: str = "six", rule: str = "max",
                 fp8_max: float | None = None, out: NVFP4Tensor | None = None, stream=None) -> NVFP4Tensor:
    """ARCQuant augmented quantization of a CUDA bf16 matrix x [rows, K]:
    channels in the order ``perm`` (an int32 CUDA tensor, a permutation of
    0..K-1), then S appended channels -- the residual of the first S
    reordered channels (AUG_RESIDUAL, activations) or their copy
    (AUG_DUPLICATE, weights).  The result is the [rows, K + S] operand."""
    import torch

    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise ValueError("x must be a 2-D bfloat16 CUDA tensor")
    if x.stride(1) != 1:
        raise ValueError("x must have unit stride along K")
    rows, K = x.shape
    if perm.dtype != torch.int32 or perm.numel() != K or not perm.is_cuda:
        raise ValueError("perm must be an int32 CUDA tensor with K entries")
    F = DEFAULT_FP8_MAX[mode] if fp8_max is None else float(fp8_max)
    KA = K + S
    if out is None:
        dev = x.device
        out = NVFP4Tensor(
            codes=torch.empty(rows, KA // 2, dtype=torch.uint8, device=dev),
            scales=torch.empty(max(1, nvfp4_scales_bytes(rows, KA)), dtype=torch.uint8, device=dev),
            global_scale=torch.empty(1, dtype=torch.float32, device=dev),
            workspace=torch.empty(nvfp4_quantize_workspace_bytes(rows, K), dtype=torch.uint8, device=dev),
            rows=rows, K=KA)
    if perm.device != x.device:
        raise ValueError("perm must be on x's device")
    _check_operand(out, "out", rows, KA, x.device, workspace=True)
    st = nvfp4_quantize_arc(x.data_ptr(), rows, K, _row_pitch(x), perm.data_ptr(), S, augment, MODES[mode],
                            RULES[rule], F, out.codes.data_ptr(), out.scales.data_ptr(),
                            out.global_scale.data_ptr(), out.workspace.data_ptr(), out.workspace.numel(),
                            _stream_handle(stream))
    _check(st, "nvfp4_quantize_arc")
    return out


def quantize_arc_rmsnorm(x, gamma, eps: float, perm, S: int, mode: str = "six", rule: str = "max",
                         fp8_max: float | None = None, out: NVFP4Tensor | None = None, stream=None) -> NVFP4Tensor:
    """``quantize_arc`` (residual channels) of the RMSNorm of x: the rows of
    the bf16 CUDA matrix x [rows, K] are normalized by their root mean square
    (plus eps) and scaled by the bf16 gains ``gamma`` [K], rounded to bf16,
    reordered by ``perm`` and quantized with S residual channels, all in the
    library's two kernels (the normalized tensor is never written)."""
    import torch

    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise ValueError("x must be a 2-D bfloat16 CUDA tensor")
    if x.stride(1) != 1:
        raise ValueError("x must have unit stride along K")
    rows, K = x.shape
    if perm.dtype != torch.int32 or perm.numel() != K or not perm.is_cuda or perm.device != x.device:
        raise ValueError("perm must be an int32 tensor with K entries on x's device")
    if gamma.dtype != torch.bfloat16 or gamma.numel() != K or not gamma.is_cuda or gamma.device != x.device:
        raise ValueError("gamma must be a bfloat16 tensor with K entries on x's device")
    gamma = gamma.contiguous()
    F = DEFAULT_FP8_MAX[mode] if fp8_max is None else float(fp8_max)
    KA = K + S
    if out is None:
        dev = x.device
        out = NVFP4Tensor(
            codes=torch.empty(rows, KA // 2, dtype=torch.uint8, device=dev),
            scales=torch.empty(max(1, nvfp4_scales_bytes(rows, KA)), dtype=torch.uint8, device=dev),
            global_scale=torch.empty(1, dtype=torch.float32, device=dev),
            workspace=torch.empty(nvfp4_quantize_arc_rmsnorm_workspace_bytes(rows, K), dtype=torch.uint8,
                                  device=dev),
            rows=rows, K=KA)
    _check_operand(out, "out", rows, KA, x.device, workspace=True)
    st = nvfp4_quantize_arc_rmsnorm(x.data_ptr(), rows, K, _row_pitch(x), gamma.data_ptr(), float(eps),
                                    perm.data_ptr(), S, MODES[mode], RULES[rule], F, out.codes.data_ptr(),
                                    out.scales.data_ptr(), out.global_scale.data_ptr(), out.workspace.data_ptr(),
                                    out.workspace.numel(), _stream_handle(stream))
    _check(st, "nvfp4_quantize_arc_rmsnorm")
    return out


def quantize_t(x, mode: str = "six", rule: str = "max", fp8_max: float | None = None,
               out: NVFP4Tensor | None = None, stream=None) -> NVFP4Tensor:
    """NVFP4-quantize x^T for a CUDA bf16 matrix x [rows, K] (rows % 64 == 0,
    K % 8 == 0): the result is the [K, rows] operand, blocks along rows of x."""
    import torch

    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise ValueError("x must be a 2-D bfloat16 CUDA tensor")
    if x.stride(1) != 1:
        raise ValueError("x must have unit stride along K")
    rows, K = x.shape
    F = DEFAULT_FP8_MAX[mode] if fp8_max is None else float(fp8_max)
    if out is None:
        dev = x.device
        out = NVFP4Tensor(
            codes=torch.empty(K, rows // 2, dtype=torch.uint8, device=dev),
            scales=torch.empty(max(1, nvfp4_scales_bytes(K, rows)), dtype=torch.uint8, device=dev),
            global_scale=torch.empty(1, dtype=torch.float32, device=dev),
            workspace=torch.empty(nvfp4_quantize_workspace_bytes(rows, K), dtype=torch.uint8, device=dev),
            rows=K, K=rows)
    _check_operand(out, "out", K, rows, x.device, workspace=True)
    st = nvfp4_quantize_t(x.data_ptr(), rows, K, _row_pitch(x), MODES[mode], RULES[rule], F,
                          out.codes.data_ptr(), out.scales.data_ptr(), out.global_scale.data_ptr(),
                          out.workspace.data_ptr(), out.workspace.numel(), _stream_handle(stream))
    _check(st, "nvfp4_quantize_t")
    return out


def gemm(a: NVFP4Tensor, b: NVFP4Tensor, out_dtype=None, out=None, workspace=None,
         stream=None):
    """Y[M, N] = A_hat @ B_hat^T for two NVFP4 operands with the same K."""
    import torch

    if a.K != b.K:
        raise ValueError("operands disagree on K")
    out_dtype, code = _out_code(out_dtype, out)
    M, N, K = a.rows, b.rows, a.K
    dev = a.codes.device
    _check_operand(a, "a", M, K, dev)
    _check_operand(b, "b", N, K, dev)
    if out is None:
        out = torch.empty(M, N, dtype=out_dtype, device=dev)
    if workspace is None:
        workspace = torch.empty(nvfp4_gemm_workspace_bytes(), dtype=torch.uint8, device=dev)
    _check_output(out, M, N, out_dtype, dev)
    _require(workspace, "workspace", torch.uint8, 0, dev)
    st = nvfp4_gemm(a.codes.data_ptr(), a.scales.data_ptr(), a.global_scale.data_ptr(),
                    b.codes.data_ptr(), b.scales.data_ptr(), b.global_scale.data_ptr(), M, N, K,
                    out.data_ptr(), _row_pitch(out), code, workspace.data_ptr(), workspace.numel(),
                    _stream_handle(stream))
    _check(st, "nvfp4_gemm")
    return out


def quantize_gemm(x, w: NVFP4Tensor, mode: str = "six", rule: str = "max", fp8_max: float | None = None,
                  out_dtype=None, x_out: NVFP4Tensor | None = None, out=None, workspace=None, stream=None):
    """The W4A4 linear layer in one call: quantize the bf16 CUDA activations
    x [M, K] (into ``x_out``, which then holds the NVFP4 operand of x), then
    Y = X_hat @ W_hat^T against the pre-quantized weight ``w`` [N, K].  The
    quantize and GEMM kernels run as programmatic dependents of the kernel
    before them.  Returns (x_out, Y)."""
    import torch

    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise ValueError("x must be a 2-D bfloat16 CUDA tensor")
    if x.stride(1) != 1:
        raise ValueError("x must have unit stride along K")
    M, K = x.shape
    if w.K != K:
        raise ValueError("x and w disagree on K")
    N = w.rows
    dev = x.device
    F = DEFAULT_FP8_MAX[mode] if fp8_max is None else float(fp8_max)
    out_dtype, code = _out_code(out_dtype, out)
    if x_out is None:
        x_out = NVFP4Tensor(
            codes=torch.empty(M, K // 2, dtype=torch.uint8, device=dev),
            scales=torch.empty(max(1, nvfp4_scales_bytes(M, K)), dtype=torch.uint8, device=dev),
            global_scale=torch.empty(1, dtype=torch.float32, device=dev),
            workspace=torch.empty(nvfp4_quantize_workspace_bytes(M, K), dtype=torch.uint8, device=dev),
            rows=M, K=K)
    _check_operand(x_out, "x_out", M, K, dev, workspace=True)
    _check_operand(w, "w", N, K, dev)
    if out is None:
        out = torch.empty(M, N, dtype=out_dtype, device=dev)
    if workspace is None:
        workspace = torch.empty(nvfp4_gemm_workspace_bytes(), dtype=torch.uint8, device=dev)
    _check_output(out, M, N, out_dtype, dev)
    _require(workspace, "workspace", torch.uint8, 0, dev)
    st = nvfp4_quantize_gemm(x.data_ptr(), M, K, _row_pitch(x), MODES[mode], RULES[rule], F,
                             x_out.codes.data_ptr(), x_out.scales.data_ptr(), x_out.global_scale.data_ptr(),
                             x_out.workspace.data_ptr(), x_out.workspace.numel(), w.codes.data_ptr(),
                             w.scales.data_ptr(), w.global_scale.data_ptr(), N, out.data_ptr(), _row_pitch(out),
                             code, workspace.data_ptr(), workspace.numel(), _stream_handle(stream))
    _check(st, "nvfp4_quantize_gemm")
    return x_out, out


def quantize_arc_gemm(x, perm, S: int, w: NVFP4Tensor, mode: str = "six", rule: str = "max",
                      fp8_max: float | None = None, out_dtype=None, x_out: NVFP4Tensor | None = None, out=None,
                      workspace=None, stream=None, gamma=None, eps: float = 1e-6):
    """The augmented-channel W4A4 linear layer in one call: quantize the bf16
    CUDA activations x [M, K] with channel order ``perm`` and S residual
    channels (as ``quantize_arc`` with AUG_RESIDUAL, into ``x_out``; with
    ``gamma``, as ``quantize_arc_rmsnorm``: RMSNorm with those bf16 gains and
    ``eps`` fused ahead), then Y = X_aug @ W_aug^T over K + S against ``w``,
    the weight quantized by ``quantize_arc`` with the same perm and S and
    AUG_DUPLICATE.  The kernels run as programmatic dependents of the kernel
    before them.  Returns (x_out, Y)."""
    import torch

    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise ValueError("x must be a 2-D bfloat16 CUDA tensor")
    if x.stride(1) != 1:
        raise ValueError("x must have unit stride along K")
    M, K = x.shape
    if perm.dtype != torch.int32 or perm.numel() != K or not perm.is_cuda or perm.device != x.device:
        raise ValueError("perm must be an int32 tensor with K entries on x's device")
    KA = K + S
    if w.K != KA:
        raise ValueError("w must have K + S columns")
    N = w.rows
    dev = x.device
    F = DEFAULT_FP8_MAX[mode] if fp8_max is None else float(fp8_max)
    out_dtype, code = _out_code(out_dtype, out)
    if gamma is not None:
        if gamma.dtype != torch.bfloat16 or gamma.numel() != K or not gamma.is_cuda or gamma.device != x.device:
            raise ValueError("gamma must be a bfloat16 tensor with K entries on x's device")
        gamma = gamma.contiguous()
    if x_out is None:
        ws_bytes = (nvfp4_quantize_arc_rmsnorm_workspace_bytes(M, K) if gamma is not None
                    else nvfp4_quantize_workspace_bytes(M, K))
        x_out = NVFP4Tensor(
            codes=torch.empty(M, KA // 2, dtype=torch.uint8, device=dev),
            scales=torch.empty(max(1, nvfp4_scales_bytes(M, KA)), dtype=torch.uint8, device=dev),
            global_scale=torch.empty(1, dtype=torch.float32, device=dev),
            workspace=torch.empty(ws_bytes, dtype=torch.uint8, device=dev),
            rows=M, K=KA)
    _check_operand(x_out, "x_out", M, KA, dev, workspace=True)
    _check_operand(w, "w", N, KA, dev)
    if out is None:
        out = torch.empty(M, N, dtype=out_dtype, device=dev)
    if workspace is None:
        workspace = torch.empty(nvfp4_gemm_workspace_bytes(), dtype=torch.uint8, device=dev)
    _check_output(out, M, N, out_dtype, dev)
    _require(workspace, "workspace", torch.uint8, 0, dev)
    if gamma is not None:
        st = nvfp4_quantize_arc_rmsnorm_gemm(
            x.data_ptr(), M, K, _row_pitch(x), gamma.data_ptr(), float(eps), perm.data_ptr(), S, MODES[mode],
            RULES[rule], F, x_out.codes.data_ptr(), x_out.scales.data_ptr(), x_out.global_scale.data_ptr(),
            x_out.workspace.data_ptr(), x_out.workspace.numel(), w.codes.data_ptr(), w.scales.data_ptr(),
            w.global_scale.data_ptr(), N, out.data_ptr(), _row_pitch(out), code, workspace.data_ptr(),
            workspace.numel(), _stream_handle(stream))
        _check(st, "nvfp4_quantize_arc_rmsnorm_gemm")
        return x_out, out
    st = nvfp4_quantize_arc_gemm(x.data_ptr(), M, K, _row_pitch(x), perm.data_ptr(), S, MODES[mode], RULES[rule],
                                 F, x_out.codes.data_ptr(), x_out.scales.data_ptr(), x_out.global_scale.data_ptr(),
                                 x_out.workspace.data_ptr(), x_out.workspace.numel(), w.codes.data_ptr(),
                                 w.scales.data_ptr(), w.global_scale.data_ptr(), N, out.data_ptr(), _row_pitch(out),
                                 code, workspace.data_ptr(), workspace.numel(), _stream_handle(stream))
    _check(st, "nvfp4_quantize_arc_gemm")
    return x_out, out


def gemm_quantized(a: NVFP4Tensor, b: NVFP4Tensor, y_alpha, mode: str = "six", rule: str = "max",
                   out: NVFP4Tensor | None = None, stream=None) -> NVFP4Tensor:
    """Y = A_hat @ B_hat^T written directly as an NVFP4 [M, N] operand,
    quantized against the float32 CUDA tensor ``y_alpha`` (one element)."""
    import torch

    if a.K != b.K:
        raise ValueError("operands disagree on K")
    M, N = a.rows, b.rows
    dev = a.codes.device
    _check_operand(a, "a", M, a.K, dev)
    _check_operand(b, "b", N, b.K, dev)
    _require(y_alpha, "y_alpha", torch.float32, 1, dev, contiguous=False)
    if out is None:
        out = NVFP4Tensor(
            codes=torch.empty(M, N // 2, dtype=torch.uint8, device=dev),
            scales=torch.empty(max(1, nvfp4_scales_bytes(M, N)), dtype=torch.uint8, device=dev),
            global_scale=y_alpha.reshape(1),
            workspace=torch.empty(nvfp4_gemm_workspace_bytes(), dtype=torch.uint8, device=dev),
            rows=M, K=N)
    _check_operand(out, "out", M, N, dev, global_scale=False, workspace=True)
    st = nvfp4_gemm_quantized(a.codes.data_ptr(), a.scales.data_ptr(), a.global_scale.data_ptr(),
                              b.codes.data_ptr(), b.scales.data_ptr(), b.global_scale.data_ptr(), M, N, a.K,
                              MODES[mode], RULES[rule], y_alpha.data_ptr(), out.codes.data_ptr(),
                              out.scales.data_ptr(), out.workspace.data_ptr(), out.workspace.numel(),
                              _stream_handle(stream))
    _check(st, "nvfp4_gemm_quantized")
    return out


def gemm_segmented(a: NVFP4Tensor, b: NVFP4Tensor, b_globals, seg_ends, out_dtype=None, out=None,
                   workspace=None, stream=None):
    """Y = A_hat @ B_hat^T where B is several weights fused along N: columns
    [seg_ends[s-1], seg_ends[s]) of Y are scaled by alpha_A * b_globals[s]
    (b_globals: float32 CUDA tensor [nseg]; b.global_scale is not used)."""
    import torch

    if a.K != b.K:
        raise ValueError("operands disagree on K")
    ends = (ctypes.c_int64 * len(seg_ends))(*[int(e) for e in seg_ends])
    if b_globals.dtype != torch.float32 or b_globals.numel() != len(seg_ends) or not b_globals.is_cuda:
        raise ValueError("b_globals must be a float32 CUDA tensor with one entry per segment")
    out_dtype, code = _out_code(out_dtype, out)
    M, N, K = a.rows, b.rows, a.K
    dev = a.codes.device
    _check_operand(a, "a", M, K, dev)
    _check_operand(b, "b", N, K, dev, global_scale=False)
    if b_globals.device != dev:
        raise ValueError("b_globals must be on the operands' device")
    if out is None:
        out = torch.empty(M, N, dtype=out_dtype, device=dev)
    if workspace is None:
        workspace = torch.empty(nvfp4_gemm_workspace_bytes(), dtype=torch.uint8, device=dev)
    _check_output(out, M, N, out_dtype, dev)
    _require(workspace, "workspace", torch.uint8, 0, dev)
    st = nvfp4_gemm_segmented(a.codes.data_ptr(), a.scales.data_ptr(), a.global_scale.data_ptr(),
                              b.codes.data_ptr(), b.scales.data_ptr(), b_globals.data_ptr(),
                              ctypes.addressof(ends), len(seg_ends), M, N, K, out.data_ptr(),
                              _row_pitch(out), code, workspace.data_ptr(), workspace.numel(),
                              _stream_handle(stream))
    _check(st, "nvfp4_gemm_segmented")
    return out


def device_status(workspace, stream=None) -> int:
    """Synchronize the stream and read a call's device status word."""
    return nvfp4_get_device_status(workspace.data_ptr(), _stream_handle(stream))
