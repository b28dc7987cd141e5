"""CPU oracle for NVFP4 quantization and the W4A4 GEMM -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  The product library under
``w4a4_gemm_nvfp4_b200/`` never imports it and shares no code with it.

What it computes (page = "Four Over Six (4/6)" technical summary,
gist.science/ko/paper/2512.02010, unless stated otherwise):

* ``quantize`` -- NVFP4 16-element block quantization, scale-to-6 ("문제 제기"
  section) and Four-Over-Six ("적응형 블록 스케일링 알고리즘" section: quantize
  twice, compare errors under max / MAE / MSE, keep the smaller), with the
  FP32 tensor scale alpha = amax / (fp8_max * 6) and fp8_max = 256 for 4/6
  ("구현 세부 사항" section).  The arithmetic lives in ``nvfp4_oracle.c`` and
  follows the steps in that order, one binary32 operation at a time.
* ``gemm_reference`` -- Y = A_hat @ B_hat^T in binary64 on the dequantized
  operands (ARCQuant summary, gist.science/ko/paper/2601.07475, "방법론"
  section: one uniform NVFP4 GEMM over the K dimension).  Dequantization is
  exact in binary64; the product uses numpy's float64 matmul as a library
  primitive.

Every function here is pinned by ``tests/test_oracle_*.py`` against values the
pages print, closed forms, brute force or library routines (torch's FP8 cast),
never against the CUDA path.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC"]

MODE_SIX = 0
MODE_FOUR_OVER_SIX = 1
RULE_MAX = 0
RULE_MAE = 1
RULE_MSE = 2

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile nvfp4_oracle.c into liboracle.so next to it (gcc)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            u8p = ctypes.POINTER(ctypes.c_uint8)
            u16p = ctypes.POINTER(ctypes.c_uint16)
            f32p = ctypes.POINTER(ctypes.c_float)
            f64p = ctypes.POINTER(ctypes.c_double)
            i32p = ctypes.POINTER(ctypes.c_int)
            i64 = ctypes.c_int64
            sig = {
                "or_e2m1_value": (ctypes.c_float, [ctypes.c_uint8]),
                "or_e2m1_encode": (ctypes.c_uint8, [ctypes.c_float]),
                "or_e4m3_value": (ctypes.c_float, [ctypes.c_uint8]),
                "or_e4m3_encode_satfinite": (ctypes.c_uint8, [ctypes.c_float]),
                "or_amax_bf16": (ctypes.c_float, [u16p, i64, i64, i64, i32p]),
                "or_global_scale": (ctypes.c_float, [ctypes.c_float, ctypes.c_float]),
                "or_quantize_block": (None, [f32p, ctypes.c_float, ctypes.c_int, ctypes.c_int,
                                             u8p, u8p, i32p, f32p, f32p]),
                "or_quantize_candidate": (None, [f32p, ctypes.c_float, ctypes.c_float, ctypes.c_int,
                                                 u8p, u8p, f32p]),
                "or_quantize_rows": (None, [u16p, i64, i64, i64, ctypes.c_float, ctypes.c_int,
                                            ctypes.c_int, u8p, u8p]),
                "or_quantize": (ctypes.c_int, [u16p, i64, i64, i64, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_float, u8p, u8p, f32p]),
                "or_quantize_arc": (ctypes.c_int, [u16p, i64, i64, i64, ctypes.POINTER(ctypes.c_int32), i64,
                                                   ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                                   u8p, u8p, f32p]),
                "or_rmsnorm_bf16": (ctypes.c_int, [u16p, i64, i64, i64, u16p, ctypes.c_float, u16p]),
                "or_f32_to_bf16": (ctypes.c_uint16, [ctypes.c_float]),
                "or_scales_swizzled_bytes": (i64, [i64, i64]),
                "or_swizzle_scales": (None, [u8p, i64, i64, u8p]),
                "or_unswizzle_scales": (None, [u8p, i64, i64, u8p]),
                "or_dequantize": (None, [u8p, u8p, ctypes.c_float, i64, i64, f64p]),
            }
            for name, (res, args) in sig.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def _ptr(a: np.ndarray, ctype):
    assert a.flags["C_CONTIGUOUS"] or a.ndim == 0
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def as_bf16_bits(x) -> np.ndarray:
    """Accept a torch bfloat16 tensor or a uint16 array of bf16 bit patterns."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch  # only for the conversion of caller-owned tensors

    assert x.dtype == torch.bfloat16
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


# ------------------------------------------------------------------ codecs --

def e2m1_value(code: int) -> float:
    return float(_load().or_e2m1_value(int(code)))


def e2m1_encode(v: float) -> int:
    return int(_load().or_e2m1_encode(float(v)))


def e4m3_value(code: int) -> float:
    return float(_load().or_e4m3_value(int(code)))


def e4m3_encode(v: float) -> int:
    return int(_load().or_e4m3_encode_satfinite(float(v)))


# ------------------------------------------------------------ tensor scale --

def amax(x) -> tuple[float, bool]:
    xb = as_bf16_bits(x)
    rows, K = xb.shape
    bad = ctypes.c_int(0)
    a = _load().or_amax_bf16(_ptr(xb, ctypes.c_uint16), rows, K, K, ctypes.byref(bad))
    return float(np.float32(a)), bool(bad.value)


def global_scale(amax_value: float, fp8_max: float) -> float:
    return float(np.float32(_load().or_global_scale(float(amax_value), float(fp8_max))))


# ---------------------------------------------------------------- quantize --

def quantize_block(x16, alpha: float, mode: int, rule: int):
    """One 16-element block.  Returns (codes[16] one per byte, scale byte,
    chose4, err6, err4)."""
    xb = np.ascontiguousarray(np.asarray(x16, dtype=np.float32).reshape(16))
    codes = np.zeros(16, np.uint8)
    scale = np.zeros(1, np.uint8)
    chose4 = ctypes.c_int(0)
    e6 = ctypes.c_float(0)
    e4 = ctypes.c_float(0)
    _load().or_quantize_block(_ptr(xb, ctypes.c_float), float(alpha), int(mode), int(rule),
                              _ptr(codes, ctypes.c_uint8), _ptr(scale, ctypes.c_uint8),
                              ctypes.byref(chose4), ctypes.byref(e6), ctypes.byref(e4))
    return codes, int(scale[0]), bool(chose4.value), float(np.float32(e6.value)), float(np.float32(e4.value))


def quantize_candidate(x16, alpha: float, Q: float, rule: int):
    """One scale candidate (Q = 6 or 4) of one block: (codes[16], scale byte, error)."""
    xb = np.ascontiguousarray(np.asarray(x16, dtype=np.float32).reshape(16))
    codes = np.zeros(16, np.uint8)
    scale = np.zeros(1, np.uint8)
    err = ctypes.c_float(0)
    _load().or_quantize_candidate(_ptr(xb, ctypes.c_float), float(alpha), float(Q), int(rule),
                                  _ptr(codes, ctypes.c_uint8), _ptr(scale, ctypes.c_uint8),
                                  ctypes.byref(err))
    return codes, int(scale[0]), float(np.float32(err.value))


def quantize_rows(x, alpha: float, mode: int, rule: int):
    """Quantize given rows with a given alpha.  Returns (codes [rows, K/2],
    canonical scales [rows, K/16])."""
    xb = as_bf16_bits(x)
    rows, K = xb.shape
    assert K % 16 == 0
    codes = np.zeros((rows, K // 2), np.uint8)
    scales = np.zeros((rows, K // 16), np.uint8)
    _load().or_quantize_rows(_ptr(xb, ctypes.c_uint16), rows, K, K, float(alpha), int(mode),
                             int(rule), _ptr(codes, ctypes.c_uint8), _ptr(scales, ctypes.c_uint8))
    return codes, scales


class NonFiniteInput(ValueError):
    pass


def quantize(x, mode: int, rule: int, fp8_max: float):
    """Whole-tensor quantization.  Returns (codes [rows, K/2] uint8, canonical
    scales [rows, K/16] uint8, alpha float)."""
    xb = as_bf16_bits(x)
    rows, K = xb.shape
    assert K % 16 == 0
    codes = np.zeros((rows, K // 2), np.uint8)
    scales = np.zeros((rows, K // 16), np.uint8)
    alpha = ctypes.c_float(0)
    rc = _load().or_quantize(_ptr(xb, ctypes.c_uint16), rows, K, K, int(mode), int(rule),
                             float(fp8_max), _ptr(codes, ctypes.c_uint8),
                             _ptr(scales, ctypes.c_uint8), ctypes.byref(alpha))
    if rc != 0:
        raise NonFiniteInput("tensor holds Inf or NaN")
    return codes, scales, float(np.float32(alpha.value))


AUG_RESIDUAL = 0
AUG_DUPLICATE = 1


def quantize_arc(x, perm, S: int, augment: int, mode: int, rule: int, fp8_max: float):
    """ARCQuant augmented quantization (ARCQuant page, 기술 요약 / 방법론):
    channels reordered by `perm`, primary NVFP4 stage, then S augmented
    channels -- the residual of the first S reordered channels against the
    primary stage (augment=AUG_RESIDUAL) or a copy of them (AUG_DUPLICATE, for
    weights) -- quantized with the same alpha.  Returns (codes [rows,
    (K+S)/2], canonical scales [rows, (K+S)/16], alpha)."""
    xb = as_bf16_bits(x)
    rows, K = xb.shape
    p = np.ascontiguousarray(np.asarray(perm, dtype=np.int32))
    assert p.shape == (K,) and sorted(p.tolist()) == list(range(K))
    assert K % 16 == 0 and S % 16 == 0 and 0 <= S <= K
    codes = np.zeros((rows, (K + S) // 2), np.uint8)
    scales = np.zeros((rows, (K + S) // 16), np.uint8)
    alpha = ctypes.c_float(0)
    rc = _load().or_quantize_arc(_ptr(xb, ctypes.c_uint16), rows, K, K, _ptr(p, ctypes.c_int32), S,
                                 int(augment), int(mode), int(rule), float(fp8_max),
                                 _ptr(codes, ctypes.c_uint8), _ptr(scales, ctypes.c_uint8),
                                 ctypes.byref(alpha))
    if rc != 0:
        raise NonFiniteInput("tensor holds Inf or NaN")
    return codes, scales, float(np.float32(alpha.value))


def rmsnorm(x, gamma, eps: float) -> np.ndarray:
    """RMSNorm of each row of the bf16 tensor x [rows, K] with the bf16 gain
    gamma [K] (ARCQuant page, 방법론, 커널 구현: normalization fused ahead of
    the reorder and the dual quantization): y = bf16((x * r) * gamma) with
    r = 1 / sqrt(pairwise_sum(x^2) / K + eps).  Returns the bf16 bit patterns
    of y as a uint16 [rows, K] array."""
    xb = as_bf16_bits(x)
    gb = as_bf16_bits(gamma).reshape(-1)
    rows, K = xb.shape
    assert gb.shape == (K,)
    y = np.zeros((rows, K), np.uint16)
    rc = _load().or_rmsnorm_bf16(_ptr(xb, ctypes.c_uint16), rows, K, K, _ptr(np.ascontiguousarray(gb), ctypes.c_uint16),
                                 float(np.float32(eps)), _ptr(y, ctypes.c_uint16))
    assert rc == 0
    return y


def f32_to_bf16(v: float) -> int:
    """bf16 bit pattern of the nearest bf16 to a binary32 value (ties to even)."""
    return int(_load().or_f32_to_bf16(float(np.float32(v))))


def quantize_arc_rmsnorm(x, gamma, eps: float, perm, S: int, mode: int, rule: int, fp8_max: float):
    """The augmented quantization (residual channels) of rmsnorm(x, gamma,
    eps): the normalized bf16 rows, reordered, quantized, with S residual
    channels.  Returns (codes, canonical scales, alpha) like quantize_arc."""
    return quantize_arc(rmsnorm(x, gamma, eps), perm, S, AUG_RESIDUAL, mode, rule, fp8_max)


# ------------------------------------------------------------ scale layout --

def scales_swizzled_bytes(rows: int, K: int) -> int:
    return int(_load().or_scales_swizzled_bytes(rows, K))


def swizzle_scales(canon: np.ndarray, rows: int, K: int) -> np.ndarray:
    c = np.ascontiguousarray(canon, dtype=np.uint8)
    assert c.shape == (rows, K // 16) and K % 64 == 0
    out = np.zeros(scales_swizzled_bytes(rows, K), np.uint8)
    _load().or_swizzle_scales(_ptr(c, ctypes.c_uint8), rows, K, _ptr(out, ctypes.c_uint8))
    return out


def unswizzle_scales(swz: np.ndarray, rows: int, K: int) -> np.ndarray:
    s = np.ascontiguousarray(swz, dtype=np.uint8).reshape(-1)
    assert s.size >= scales_swizzled_bytes(rows, K)
    out = np.zeros((rows, K // 16), np.uint8)
    _load().or_unswizzle_scales(_ptr(s, ctypes.c_uint8), rows, K, _ptr(out, ctypes.c_uint8))
    return out


# ----------------------------------------------------------------- dequant --

def dequantize(codes: np.ndarray, scales: np.ndarray, alpha: float) -> np.ndarray:
    """Exact binary64 values val(code) * val(scale) * alpha, [rows, K]."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    s = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, K = c.shape[0], c.shape[1] * 2
    assert s.shape == (rows, K // 16)
    out = np.zeros((rows, K), np.float64)
    _load().or_dequantize(_ptr(c, ctypes.c_uint8), _ptr(s, ctypes.c_uint8), float(alpha), rows, K,
                          _ptr(out, ctypes.c_double))
    return out


# -------------------------------------------------------------------- GEMM --

def gemm_reference(a_codes, a_scales, a_alpha, b_codes, b_scales, b_alpha):
    """Y = A_hat @ B_hat^T in binary64 plus the cancellation guard
    sum_k |A_hat[m,k]| |B_hat[n,k]| (same shapes), both [M, N]."""
    a = dequantize(a_codes, a_scales, a_alpha)
    b = dequantize(b_codes, b_scales, b_alpha)
    return a @ b.T, np.abs(a) @ np.abs(b).T
