"""Pins for the RMSNorm step of the augmented quantizer (ARCQuant page,
방법론, 커널 구현: normalization fused ahead of the reorder and the dual
quantization).  The page gives no formula; the oracle takes the standard
RMSNorm and four readings of its rounding order:

* summation: sum of squares as the contiguous pairwise tree (zero-padded to a
  power of two), not left to right;
* mean:      fl(s / K), not fl(s * fl(1/K));
* rsqrt:     fl(1 / fl(sqrt(d))), not the correctly rounded 1/sqrt(d);
* order:     fl(fl(x * r) * gamma), not fl(x * fl(r * gamma)).

tests/golden/rmsnorm_pins.txt holds one row per reading where the reading
and its alternative give a different bf16 output element; its values were
derived in exact rational arithmetic (tests/exact_binary32.py, no oracle
code, by tests/golden/make_rmsnorm_pins.py).  The tests re-derive them, check
the oracle against them on the whole row, and show that an oracle built with
the alternative line fails them.
"""
import ctypes
import os
import re
import struct
import subprocess
from fractions import Fraction

import numpy as np
import pytest
import torch

import exact_binary32 as xb
import oracle
from conftest import read_golden

ALT = {"summation": dict(summation="sequential"), "mean": dict(mean="reciprocal"),
       "rsqrt": dict(rsqrt="rsqrt"), "order": dict(order="r_gamma_first")}


def _from_bf16(b: int) -> Fraction:
    return Fraction(struct.unpack("<f", struct.pack("<I", b << 16))[0])


def _bits(v: Fraction) -> int:
    return struct.unpack("<I", struct.pack("<f", float(v)))[0] >> 16


def _cases():
    out = []
    for ln in read_golden("rmsnorm_pins.txt"):
        f = [p.strip() for p in ln.split("|")]
        out.append(dict(name=f[0], reading=f[1], K=int(f[2]), eps=float.fromhex(f[3]),
                        x=[int(v, 16) for v in f[4].split()], g=[int(v, 16) for v in f[5].split()],
                        i=int(f[6]), y=int(f[7], 16), y_alt=int(f[8], 16)))
    return out


CASES = _cases()


def test_every_reading_is_pinned():
    assert {c["reading"] for c in CASES} == set(ALT)
    assert all(len(c["x"]) == len(c["g"]) == c["K"] for c in CASES)


@pytest.mark.parametrize("case", CASES, ids=lambda c: c["name"])
def test_golden_values_follow_from_exact_arithmetic(case):
    x = [_from_bf16(b) for b in case["x"]]
    g = [_from_bf16(b) for b in case["g"]]
    eps = Fraction(case["eps"])
    i = case["i"]
    alt = ALT[case["reading"]]
    r0 = xb.rms_scale(x, eps)
    r1 = xb.rms_scale(x, eps, **{k: v for k, v in alt.items() if k != "order"})
    order = {k: v for k, v in alt.items() if k == "order"}
    assert _bits(xb.rms_out(x[i], r0, g[i])) == case["y"]
    assert _bits(xb.rms_out(x[i], r1, g[i], **order)) == case["y_alt"]
    assert case["y"] != case["y_alt"]


def _row_arrays(case):
    x = np.array(case["x"], np.uint16).reshape(1, -1)
    g = np.array(case["g"], np.uint16)
    return x, g


@pytest.mark.parametrize("case", CASES, ids=lambda c: c["name"])
def test_oracle_matches_exact_model_on_the_whole_row(case):
    x, g = _row_arrays(case)
    y = oracle.rmsnorm(x, g, case["eps"])
    assert int(y[0, case["i"]]) == case["y"]
    xs = [_from_bf16(b) for b in case["x"]]
    gs = [_from_bf16(b) for b in case["g"]]
    r = xb.rms_scale(xs, Fraction(case["eps"]))
    assert [int(v) for v in y[0]] == [_bits(xb.rms_out(v, r, gv)) for v, gv in zip(xs, gs)]


# ------------------------------------------------------------- mutants --
MUTATIONS = {
    "summation": (r"const float ms = pairwise_sum\(t, K\) / \(float\)K;",
                  "float s_ = 0.0f; for (int64_t k_ = 0; k_ < K; ++k_) s_ = s_ + t[k_]; "
                  "const float ms = s_ / (float)K;"),
    "mean": (r"const float ms = pairwise_sum\(t, K\) / \(float\)K;",
             "const float ms = pairwise_sum(t, K) * (1.0f / (float)K);"),
    "rsqrt": (r"const float q = sqrtf\(ms \+ eps\);\s*const float rinv = 1\.0f / q;",
              "const float rinv = (float)(1.0 / sqrt((double)(ms + eps)));"),
    "order": (r"const float xr = bf16_to_f32\(row\[k\]\) \* rinv;\s*"
              r"y\[r \* K \+ k\] = or_f32_to_bf16\(xr \* bf16_to_f32\(gamma\[k\]\)\);",
              "y[r * K + k] = or_f32_to_bf16(bf16_to_f32(row[k]) * (rinv * bf16_to_f32(gamma[k])));"),
}


@pytest.mark.parametrize("reading", sorted(MUTATIONS))
def test_alternative_reading_fails_the_pins(tmp_path, reading):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "nvfp4_oracle.c")).read()
    pattern, repl = MUTATIONS[reading]
    mutated, n = re.subn(pattern, repl, src)
    assert n == 1, f"the {reading} line was not found in the oracle source"
    (tmp_path / "m.c").write_text(mutated)
    so = tmp_path / "libm.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
                    str(tmp_path / "m.c"), "-o", str(so), "-lm"], check=True)
    lib = ctypes.CDLL(str(so))
    u16p = ctypes.POINTER(ctypes.c_uint16)
    lib.or_rmsnorm_bf16.restype = ctypes.c_int
    lib.or_rmsnorm_bf16.argtypes = [u16p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, u16p,
                                    ctypes.c_float, u16p]
    caught = 0
    for case in CASES:
        x, g = _row_arrays(case)
        y = np.zeros_like(x)
        lib.or_rmsnorm_bf16(x.ctypes.data_as(u16p), 1, case["K"], case["K"], g.ctypes.data_as(u16p),
                            case["eps"], y.ctypes.data_as(u16p))
        if case["reading"] == reading:
            assert int(y[0, case["i"]]) == case["y_alt"], case["name"]
            caught += 1
    assert caught >= 1


def test_bf16_rounding_matches_torch():
    """The oracle's binary32 -> bf16 rounding against torch's cast, on values
    across the range, the exact midpoints between bf16 neighbours (ties to the
    even significand), and values past the largest bf16 (to infinity)."""
    rng = np.random.default_rng(3)
    v = (rng.standard_normal(20000) * np.exp2(rng.integers(-130, 120, 20000))).astype(np.float32)
    mids = (np.arange(0x3F80, 0x4000, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    big = np.array([3.3895314e38, 3.39e38, 3.4e38, -3.4e38], np.float32)
    for arr in (v, mids, -mids, big):
        ref = torch.from_numpy(arr.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        got = np.array([oracle.f32_to_bf16(float(a)) for a in arr], np.uint16)
        assert np.array_equal(got, ref)
