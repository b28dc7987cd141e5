"""Pins for the three readings of the block step whose rounding order the
pages leave open ("Four Over Six (4/6)" technical summary,
gist.science/ko/paper/2512.02010, sections "적응형 블록 스케일링 알고리즘" and
"구현 세부 사항"):

* quotient:  s_raw = fl(b / fl(alpha * Q)), not fl(fl(b / alpha) / Q);
* scaling:   v = fl(x * fl(1 / d)), not fl(x / d);
* summation: MAE / MSE terms summed as the contiguous pairwise tree, not
  left to right.

tests/golden/reading_pins.txt holds blocks for which each reading and its
alternative give different codes or scales.  Their expected bits were derived
by hand in exact rational arithmetic (tests/exact_binary32.py, which shares
nothing with the oracle); the tests below re-derive them, check the oracle
against them, and show that an oracle built with the alternative line fails
them (the mutant is compiled from the oracle's source with that one line
replaced).
"""
import ctypes
import os
import re
import subprocess
from fractions import Fraction

import numpy as np
import pytest
import torch

import exact_binary32 as xb
import oracle
from conftest import read_golden

RULES = {"max": oracle.RULE_MAX, "mae": oracle.RULE_MAE, "mse": oracle.RULE_MSE}
MODES = {"six": oracle.MODE_SIX, "four_over_six": oracle.MODE_FOUR_OVER_SIX}
ALT = {"quotient": dict(quotient="alpha_first"), "scaling": dict(scaling="divide"),
       "summation": dict(summation="sequential")}


def _cases():
    out = []
    for ln in read_golden("reading_pins.txt"):
        f = [p.strip() for p in ln.split("|")]
        vals = [float(v) for v in f[6].split()]
        out.append(dict(name=f[0], reading=f[1], F=float(f[2]), mode=f[3], rule=f[4], amax=float(f[5]),
                        block=vals + [0.0] * (16 - len(vals)), scale=int(f[7], 16),
                        codes=[int(c) for c in f[8].split()], keep=int(f[9]), alt_scale=int(f[10], 16),
                        alt_codes=[int(c) for c in f[11].split()], alt_keep=int(f[12])))
    return out


CASES = _cases()


def _tensor(case) -> torch.Tensor:
    """The 1 x 64 bf16 tensor [amax, 0 x 15 | block | 0 x 32]."""
    row = np.zeros(64, np.float32)
    row[0] = case["amax"]
    row[16:32] = case["block"]
    t = torch.from_numpy(row.reshape(1, 64).copy()).to(torch.bfloat16)
    assert np.array_equal(t.float().numpy(), row[None, :]), "golden values must be bf16-exact"
    return t


def _exact(case, **reading):
    alpha = xb.rn32(Fraction(case["amax"]) / Fraction(int(case["F"]) * 6))
    blk = [Fraction(v) for v in case["block"]]
    if case["mode"] == "six":
        codes, s, _, _ = xb.candidate(blk, alpha, 6, case["rule"], **reading)
        return codes, s, 6
    codes, s, pick4, _, _ = xb.block(blk, alpha, case["rule"], **reading)
    return codes, s, 4 if pick4 else 6


def test_every_reading_is_pinned():
    assert {c["reading"] for c in CASES} == {"quotient", "scaling", "summation"}
    assert {(c["reading"], c["F"]) for c in CASES if c["reading"] != "summation"} == {
        ("quotient", 448.0), ("quotient", 256.0), ("scaling", 448.0), ("scaling", 256.0)}
    assert {c["rule"] for c in CASES if c["reading"] == "summation"} == {"mae", "mse"}


@pytest.mark.parametrize("case", CASES, ids=lambda c: c["name"])
def test_golden_values_follow_from_exact_arithmetic(case):
    """The stored bits are what the stated reading gives, and the rejected
    alternative gives the stored, different, bits."""
    codes, s, keep = _exact(case)
    assert (codes, s, keep) == (case["codes"], case["scale"], case["keep"])
    a_codes, a_s, a_keep = _exact(case, **ALT[case["reading"]])
    assert (a_codes, a_s, a_keep) == (case["alt_codes"], case["alt_scale"], case["alt_keep"])
    assert (a_codes, a_s) != (codes, s)


def _quantize_with(lib, x: torch.Tensor, mode: int, rule: int, F: float):
    """or_quantize of `lib` (the oracle, or a mutant built from its source)
    on a 1 x 64 tensor: (codes of block 1 unpacked, scale of block 1, alpha)."""
    xb16 = np.ascontiguousarray(x.view(torch.int16).numpy().view(np.uint16))
    codes = np.zeros((1, 32), np.uint8)
    scales = np.zeros((1, 4), np.uint8)
    alpha = ctypes.c_float(0)
    u8p = ctypes.POINTER(ctypes.c_uint8)
    rc = lib.or_quantize(xb16.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16)), ctypes.c_int64(1),
                         ctypes.c_int64(64), ctypes.c_int64(64), mode, rule, ctypes.c_float(F),
                         codes.ctypes.data_as(u8p), scales.ctypes.data_as(u8p), ctypes.byref(alpha))
    assert rc == 0
    packed = codes[0, 8:16]
    unpacked = [int(v) for b in packed for v in (b & 15, b >> 4)]
    return unpacked, int(scales[0, 1]), alpha.value


@pytest.mark.parametrize("case", CASES, ids=lambda c: c["name"])
def test_oracle_matches_golden(case):
    x = _tensor(case)
    # whole-tensor path: amax -> alpha -> block step, packing and canonical scales
    codes, scales, alpha = oracle.quantize(x, MODES[case["mode"]], RULES[case["rule"]], case["F"])
    assert np.float32(alpha) == np.float32(float(xb.rn32(Fraction(case["amax"]) / Fraction(int(case["F"]) * 6))))
    unpacked = [int(v) for b in codes[0, 8:16] for v in (b & 15, b >> 4)]
    assert unpacked == case["codes"] and int(scales[0, 1]) == case["scale"]
    # block-level path, with the choice
    blk = np.array(case["block"], np.float32)
    c, s, chose4, _, _ = oracle.quantize_block(blk, alpha, MODES[case["mode"]], RULES[case["rule"]])
    assert list(c) == case["codes"] and s == case["scale"] and (4 if chose4 else 6) == case["keep"]


# ------------------------------------------------------------- mutants --
# Each mutant is the oracle's own source with the one line of a reading
# replaced by its alternative; the golden blocks of that reading must catch it.
MUTATIONS = {
    "quotient": (r"float aq = alpha \* Q;\s*float s_raw = b / aq;", "float s_raw = (b / alpha) / Q;"),
    "scaling": (r"float v = x\[i\] \* r;", "float v = x[i] / d;"),
    "summation": (r"for \(int n = 16; n > 1; n /= 2\)\s*for \(int i = 0; i < n / 2; \+\+i\) a\[i\] = a\[2 \* i\] \+ a\[2 \* i \+ 1\];",
                  "for (int i = 1; i < 16; ++i) a[0] = a[0] + a[i];"),
}


def _build_mutant(tmp_path, reading):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "nvfp4_oracle.c")).read()
    pattern, repl = MUTATIONS[reading]
    mutated, n = re.subn(pattern, repl, src)
    assert n == 1, f"the {reading} line was not found in the oracle source"
    path_c = tmp_path / f"mutant_{reading}.c"
    path_so = tmp_path / f"libmutant_{reading}.so"
    path_c.write_text(mutated)
    subprocess.run(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
                    str(path_c), "-o", str(path_so), "-lm"], check=True)
    lib = ctypes.CDLL(str(path_so))
    lib.or_quantize.restype = ctypes.c_int
    return lib


@pytest.mark.parametrize("reading", sorted(MUTATIONS))
def test_alternative_reading_fails_the_pins(tmp_path, reading):
    lib = _build_mutant(tmp_path, reading)
    caught = 0
    for case in CASES:
        codes, scale, _ = _quantize_with(lib, _tensor(case), MODES[case["mode"]], RULES[case["rule"]], case["F"])
        if case["reading"] == reading:
            # the mutant reproduces the derived alternative, so the pin fails on it
            assert (codes, scale) == (case["alt_codes"], case["alt_scale"]), case["name"]
            caught += 1
    assert caught >= 2


# ------------------------------------------- the exact model, checked --

def test_exact_model_rounds_like_ieee_binary32():
    """rn32 of the exact result equals numpy's binary32 multiply, add and
    divide on random operands spanning normal, subnormal and overflowing
    results."""
    rng = np.random.default_rng(7)
    a = (rng.standard_normal(3000) * np.exp2(rng.integers(-140, 120, 3000))).astype(np.float32)
    b = (rng.standard_normal(3000) * np.exp2(rng.integers(-20, 20, 3000))).astype(np.float32)
    with np.errstate(all="ignore"):
        for x, y in zip(a, b):
            fx, fy = Fraction(float(x)), Fraction(float(y))
            for exact, got in ((fx * fy, x * y), (fx + fy, x + y), (fx / fy, x / y)):
                want = xb.rn32(exact)
                if np.isinf(got):
                    assert want in (xb.INF, -xb.INF)
                else:
                    assert want == Fraction(float(got)), (x, y)


def test_exact_model_e4m3_matches_torch_cast():
    rng = np.random.default_rng(8)
    vals = np.concatenate([np.exp2(rng.uniform(-12, 9.5, 4000)), [2.0 ** -10, 3 * 2.0 ** -11, 464.0, 449.0]])
    vals = vals.astype(np.float32)
    ref = torch.from_numpy(np.minimum(vals, 448.0)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for v, r in zip(vals, ref):
        assert xb.e4m3_rne_satfinite(Fraction(float(v))) == r, v


def test_exact_model_e2m1_is_nearest_with_even_ties():
    for v, want in ((0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6), (7.0, 7),
                    (0.2499, 0), (0.2501, 1), (4.99, 6), (5.01, 7)):
        assert xb.e2m1_rne_satfinite(Fraction(v), False) == want, v
    assert xb.e2m1_rne_satfinite(Fraction(1, 10), True) == 8
