"""Pins for the oracle's NVFP4 block quantization (scale-6 and Four-Over-Six).

Pinned against (all from the Four-Over-Six summary, gist.science/ko/paper/2512.02010):
* worked examples of section "문제 제기" (66.6 %) and "핵심 메커니즘" (75 % -> 3),
  in tests/golden/worked_examples.txt;
* the selection definition of "적응형 블록 스케일링 알고리즘": the kept scale
  never has the larger error, recomputed here in binary64 from the emitted codes;
* the headroom statement of "구현 세부 사항" (fp8_max 256 vs 448);
* alpha = amax / (fp8_max * 6) against numpy's IEEE float32 division;
* special cases (zero block, single value, values already on the grid).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from conftest import read_golden

RULES = {"max": oracle.RULE_MAX, "mae": oracle.RULE_MAE, "mse": oracle.RULE_MSE}
MAGS = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def _val(codes):
    codes = np.asarray(codes, np.int64)
    v = MAGS[codes & 7]
    return np.where(codes & 8, -v, v)


def _e4m3_val(code):
    return float(torch.tensor([code], dtype=torch.uint8).view(torch.float8_e4m3fn).float()[0])


def _examples():
    out = []
    for ln in read_golden("worked_examples.txt"):
        f = [p.strip() for p in ln.split("|")]
        lead = [float(v) for v in f[2].split()]
        block = np.zeros(16, np.float32)
        block[: len(lead)] = lead
        out.append(dict(name=f[0], F=float(f[1]), block=block, alpha=float(f[3]), s6=float(f[4]),
                        d6=float(f[5]), c6=[int(c) for c in f[6].split()], s4=float(f[7]),
                        d4=float(f[8]), c4=[int(c) for c in f[9].split()],
                        choice=[int(c) for c in f[10].split()]))
    return out


@pytest.mark.parametrize("ex", _examples(), ids=lambda e: e["name"])
def test_worked_examples(ex):
    amax = float(np.max(np.abs(ex["block"])))
    alpha = oracle.global_scale(amax, ex["F"])
    assert alpha == ex["alpha"]
    for Q, s_exp, d_exp, c_exp in ((6.0, ex["s6"], ex["d6"], ex["c6"]), (4.0, ex["s4"], ex["d4"], ex["c4"])):
        codes, s, _ = oracle.quantize_candidate(ex["block"], alpha, Q, oracle.RULE_MSE)
        assert _e4m3_val(s) == s_exp
        assert _e4m3_val(s) * alpha == d_exp
        n = len(c_exp)
        assert list(codes[:n]) == c_exp
        assert all(c in (0, 8) for c in codes[n:])
    for rule, want in zip(("max", "mae", "mse"), ex["choice"]):
        codes, s, chose4, e6, e4 = oracle.quantize_block(ex["block"], alpha, oracle.MODE_FOUR_OVER_SIX, RULES[rule])
        assert chose4 == (want == 4), (rule, e6, e4)
        assert _e4m3_val(s) == (ex["s4"] if want == 4 else ex["s6"])


def test_66pct_and_gap():
    """Scale 6: FP4 value 4 is 2/3 of the block max; every x in (8, 12) lands on
    4 or 6 only (x < 10 -> 4, the tie 10 -> 4, x > 10 -> 6)."""
    alpha = 2.0 ** -7
    for x in np.arange(8.0, 12.01, 0.0625, dtype=np.float32):
        block = np.zeros(16, np.float32)
        block[0], block[1] = 12.0, x
        codes, s, _, _, _ = oracle.quantize_block(block, alpha, oracle.MODE_SIX, oracle.RULE_MAX)
        assert _e4m3_val(s) * alpha == 2.0
        v = oracle.e2m1_value(codes[1]) * 2.0
        assert v in (8.0, 12.0)
        assert v == (8.0 if x <= 10.0 else 12.0)
    assert 4.0 / 6.0 == pytest.approx(0.666, abs=1e-3)


def test_headroom_fp8_max():
    """With fp8_max = 448 the scale-4 candidate of a full-scale block saturates
    E4M3 (raw 672 > 448) and collapses onto the scale-6 one; with 256 it fits."""
    block = np.zeros(16, np.float32)
    block[0], block[1] = 12.0, 9.0
    a448 = oracle.global_scale(12.0, 448.0)
    c6, s6, e6 = oracle.quantize_candidate(block, a448, 6.0, oracle.RULE_MSE)
    c4, s4, e4 = oracle.quantize_candidate(block, a448, 4.0, oracle.RULE_MSE)
    assert s4 == 0x7E and _e4m3_val(s4) == 448.0
    assert s6 == s4 and list(c6) == list(c4) and e6 == e4
    _, _, chose4, _, _ = oracle.quantize_block(block, a448, oracle.MODE_FOUR_OVER_SIX, oracle.RULE_MSE)
    assert not chose4
    a256 = oracle.global_scale(12.0, 256.0)
    _, s4, _ = oracle.quantize_candidate(block, a256, 4.0, oracle.RULE_MSE)
    assert _e4m3_val(s4) == 384.0


def test_scale4_never_saturates_with_256():
    x = workloads.sweep_operand(64, 1024, seed=3).make()
    amax, _ = oracle.amax(x)
    alpha = oracle.global_scale(amax, 256.0)
    xf = x.float().numpy().reshape(-1, 16)
    for blk in xf[:: 7]:
        _, s6, _ = oracle.quantize_candidate(blk, alpha, 6.0, oracle.RULE_MSE)
        _, s4, _ = oracle.quantize_candidate(blk, alpha, 4.0, oracle.RULE_MSE)
        assert _e4m3_val(s4) <= 384.0 and _e4m3_val(s6) <= 256.0
        # s4 is within one E4M3 rounding of 1.5 * s6's raw value
        if _e4m3_val(s6) >= 2.0 ** -6:
            assert _e4m3_val(s4) == pytest.approx(1.5 * _e4m3_val(s6), rel=2 * 2.0 ** -4)


@pytest.mark.parametrize("F", [448.0, 256.0])
def test_alpha_is_amax_over_f6(F):
    x = workloads.small_operand(32, 256, seed=5).make()
    amax, bad = oracle.amax(x)
    assert not bad
    ref_amax = np.float32(np.max(np.abs(x.float().numpy())))
    assert np.float32(amax) == ref_amax
    alpha = oracle.global_scale(amax, F)
    assert np.float32(alpha) == np.float32(ref_amax) / np.float32(F * 6)


def _fp64_error(x, codes, scale_code, alpha, rule):
    d = _e4m3_val(scale_code) * alpha
    e = x.astype(np.float64) - _val(codes) * d
    if rule == oracle.RULE_MAX:
        return np.max(np.abs(e))
    if rule == oracle.RULE_MAE:
        return np.sum(np.abs(e))
    return np.sum(e * e)


@pytest.mark.parametrize("rule", ["max", "mae", "mse"])
@pytest.mark.parametrize("kind", ["t", "normal"])
def test_four_over_six_keeps_smaller_error(rule, kind):
    """The kept scale's error, recomputed in binary64 from the emitted codes,
    is never larger than the other candidate's (binary32 rounding may only
    flip exact near-ties, which are counted and must be rare)."""
    r = RULES[rule]
    x = workloads.small_operand(64, 512, seed=11, kind=kind).make()
    amax, _ = oracle.amax(x)
    alpha = oracle.global_scale(amax, 256.0)
    blocks = x.float().numpy().reshape(-1, 16)
    near, n4 = 0, 0
    for blk in blocks:
        c6, s6, _ = oracle.quantize_candidate(blk, alpha, 6.0, r)
        c4, s4, _ = oracle.quantize_candidate(blk, alpha, 4.0, r)
        codes, s, chose4, _, _ = oracle.quantize_block(blk, alpha, oracle.MODE_FOUR_OVER_SIX, r)
        E6 = _fp64_error(blk, c6, s6, alpha, r)
        E4 = _fp64_error(blk, c4, s4, alpha, r)
        Ek = E4 if chose4 else E6
        Eo = E6 if chose4 else E4
        assert list(codes) == list(c4 if chose4 else c6) and s == (s4 if chose4 else s6)
        n4 += chose4
        if Ek > Eo:
            assert Ek - Eo <= 1e-6 * max(Ek, Eo), (blk, E6, E4, chose4)
            near += 1
    assert near <= len(blocks) // 1000 + 1
    assert 0 < n4 < len(blocks)  # both scales get used on real-looking data


def test_mode_six_is_four_over_six_restricted():
    x = workloads.small_operand(16, 512, seed=2).make()
    amax, _ = oracle.amax(x)
    alpha = oracle.global_scale(amax, 256.0)
    for blk in x.float().numpy().reshape(-1, 16):
        c_six, s_six, chose4, _, _ = oracle.quantize_block(blk, alpha, oracle.MODE_SIX, oracle.RULE_MAX)
        assert not chose4
        c6, s6, _ = oracle.quantize_candidate(blk, alpha, 6.0, oracle.RULE_MAX)
        assert list(c_six) == list(c6) and s_six == s6
        c, s, chose4, _, _ = oracle.quantize_block(blk, alpha, oracle.MODE_FOUR_OVER_SIX, oracle.RULE_MAX)
        if not chose4:
            assert list(c) == list(c6) and s == s6


def test_special_cases():
    alpha = 2.0 ** -7
    zero = np.zeros(16, np.float32)
    for mode in (oracle.MODE_SIX, oracle.MODE_FOUR_OVER_SIX):
        codes, s, chose4, e6, e4 = oracle.quantize_block(zero, alpha, mode, oracle.RULE_MSE)
        assert s == 0 and not codes.any() and not chose4 and e6 == 0
    for sign in (1.0, -1.0):
        one = np.zeros(16, np.float32)
        one[5] = sign * 12.0
        c6, _, e6 = oracle.quantize_candidate(one, alpha, 6.0, oracle.RULE_MAE)
        c4, _, e4 = oracle.quantize_candidate(one, alpha, 4.0, oracle.RULE_MAE)
        assert c6[5] == (7 if sign > 0 else 15) and c4[5] == (6 if sign > 0 else 14)
        assert e6 == 0 and e4 == 0
        _, _, chose4, _, _ = oracle.quantize_block(one, alpha, oracle.MODE_FOUR_OVER_SIX, oracle.RULE_MAE)
        assert not chose4  # a tie keeps scale 6
    # values already on the grid under a power-of-two decode scale round-trip exactly
    grid = np.array([12, -8, 6, 4, 3, 2, 1, -0.0, 0, -12, 8, -6, -4, -3, -2, -1], np.float32)
    codes, s, _, _, _ = oracle.quantize_block(grid, alpha, oracle.MODE_SIX, oracle.RULE_MSE)
    assert np.array_equal(_val(codes) * _e4m3_val(s) * alpha, grid.astype(np.float64))


def test_negative_small_values_keep_sign():
    alpha = 2.0 ** -7
    blk = np.zeros(16, np.float32)
    blk[0], blk[1], blk[2] = 12.0, -0.1, -0.0
    codes, _, _, _, _ = oracle.quantize_block(blk, alpha, oracle.MODE_SIX, oracle.RULE_MSE)
    assert codes[1] == 8 and codes[2] == 8 and codes[3] == 0


def test_tiny_alpha_gives_zero_codes_not_nan():
    """amax so small that 1/d overflows binary32: r is taken as 0 (reading),
    every code becomes +-0 and the error is the input itself."""
    blk = np.zeros(16, np.float32)
    blk[0] = np.float32(2.0 ** -130)
    blk[1] = np.float32(-(2.0 ** -131))
    alpha = oracle.global_scale(float(blk[0]), 448.0)
    d = _e4m3_val(oracle.quantize_candidate(blk, alpha, 6.0, oracle.RULE_MAX)[1]) * alpha
    with np.errstate(over="ignore"):  # the overflow is the point of this case
        assert np.isinf(np.float32(1.0) / np.float32(d))
    codes, s, chose4, e6, e4 = oracle.quantize_block(blk, alpha, oracle.MODE_FOUR_OVER_SIX, oracle.RULE_MAX)
    assert list(codes[:2]) == [0, 8] and not codes[2:].any()
    assert e6 == np.float32(2.0 ** -130) and e4 == e6 and not chose4


def test_amax_zero_tensor_alpha_one():
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    codes, scales, alpha = oracle.quantize(x, oracle.MODE_FOUR_OVER_SIX, oracle.RULE_MSE, 256.0)
    assert alpha == 1.0 and not codes.any() and not scales.any()


@pytest.mark.parametrize("bad", [float("inf"), float("-inf"), float("nan")])
def test_nonfinite_input_is_an_error(bad):
    x = torch.ones(4, 64, dtype=torch.bfloat16)
    x[2, 17] = bad
    _, nonfinite = oracle.amax(x)
    assert nonfinite
    with pytest.raises(oracle.NonFiniteInput):
        oracle.quantize(x, oracle.MODE_SIX, oracle.RULE_MAX, 448.0)


def test_code_packing_low_nibble_first():
    """Element 2j is the low nibble of byte j (reading: the FP4 operand's
    little-endian packing)."""
    row = np.zeros(32, np.float32)
    row[0], row[1] = 12.0, 2.0       # codes 7 and 2 with d = 2
    row[16], row[17] = -12.0, 3.0    # codes 15 and 3 with d = 2
    x = torch.from_numpy(row[None, :]).to(torch.bfloat16)
    codes, scales, alpha = oracle.quantize(x, oracle.MODE_SIX, oracle.RULE_MAX, 256.0)
    assert alpha == 2.0 ** -7
    assert codes[0, 0] == 7 | (2 << 4)
    assert codes[0, 8] == 15 | (3 << 4)
    assert list(scales[0]) == [0x78, 0x78]  # 256 = 2^8: exponent field 15, mantissa 0


# ---------------------------------------------------------------- layout --

def _swizzle_by_reshape(canon, rows, K):
    """Independent formulation of the block-scaled MMA scale layout: pad rows
    to 128, view as [row-block, 4 row-groups of 32, 32, K-group, 4] and
    permute to [row-block, K-group, 32, 4 row-groups, 4]."""
    rp = -(-rows // 128) * 128
    pad = np.zeros((rp, K // 16), np.uint8)
    pad[:rows] = canon
    t = pad.reshape(rp // 128, 4, 32, K // 64, 4).transpose(0, 3, 2, 1, 4)
    return np.ascontiguousarray(t).reshape(-1)


@pytest.mark.parametrize("rows,K", [(1, 64), (64, 512), (129, 128), (300, 192), (256, 1024)])
def test_swizzle_layout(rows, K):
    rng = np.random.default_rng(rows * K)
    canon = rng.integers(1, 255, size=(rows, K // 16), dtype=np.uint8)
    swz = oracle.swizzle_scales(canon, rows, K)
    assert swz.size == -(-rows // 128) * 128 * (K // 16)
    assert np.array_equal(swz, _swizzle_by_reshape(canon, rows, K))
    assert np.array_equal(oracle.unswizzle_scales(swz, rows, K), canon)


def test_swizzle_hand_positions():
    rows, K = 256, 256
    canon = np.zeros((rows, K // 16), np.uint8)
    canon[33, 5] = 1     # atom (0, 1): 512 + 1*16 + 1*4 + 1 = 533
    canon[130, 14] = 2   # atom (1, 3): (1*4 + 3)*512 + 2*16 + 0*4 + 2 = 3618
    canon[127, 0] = 3    # atom (0, 0): 31*16 + 3*4 + 0 = 508
    swz = oracle.swizzle_scales(canon, rows, K)
    assert swz[533] == 1 and swz[3618] == 2 and swz[508] == 3
    assert np.count_nonzero(swz) == 3
