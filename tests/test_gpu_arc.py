"""Parity of nvfp4_quantize_arc (ARCQuant augmented residual channels) with
the oracle, bit-exact, and of the augmented GEMM over K + S with the fp64
oracle; the augmented product must also be closer to the exact bf16 product
than the plain W4A4 one on outlier-heavy activations."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import w4a4_gemm_nvfp4_b200 as nv
from gpu_util import MODE, RULE, assert_gemm_close, to_np

pytestmark = pytest.mark.gpu

RECIPES = [("six", "max", 448.0), ("four_over_six", "mse", 256.0), ("four_over_six", "mae", 256.0),
           ("four_over_six", "max", 256.0)]


def outlier_perm(x: torch.Tensor) -> np.ndarray:
    """Channels by descending column absmax (the calibration ranking)."""
    amax = x.float().abs().amax(dim=0).numpy()
    return np.argsort(-amax, kind="stable").astype(np.int32)


def gpu_arc(x_cpu, perm, S, augment, mode, rule, F, canary=0xA5):
    rows, K = x_cpu.shape
    KA = K + S
    out = nv.NVFP4Tensor(
        codes=torch.full((rows, KA // 2), canary, dtype=torch.uint8, device="cuda"),
        scales=torch.full((nv.nvfp4_scales_bytes(rows, KA),), canary, dtype=torch.uint8, device="cuda"),
        global_scale=torch.full((1,), -1.0, dtype=torch.float32, device="cuda"),
        workspace=torch.full((nv.nvfp4_quantize_workspace_bytes(rows, K),), 0xFF, dtype=torch.uint8,
                             device="cuda"),
        rows=rows, K=KA)
    nv.quantize_arc(x_cpu.cuda(), torch.from_numpy(perm).cuda(), S, augment, mode, rule, F, out=out)
    return out, nv.device_status(out.workspace)


def assert_arc_equal(q, x, perm, S, augment, mode, rule, F):
    rows, K = x.shape
    oc, os_, oa = oracle.quantize_arc(x, perm, S, augment, MODE[mode], RULE[rule], F)
    assert float(q.global_scale.cpu()[0]) == np.float32(oa)
    gc = to_np(q.codes)
    bad = np.argwhere(gc != oc)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first {bad[:5].tolist()}"
    swz = oracle.swizzle_scales(os_, rows, K + S)
    gs = to_np(q.scales)
    bad = np.nonzero(gs != swz)[0]
    assert bad.size == 0, f"{bad.size} scale bytes differ, first {bad[:5].tolist()}"


@pytest.mark.parametrize("recipe", RECIPES, ids=lambda r: "-".join(map(str, r)))
@pytest.mark.parametrize("shape,S", [((1, 64), 64), ((129, 256), 64), ((300, 512), 128), ((64, 1024), 0),
                                     ((200, 5120), 256)], ids=lambda v: str(v))
@pytest.mark.parametrize("augment", [nv.AUG_RESIDUAL, nv.AUG_DUPLICATE])
def test_quantize_arc_matches_oracle(shape, S, recipe, augment):
    x = workloads.small_operand(*shape, seed=shape[0] + shape[1] + S, kind="t").make()
    perm = outlier_perm(x)
    q, st = gpu_arc(x, perm, S, augment, *recipe)
    assert st == nv.OK
    assert_arc_equal(q, x, perm, S, augment, *recipe)


def test_random_permutation_and_full_augment():
    x = workloads.small_operand(70, 192, seed=9, kind="normal").make()
    perm = torch.randperm(192, generator=torch.Generator().manual_seed(4)).numpy().astype(np.int32)
    q, st = gpu_arc(x, perm, 192, nv.AUG_RESIDUAL, "four_over_six", "mse", 256.0)
    assert st == nv.OK
    assert_arc_equal(q, x, perm, 192, nv.AUG_RESIDUAL, "four_over_six", "mse", 256.0)


def test_augmented_gemm_matches_oracle_and_beats_plain():
    """Y = [X_p | R] . [W_p | W_S]^T over K + S: parity with the fp64 oracle
    on the same operands, and a smaller error against the bf16 product than
    plain W4A4 on outlier-heavy activations."""
    M, N, K, S = 256, 384, 1024, 128
    x = workloads.Operand(M, K, "normal", 1.0, outliers="channels", out_frac=0.02, out_mult=60.0,
                          seed=21).make()
    w = workloads.Operand(N, K, "normal", 0.02, seed=22).make()
    perm = outlier_perm(x)
    qx, st = gpu_arc(x, perm, S, nv.AUG_RESIDUAL, "six", "max", 448.0)
    assert st == nv.OK
    qw, st = gpu_arc(w, perm, S, nv.AUG_DUPLICATE, "six", "max", 448.0)
    assert st == nv.OK
    y = to_np(nv.gemm(qx, qw, out_dtype=torch.float32))
    xc, xs, xa = oracle.quantize_arc(x, perm, S, oracle.AUG_RESIDUAL, oracle.MODE_SIX, oracle.RULE_MAX, 448.0)
    wc, ws, wa = oracle.quantize_arc(w, perm, S, oracle.AUG_DUPLICATE, oracle.MODE_SIX, oracle.RULE_MAX, 448.0)
    ref, guard = oracle.gemm_reference(xc, xs, xa, wc, ws, wa)
    assert_gemm_close(y, ref, guard)
    exact = x.double().numpy() @ w.double().numpy().T
    pc, ps, pa = oracle.quantize(x, oracle.MODE_SIX, oracle.RULE_MAX, 448.0)
    qc, qs, qa = oracle.quantize(w, oracle.MODE_SIX, oracle.RULE_MAX, 448.0)
    plain, _ = oracle.gemm_reference(pc, ps, pa, qc, qs, qa)
    err_aug = np.abs(y - exact).mean()
    err_plain = np.abs(plain - exact).mean()
    assert err_aug < err_plain, (err_aug, err_plain)


# ------------------------------------------------- RMSNorm fused ahead --

def _gains(K, seed):
    g = torch.Generator().manual_seed(seed)
    return (1.0 + 0.25 * torch.randn(K, generator=g)).to(torch.bfloat16)


def gpu_arc_rmsnorm(x_cpu, gamma, eps, perm, S, mode, rule, F, canary=0xA5):
    rows, K = x_cpu.shape
    KA = K + S
    out = nv.NVFP4Tensor(
        codes=torch.full((rows, KA // 2), canary, dtype=torch.uint8, device="cuda"),
        scales=torch.full((nv.nvfp4_scales_bytes(rows, KA),), canary, dtype=torch.uint8, device="cuda"),
        global_scale=torch.full((1,), -1.0, dtype=torch.float32, device="cuda"),
        workspace=torch.full((nv.nvfp4_quantize_arc_rmsnorm_workspace_bytes(rows, K),), 0xFF, dtype=torch.uint8,
                             device="cuda"),
        rows=rows, K=KA)
    nv.quantize_arc_rmsnorm(x_cpu.cuda(), gamma.cuda(), eps, torch.from_numpy(perm).cuda(), S, mode, rule, F,
                            out=out)
    return out, nv.device_status(out.workspace)


@pytest.mark.parametrize("recipe", RECIPES, ids=lambda r: "-".join(map(str, r)))
@pytest.mark.parametrize("shape,S", [((1, 64), 64), ((129, 256), 64), ((300, 512), 128), ((64, 1024), 0),
                                     ((33, 2112), 64), ((37, 5120), 128), ((9, 7168), 128), ((6, 8192), 0),
                                     ((4, 8256), 64), ((5, 16384), 256)], ids=str)
def test_quantize_arc_rmsnorm_matches_oracle(shape, S, recipe):
    """Bit-exact with the oracle's RMSNorm (pinned in test_oracle_rmsnorm.py)
    followed by its augmented quantization; every byte, padding included."""
    rows, K = shape
    mode, rule, F = recipe
    x = workloads.small_operand(rows, K, seed=rows + K).make()
    gamma = _gains(K, K)
    perm = outlier_perm(x)
    q, status = gpu_arc_rmsnorm(x, gamma, 1e-6, perm, S, mode, rule, F)
    assert status == nv.OK
    y = torch.from_numpy(oracle.rmsnorm(x, gamma, 1e-6).view(np.int16)).view(torch.bfloat16)
    assert_arc_equal(q, y, perm, S, nv.AUG_RESIDUAL, mode, rule, F)


def test_quantize_arc_rmsnorm_more_rows_than_warps():
    """More rows than the RMS pass has warps in one wave at K = 5120 (each warp
    takes several rows in turn)."""
    rows, K, S = 2600, 5120, 128
    x = workloads.small_operand(rows, K, seed=11).make()
    gamma = _gains(K, 3)
    perm = outlier_perm(x)
    q, status = gpu_arc_rmsnorm(x, gamma, 1e-6, perm, S, "four_over_six", "mse", 256.0)
    assert status == nv.OK
    y = torch.from_numpy(oracle.rmsnorm(x, gamma, 1e-6).view(np.int16)).view(torch.bfloat16)
    assert_arc_equal(q, y, perm, S, nv.AUG_RESIDUAL, "four_over_six", "mse", 256.0)


def _f32_rms_and_peak(x: torch.Tensor, gamma: torch.Tensor, eps: float):
    """For choosing inputs only (expected values come from the oracle): each
    row's r = 1 / sqrt(pairwise_sum(x^2) / K + eps) in binary32 numpy
    arithmetic (the zero-padded pairwise tree, one rounding per step) and
    T = max_k |x_k * gamma_k| (exact in binary32 for these values)."""
    xf = x.float().numpy()
    gf = gamma.float().numpy()
    rows, K = xf.shape
    n = 1 << (K - 1).bit_length()
    a = np.zeros((rows, n), np.float32)
    a[:, :K] = xf * xf
    while a.shape[1] > 1:
        a = a[:, 0::2] + a[:, 1::2]
    r = np.float32(1.0) / np.sqrt(a[:, 0] / np.float32(K) + np.float32(eps))
    T = np.abs(xf * gf[None, :]).max(axis=1)
    return r, T


def _bf16_of(v: float) -> int:
    """bf16 bits of the nearest bf16 to the real number v >= 0 (ties to even)."""
    from fractions import Fraction
    import exact_binary32 as xb
    return xb.bf16_rne(Fraction(v))


@pytest.mark.parametrize("K,rows", [(256, 32768), (5120, 8192)], ids=str)
def test_quantize_arc_rmsnorm_rows_whose_max_y_sits_on_a_bf16_boundary(K, rows):
    """The RMS pass bounds a row's max |y| by P r (1 -+ 2^-20), P = max |x * gamma|,
    and computes the row's y one by one only when the two bounds round to
    different bf16 values.  Rows chosen so that they do (a few in ten thousand)
    are quantized alone, so that each decides alpha, and compared with the
    oracle bit for bit."""
    x = workloads.small_operand(rows, K, seed=2 * K + 1).make()
    gamma = _gains(K, K + 1)
    r, T = _f32_rms_and_peak(x, gamma, 1e-6)
    picked = []
    for i in range(rows):
        pr = float(T[i]) * float(r[i])
        if _bf16_of(pr * (1 - 2.0 ** -20)) != _bf16_of(pr * (1 + 2.0 ** -20)):
            picked.append(i)
        if len(picked) == 6:
            break
    assert picked, "no row near a bf16 rounding boundary among the candidates"
    perm = np.arange(K, dtype=np.int32)[::-1].copy()
    for i in picked:
        xi = x[i:i + 1].clone()
        q, status = gpu_arc_rmsnorm(xi, gamma, 1e-6, perm, 64, "four_over_six", "mse", 256.0)
        assert status == nv.OK
        y = torch.from_numpy(oracle.rmsnorm(xi, gamma, 1e-6).view(np.int16)).view(torch.bfloat16)
        assert_arc_equal(q, y, perm, 64, nv.AUG_RESIDUAL, "four_over_six", "mse", 256.0)


@pytest.mark.parametrize("K", [256, 5120, 16384], ids=str)
@pytest.mark.parametrize("case", ["large_gain", "tiny_rows"])
def test_quantize_arc_rmsnorm_outside_the_bound_s_range(K, case):
    """Where the RMS pass's bound on max |y| does not hold (a gain above 2^20,
    or y near the bottom of the binary32 range) every y is computed; the result
    is still the oracle's.  K = 16384 takes the round-by-round pass."""
    rows = 64
    x = workloads.small_operand(rows, K, seed=K + 5).make()
    gamma = _gains(K, K + 2)
    if case == "large_gain":
        gamma[K // 3] = 2.0 ** 21
    else:
        x = (x.float() * 2.0 ** -120).to(torch.bfloat16)
    perm = outlier_perm(x)
    q, status = gpu_arc_rmsnorm(x, gamma, 1e-6, perm, 64, "four_over_six", "mae", 256.0)
    assert status == nv.OK
    y = torch.from_numpy(oracle.rmsnorm(x, gamma, 1e-6).view(np.int16)).view(torch.bfloat16)
    assert_arc_equal(q, y, perm, 64, nv.AUG_RESIDUAL, "four_over_six", "mae", 256.0)


def test_quantize_arc_rmsnorm_reading_pins():
    """The rows of tests/golden/rmsnorm_pins.txt (each separates one reading of
    the RMSNorm rounding order from its alternative) quantized on the GPU:
    the operand equals the oracle's on the pinned normalized rows."""
    import test_oracle_rmsnorm as tr

    for case in tr.CASES:
        x_bits, g_bits = tr._row_arrays(case)
        x = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16)
        gamma = torch.from_numpy(g_bits.view(np.int16)).view(torch.bfloat16)
        perm = np.arange(case["K"], dtype=np.int32)
        q, status = gpu_arc_rmsnorm(x, gamma, case["eps"], perm, 0, "six", "max", 448.0)
        assert status == nv.OK
        y = oracle.rmsnorm(x_bits, g_bits, case["eps"])
        assert int(y[0, case["i"]]) == case["y"]
        assert_arc_equal(q, torch.from_numpy(y.view(np.int16)).view(torch.bfloat16), perm, 0,
                         nv.AUG_RESIDUAL, "six", "max", 448.0)


def test_quantize_arc_rmsnorm_nonfinite_input_is_reported():
    x = workloads.small_operand(8, 256, seed=3).make()
    x[5, 17] = float("inf")
    q, status = gpu_arc_rmsnorm(x, _gains(256, 1), 1e-6, np.arange(256, dtype=np.int32), 64, "six", "max", 448.0)
    assert status == nv.ERR_NONFINITE
    assert np.isnan(float(q.global_scale.cpu()[0]))


def test_quantize_arc_rmsnorm_gemm_uses_the_normalized_activations():
    """The augmented GEMM over K + S on the fused operand matches the fp64
    oracle GEMM of the normalized activations against the duplicated weight."""
    M, K, N, S = 256, 1024, 384, 128
    x = workloads.small_operand(M, K, seed=11).make()
    w = workloads.small_operand(N, K, seed=12, kind="normal").make()
    gamma = _gains(K, 13)
    perm = outlier_perm(x)
    qx, status = gpu_arc_rmsnorm(x, gamma, 1e-5, perm, S, "four_over_six", "mse", 256.0)
    assert status == nv.OK
    qw = nv.quantize_arc(w.cuda(), torch.from_numpy(perm).cuda(), S, nv.AUG_DUPLICATE, "six", "max", 448.0)
    y_gpu = nv.gemm(qx, qw, out_dtype=torch.float32)
    yb = torch.from_numpy(oracle.rmsnorm(x, gamma, 1e-5).view(np.int16)).view(torch.bfloat16)
    xc, xs, xa = oracle.quantize_arc(yb, perm, S, oracle.AUG_RESIDUAL, oracle.MODE_FOUR_OVER_SIX,
                                     oracle.RULE_MSE, 256.0)
    wc, ws_, wa = oracle.quantize_arc(w, perm, S, oracle.AUG_DUPLICATE, oracle.MODE_SIX, oracle.RULE_MAX, 448.0)
    ref, guard = oracle.gemm_reference(xc[:64], xs[:64], xa, wc, ws_, wa)
    assert_gemm_close(to_np(y_gpu)[:64], ref, guard, bf16=False)


@pytest.mark.parametrize("recipe", RECIPES[:2], ids=lambda r: "-".join(map(str, r)))
@pytest.mark.parametrize("offset", [32, 8], ids=["32-byte-aligned", "16-byte-aligned"])
def test_quantize_arc_rmsnorm_pitched_rows(recipe, offset):
    """x as a view with a row pitch above K (the RMS pass and the bulk row
    copies both follow the pitch); with an 8-element column offset and gains
    at a 16-byte (not 32-byte) boundary the RMS pass takes 128-bit loads."""
    mode, rule, F = recipe
    rows, K, S = 200, 1024, 128
    wide = workloads.small_operand(rows, K + 96, seed=21).make()  # a pitch of 70 x 32 bytes
    x = wide[:, offset:offset + K]
    gamma = _gains(K, 22)
    g_dev = torch.empty(K + 8, dtype=torch.bfloat16, device="cuda")
    g_off = g_dev[8:] if offset == 8 else g_dev[:K]
    g_off.copy_(gamma.cuda())
    perm = outlier_perm(x)
    out = nv.quantize_arc_rmsnorm(wide.cuda()[:, offset:offset + K], g_off, 1e-6, torch.from_numpy(perm).cuda(), S,
                                  mode, rule, F)
    assert nv.device_status(out.workspace) == nv.OK
    y = torch.from_numpy(oracle.rmsnorm(x.contiguous(), gamma, 1e-6).view(np.int16)).view(torch.bfloat16)
    assert_arc_equal(out, y, perm, S, nv.AUG_RESIDUAL, mode, rule, F)


def test_quantize_arc_rmsnorm_gemm_equals_the_two_calls():
    """nvfp4_quantize_arc_rmsnorm_gemm: RMSNorm, augmented quantization and the
    GEMM over K + S in one call, bit-equal to the two calls."""
    M, K, N, S = 300, 2048, 384, 128
    x = workloads.small_operand(M, K, seed=31).make().cuda()
    w = workloads.small_operand(N, K, seed=32, kind="normal").make().cuda()
    gamma = _gains(K, 33).cuda()
    perm = torch.from_numpy(outlier_perm(x.cpu())).cuda()
    qw = nv.quantize_arc(w, perm, S, nv.AUG_DUPLICATE, "six", "max", 448.0)
    qx_ref = nv.quantize_arc_rmsnorm(x, gamma, 1e-6, perm, S, "four_over_six", "mse", 256.0)
    y_ref = nv.gemm(qx_ref, qw, out_dtype=torch.bfloat16)
    ws = torch.zeros(nv.nvfp4_gemm_workspace_bytes(), dtype=torch.uint8, device="cuda")
    qx, y = nv.quantize_arc_gemm(x, perm, S, qw, "four_over_six", "mse", 256.0, out_dtype=torch.bfloat16,
                                 workspace=ws, gamma=gamma, eps=1e-6)
    torch.cuda.synchronize()
    assert nv.device_status(qx.workspace) == nv.OK and nv.device_status(ws) == nv.OK
    assert torch.equal(qx.codes, qx_ref.codes) and torch.equal(qx.scales, qx_ref.scales)
    assert torch.equal(qx.global_scale, qx_ref.global_scale)
    assert torch.equal(y, y_ref)


# ------------------------------------------------ full size, sampled rows --
# The augmented quantizers on the 32768 x 5120 prefill activations with the
# bench's recipe (4/6-MSE, fp8_max 256, S = 128, channels by descending column
# amax).  alpha comes from the whole tensor: the oracle checks it from the
# whole tensor's amax, and quantizes the sampled rows together with one extra
# row that carries that amax, so that its alpha is the tensor's.

def _amax_row(bits_u16: np.ndarray) -> np.ndarray:
    """A row of zeros holding the largest |value| of the bf16 bit patterns."""
    flat = bits_u16.reshape(-1)
    mag = flat & 0x7FFF
    row = np.zeros((1, bits_u16.shape[1]), np.uint16)
    row[0, 0] = flat[int(np.argmax(mag))]
    return row


def _check_arc_sampled(q, y_bits: np.ndarray, perm, S, nsample=48, seed=3):
    rows, K = y_bits.shape
    mode, rule, F = "four_over_six", "mse", 256.0
    idx = workloads.sample_rows(rows, nsample, seed).numpy()
    sample = np.concatenate([y_bits[idx], _amax_row(y_bits)])
    ys = torch.from_numpy(sample.view(np.int16)).view(torch.bfloat16)
    oc, os_, oa = oracle.quantize_arc(ys, perm, S, nv.AUG_RESIDUAL, MODE[mode], RULE[rule], F)
    amax, bad = oracle.amax(torch.from_numpy(y_bits.view(np.int16)).view(torch.bfloat16))
    assert not bad and np.float32(oa) == np.float32(oracle.global_scale(amax, F))
    assert float(q.global_scale.cpu()[0]) == np.float32(oa)
    gc = to_np(q.codes[torch.from_numpy(idx).cuda()])
    assert np.array_equal(gc, oc[:-1])
    gs = oracle.unswizzle_scales(to_np(q.scales), rows, K + S)[idx]
    assert np.array_equal(gs, os_[:-1])


@pytest.mark.slow
@pytest.mark.parametrize("rmsnorm", [False, True], ids=["plain", "rmsnorm"])
def test_quantize_arc_prefill_full_size_sampled(rmsnorm):
    x = workloads.WORKLOADS["prefill"].x.make()
    K, S = x.shape[1], 128
    perm = outlier_perm(x)
    xd, pd = x.cuda(), torch.from_numpy(perm).cuda()
    if rmsnorm:
        gamma = _gains(K, 5)
        q = nv.quantize_arc_rmsnorm(xd, gamma.cuda(), 1e-6, pd, S, "four_over_six", "mse", 256.0)
        y_bits = oracle.rmsnorm(x, gamma, 1e-6)
    else:
        q = nv.quantize_arc(xd, pd, S, nv.AUG_RESIDUAL, "four_over_six", "mse", 256.0)
        y_bits = oracle.as_bf16_bits(x)
    assert nv.device_status(q.workspace) == nv.OK
    _check_arc_sampled(q, y_bits, perm, S)


@pytest.mark.slow
def test_quantize_arc_gemm_prefill_full_size_sampled():
    """The bench's augmented layer in one call on the prefill case: X
    (32768x5120, 4/6-MSE) with 128 residual channels, W (17408x5120, scale-6)
    with those channels duplicated, bf16 Y over K + 128.  W's operand equals the
    oracle's in full; sampled rows of Y match the fp64 product of the oracle's
    operands (X's rows quantized with the whole tensor's alpha)."""
    wl = workloads.WORKLOADS["prefill"]
    x, w = wl.x.make(), wl.w.make()
    K, S = x.shape[1], 128
    perm = outlier_perm(x)
    pd = torch.from_numpy(perm).cuda()
    wm, wr, wF = wl.w_recipe
    qw = nv.quantize_arc(w.cuda(), pd, S, nv.AUG_DUPLICATE, wm, wr, wF)
    assert nv.device_status(qw.workspace) == nv.OK
    wc, ws, wa = oracle.quantize_arc(w, perm, S, nv.AUG_DUPLICATE, MODE[wm], RULE[wr], wF)
    assert np.array_equal(to_np(qw.codes), wc)
    qx, y = nv.quantize_arc_gemm(x.cuda(), pd, S, qw, "four_over_six", "mse", 256.0, out_dtype=torch.bfloat16)
    assert nv.device_status(qx.workspace) == nv.OK
    xb = oracle.as_bf16_bits(x)
    idx = workloads.sample_rows(x.shape[0], 32, 4).numpy()
    sample = np.concatenate([xb[idx], _amax_row(xb)])
    xs_t = torch.from_numpy(sample.view(np.int16)).view(torch.bfloat16)
    xc, xs, xa = oracle.quantize_arc(xs_t, perm, S, nv.AUG_RESIDUAL, MODE["four_over_six"], RULE["mse"], 256.0)
    assert float(qx.global_scale.cpu()[0]) == np.float32(xa)
    assert np.array_equal(to_np(qx.codes[torch.from_numpy(idx).cuda()]), xc[:-1])
    ref, guard = oracle.gemm_reference(xc[:-1], xs[:-1], xa, wc, ws, wa)
    assert_gemm_close(to_np(y[torch.from_numpy(idx).cuda()].float()), ref, guard, bf16=True)
