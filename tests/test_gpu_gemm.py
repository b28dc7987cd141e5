"""Parity of the CUDA W4A4 GEMM (nvfp4_gemm through the C ABI) with the fp64
oracle product of the dequantized operands.  Operands are made by the oracle
(quantizer output or arbitrary codes/scales) and uploaded, so these tests
exercise the GEMM alone; the full-size cases run the quantize -> GEMM
pipeline as the benchmark does and check sampled output rows."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import w4a4_gemm_nvfp4_b200 as nv
from gpu_util import MODE, RULE, assert_gemm_close, gpu_quantize, to_np, upload_operand

pytestmark = pytest.mark.gpu


def _run(a, b, out_dtype):
    y = nv.gemm(a, b, out_dtype=out_dtype)
    ws = torch.zeros(nv.nvfp4_gemm_workspace_bytes(), dtype=torch.uint8, device="cuda")
    y = nv.gemm(a, b, out_dtype=out_dtype, out=y, workspace=ws)
    assert nv.device_status(ws) == nv.OK
    return to_np(y.float()) if out_dtype == torch.bfloat16 else to_np(y)


def _quantized(rows, K, seed, recipe, kind="t"):
    x = workloads.small_operand(rows, K, seed, kind=kind).make()
    mode, rule, F = recipe
    c, s, a = oracle.quantize(x, MODE[mode], RULE[rule], F)
    return c, s, a


def _random_operand(rows, K, rng, max_scale_code=0x60):
    codes = rng.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)
    scales = rng.integers(0, max_scale_code, size=(rows, K // 16), dtype=np.uint8)
    return codes, scales


def _check(ac, as_, aa, bc, bs, ba):
    ref, guard = oracle.gemm_reference(ac, as_, aa, bc, bs, ba)
    A, B = upload_operand(ac, as_, aa), upload_operand(bc, bs, ba)
    rel32 = assert_gemm_close(_run(A, B, torch.float32), ref, guard)
    assert_gemm_close(_run(A, B, torch.bfloat16), ref, guard, bf16=True)
    return rel32


SHAPES = [(64, 256, 512), (1, 1, 64), (3, 5, 128), (127, 129, 192), (128, 256, 256),
          (200, 300, 320), (257, 513, 1024), (130, 1000, 2048), (1024, 768, 64)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_gemm_quantized_operands(M, N, K):
    ac, as_, aa = _quantized(M, K, 1, ("four_over_six", "mse", 256.0))
    bc, bs, ba = _quantized(N, K, 2, ("six", "max", 448.0), kind="normal")
    _check(ac, as_, aa, bc, bs, ba)


@pytest.mark.parametrize("M,N,K", [(64, 256, 512), (130, 260, 576), (256, 512, 4096)])
def test_gemm_random_codes_and_scales(M, N, K):
    rng = np.random.default_rng(M + N + K)
    ac, as_ = _random_operand(M, K, rng)
    bc, bs = _random_operand(N, K, rng)
    _check(ac, as_, 0.75, bc, bs, 1.25)


def test_pr1():
    wl = workloads.WORKLOADS["pr1"]
    x, w = wl.x.make(), wl.w.make()
    for mode, rule, F in wl.x_recipes:
        xc, xs, xa = oracle.quantize(x, MODE[mode], RULE[rule], F)
        wc, ws, wa = oracle.quantize(w, MODE[mode], RULE[rule], F)
        _check(xc, xs, xa, wc, ws, wa)


def test_closed_form_all_half():
    """All codes +1 (0.5), constant scales: every output equals
    K * 0.25 * sA * sB * alphaA * alphaB exactly."""
    M, N, K = 200, 300, 1024
    ac = np.full((M, K // 2), 0x11, np.uint8)
    bc = np.full((N, K // 2), 0x11, np.uint8)
    as_ = np.full((M, K // 16), 0x38, np.uint8)   # 1.0
    bs = np.full((N, K // 16), 0x41, np.uint8)    # 2.25
    A, B = upload_operand(ac, as_, 0.5), upload_operand(bc, bs, 0.25)
    y = _run(A, B, torch.float32)
    assert np.all(y == K * 0.25 * 2.25 * 0.5 * 0.25)


@pytest.mark.parametrize("kb", [0, 1, 2, 3, 4, 7, 13, 31])
def test_one_hot_k_block_pins_scale_layout(kb):
    """Only K block kb is nonzero and every row/column gets its own scale:
    Y[m,n] = sA[m,kb] sB[n,kb] * sum_k qA qB exactly, which fails for any
    misplaced scale byte (row, K group or atom order)."""
    M, N, K = 256, 256, 512
    rng = np.random.default_rng(kb)
    ac, as_ = _random_operand(M, K, rng)
    bc, bs = _random_operand(N, K, rng)
    mask = np.zeros((1, K // 2), np.uint8)
    mask[0, kb * 8:(kb + 1) * 8] = 0xFF
    ac &= mask
    bc &= mask
    as_ = rng.integers(0x30, 0x50, size=as_.shape, dtype=np.uint8)
    bs = rng.integers(0x30, 0x50, size=bs.shape, dtype=np.uint8)
    ref, _ = oracle.gemm_reference(ac, as_, 1.0, bc, bs, 1.0)
    y = _run(upload_operand(ac, as_, 1.0), upload_operand(bc, bs, 1.0), torch.float32)
    assert np.array_equal(y.astype(np.float64), ref)


def test_tile_order_with_partial_last_group():
    """The output tiles are walked in groups of 32 rows of 256-row tiles.
    M = 8488 gives 34 rows of tiles: one full group and a ragged group of two.
    Every output element is checked, so a tile that is skipped or computed
    twice in the last group fails."""
    M, N, K = 33 * 256 + 40, 3 * 256 + 64, 256
    rng = np.random.default_rng(8488)
    ac, as_ = _random_operand(M, K, rng)
    bc, bs = _random_operand(N, K, rng)
    ref, guard = oracle.gemm_reference(ac, as_, 0.5, bc, bs, 2.0)
    y = _run(upload_operand(ac, as_, 0.5), upload_operand(bc, bs, 2.0), torch.float32)
    assert_gemm_close(y, ref, guard)


# ------------------------------------------------ full sizes, sampled rows --

@pytest.mark.slow
@pytest.mark.parametrize("name", ["mlp8b", "attn27b", "prefill"])
def test_pipeline_full_size_sampled(name):
    """quantize X (each recipe) and W on the GPU, GEMM, and compare sampled
    rows of Y with the oracle's fp64 product of its own quantized operands;
    the one-call layer must give the same bytes as the two calls."""
    wl = workloads.WORKLOADS[name]
    x, w = wl.x.make(), wl.w.make()
    wm, wr, wF = wl.w_recipe
    qw, st = gpu_quantize(w, wm, wr, wF, canary=0)
    assert st == nv.OK
    wc, ws, wa = oracle.quantize(w, MODE[wm], RULE[wr], wF)
    assert np.array_equal(to_np(qw.codes), wc)
    xamax, _ = oracle.amax(x)
    idx = workloads.sample_rows(wl.M, 64, 1).numpy()
    for xm, xr, xF in wl.x_recipes:
        qx, st = gpu_quantize(x, xm, xr, xF, canary=0)
        assert st == nv.OK
        y = nv.gemm(qx, qw, out_dtype=torch.bfloat16)
        y32 = nv.gemm(qx, qw, out_dtype=torch.float32)
        xa = oracle.global_scale(xamax, xF)
        xc, xs = oracle.quantize_rows(x[idx], xa, MODE[xm], RULE[xr])
        ref, guard = oracle.gemm_reference(xc, xs, xa, wc, ws, wa)
        rows = torch.from_numpy(idx).cuda()
        assert_gemm_close(to_np(y32[rows]), ref, guard)
        assert_gemm_close(to_np(y[rows].float()), ref, guard, bf16=True)
        # the one-call layer (the bench's timed step) gives the same bytes
        ws1 = torch.zeros(nv.nvfp4_gemm_workspace_bytes(), dtype=torch.uint8, device="cuda")
        qx1, y1 = nv.quantize_gemm(x.cuda(), qw, xm, xr, xF, out_dtype=torch.bfloat16, workspace=ws1)
        assert nv.device_status(qx1.workspace) == nv.OK and nv.device_status(ws1) == nv.OK
        assert torch.equal(qx1.codes, qx.codes) and torch.equal(y1, y)


@pytest.mark.parametrize("ldy_pad", [3, 8, 130])
def test_strided_output(ldy_pad):
    M, N, K = 150, 200, 256
    ac, as_, aa = _quantized(M, K, 3, ("four_over_six", "max", 256.0))
    bc, bs, ba = _quantized(N, K, 4, ("six", "max", 448.0))
    ref, guard = oracle.gemm_reference(ac, as_, aa, bc, bs, ba)
    A, B = upload_operand(ac, as_, aa), upload_operand(bc, bs, ba)
    for dt in (torch.float32, torch.bfloat16):
        big = torch.full((M, N + ldy_pad), 7.0, dtype=dt, device="cuda")
        nv.gemm(A, B, out_dtype=dt, out=big[:, :N])
        got = to_np(big.float())
        assert_gemm_close(got[:, :N], ref, guard, bf16=dt == torch.bfloat16)
        assert (got[:, N:] == 7.0).all()  # nothing written past N


# ------------------------------------------- per-segment B global scales --

@pytest.mark.parametrize("M,K,seg_rows", [
    (200, 512, [128, 64, 192, 80]),            # boundaries inside a 256-column tile and a half
    (64, 256, [64] * 16),                       # the most segments, 64 columns each
    (130, 1024, [1024, 640, 320]),              # a fused Q / K / V-like split
])
def test_gemm_segmented_matches_oracle(M, K, seg_rows):
    ac, as_, aa = _quantized(M, K, 5, ("four_over_six", "mse", 256.0))
    parts = [_quantized(n, K, 40 + i, ("six", "max", 448.0), kind="normal") for i, n in enumerate(seg_rows)]
    bc = np.concatenate([p[0] for p in parts])
    bs = np.concatenate([p[1] for p in parts])
    alphas = np.array([p[2] for p in parts], np.float32)
    ends = np.cumsum(seg_rows).tolist()
    A = upload_operand(ac, as_, aa)
    B = upload_operand(bc, bs, 1.0)
    bg = torch.from_numpy(alphas).cuda()
    ws = torch.zeros(nv.nvfp4_gemm_workspace_bytes(), dtype=torch.uint8, device="cuda")
    refs, guards = [], []
    for (c, s, a), lo, hi in zip(parts, [0] + ends[:-1], ends):
        r, g = oracle.gemm_reference(ac, as_, aa, c, s, a)
        refs.append(r)
        guards.append(g)
    ref, guard = np.concatenate(refs, axis=1), np.concatenate(guards, axis=1)
    for dt, bf16 in ((torch.float32, False), (torch.bfloat16, True)):
        y = nv.gemm_segmented(A, B, bg, ends, out_dtype=dt, workspace=ws)
        assert nv.device_status(ws) == nv.OK
        assert_gemm_close(to_np(y.float()), ref, guard, bf16=bf16)


def test_gemm_segmented_one_segment_is_gemm():
    ac, as_, aa = _quantized(300, 640, 7, ("four_over_six", "mae", 256.0))
    bc, bs, ba = _quantized(520, 640, 8, ("six", "max", 448.0), kind="normal")
    A, B = upload_operand(ac, as_, aa), upload_operand(bc, bs, ba)
    y1 = nv.gemm(A, B, out_dtype=torch.float32)
    y2 = nv.gemm_segmented(A, B, B.global_scale.clone(), [520], out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


# ----------------------------------------------- NVFP4 output (static alpha) --

@pytest.mark.parametrize("M,N,K", [(64, 128, 512), (200, 320, 256), (300, 1024, 1024)])
@pytest.mark.parametrize("recipe", [("six", "max"), ("four_over_six", "mse"), ("four_over_six", "mae"),
                                    ("four_over_six", "max")], ids=lambda r: "-".join(r))
def test_gemm_quantized_output_equals_gemm_then_quantize(M, N, K, recipe):
    """The fused epilogue equals nvfp4_gemm (bf16 Y) followed by
    nvfp4_quantize_with_scale, bit for bit, and the oracle's row quantizer on
    that bf16 Y at the same alpha."""
    mode, rule = recipe
    ac, as_, aa = _quantized(M, K, 31, ("four_over_six", "mse", 256.0))
    bc, bs, ba = _quantized(N, K, 32, ("six", "max", 448.0), kind="normal")
    A, B = upload_operand(ac, as_, aa), upload_operand(bc, bs, ba)
    y = nv.gemm(A, B, out_dtype=torch.bfloat16)
    alpha = torch.tensor([float(y.float().abs().max()) / (6 * 448.0) * 1.3], dtype=torch.float32, device="cuda")
    ref = nv.quantize(y, mode, rule, out=None, global_scale=alpha)
    q = nv.gemm_quantized(A, B, alpha, mode, rule)
    assert nv.device_status(q.workspace) == nv.OK
    assert torch.equal(q.codes, ref.codes) and torch.equal(q.scales, ref.scales)
    oc, os_ = oracle.quantize_rows(y.cpu(), float(alpha.cpu()[0]), MODE[mode], RULE[rule])
    assert np.array_equal(to_np(q.codes), oc)
    assert np.array_equal(to_np(q.scales), oracle.swizzle_scales(os_, M, N))


@pytest.mark.slow
def test_prefill_nvfp4_output_and_static_alpha_full_size():
    """The bench's prefill case (X 32768x5120 4/6-MSE, W 17408x5120 scale-6):
    the GEMM writing Y as NVFP4 (4/6-MSE) equals the bf16 GEMM followed by the
    static-alpha quantizer over the whole 32768x17408 output, and sampled rows
    equal the oracle's row quantizer on that Y at the same alpha; X quantized
    at a static alpha equal to its dynamic one reproduces the dynamic call."""
    wl = workloads.WORKLOADS["prefill"]
    x, w = wl.x.make(), wl.w.make()
    xm, xr, xF = "four_over_six", "mse", 256.0
    qx, st = gpu_quantize(x, xm, xr, xF, canary=0)
    assert st == nv.OK
    qs = nv.quantize(x.cuda(), xm, xr, global_scale=qx.global_scale.clone())
    assert nv.device_status(qs.workspace) == nv.OK
    assert torch.equal(qs.codes, qx.codes) and torch.equal(qs.scales, qx.scales)
    wm, wr, wF = wl.w_recipe
    qw, st = gpu_quantize(w, wm, wr, wF, canary=0)
    assert st == nv.OK
    y = nv.gemm(qx, qw, out_dtype=torch.bfloat16)
    alpha = torch.tensor([float(y.float().abs().max()) / (6 * 256.0)], dtype=torch.float32, device="cuda")
    q = nv.gemm_quantized(qx, qw, alpha, "four_over_six", "mse")
    assert nv.device_status(q.workspace) == nv.OK
    ref = nv.quantize(y, "four_over_six", "mse", global_scale=alpha)
    assert torch.equal(q.codes, ref.codes) and torch.equal(q.scales, ref.scales)
    M, N = y.shape
    idx = workloads.sample_rows(M, 32, 2).numpy()
    oc, os_ = oracle.quantize_rows(y[torch.from_numpy(idx).cuda()].cpu(), float(alpha.cpu()[0]), MODE["four_over_six"],
                                   RULE["mse"])
    assert np.array_equal(to_np(q.codes[torch.from_numpy(idx).cuda()]), oc)
    assert np.array_equal(oracle.unswizzle_scales(to_np(q.scales), M, N)[idx], os_)


@pytest.mark.skipif(torch.cuda.device_count() < 2, reason="needs two visible GPUs")
def test_second_device_after_the_first():
    """Kernel attributes (the GEMM's and the augmented quantizer's shared-memory
    opt-in) belong to each device's context: a call on device 1 after calls on
    device 0 must launch and be right."""
    ac, as_, aa = _quantized(256, 512, 51, ("four_over_six", "mse", 256.0))
    bc, bs, ba = _quantized(384, 512, 52, ("six", "max", 448.0), kind="normal")
    ref, guard = oracle.gemm_reference(ac, as_, aa, bc, bs, ba)
    x = workloads.small_operand(128, 512, seed=53).make()
    perm = torch.arange(512, dtype=torch.int32)
    for dev in (0, 1):
        with torch.cuda.device(dev):
            A, B = upload_operand(ac, as_, aa), upload_operand(bc, bs, ba)
            assert A.codes.device.index == dev
            y = nv.gemm(A, B, out_dtype=torch.float32)
            ws = torch.zeros(nv.nvfp4_gemm_workspace_bytes(), dtype=torch.uint8, device="cuda")
            nv.gemm(A, B, out_dtype=torch.float32, out=y, workspace=ws)
            assert nv.device_status(ws) == nv.OK
            assert_gemm_close(to_np(y), ref, guard)
            qa = nv.quantize_arc(x.cuda(), perm.cuda(), 64, nv.AUG_RESIDUAL, "four_over_six", "mse", 256.0)
            assert nv.device_status(qa.workspace) == nv.OK
