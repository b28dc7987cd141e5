"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
on seeded inputs and bring results back for comparison with the oracle."""
import numpy as np
import torch

import oracle
import w4a4_gemm_nvfp4_b200 as nv

MODE = {"six": oracle.MODE_SIX, "four_over_six": oracle.MODE_FOUR_OVER_SIX}
RULE = {"max": oracle.RULE_MAX, "mae": oracle.RULE_MAE, "mse": oracle.RULE_MSE}


def gpu_quantize(x_cpu: torch.Tensor, mode: str, rule: str, fp8_max: float, ldx_pad: int = 0,
                 canary: int = 0xA5):
    """Quantize a CPU bf16 tensor on cuda:0 through nvfp4_quantize.  Output
    buffers are pre-filled with a canary so unwritten bytes show up."""
    rows, K = x_cpu.shape
    if ldx_pad:
        big = torch.zeros(rows, K + ldx_pad, dtype=torch.bfloat16)
        big[:, :K] = x_cpu
        xd = big.cuda()[:, :K]
    else:
        xd = x_cpu.cuda()
    out = nv.NVFP4Tensor(
        codes=torch.full((rows, K // 2), canary, dtype=torch.uint8, device="cuda"),
        scales=torch.full((nv.nvfp4_scales_bytes(rows, K),), canary, dtype=torch.uint8, device="cuda"),
        global_scale=torch.full((1,), -1.0, dtype=torch.float32, device="cuda"),
        workspace=torch.full((nv.nvfp4_quantize_workspace_bytes(rows, K),), 0xFF, dtype=torch.uint8,
                             device="cuda"),
        rows=rows, K=K)
    nv.quantize(xd, mode, rule, fp8_max, out=out)
    status = nv.device_status(out.workspace)
    return out, status


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy()


def alpha_of(q) -> float:
    return float(np.float32(q.global_scale.cpu().numpy()[0]))


def assert_quant_equal(q, x_cpu, mode, rule, fp8_max):
    """Bit-exact comparison of codes, swizzled scales (padding included) and
    alpha with the oracle on the whole tensor."""
    rows, K = x_cpu.shape
    oc, os_, oa = oracle.quantize(x_cpu, MODE[mode], RULE[rule], fp8_max)
    swz = oracle.swizzle_scales(os_, rows, K)
    ga = alpha_of(q)
    assert np.float32(ga) == np.float32(oa), (ga, oa)
    gc = to_np(q.codes)
    bad = np.argwhere(gc != oc)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first {bad[:5].tolist()}: gpu {gc[tuple(bad[0])]:#x} oracle {oc[tuple(bad[0])]:#x}"
    gs = to_np(q.scales)
    bad = np.nonzero(gs != swz)[0]
    assert bad.size == 0, f"{bad.size} scale bytes differ, first {bad[:5].tolist()}: gpu {gs[bad[:5]]} oracle {swz[bad[:5]]}"


def upload_operand(codes: np.ndarray, scales_canon: np.ndarray, alpha: float) -> "nv.NVFP4Tensor":
    """Put an oracle-made operand on the GPU in the C ABI layout."""
    rows, half = codes.shape
    K = half * 2
    swz = oracle.swizzle_scales(scales_canon, rows, K)
    return nv.NVFP4Tensor(
        codes=torch.from_numpy(np.ascontiguousarray(codes)).cuda(),
        scales=torch.from_numpy(swz).cuda(),
        global_scale=torch.tensor([alpha], dtype=torch.float32, device="cuda"),
        workspace=torch.zeros(nv.nvfp4_quantize_workspace_bytes(rows, K), dtype=torch.uint8, device="cuda"),
        rows=rows, K=K)


# GEMM tolerance (max relative error 1e-3 against the fp64 product
# of the dequantized operands).  Entries whose |ref| is below 1e-3 of the sum
# of |products| are cancellation-dominated; they must be within 1e-6 of that
# sum instead.  bf16 output adds its own rounding (2^-9 relative).
REL_TOL = 1e-3
ABS_GUARD = 1e-6


def assert_gemm_close(y: np.ndarray, ref: np.ndarray, guard: np.ndarray, bf16: bool = False):
    y = y.astype(np.float64)
    err = np.abs(y - ref)
    rel = REL_TOL + (2.0 ** -8 if bf16 else 0.0)
    big = np.abs(ref) >= 1e-3 * guard
    ok = np.where(big, err <= rel * np.abs(ref), err <= ABS_GUARD * guard + rel * np.abs(ref))
    if not ok.all():
        idx = np.argwhere(~ok)[:5]
        details = [(tuple(i), float(y[tuple(i)]), float(ref[tuple(i)]), float(guard[tuple(i)])) for i in idx]
        raise AssertionError(f"{(~ok).sum()} of {ok.size} outputs out of tolerance, e.g. {details}")
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(big, err / np.abs(ref), 0.0)
    return float(r.max()) if r.size else 0.0


def hard_block_maxima(alpha: float, Q: float, limit: int = 512) -> np.ndarray:
    """bf16 block maxima b (as float32) for which b * fl(1/(alpha*Q)) and the
    correctly rounded quotient b / (alpha*Q) round to different E4M3 scales,
    plus those whose quotient sits within two units of an E4M3 rounding
    midpoint: the blocks on which a reciprocal-multiply shortcut for the scale
    quotient would go wrong."""
    bits = np.arange(1, 0x7F80, dtype=np.uint32)          # positive finite bf16
    b = (bits << 16).view(np.float32)
    a = np.float32(alpha) * np.float32(Q)
    with np.errstate(over="ignore", divide="ignore", invalid="ignore"):
        q_true = b / a
        q_fast = b * (np.float32(1.0) / a)
    low20 = q_true.view(np.uint32) & np.uint32(0xFFFFF)
    near_mid = np.abs(low20.astype(np.int64) - 0x80000) <= 2
    cand = np.nonzero((q_true != q_fast) | near_mid)[0]
    hard = [i for i in cand
            if near_mid[i] or oracle.e4m3_encode(float(q_true[i])) != oracle.e4m3_encode(float(q_fast[i]))]
    return b[np.array(hard[:limit], dtype=np.int64)] if hard else np.zeros(0, np.float32)


def blocks_with_maxima(maxima: np.ndarray, K: int, seed: int) -> torch.Tensor:
    """A bf16 [rows, K] tensor, one 16-element block per entry of `maxima`
    (row-major over blocks), whose block max |x| is exactly that value: one
    element is +-max, the rest uniform in (-max, max) and rounded toward zero
    so they stay below it."""
    g = np.random.default_rng(seed)
    nb = len(maxima)
    per_row = K // 16
    rows = (nb + per_row - 1) // per_row
    blocks = np.zeros((rows * per_row, 16), np.float32)
    m = np.asarray(maxima, np.float32)
    blocks[:nb] = (g.uniform(-1, 1, (nb, 16)) * m[:, None]).astype(np.float32)
    # truncate to bf16 (toward zero) so |x| <= max keeps holding
    blocks = (blocks.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)
    pos = g.integers(0, 16, nb)
    sign = np.where(g.random(nb) < 0.5, -1.0, 1.0).astype(np.float32)
    blocks[np.arange(nb), pos] = sign * m
    return torch.from_numpy(blocks.reshape(rows, K).copy()).to(torch.bfloat16)
