"""The Python binding's buffer checks (host only, no GPU).  The C ABI takes
raw pointers and cannot see buffer sizes, so the wrappers check every torch
buffer against the shape the call reads or writes; these tests run those
checks on CPU tensors (a tensor on the `meta` device stands in for a buffer on
another device)."""
import pytest
import torch

import w4a4_gemm_nvfp4_b200 as nv
from w4a4_gemm_nvfp4_b200 import _lib as L

CPU = torch.device("cpu")


def _operand(rows, K, codes_rows=None, scales_bytes=None, dtype=torch.uint8, device="cpu"):
    codes_rows = rows if codes_rows is None else codes_rows
    scales_bytes = nv.nvfp4_scales_bytes(rows, K) if scales_bytes is None else scales_bytes
    return nv.NVFP4Tensor(
        codes=torch.empty(codes_rows, K // 2, dtype=dtype, device=device),
        scales=torch.empty(scales_bytes, dtype=torch.uint8, device=device),
        global_scale=torch.empty(1, dtype=torch.float32, device=device),
        workspace=torch.empty(nv.nvfp4_quantize_workspace_bytes(rows, K), dtype=torch.uint8, device=device),
        rows=rows, K=K)


@pytest.mark.parametrize("rows,K", [(1, 64), (129, 192), (300, 1024)])
def test_exact_operand_buffers_pass(rows, K):
    L._check_operand(_operand(rows, K), "q", rows, K, CPU, workspace=True)


def test_short_codes_are_rejected():
    with pytest.raises(ValueError, match="codes"):
        L._check_operand(_operand(130, 256, codes_rows=129), "q", 130, 256, CPU)


def test_short_scales_are_rejected():
    # 130 rows pad to 256 in the swizzled layout: 128 rows' worth is too short
    with pytest.raises(ValueError, match="scales"):
        L._check_operand(_operand(130, 256, scales_bytes=nv.nvfp4_scales_bytes(128, 256)), "q", 130, 256, CPU)


def test_wrong_dtype_device_and_shape_metadata_are_rejected():
    with pytest.raises(ValueError, match="must be torch.uint8"):
        L._check_operand(_operand(64, 128, dtype=torch.int8), "q", 64, 128, CPU)
    with pytest.raises(ValueError, match="is on meta"):
        L._check_operand(_operand(64, 128, device="meta"), "q", 64, 128, CPU)
    with pytest.raises(ValueError, match=r"\[64, 128\] operand"):
        L._check_operand(_operand(64, 128), "q", 64, 256, CPU)


def test_non_contiguous_codes_are_rejected():
    q = _operand(64, 128)
    q.codes = torch.empty(64, 128, dtype=torch.uint8)[:, :64]
    with pytest.raises(ValueError, match="contiguous"):
        L._check_operand(q, "q", 64, 128, CPU)


def test_output_checks():
    L._check_output(torch.empty(5, 7, dtype=torch.float32), 5, 7, torch.float32, CPU)
    L._check_output(torch.empty(5, 10, dtype=torch.bfloat16)[:, :7], 5, 7, torch.bfloat16, CPU)  # padded rows
    L._check_output(torch.empty(1, 1, dtype=torch.bfloat16), 1, 1, torch.bfloat16, CPU)
    with pytest.raises(ValueError, match="must be torch.float32"):
        # a bf16 buffer would be overrun by fp32 stores
        L._check_output(torch.empty(5, 7, dtype=torch.bfloat16), 5, 7, torch.float32, CPU)
    with pytest.raises(ValueError, match="shape"):
        L._check_output(torch.empty(5, 6, dtype=torch.float32), 5, 7, torch.float32, CPU)
    with pytest.raises(ValueError, match="unit stride"):
        L._check_output(torch.empty(7, 5, dtype=torch.float32).t(), 5, 7, torch.float32, CPU)
    with pytest.raises(ValueError, match="is on meta"):
        L._check_output(torch.empty(5, 7, dtype=torch.float32, device="meta"), 5, 7, torch.float32, CPU)


def test_output_dtype_defaults_to_the_out_buffer():
    assert L._out_code(None, None) == (torch.bfloat16, nv.OUT_BF16)
    assert L._out_code(None, torch.empty(2, 2, dtype=torch.float32)) == (torch.float32, nv.OUT_FP32)
    assert L._out_code(torch.bfloat16, None) == (torch.bfloat16, nv.OUT_BF16)
    with pytest.raises(ValueError, match="out_dtype"):
        L._out_code(torch.float16, None)


def test_scalar_buffers():
    L._require(torch.empty(1, dtype=torch.float32), "alpha", torch.float32, 1, CPU, contiguous=False)
    with pytest.raises(ValueError, match="needs 1"):
        L._require(torch.empty(0, dtype=torch.float32), "alpha", torch.float32, 1, CPU, contiguous=False)
    with pytest.raises(TypeError):
        L._require(0.5, "alpha", torch.float32, 1, CPU)


def test_row_pitch_of_a_single_row_is_its_length():
    """torch may give a size-1 dimension any stride (0 after some views); the
    binding passes the row length as the pitch of a one-row tensor."""
    from w4a4_gemm_nvfp4_b200._lib import _row_pitch

    one = torch.zeros(64, dtype=torch.bfloat16).as_strided((1, 64), (0, 1))
    assert one.stride(0) == 0 and _row_pitch(one) == 64
    many = torch.zeros(3, 80, dtype=torch.bfloat16)[:, :64]
    assert _row_pitch(many) == 80
