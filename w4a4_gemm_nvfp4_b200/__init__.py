"""NVFP4 W4A4 linear-layer kernels for NVIDIA B200 (sm_100a).

``quantize`` -- 16-element block-scaled NVFP4 quantization (scale-to-6 or
Four-Over-Six with a max / MAE / MSE selection rule) of a bf16 CUDA matrix,
writing codes and scales in the layout the block-scaled tensor-core MMA reads;
with ``global_scale=`` a caller-supplied (e.g. calibrated) tensor scale
replaces the amax pass.
``quantize_t`` -- the same for x^T (blocks down the columns of x), the layout
of the gradient GEMMs in training.
``quantize_arc`` -- ARCQuant augmented residual channels: channels in a
calibration order plus S appended channels holding the residual of the first
S (activations) or a copy of them (weights), for one GEMM over K + S;
``quantize_arc_rmsnorm`` the same for activations with their RMSNorm fused in.
``gemm`` -- Y = A_hat @ B_hat^T on two NVFP4 operands (tcgen05 block-scaled FP4
MMA, fp32 accumulation, bf16 or fp32 output); ``gemm_segmented`` applies one
B global scale per output-column segment (fused projections);
``gemm_quantized`` writes Y directly as an NVFP4 operand against a static
output scale.
``quantize_gemm`` -- the linear layer in one call: quantize the activations,
then the GEMM against a pre-quantized weight, each kernel starting as a
programmatic dependent of the one before it; ``quantize_arc_gemm`` the same
with the augmented-channel quantizer and a GEMM over K + S.

All of it runs in libnvfp4.so (CUDA, built in-tree by ``build.py``); this
package is a ctypes binding around its C ABI (``include/nvfp4.h``).
"""
from ._lib import (  # noqa: F401
    DEFAULT_FP8_MAX, ERR_CUDA, ERR_INVALID_ARG, ERR_NONFINITE, ERR_TIMEOUT, ERR_UNSUPPORTED_DEVICE,
    LIB_PATH, MODES, OK, OUT_BF16, OUT_FP32, RULES, NVFP4Error, NVFP4Tensor, device_status, gemm,
    gemm_segmented, nvfp4_gemm_segmented, gemm_quantized, nvfp4_gemm_quantized,
    last_error_message, load, nvfp4_codes_bytes, nvfp4_gemm, nvfp4_gemm_workspace_bytes,
    nvfp4_get_device_status, nvfp4_quantize, nvfp4_quantize_noalloc, nvfp4_quantize_with_scale,
    nvfp4_quantize_workspace_bytes, nvfp4_scales_bytes,
    quantize, quantize_t, nvfp4_quantize_t, quantize_gemm, nvfp4_quantize_gemm, quantize_arc_gemm,
    nvfp4_quantize_arc_gemm, quantize_arc_rmsnorm, nvfp4_quantize_arc_rmsnorm,
    nvfp4_quantize_arc_rmsnorm_workspace_bytes, nvfp4_quantize_arc_rmsnorm_gemm, quantize_arc, nvfp4_quantize_arc, AUG_RESIDUAL, AUG_DUPLICATE, status_string, testing_set_gemm_wait)
