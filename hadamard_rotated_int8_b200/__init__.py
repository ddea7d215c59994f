"""Hadamard-rotated ("ConvRot") INT8 linear layer for NVIDIA B200 (sm_100a).

The compute lives in ``libsdnq.so`` (hand-written CUDA behind the C ABI of
``include/sdnq.h``); this package is the thin Python binding over it, with the same names:

* ``sdnq_rotate_quant_weight``  weight rotate + row-wise int8 quantize (offline)
* ``sdnq_rotquant_act``         online activation rotate + per-token int8 quantize
* ``sdnq_int8_linear``          int8 x int8 -> int32 tensor-core matmul + fp32 de-quant epilogue
* ``sdnq_int8_linear_fused``    rotate + quantize and the int8 linear in one launch
* ``sdnq_int8_linear_fused_plan`` whether that call takes one launch or two for a shape
* ``sdnq_int8_linear_gelu``     the same with GELU fused into the epilogue (MLP up-projection)
* ``sdnq_int8_linear_lora``     the same plus the bf16 LoRA side term
  (= ``sdnq_lora_down`` then ``sdnq_int8_linear_lora_up``)
* ``sdnq_int8_linear_grad_input`` input gradient through the frozen rotated int8 base
  (= ``sdnq_quant_grad_output`` then ``sdnq_int8_grad_input_gemm``)
* ``sdnq_gelu_bf16``            exact-erf GELU (MLP glue)
* ``sdnq_rotquant_fp8``, ``sdnq_fp8_linear``  the FP8 (e4m3) variant of the same path
* ``sdnq_attention_int8qk``     attention with Hadamard-rotated int8 QK and a bf16 PV

``linear`` composes the online path (rotate + quantize, then the int8 linear).
"""
from ._native import (SdnqError, lib, sdnq_attention_int8qk, sdnq_device_status,
                      sdnq_fp8_linear, sdnq_gelu_bf16,
                      sdnq_int8_linear, sdnq_rotquant_fp8,
                      sdnq_int8_grad_input_gemm, sdnq_int8_linear_fused,
                      sdnq_int8_linear_fused_plan, sdnq_int8_linear_gelu,
                      sdnq_int8_linear_grad_input, sdnq_int8_linear_lora,
                      sdnq_int8_linear_lora_noalloc, sdnq_int8_linear_lora_up,
                      sdnq_lora_down, sdnq_rotate_quant_weight,
                      sdnq_quant_grad_output, sdnq_rotquant_act, sdnq_selftest_wait_timeout,
                      status_string, version)

__all__ = [
    "SdnqError", "lib", "linear", "sdnq_attention_int8qk", "sdnq_device_status",
    "sdnq_fp8_linear", "sdnq_gelu_bf16",
    "sdnq_int8_linear", "sdnq_rotquant_fp8",
    "sdnq_int8_grad_input_gemm", "sdnq_int8_linear_fused", "sdnq_int8_linear_fused_plan",
    "sdnq_int8_linear_gelu",
    "sdnq_int8_linear_grad_input",
    "sdnq_int8_linear_lora", "sdnq_quant_grad_output",
    "sdnq_int8_linear_lora_noalloc", "sdnq_int8_linear_lora_up", "sdnq_lora_down",
    "sdnq_rotate_quant_weight", "sdnq_rotquant_act", "sdnq_selftest_wait_timeout",
    "status_string", "version",
]


def linear(x, qW, sW, group=256, bias=None, lora=None, gelu=False, out=None, stream=None):
    """y = rotated-int8 linear of x [M, K] bf16 against pre-quantized weights (qW, sW).
    ``lora`` = (A, B, lora_scale) adds the bf16 adapter term; ``gelu`` applies GELU to the
    output inside the GEMM epilogue (not combined with ``lora``)."""
    if gelu and lora is not None:
        raise ValueError("gelu with lora is not provided")
    if not gelu and lora is None:
        return sdnq_int8_linear_fused(x, group, qW, sW, bias, out=out, stream=stream)
    qx, sx = sdnq_rotquant_act(x, group, stream=stream)
    if gelu:
        return sdnq_int8_linear_gelu(qx, sx, qW, sW, bias, out=out, stream=stream)
    A, B, scale = lora
    return sdnq_int8_linear_lora(qx, sx, qW, sW, bias, x, A, B, scale, out=out, stream=stream)
