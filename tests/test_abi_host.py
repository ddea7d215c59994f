"""Host-only checks of the C ABI: the library loads, exports every entry point that
include/sdnq.h declares, and rejects bad arguments before touching a GPU. Nothing here
launches a kernel: every call either fails validation or (on a machine without a B200)
fails the device check."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

from hadamard_rotated_int8_b200 import _build, _native

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sdnq.h")

A16 = 0x10000      # 16-byte aligned fake address: never dereferenced (validation fails first)
MIS = 0x10001      # misaligned fake address
S = 0              # stream: NULL


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"\b(sdnq_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return _native.lib()


def test_header_declares_the_four_layer_calls():
    syms = declared_symbols()
    for name in ("sdnq_rotate_quant_weight", "sdnq_rotquant_act", "sdnq_int8_linear",
                 "sdnq_int8_linear_lora", "sdnq_status_string"):
        assert name in syms


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", _build.LIB], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (sdnq_\w+)", out))
    assert set(declared_symbols()) <= exported
    # nothing but the ABI is exported under the sdnq_ prefix
    assert exported == set(declared_symbols())


def test_binding_names_match_the_abi(lib):
    import hadamard_rotated_int8_b200 as pkg
    for name in ("sdnq_rotate_quant_weight", "sdnq_rotquant_act", "sdnq_int8_linear",
                 "sdnq_int8_linear_lora", "sdnq_gelu_bf16"):
        assert callable(getattr(pkg, name))
    assert set(_native.SIGNATURES) == set(declared_symbols())


def test_status_strings(lib):
    for code in range(7):
        s = _native.status_string(code)
        assert s.startswith("SDNQ_")
    assert _native.status_string(99) == "SDNQ_ERR_UNKNOWN"
    assert "sm_100a" in _native.version()


def rq(lib, x=A16, M=4, K=256, ld=256, g=256, q=A16, s=A16):
    return lib.sdnq_rotquant_act(x, M, K, ld, g, q, s, S)


def test_rotquant_validation(lib):
    assert rq(lib, x=0) == _native.SDNQ_ERR_NULL
    assert rq(lib, q=0) == _native.SDNQ_ERR_NULL
    assert rq(lib, s=0) == _native.SDNQ_ERR_NULL
    assert rq(lib, M=-1) == _native.SDNQ_ERR_SHAPE
    assert rq(lib, K=0) == _native.SDNQ_ERR_SHAPE
    assert rq(lib, K=264, ld=264) == _native.SDNQ_ERR_SHAPE        # K % 16
    assert rq(lib, K=256, ld=128) == _native.SDNQ_ERR_SHAPE        # ld < K
    assert rq(lib, K=262144, ld=262144) == _native.SDNQ_ERR_SHAPE  # K > max
    assert rq(lib, g=4) == _native.SDNQ_ERR_UNSUPPORTED
    assert rq(lib, g=512) == _native.SDNQ_ERR_UNSUPPORTED
    assert rq(lib, g=96) == _native.SDNQ_ERR_UNSUPPORTED           # not a power of two
    assert rq(lib, K=384, ld=384, g=256) == _native.SDNQ_ERR_SHAPE  # K % g
    assert rq(lib, ld=260) == _native.SDNQ_ERR_ALIGN
    assert rq(lib, x=MIS) == _native.SDNQ_ERR_ALIGN
    assert rq(lib, q=A16 + 8) == _native.SDNQ_ERR_ALIGN
    assert lib.sdnq_rotate_quant_weight(A16, 4, 256, 256, 256, 0, A16, S) == _native.SDNQ_ERR_NULL


def lin(lib, qx=A16, sx=A16, qw=A16, sw=A16, bias=0, M=128, N=256, K=256, out=A16, ldo=256,
        acc=0):
    return lib.sdnq_int8_linear(qx, sx, qw, sw, bias, M, N, K, out, ldo, acc, S)


def test_linear_validation(lib):
    assert lin(lib, qx=0) == _native.SDNQ_ERR_NULL
    assert lin(lib, sw=0) == _native.SDNQ_ERR_NULL
    assert lin(lib, out=0) == _native.SDNQ_ERR_NULL
    assert lin(lib, M=-3) == _native.SDNQ_ERR_SHAPE
    assert lin(lib, N=0) == _native.SDNQ_ERR_SHAPE
    assert lin(lib, K=8) == _native.SDNQ_ERR_SHAPE
    assert lin(lib, K=200) == _native.SDNQ_ERR_SHAPE
    assert lin(lib, ldo=128) == _native.SDNQ_ERR_SHAPE
    assert lin(lib, ldo=260) == _native.SDNQ_ERR_ALIGN
    assert lin(lib, qx=MIS) == _native.SDNQ_ERR_ALIGN
    assert lin(lib, sx=A16 + 2) == _native.SDNQ_ERR_ALIGN
    assert lin(lib, sw=A16 + 4) == _native.SDNQ_ERR_ALIGN
    assert lin(lib, bias=A16 + 8) == _native.SDNQ_ERR_ALIGN
    assert lin(lib, acc=A16 + 4) == _native.SDNQ_ERR_ALIGN


def lora(lib, x=A16, A=A16, B=A16, rank=64, u=A16, N=256, ldx=256):
    return lib.sdnq_int8_linear_lora(A16, A16, A16, A16, 0, x, ldx, A, B, rank, 1.0, u, 128, N,
                                     256, A16, 256, 0, S)


def test_lora_validation(lib):
    assert lora(lib, x=0) == _native.SDNQ_ERR_NULL
    assert lora(lib, u=0) == _native.SDNQ_ERR_NULL
    assert lora(lib, rank=8) == _native.SDNQ_ERR_UNSUPPORTED
    assert lora(lib, rank=24) == _native.SDNQ_ERR_UNSUPPORTED
    assert lora(lib, rank=512) == _native.SDNQ_ERR_UNSUPPORTED
    assert lora(lib, ldx=128) == _native.SDNQ_ERR_SHAPE
    assert lora(lib, N=252) == _native.SDNQ_ERR_SHAPE  # B rows must be 16-byte strided
    assert lora(lib, A=MIS) == _native.SDNQ_ERR_ALIGN


def lora_down(lib, x=A16, ldx=256, A=A16, rank=64, M=128, K=256, u=A16):
    return lib.sdnq_lora_down(x, ldx, A, rank, M, K, u, S)


def lora_up(lib, u=A16, B=A16, rank=64, N=256, M=128):
    return lib.sdnq_int8_linear_lora_up(A16, A16, A16, A16, 0, u, B, rank, 1.0, M, N, 256, A16,
                                        256, 0, S)


def test_lora_halves_validation(lib):
    """The down-projection and the up-projection GEMM as calls of their own refuse what the
    whole LoRA call refuses, before any device work."""
    assert lora_down(lib, x=0) == _native.SDNQ_ERR_NULL
    assert lora_down(lib, A=0) == _native.SDNQ_ERR_NULL
    assert lora_down(lib, u=0) == _native.SDNQ_ERR_NULL
    assert lora_down(lib, M=-1) == _native.SDNQ_ERR_SHAPE
    assert lora_down(lib, K=8) == _native.SDNQ_ERR_SHAPE
    assert lora_down(lib, K=264) == _native.SDNQ_ERR_SHAPE      # K % 16
    assert lora_down(lib, ldx=128) == _native.SDNQ_ERR_SHAPE
    assert lora_down(lib, rank=24) == _native.SDNQ_ERR_UNSUPPORTED
    assert lora_down(lib, rank=512) == _native.SDNQ_ERR_UNSUPPORTED
    assert lora_down(lib, ldx=260) == _native.SDNQ_ERR_ALIGN     # rows not 16-byte strided
    assert lora_down(lib, u=MIS) == _native.SDNQ_ERR_ALIGN
    assert lora_up(lib, u=0) == _native.SDNQ_ERR_NULL
    assert lora_up(lib, B=0) == _native.SDNQ_ERR_NULL
    assert lora_up(lib, rank=8) == _native.SDNQ_ERR_UNSUPPORTED
    assert lora_up(lib, N=252) == _native.SDNQ_ERR_SHAPE
    assert lora_up(lib, B=MIS) == _native.SDNQ_ERR_ALIGN
    assert lora_up(lib, u=MIS) == _native.SDNQ_ERR_ALIGN


def grad(lib, dy=A16, lddy=256, qW=A16, sW=A16, M=128, N=256, K=512, g=256, qg=A16, sg=A16,
         dx=A16, lddx=512, acc=0):
    return lib.sdnq_int8_linear_grad_input(dy, lddy, qW, sW, M, N, K, g, qg, sg, dx, lddx, acc, S)


def test_grad_input_validation(lib):
    assert grad(lib, dy=0) == _native.SDNQ_ERR_NULL
    assert grad(lib, qg=0) == _native.SDNQ_ERR_NULL
    assert grad(lib, sW=0) == _native.SDNQ_ERR_NULL
    assert grad(lib, M=-1) == _native.SDNQ_ERR_SHAPE
    assert grad(lib, N=8) == _native.SDNQ_ERR_SHAPE
    assert grad(lib, N=264, lddy=264) == _native.SDNQ_ERR_SHAPE   # contraction % 16
    assert grad(lib, K=520, lddx=520) == _native.SDNQ_ERR_SHAPE   # K % group
    assert grad(lib, lddy=128) == _native.SDNQ_ERR_SHAPE
    assert grad(lib, lddx=256) == _native.SDNQ_ERR_SHAPE
    assert grad(lib, g=48) == _native.SDNQ_ERR_UNSUPPORTED
    assert grad(lib, g=512) == _native.SDNQ_ERR_UNSUPPORTED
    assert grad(lib, lddy=260) == _native.SDNQ_ERR_ALIGN
    assert grad(lib, sW=A16 + 4) == _native.SDNQ_ERR_ALIGN
    assert grad(lib, qg=MIS) == _native.SDNQ_ERR_ALIGN
    assert grad(lib, acc=A16 + 4) == _native.SDNQ_ERR_ALIGN


def fused(lib, x=A16, ldx=256, g=256, sync=A16, qx=A16, sx=A16, out=A16, M=128, K=256, policy=0):
    return lib.sdnq_int8_linear_fused(x, ldx, g, A16, A16, 0, M, 256, K, qx, sx, sync, out, 256,
                                      0, policy, S)


def test_fused_validation(lib):
    assert fused(lib, x=0) == _native.SDNQ_ERR_NULL
    assert fused(lib, sync=0) == _native.SDNQ_ERR_NULL
    assert fused(lib, qx=0) == _native.SDNQ_ERR_NULL
    assert fused(lib, sync=A16 + 2) == _native.SDNQ_ERR_ALIGN
    assert fused(lib, g=48) == _native.SDNQ_ERR_UNSUPPORTED
    assert fused(lib, ldx=128) == _native.SDNQ_ERR_SHAPE
    assert fused(lib, K=200, ldx=200) == _native.SDNQ_ERR_SHAPE
    assert fused(lib, x=MIS) == _native.SDNQ_ERR_ALIGN
    assert fused(lib, policy=3) == _native.SDNQ_ERR_UNSUPPORTED


def test_fused_plan_validation(lib):
    import ctypes
    one = ctypes.c_int32(7)
    ref = ctypes.byref(one)
    assert lib.sdnq_int8_linear_fused_plan(4096, 3072, 3072, 0, None) == _native.SDNQ_ERR_NULL
    assert lib.sdnq_int8_linear_fused_plan(-1, 3072, 3072, 0, ref) == _native.SDNQ_ERR_SHAPE
    assert lib.sdnq_int8_linear_fused_plan(4096, 0, 3072, 0, ref) == _native.SDNQ_ERR_SHAPE
    assert lib.sdnq_int8_linear_fused_plan(4096, 3072, 3000, 0, ref) == _native.SDNQ_ERR_SHAPE
    assert lib.sdnq_int8_linear_fused_plan(4096, 3072, 3072, 5, ref) == \
        _native.SDNQ_ERR_UNSUPPORTED
    assert one.value == 7   # nothing written on an error
    if not torch.cuda.is_available():
        assert lib.sdnq_int8_linear_fused_plan(4096, 3072, 3072, 0, ref) == \
            _native.SDNQ_ERR_UNSUPPORTED


def test_gelu_and_selftest_validation(lib):
    assert lib.sdnq_gelu_bf16(0, 4, 8, 8, A16, 8, S) == _native.SDNQ_ERR_NULL
    assert lib.sdnq_gelu_bf16(A16, 4, 0, 8, A16, 8, S) == _native.SDNQ_ERR_SHAPE
    assert lib.sdnq_gelu_bf16(A16, 4, 8, 12, A16, 16, S) == _native.SDNQ_ERR_ALIGN
    assert lib.sdnq_gelu_bf16(A16, 4, 8, 8, A16, 16, S) == _native.SDNQ_ERR_SHAPE  # alias, ld differ
    assert lib.sdnq_selftest_wait_timeout(10, S) == _native.SDNQ_ERR_SHAPE


W256 = 0x100000    # 256-byte aligned fake workspace address


def attn(lib, q=A16, k=A16, v=A16, B=1, Lq=64, Lk=96, H=2, D=128, g=256, scale=0.088,
         smooth=1, ws=W256, ws_bytes=None, o=A16):
    if ws_bytes is None:
        ws_bytes = lib.sdnq_attention_workspace(B, Lq, Lk, H, 128, None)
    return lib.sdnq_attention_int8qk(q, k, v, B, Lq, Lk, H, D, g, scale, smooth, ws, ws_bytes,
                                     o, S)


def test_attention_validation(lib):
    assert attn(lib, q=0) == _native.SDNQ_ERR_NULL
    assert attn(lib, ws=0) == _native.SDNQ_ERR_NULL
    assert attn(lib, D=64) == _native.SDNQ_ERR_UNSUPPORTED
    assert attn(lib, g=96) == _native.SDNQ_ERR_UNSUPPORTED
    assert attn(lib, Lk=0) == _native.SDNQ_ERR_SHAPE
    assert attn(lib, ws_bytes=1024) == _native.SDNQ_ERR_SHAPE
    assert attn(lib, ws=W256 + 16) == _native.SDNQ_ERR_ALIGN
    assert attn(lib, v=MIS) == _native.SDNQ_ERR_ALIGN
    # the softmax scale must be finite and >= 0 (the kernel takes the row maximum of
    # acc * s_k and scales it afterwards, which needs a nonnegative factor)
    for bad in (-0.5, float("nan"), float("inf")):
        assert attn(lib, scale=bad) == _native.SDNQ_ERR_UNSUPPORTED
    ws_bytes = lib.sdnq_attention_workspace(1, 64, 96, 2, 128, None)
    assert lib.sdnq_attention_core(A16, 1, 64, 96, 2, 128, -1.0, W256, ws_bytes, A16, S) == \
        _native.SDNQ_ERR_UNSUPPORTED
    assert lib.sdnq_attention_workspace(1, 0, 96, 2, 128, None) < 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path only")
def test_valid_arguments_without_a_b200_are_refused(lib):
    # no silent CPU path: a well-formed call on a machine without an sm_100 GPU is refused
    assert rq(lib) == _native.SDNQ_ERR_UNSUPPORTED
    assert rq(lib, M=0) == _native.SDNQ_ERR_UNSUPPORTED
    assert lin(lib) == _native.SDNQ_ERR_UNSUPPORTED
    assert lora(lib) == _native.SDNQ_ERR_UNSUPPORTED
    assert lib.sdnq_gelu_bf16(A16, 4, 8, 8, A16, 8, S) == _native.SDNQ_ERR_UNSUPPORTED
    assert grad(lib) == _native.SDNQ_ERR_UNSUPPORTED
    assert fused(lib) == _native.SDNQ_ERR_UNSUPPORTED
    assert attn(lib) == _native.SDNQ_ERR_UNSUPPORTED
    assert attn(lib, scale=0.0) == _native.SDNQ_ERR_UNSUPPORTED


def test_binding_refuses_cpu_tensors(lib):
    import hadamard_rotated_int8_b200 as pkg
    with pytest.raises(ValueError):
        pkg.sdnq_rotquant_act(torch.zeros(4, 256, dtype=torch.bfloat16))
