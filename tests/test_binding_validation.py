"""Argument checks of the Python binding (CPU only).

Every wrapper must refuse a tensor of the wrong dtype, length or shape before it reaches the
library: a short scale or bias vector would otherwise become an out-of-bounds device read.
The library is replaced by a fake that fails the test if any call gets through, and the
current-device check is stubbed so that CPU tensors stand in for device tensors.
"""
import pytest
import torch

from hadamard_rotated_int8_b200 import _native


class _NoLibrary:
    def __getattr__(self, name):
        raise AssertionError(f"{name} reached the library despite invalid arguments")


@pytest.fixture(autouse=True)
def no_library(monkeypatch):
    monkeypatch.setattr(_native, "lib", lambda: _NoLibrary())
    monkeypatch.setattr(_native, "_on_current_device", lambda t, name: None)


M, N, K, R = 64, 48, 256, 16


def t8(*shape):
    return torch.zeros(shape, dtype=torch.int8)


def f32(*shape):
    return torch.zeros(shape, dtype=torch.float32)


def bf(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def linear_args(**over):
    a = dict(qx=t8(M, K), sx=f32(M), qW=t8(N, K), sW=f32(N), bias=bf(N), out=bf(M, N),
             acc_out=None)
    a.update(over)
    return a


@pytest.mark.parametrize("over,err", [
    (dict(sx=f32(M - 1)), ValueError),                 # short token scales
    (dict(sx=torch.zeros(M, dtype=torch.float64)), TypeError),
    (dict(sx=f32(M, 1)), ValueError),                  # not 1-D
    (dict(sx=None), ValueError),
    (dict(sW=f32(N - 1)), ValueError),                 # short row scales
    (dict(sW=bf(N)), TypeError),
    (dict(bias=bf(N - 1)), ValueError),                # short bias
    (dict(bias=f32(N)), TypeError),
    (dict(out=bf(M, N + 1)), ValueError),
    (dict(out=f32(M, N)), TypeError),
    (dict(acc_out=torch.zeros(M, N - 1, dtype=torch.int32)), ValueError),
    (dict(acc_out=f32(M, N)), TypeError),
    (dict(qW=t8(N, K + 16)), ValueError),              # K mismatch
])
def test_linear_refuses_bad_operands(over, err):
    a = linear_args(**over)
    for fn in (_native.sdnq_int8_linear, _native.sdnq_int8_linear_gelu):
        with pytest.raises(err):
            fn(a["qx"], a["sx"], a["qW"], a["sW"], a["bias"], out=a["out"], acc_out=a["acc_out"])


def test_fp8_linear_refuses_short_scales_and_int_accumulators():
    qx, qW = torch.zeros(M, K, dtype=torch.uint8), torch.zeros(N, K, dtype=torch.uint8)
    with pytest.raises(ValueError):
        _native.sdnq_fp8_linear(qx, f32(M), qW, f32(N - 4))
    with pytest.raises(TypeError):   # the e4m3 accumulators are fp32
        _native.sdnq_fp8_linear(qx, f32(M), qW, f32(N),
                                acc_out=torch.zeros(M, N, dtype=torch.int32))


@pytest.mark.parametrize("what", ["A_dtype", "B_shape", "x_shape", "u_ws", "sx", "bias"])
def test_lora_refuses_bad_operands(what):
    a = dict(qx=t8(M, K), sx=f32(M), qW=t8(N, K), sW=f32(N), bias=bf(N), x=bf(M, K),
             A=bf(K, R), B=bf(R, N), u_ws=bf(M, R))
    if what == "A_dtype":
        a["A"] = f32(K, R)
    elif what == "B_shape":
        a["B"] = bf(R, N + 8)
    elif what == "x_shape":
        a["x"] = bf(M + 1, K)
    elif what == "u_ws":
        a["u_ws"] = bf(M, R - 1)
    elif what == "sx":
        a["sx"] = f32(M // 2)
    else:
        a["bias"] = bf(N // 2)
    with pytest.raises((TypeError, ValueError)):
        _native.sdnq_int8_linear_lora(a["qx"], a["sx"], a["qW"], a["sW"], a["bias"], a["x"],
                                      a["A"], a["B"], 1.0, u_ws=a["u_ws"])
    if what != "u_ws":
        with pytest.raises((TypeError, ValueError)):
            _native.sdnq_int8_linear_lora_noalloc(a["qx"], a["sx"], a["qW"], a["sW"],
                                                  a["bias"], a["x"], a["A"], a["B"], 1.0)


def test_lora_halves_refuse_bad_operands():
    with pytest.raises(ValueError):   # A rows != K
        _native.sdnq_lora_down(bf(M, K), bf(K + 16, R))
    with pytest.raises(ValueError):   # u of the wrong shape
        _native.sdnq_lora_down(bf(M, K), bf(K, R), u=bf(M, R + 16))
    with pytest.raises(TypeError):
        _native.sdnq_lora_down(f32(M, K), bf(K, R))
    a = dict(qx=t8(M, K), sx=f32(M), qW=t8(N, K), sW=f32(N), bias=bf(N), u=bf(M, R), B=bf(R, N))
    for key, bad, err in (("u", bf(M - 1, R), ValueError), ("B", bf(R, N + 8), ValueError),
                          ("u", f32(M, R), TypeError), ("sx", f32(M - 1), ValueError)):
        b = dict(a, **{key: bad})
        with pytest.raises(err):
            _native.sdnq_int8_linear_lora_up(b["qx"], b["sx"], b["qW"], b["sW"], b["bias"],
                                             b["u"], b["B"], 1.0)


def test_noalloc_refuses_more_rows_than_its_scratch_holds():
    rows = _native.NOALLOC_MAX_U_ELEMS // R + 1
    with pytest.raises(ValueError, match="scratch"):
        _native.sdnq_int8_linear_lora_noalloc(t8(rows, K), f32(rows), t8(N, K), f32(N), None,
                                              bf(rows, K), bf(K, R), bf(R, N), 1.0)


def test_fused_refuses_short_counter_buffer_and_workspaces():
    x = bf(M, K)
    with pytest.raises(ValueError):
        _native.sdnq_int8_linear_fused(x, 256, t8(N, K), f32(N),
                                       sync_ws=torch.zeros(1, dtype=torch.int32))
    sync = torch.zeros(64, dtype=torch.int32)
    with pytest.raises(ValueError):
        _native.sdnq_int8_linear_fused(x, 256, t8(N, K), f32(N), sx_ws=f32(M - 1), sync_ws=sync)
    with pytest.raises(ValueError):
        _native.sdnq_int8_linear_fused(x, 256, t8(N, K), f32(N), qx_ws=t8(M, K - 16),
                                       sync_ws=sync)


def test_rotquant_refuses_wrong_outputs():
    with pytest.raises(ValueError):
        _native.sdnq_rotquant_act(bf(M, K), 256, qx=t8(M, K), sx=f32(M - 1))
    with pytest.raises(ValueError):
        _native.sdnq_rotate_quant_weight(bf(N, K), 256, qW=t8(N, K // 2))
    with pytest.raises(TypeError):
        _native.sdnq_rotquant_fp8(bf(M, K), 256, q=t8(M, K))


def test_grad_refuses_short_row_scales_and_outputs():
    dy, qW = bf(M, N), t8(N, K)
    with pytest.raises(ValueError):
        _native.sdnq_int8_linear_grad_input(dy, qW, f32(N - 1), 256)
    with pytest.raises(ValueError):
        _native.sdnq_quant_grad_output(dy, f32(N - 1))
    with pytest.raises(ValueError):
        _native.sdnq_int8_grad_input_gemm(t8(M, N), f32(M - 1), qW, 256)
    with pytest.raises(ValueError):
        _native.sdnq_int8_grad_input_gemm(t8(M, N), f32(M), qW, 256, out=bf(M, K - 8))


def test_cpu_tensors_are_refused_without_a_device(monkeypatch):
    monkeypatch.undo()   # the real device check
    with pytest.raises(ValueError, match="CUDA"):
        _native.sdnq_rotquant_act(bf(M, K), 256)
