"""The no-allocation LoRA entry point, checked against the regular one and the oracle.

Some callers cannot hand the library a workspace: their framework owns all device memory
(a caching allocator or a fixed memory plan) and does not permit allocations from outside
it, or a cudaMalloc, with its possible device synchronisation and unpredictable latency, is
not acceptable where they run. sdnq_int8_linear_lora_noalloc serves them by keeping the
LoRA intermediate u in a fixed array inside the library. Here it is called through the C ABI
twice in a row, on two different problems, and each result must be bit for bit that of
sdnq_int8_linear_lora given a caller-allocated u_ws (both run the same kernels on the same
inputs), and within the LoRA bound of the CPU oracle that the parity tests use. The Python
wrapper is exercised too.

This file is collected last so that a run stopping at its first failure has run every
other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import hadamard_rotated_int8_b200 as sd
from hadamard_rotated_int8_b200 import _build, _native, synthetic
from tests.test_gpu_parity import check_lora_tolerance

pytestmark = pytest.mark.gpu

P = ctypes.c_void_p


def _ulp_diff(a_bits, b_bits):
    def key(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, 0x8000 - (b & 0x7fff), 0x8000 + b)
    return np.abs(key(a_bits) - key(b_bits))


def _bits(t):
    return synthetic.bits(t.detach().cpu().contiguous())


def _prepared(M, N, K, rank, seed):
    case = synthetic.make_case(M=M, N=N, K=K, g=256, seed=seed, outlier_count=K // 100,
                               outlier_factor=30.0, bias_std=0.01, lora_rank=rank,
                               lora_scale=0.5)
    x = case.x.cuda()
    qW, sW = sd.sdnq_rotate_quant_weight(case.W.cuda(), 256)
    qx, sx = sd.sdnq_rotquant_act(x, 256)
    return dict(case=case, x=x, qx=qx, sx=sx, qW=qW, sW=sW, bias=case.bias.cuda(),
                A=case.A.cuda(), B=case.B.cuda(), scale=case.lora_scale, M=M, N=N, K=K,
                rank=rank)


def _noalloc_via_cabi(p):
    """Call sdnq_int8_linear_lora_noalloc through ctypes with raw device pointers."""
    out = torch.empty((p["M"], p["N"]), dtype=torch.bfloat16, device="cuda")
    st = _native.lib().sdnq_int8_linear_lora_noalloc(
        P(p["qx"].data_ptr()), P(p["sx"].data_ptr()), P(p["qW"].data_ptr()),
        P(p["sW"].data_ptr()), P(p["bias"].data_ptr()), P(p["x"].data_ptr()),
        p["x"].stride(0), P(p["A"].data_ptr()), P(p["B"].data_ptr()), p["rank"],
        float(p["scale"]), p["M"], p["N"], p["K"], P(out.data_ptr()), out.stride(0), P(0),
        P(torch.cuda.current_stream().cuda_stream))
    assert st == _native.SDNQ_OK, _native.status_string(st)
    return out


def _with_workspace(p):
    u = torch.empty((p["M"], p["rank"]), dtype=torch.bfloat16, device="cuda")
    return sd.sdnq_int8_linear_lora(p["qx"], p["sx"], p["qW"], p["sW"], p["bias"], p["x"],
                                    p["A"], p["B"], p["scale"], u_ws=u)


def _oracle(p):
    c = p["case"]
    return oracle.linear(synthetic.bits(c.x), *oracle.rotate_quantize(synthetic.bits(c.W), 256),
                         256, bias_bits=synthetic.bits(c.bias), A_bits=synthetic.bits(c.A),
                         B_bits=synthetic.bits(c.B), lora_scale=c.lora_scale)


def test_noalloc_matches_workspace_entry_point_twice():
    _build.build()
    oracle.build()
    first = _prepared(M=300, N=264, K=512, rank=64, seed=31)
    second = _prepared(M=1024, N=520, K=1024, rank=32, seed=32)
    # two calls in a row on the shared scratch array, then the workspace calls
    got1 = _noalloc_via_cabi(first)
    got2 = _noalloc_via_cabi(second)
    want1 = _with_workspace(first)
    want2 = _with_workspace(second)
    torch.cuda.synchronize()
    assert sd.sdnq_device_status() == 0
    for p, got, want in ((first, got1, want1), (second, got2, want2)):
        g, w = _bits(got), _bits(want)
        assert np.array_equal(g, w), \
            f"no-alloc output differs from the workspace call in {np.count_nonzero(g != w)} places"
        # against the oracle: the LoRA bound of the parity tests (one bf16 ulp plus the fp32
        # accumulation bound of the adapter terms; outputs where the sum cancels may sit more
        # than one ulp away)
        ref = _oracle(p)
        u = torch.empty((p["M"], p["rank"]), dtype=torch.bfloat16, device="cuda")
        sd.sdnq_int8_linear_lora(p["qx"], p["sx"], p["qW"], p["sW"], p["bias"], p["x"], p["A"],
                                 p["B"], p["scale"], u_ws=u)
        torch.cuda.synchronize()
        check_lora_tolerance(p["case"], _bits(u), g, ref, p["scale"])


def test_noalloc_python_wrapper_after_a_larger_call():
    """The wrapper on a small problem right after a larger one left the shared array full of
    other rows: its rows of u are rewritten before they are read."""
    _build.build()
    big = _prepared(M=2048, N=256, K=512, rank=128, seed=33)
    small = _prepared(M=130, N=136, K=256, rank=16, seed=34)
    _noalloc_via_cabi(big)
    got = sd._native.sdnq_int8_linear_lora_noalloc(small["qx"], small["sx"], small["qW"],
                                                   small["sW"], small["bias"], small["x"],
                                                   small["A"], small["B"], small["scale"])
    want = _with_workspace(small)
    torch.cuda.synchronize()
    assert sd.sdnq_device_status() == 0
    assert np.array_equal(_bits(got), _bits(want))


def test_noalloc_rejects_problems_larger_than_its_scratch():
    _build.build()
    rank = 64
    M = _native.NOALLOC_MAX_U_ELEMS // rank + 1
    st = _native.lib().sdnq_int8_linear_lora_noalloc(
        P(0), P(0), P(0), P(0), P(0), P(0), 256, P(0), P(0), rank, 1.0, M, 256, 256, P(0),
        256, P(0), P(0))
    assert st == _native.SDNQ_ERR_SHAPE
    # a row count whose product with the rank overflows 64 bits is refused the same way
    st = _native.lib().sdnq_int8_linear_lora_noalloc(
        P(0), P(0), P(0), P(0), P(0), P(0), 256, P(0), P(0), rank, 1.0, 2 ** 62, 256, 256, P(0),
        256, P(0), P(0))
    assert st == _native.SDNQ_ERR_SHAPE
