"""GPU parity of the FP8 (e4m3) variant against the oracle: e4m3 codes and fp32 scales
bit-exact (both sides take the same fp32 quotient and round it once to e4m3); accumulators
within the fp32 summation bound (the tensor cores sum in their own order: |acc - exact| <=
(K - 1) 2^-24 sum_k |products|); bf16 outputs within one ulp plus that bound carried through
the scales. Every input is seeded; every expected value and every bound comes from the oracle
and the arithmetic."""
import numpy as np
import pytest
import torch

import oracle
import hadamard_rotated_int8_b200 as sd
from hadamard_rotated_int8_b200 import _build, synthetic
from tests.test_gpu_parity import assert_equal, bf16_val, bits_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    _build.build()
    oracle.build()
    torch.cuda.init()
    yield
    assert sd.sdnq_device_status() == 0


def run_fp8(case):
    xg = case.x.cuda()
    qW, sW = sd.sdnq_rotquant_fp8(case.W.cuda(), case.g)
    qx, sx = sd.sdnq_rotquant_fp8(xg, case.g)
    bias = case.bias.cuda() if case.bias is not None else None
    acc = torch.empty((case.M, case.N), dtype=torch.float32, device="cuda")
    out = sd.sdnq_fp8_linear(qx, sx, qW, sW, bias, acc_out=acc)
    torch.cuda.synchronize()
    return {"qx": qx.cpu().numpy(), "sx": sx.cpu().numpy(), "qW": qW.cpu().numpy(),
            "sW": sW.cpu().numpy(), "acc": acc.cpu().numpy(), "out": bits_of(out)}


def check_against_oracle(case, got, rows=None):
    xb = synthetic.bits(case.x)
    if rows is not None:
        xb = xb[rows]
    qw_r, sw_r = oracle.rotate_quantize_fp8(synthetic.bits(case.W), case.g)
    bias = synthetic.bits(case.bias) if case.bias is not None else None
    ref = oracle.linear_fp8(xb, qw_r, sw_r, case.g, bias_bits=bias)
    sel = slice(None) if rows is None else rows
    assert_equal(got["qW"], qw_r, "weight e4m3 codes")
    assert_equal(got["sW"].view(np.uint32), sw_r.view(np.uint32), "weight scales")
    assert_equal(got["qx"][sel], ref["qx"], "activation e4m3 codes")
    assert_equal(got["sx"][sel].view(np.uint32), ref["sx"].view(np.uint32), "activation scales")
    # accumulators: fp32 summation bound
    ax = np.abs(oracle.e4m3_decode(ref["qx"]).astype(np.float64))
    aw = np.abs(oracle.e4m3_decode(qw_r).astype(np.float64))
    mag = ax @ aw.T
    K = case.K
    acc_bound = (K - 1) * 2.0 ** -24 * mag + np.abs(ref["acc"]).astype(np.float64) * 2.0 ** -24
    acc_err = np.abs(got["acc"][sel].astype(np.float64) - ref["acc"].astype(np.float64))
    assert np.all(acc_err <= acc_bound), float((acc_err / np.maximum(acc_bound, 1e-30)).max())
    # outputs: one bf16 ulp of the reference plus the accumulator bound through the scales
    t = ref["sx"].astype(np.float64)[:, None] * sw_r.astype(np.float64)[None, :]
    ref_v = bf16_val(ref["out"]).astype(np.float64)
    got_v = bf16_val(got["out"][sel]).astype(np.float64)
    bound = np.abs(ref_v) * 2.0 ** -7 + 2 * acc_bound * t + 1e-30
    assert np.all(np.abs(got_v - ref_v) <= bound)
    return acc_err, acc_bound


CASES = [(128, 256, 256, 256), (300, 520, 768, 256), (257, 136, 1024, 64), (130, 300, 1040, 16),
         (64, 1000, 4096, 128), (1, 8, 256, 8), (512, 768, 3072, 256)]


@pytest.mark.parametrize("M,N,K,g", CASES)
@pytest.mark.parametrize("bias", [False, True])
def test_fp8_parity(M, N, K, g, bias):
    case = synthetic.make_case(M=M, N=N, K=K, g=g, seed=M + 5 * N + K, outlier_count=K // 64,
                               outlier_factor=30.0, bias_std=0.01 if bias else None)
    check_against_oracle(case, run_fp8(case))


def test_fp8_zero_and_extreme_rows():
    case = synthetic.make_case(M=200, N=136, K=512, g=256, seed=7, bias_std=0.01)
    x = case.x.float()
    x[4] = 0.0
    x[9] *= 1e30
    x[11] *= 1e-30
    case.x = x.to(torch.bfloat16)
    got = run_fp8(case)
    assert got["sx"][4] == 0 and np.all(got["qx"][4] == 0)
    check_against_oracle(case, got)
