"""GPU parity of the one-launch online path (sdnq_int8_linear_fused: the activation rotate +
quantize runs on warps inside the int8 GEMM kernel) against the oracle: bit-exact activation
codes, scales, int32 accumulators and bf16 outputs on ragged shapes, every group size, with
and without bias, rows longer than the fused limit (two launches), repeated calls on one
counter buffer. The full-size workloads are compared on every element in
tests/test_gpu_fullsize.py. Every input is seeded; every expected value comes from the
oracle."""
import numpy as np
import pytest
import torch

import oracle
import hadamard_rotated_int8_b200 as sd
from hadamard_rotated_int8_b200 import _build, _native, synthetic
from tests.test_gpu_parity import assert_equal, bits_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    _build.build()
    oracle.build()
    torch.cuda.init()
    yield
    assert sd.sdnq_device_status() == 0


def run_fused(case, sync=None):
    xg = case.x.cuda()
    qW, sW = sd.sdnq_rotate_quant_weight(case.W.cuda(), case.g)
    bias = case.bias.cuda() if case.bias is not None else None
    M, K = case.M, case.K
    qx = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sx = torch.empty((M,), dtype=torch.float32, device="cuda")
    acc = torch.empty((M, case.N), dtype=torch.int32, device="cuda")
    out = sd.sdnq_int8_linear_fused(xg, case.g, qW, sW, bias, qx_ws=qx, sx_ws=sx, sync_ws=sync,
                                    acc_out=acc, policy=_native.FUSE_ALWAYS)
    torch.cuda.synchronize()
    return {"qx": qx.cpu().numpy(), "sx": sx.cpu().numpy(), "acc": acc.cpu().numpy(),
            "out": bits_of(out)}


def oracle_ref(case, rows=None):
    xb = synthetic.bits(case.x)
    if rows is not None:
        xb = xb[rows]
    qW, sW = oracle.rotate_quantize(synthetic.bits(case.W), case.g)
    bias = synthetic.bits(case.bias) if case.bias is not None else None
    return oracle.linear(xb, qW, sW, case.g, bias_bits=bias)


CASES = [
    (128, 256, 256, 256), (300, 520, 768, 256), (257, 8, 256, 64), (130, 300, 1040, 16),
    (129, 257, 4096, 128), (64, 1000, 512, 8), (512, 768, 3072, 256), (1, 1, 256, 256),
    (700, 384, 8192, 256), (200, 136, 9216, 128), (64, 128, 13312, 64),
]


@pytest.mark.parametrize("M,N,K,g", CASES)
@pytest.mark.parametrize("bias", [False, True])
def test_fused_bit_exact(M, N, K, g, bias):
    case = synthetic.make_case(M=M, N=N, K=K, g=g, seed=M * 3 + N + K, outlier_count=K // 64,
                               outlier_factor=30.0, bias_std=0.01 if bias else None)
    got = run_fused(case)
    ref = oracle_ref(case)
    assert_equal(got["qx"], ref["qx"], "activation codes")
    assert_equal(got["sx"].view(np.uint32), ref["sx"].view(np.uint32), "activation scales")
    assert_equal(got["acc"], ref["acc"], "int32 accumulators")
    assert_equal(got["out"], ref["out"], "bf16 outputs")


def test_auto_policy_matches_both_paths():
    """The automatic choice (two launches for this 2.6-wave shape, one launch for the larger
    one) gives the same bits as forcing either path."""
    for M, N, K in ((4096, 3072, 3072), (8192, 6144, 3072)):
        case = synthetic.make_case(M=M, N=N, K=K, g=256, seed=M + N, outlier_count=31,
                                   outlier_factor=30.0, bias_std=0.01)
        xg = case.x.cuda()
        qW, sW = sd.sdnq_rotate_quant_weight(case.W.cuda(), 256)
        bias = case.bias.cuda()
        outs = [sd.sdnq_int8_linear_fused(xg, 256, qW, sW, bias, policy=pol)
                for pol in (_native.FUSE_AUTO, _native.FUSE_ALWAYS, _native.FUSE_NEVER)]
        torch.cuda.synchronize()
        assert_equal(bits_of(outs[0]), bits_of(outs[1]), "auto vs one launch")
        assert_equal(bits_of(outs[0]), bits_of(outs[2]), "auto vs two launches")


def test_counter_buffer_is_left_zero_and_reused():
    case = synthetic.make_case(M=1000, N=512, K=3072, g=256, seed=77, outlier_count=30,
                               outlier_factor=30.0, bias_std=0.01)
    sync = torch.zeros(_native.fused_sync_words(case.M), dtype=torch.int32, device="cuda")
    first = run_fused(case, sync)
    assert int(sync.abs().sum()) == 0
    second = run_fused(case, sync)
    assert int(sync.abs().sum()) == 0
    assert_equal(first["out"], second["out"], "repeat")
    ref = oracle_ref(case)
    assert_equal(second["out"], ref["out"], "bf16 outputs")


def test_fused_equals_two_launches_on_zero_and_huge_rows():
    case = synthetic.make_case(M=333, N=264, K=2048, g=256, seed=5, bias_std=0.01)
    x = case.x.clone()
    x[7] = 0.0
    x[100] = (torch.randn(2048, generator=torch.Generator().manual_seed(1)) * 1e30).to(torch.bfloat16)
    case.x = x
    got = run_fused(case)
    xg = x.cuda()
    qW, sW = sd.sdnq_rotate_quant_weight(case.W.cuda(), 256)
    qx, sx = sd.sdnq_rotquant_act(xg, 256)
    two = sd.sdnq_int8_linear(qx, sx, qW, sW, case.bias.cuda())
    torch.cuda.synchronize()
    assert got["sx"][7] == 0
    assert_equal(got["qx"], qx.cpu().numpy(), "codes against the two-launch path")
    assert_equal(got["out"], bits_of(two), "outputs against the two-launch path")
