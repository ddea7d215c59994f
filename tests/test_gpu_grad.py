"""GPU parity of the input gradient through the frozen rotated int8 base
(sdnq_int8_linear_grad_input) against the oracle's three steps: bit-exact int8 codes of
dy * sW, fp32 scales, int32 accumulators and bf16 dx, on ragged shapes (M, the contraction N
and the output width K not multiples of the tiles), every group size, strided dy, zero rows,
and the split calls against the composed one (the full-size attention and PEFT layers are
compared on every element in tests/test_gpu_fullsize.py). Every input is seeded; every
expected value comes from the oracle."""
import numpy as np
import pytest
import torch

import oracle
import hadamard_rotated_int8_b200 as sd
from hadamard_rotated_int8_b200 import _build, synthetic
from tests.test_gpu_parity import assert_equal, bits_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    _build.build()
    oracle.build()
    torch.cuda.init()
    yield
    assert sd.sdnq_device_status() == 0


def grad_case(M, N, K, g, seed, outlier_cols=0, ld_pad=0):
    """dy [M, N] (optionally inside a wider buffer), the layer's weight W [N, K]."""
    c = synthetic.make_grad_case(M, N, K, g, seed=seed, outlier_count=outlier_cols,
                                 outlier_factor=40.0, ld_pad=ld_pad)
    return c.x, c.W


def run_gpu(dy_full, W, g, N):
    dyg = dy_full.cuda()[:, :N]
    qW, sW = sd.sdnq_rotate_quant_weight(W.cuda(), g)
    M, K = dyg.shape[0], W.shape[1]
    acc = torch.empty((M, K), dtype=torch.int32, device="cuda")
    qg = torch.empty((M, N), dtype=torch.int8, device="cuda")
    sg = torch.empty((M,), dtype=torch.float32, device="cuda")
    dx = sd.sdnq_int8_linear_grad_input(dyg, qW, sW, g, qg_ws=qg, sg_ws=sg, acc_out=acc)
    torch.cuda.synchronize()
    return {"qg": qg.cpu().numpy(), "sg": sg.cpu().numpy(), "acc": acc.cpu().numpy(),
            "dx": bits_of(dx)}


def oracle_ref(dy_full, W, g, N, rows=None):
    dyb = synthetic.bits(dy_full[:, :N].contiguous())
    if rows is not None:
        dyb = dyb[rows]
    qW, sW = oracle.rotate_quantize(synthetic.bits(W), g)
    return oracle.grad_input(dyb, qW, sW, g)


CASES = [
    (128, 256, 256, 256), (300, 512, 768, 256), (257, 96, 512, 64), (130, 160, 384, 128),
    (64, 48, 256, 8), (200, 1040, 1024, 32), (1, 16, 16, 16), (129, 272, 2304, 256),
    (77, 3072, 512, 128),
]


@pytest.mark.parametrize("M,N,K,g", CASES)
def test_grad_input_bit_exact(M, N, K, g):
    dy, W = grad_case(M, N, K, g, seed=M + N + K + g, outlier_cols=max(1, N // 100))
    got = run_gpu(dy, W, g, N)
    ref = oracle_ref(dy, W, g, N)
    assert_equal(got["qg"], ref["qg"], "codes of dy * sW")
    assert_equal(got["sg"].view(np.uint32), ref["sg"].view(np.uint32), "scales of dy * sW")
    assert_equal(got["acc"], ref["acc"], "int32 accumulators")
    assert_equal(got["dx"], ref["dx"], "bf16 dx")


def test_grad_input_strided_dy_and_zero_rows():
    M, N, K, g = 150, 512, 512, 256
    dy, W = grad_case(M, N, K, g, seed=9, ld_pad=24)
    dy[3] = 0.0
    dy[149] = 0.0
    got = run_gpu(dy, W, g, N)
    ref = oracle_ref(dy, W, g, N)
    assert got["sg"][3] == 0 and got["sg"][149] == 0
    assert_equal(got["qg"], ref["qg"], "codes")
    assert_equal(got["dx"], ref["dx"], "bf16 dx")


def test_grad_input_empty_batch_is_a_noop():
    W = torch.zeros(64, 256, dtype=torch.bfloat16, device="cuda")
    qW, sW = sd.sdnq_rotate_quant_weight(W, 256)
    dx = sd.sdnq_int8_linear_grad_input(torch.zeros(0, 64, dtype=torch.bfloat16, device="cuda"),
                                        qW, sW, 256)
    assert dx.shape == (0, 256)


def test_split_calls_equal_the_composed_call():
    M, N, K, g = 200, 512, 768, 128
    dy, W = grad_case(M, N, K, g, seed=21, outlier_cols=5)
    dyg = dy.cuda()
    qW, sW = sd.sdnq_rotate_quant_weight(W.cuda(), g)
    qg, sg = sd.sdnq_quant_grad_output(dyg, sW)
    dx_split = sd.sdnq_int8_grad_input_gemm(qg, sg, qW, g)
    qg2 = torch.empty_like(qg)
    sg2 = torch.empty_like(sg)
    dx = sd.sdnq_int8_linear_grad_input(dyg, qW, sW, g, qg_ws=qg2, sg_ws=sg2)
    torch.cuda.synchronize()
    assert_equal(qg.cpu().numpy(), qg2.cpu().numpy(), "codes")
    assert_equal(bits_of(dx_split), bits_of(dx), "dx")
