"""Launch ordering. The int8 GEMM, the attention kernel and the attention preparation are
launched programmatically: each may start while the kernel before it in the stream drains,
and waits (griddepcontrol.wait) before it reads that kernel's results. These tests run
several calls back to back on one stream, with no synchronisation between them, reusing the
same code, scale and workspace buffers on different inputs, and require every result to be
bit for bit that of the same call run alone after a synchronisation. A kernel that read a
buffer before the previous call finished writing it would see the previous input's codes.
Every input is seeded."""
import pytest
import torch

import hadamard_rotated_int8_b200 as sd
from hadamard_rotated_int8_b200 import _build, _native, synthetic
from tests.test_gpu_parity import assert_equal, bits_of

pytestmark = pytest.mark.gpu

ROUNDS = 4


@pytest.fixture(scope="module", autouse=True)
def built():
    _build.build()
    torch.cuda.init()
    yield
    assert sd.sdnq_device_status() == 0


def inputs(M, K, seed):
    return [synthetic.make_case(M=M, N=8, K=K, g=256, seed=seed + i, outlier_count=8,
                                outlier_factor=20.0).x.cuda() for i in range(ROUNDS)]


def layer(N, K, seed, bias=True):
    case = synthetic.make_case(M=8, N=N, K=K, g=256, seed=seed, bias_std=0.01 if bias else None)
    qW, sW = sd.sdnq_rotate_quant_weight(case.W.cuda(), 256)
    return qW, sW, case.bias.cuda() if bias else None


@pytest.mark.parametrize("M,N,K", [(4096, 3072, 3072), (700, 520, 1024)])
def test_linear_back_to_back(M, N, K):
    xs = inputs(M, K, 100)
    qW, sW, bias = layer(N, K, 7)
    alone = []
    for x in xs:
        qx, sx = sd.sdnq_rotquant_act(x, 256)
        alone.append(sd.sdnq_int8_linear(qx, sx, qW, sW, bias))
        torch.cuda.synchronize()
    qx = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sx = torch.empty((M,), dtype=torch.float32, device="cuda")
    outs = [torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for _ in xs]
    for x, out in zip(xs, outs):   # one stream, no synchronisation, qx / sx reused
        sd.sdnq_rotquant_act(x, 256, qx, sx)
        sd.sdnq_int8_linear(qx, sx, qW, sW, bias, out=out)
    torch.cuda.synchronize()
    for i, (a, b) in enumerate(zip(alone, outs)):
        assert_equal(bits_of(b), bits_of(a), f"round {i}")


def test_gelu_lora_fp8_grad_back_to_back():
    M, N, K, rank = 640, 768, 1024, 32
    xs = inputs(M, K, 200)
    qW, sW, bias = layer(N, K, 8)
    gen = torch.Generator().manual_seed(9)
    A = (0.02 * torch.randn(K, rank, generator=gen)).to(torch.bfloat16).cuda()
    B = (0.02 * torch.randn(rank, N, generator=gen)).to(torch.bfloat16).cuda()
    dys = [(0.01 * torch.randn(M, N, generator=gen)).to(torch.bfloat16).cuda() for _ in xs]
    W8 = synthetic.make_case(M=8, N=N, K=K, g=256, seed=8).W.cuda()
    qW8, sW8 = sd.sdnq_rotquant_fp8(W8, 256)

    def round_(x, dy, bufs):
        qx, sx, u, q8, s8, qg, sg = bufs
        sd.sdnq_rotquant_act(x, 256, qx, sx)
        r = [sd.sdnq_int8_linear_gelu(qx, sx, qW, sW, bias),
             sd.sdnq_int8_linear_lora(qx, sx, qW, sW, bias, x, A, B, 0.5, u_ws=u)]
        sd.sdnq_rotquant_fp8(x, 256, q8, s8)
        r.append(sd.sdnq_fp8_linear(q8, s8, qW8, sW8, bias))
        r.append(sd.sdnq_int8_linear_grad_input(dy, qW, sW, 256, qg_ws=qg, sg_ws=sg))
        return r

    def bufs():
        return (torch.empty((M, K), dtype=torch.int8, device="cuda"),
                torch.empty((M,), dtype=torch.float32, device="cuda"),
                torch.empty((M, rank), dtype=torch.bfloat16, device="cuda"),
                torch.empty((M, K), dtype=torch.uint8, device="cuda"),
                torch.empty((M,), dtype=torch.float32, device="cuda"),
                torch.empty((M, N), dtype=torch.int8, device="cuda"),
                torch.empty((M,), dtype=torch.float32, device="cuda"))

    alone = []
    for x, dy in zip(xs, dys):
        alone.append(round_(x, dy, bufs()))
        torch.cuda.synchronize()
    shared = bufs()
    together = [round_(x, dy, shared) for x, dy in zip(xs, dys)]
    torch.cuda.synchronize()
    names = ["gelu", "lora", "fp8", "grad_input"]
    for i, (a, b) in enumerate(zip(alone, together)):
        for n, ra, rb in zip(names, a, b):
            assert_equal(bits_of(rb), bits_of(ra), f"round {i} {n}")


@pytest.mark.parametrize("policy", [_native.FUSE_ALWAYS, _native.FUSE_NEVER])
def test_fused_linear_back_to_back(policy):
    M, N, K = 2048, 1024, 2048
    xs = inputs(M, K, 300)
    qW, sW, bias = layer(N, K, 10)
    alone = []
    for x in xs:
        alone.append(sd.sdnq_int8_linear_fused(x, 256, qW, sW, bias, policy=policy))
        torch.cuda.synchronize()
    qx = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sx = torch.empty((M,), dtype=torch.float32, device="cuda")
    # the row counters of the one-launch path: the binding's per-stream buffer, reused
    outs = [sd.sdnq_int8_linear_fused(x, 256, qW, sW, bias, qx_ws=qx, sx_ws=sx, policy=policy)
            for x in xs]
    torch.cuda.synchronize()
    for i, (a, b) in enumerate(zip(alone, outs)):
        assert_equal(bits_of(b), bits_of(a), f"round {i}")


def test_attention_back_to_back():
    B, L, H, D = 1, 700, 4, 128
    gen = torch.Generator().manual_seed(400)
    qkv = [[torch.randn(B, L, H, D, generator=gen).to(torch.bfloat16).cuda() for _ in range(3)]
           for _ in range(ROUNDS)]
    alone = []
    for q, k, v in qkv:
        alone.append(sd.sdnq_attention_int8qk(q, k, v, 256))
        torch.cuda.synchronize()
    total, _ = _native.attention_workspace(B, L, L, H, D)
    ws = torch.empty(total, dtype=torch.uint8, device="cuda")   # one workspace for all rounds
    outs = [sd.sdnq_attention_int8qk(q, k, v, 256, ws=ws) for q, k, v in qkv]
    torch.cuda.synchronize()
    for i, (a, b) in enumerate(zip(alone, outs)):
        assert_equal(bits_of(b), bits_of(a), f"round {i}")


def test_weights_quantized_right_before_the_gemm():
    """The weight quantizer triggers its dependents at entry; the GEMM launched right after it
    must still read the finished codes and scales (a new weight every round, same buffers)."""
    M, N, K = 1024, 1536, 2048
    x = inputs(M, K, 500)[0]
    Ws = [synthetic.make_case(M=8, N=N, K=K, g=256, seed=600 + i).W.cuda() for i in range(ROUNDS)]
    qx, sx = sd.sdnq_rotquant_act(x, 256)
    torch.cuda.synchronize()
    alone = []
    for W in Ws:
        qW, sW = sd.sdnq_rotate_quant_weight(W, 256)
        torch.cuda.synchronize()
        alone.append(sd.sdnq_int8_linear(qx, sx, qW, sW))
        torch.cuda.synchronize()
    qW = torch.empty((N, K), dtype=torch.int8, device="cuda")
    sW = torch.empty((N,), dtype=torch.float32, device="cuda")
    outs = []
    for W in Ws:   # quantize the weight, then the GEMM at once, no synchronisation
        sd.sdnq_rotate_quant_weight(W, 256, qW, sW)
        outs.append(sd.sdnq_int8_linear(qx, sx, qW, sW))
    torch.cuda.synchronize()
    for i, (a, b) in enumerate(zip(alone, outs)):
        assert_equal(bits_of(b), bits_of(a), f"round {i}")
