"""GPU parity: the CUDA library against the CPU oracle, element by element, on the same
seeded bf16 inputs. Bit-exact on int8 codes, fp32 scales and int32 accumulators; bit-exact
on bf16 outputs without LoRA (same fp32 op order). With LoRA the adapter accumulates in
fp32 on the tensor cores while the oracle sums in fp64, so the bound is one bf16 ulp plus
the fp32 accumulation bound of the adapter terms (it matters only where terms cancel), and
at least 99.9% of outputs must be within one ulp. Every input comes from the seeded
generator; every expected value from the oracle."""
import numpy as np
import pytest
import torch

import oracle
import hadamard_rotated_int8_b200 as sd
from hadamard_rotated_int8_b200 import _build, synthetic
from tests.epilogue_ties import fma_sensitive_epilogue_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    _build.build()
    oracle.build()
    torch.cuda.init()
    yield
    assert sd.sdnq_device_status() == 0


def bits_of(t: torch.Tensor) -> np.ndarray:
    return synthetic.bits(t.detach().cpu().contiguous())


def bf16_val(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint32) << 16).view(np.float32)


def ulp_diff(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """Distance in bf16 ulps (monotone integer mapping of the bit patterns)."""
    def key(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, 0x8000 - (b & 0x7fff), 0x8000 + b)
    return np.abs(key(a_bits) - key(b_bits))


def assert_equal(got, want, what):
    got = np.asarray(got)
    want = np.asarray(want)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    bad = got != want
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} differ; first at {idx.tolist()}: "
                             f"got {[got[tuple(i)] for i in idx]} want {[want[tuple(i)] for i in idx]}")


def gpu_rotquant(x_cpu: torch.Tensor, g: int, weight=False):
    x = x_cpu.cuda()
    fn = sd.sdnq_rotate_quant_weight if weight else sd.sdnq_rotquant_act
    q, s = fn(x, g)
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().numpy()


# ------------------------------------------------------------------ rotate + quantize

ROTQUANT_CASES = [
    (1, 256, 256), (37, 768, 256), (300, 3072, 256), (5, 16, 8), (64, 1040, 16),
    (33, 4096, 64), (33, 4096, 128), (19, 3840, 256), (7, 10240, 256), (9, 2048, 32),
    (3, 20480, 256), (2, 131072, 256), (1000, 256, 64),
]


@pytest.mark.parametrize("M,K,g", ROTQUANT_CASES)
def test_rotquant_bit_exact(M, K, g):
    case = synthetic.make_case(M=M, N=8, K=K, g=g, seed=M + K + g, outlier_count=min(K // 100, 40),
                               outlier_factor=30.0)
    x = case.x.clone()
    if M > 4:
        x[1] = 0                      # all-zero row
        x[2, : min(K, 64)] = 1e-38    # tiny row: scale in the subnormal range
        x[2, min(K, 64):] = 0
        x[3] = x[3] * 1e30            # huge row, no overflow in the rotation
    q, s = gpu_rotquant(x, g)
    q_ref, s_ref = oracle.rotate_quantize(synthetic.bits(x), g)
    assert_equal(q, q_ref, f"codes M={M} K={K} g={g}")
    assert_equal(s.view(np.uint32), s_ref.view(np.uint32), f"scales M={M} K={K} g={g}")


@pytest.mark.parametrize("M,K,g,offset,pad", [
    (77, 3072, 256, 8, 0),      # rows 16 but not 32 bytes aligned: the 16-byte load path
    (50, 4096, 128, 0, 8),      # row stride K + 8: every other row off the 32-byte grid
    (33, 1040, 16, 8, 24),      # a partial last run (1040 = 16 runs + 16 elements)
    (129, 10240, 256, 0, 16),   # 40 groups per row, stride padded by 32 bytes
    (3, 32768, 256, 0, 0),      # the longest row of the run-per-lane kernel (512 runs)
    (2, 32768 + 256, 256, 0, 0),  # one group more: the two-pass kernel
])
def test_rotquant_offsets_and_strides(M, K, g, offset, pad):
    """Rows that start off the 32-byte grid (a view into a larger buffer), padded row
    strides, a partial last run and the row lengths where the kernel choice changes:
    codes and scales bit-exact."""
    case = synthetic.make_case(M=M, N=8, K=K, g=g, seed=K + pad + offset, outlier_count=K // 200,
                               outlier_factor=30.0)
    buf = torch.zeros((M, offset + K + pad), dtype=torch.bfloat16, device="cuda")
    buf[:, offset:offset + K] = case.x.cuda()
    x = buf[:, offset:offset + K]
    q, s = sd.sdnq_rotquant_act(x, g)
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.rotate_quantize(synthetic.bits(case.x), g)
    assert_equal(q.cpu().numpy(), q_ref, "codes")
    assert_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32), "scales")


@pytest.mark.parametrize("g", [8, 64, 256])
def test_rotquant_exact_ties_round_half_even(g):
    """Integer rows whose rotated absmax is 127 * 2^k make s_z a power of two, so many
    quotients z / s_z are exact half-integers: the codes must round those ties to even."""
    rng = np.random.default_rng(g)
    M, K = 96, 4 * max(g, 256)
    x = rng.integers(-1, 2, size=(M, K)).astype(np.float32)
    for r in range(M):
        k = r % 3                       # amax = 127 * 2^(k+1) in the first group
        target = 127 * 2 ** (k + 1)
        x[r, :g] = 0
        base, rem = divmod(target, g)
        x[r, :g] = base
        x[r, :rem] += 1
        # a few opposite pairs keep the group sum (z_0 = target) and vary the other z
        idx = rng.choice(g, size=min(8, g) // 2 * 2, replace=False)
        x[r, idx[0::2]] += 1
        x[r, idx[1::2]] -= 1
    xb = torch.from_numpy(x).to(torch.bfloat16)
    assert torch.equal(xb.float(), torch.from_numpy(x))  # small integers are exact in bf16
    q, s = gpu_rotquant(xb, g)
    q_ref, s_ref = oracle.rotate_quantize(synthetic.bits(xb), g)
    z = oracle.fwht_f32(x, g)
    sz = (np.abs(z).max(1) / np.float32(127)).astype(np.float32)
    t = z / sz[:, None]
    ties = np.count_nonzero(t - np.floor(t) == 0.5)
    assert ties > 100, ties
    assert_equal(q, q_ref, f"codes with exact ties g={g}")
    assert_equal(s.view(np.uint32), s_ref.view(np.uint32), f"scales with exact ties g={g}")


def test_rotquant_strided_input_and_weights_entry():
    case = synthetic.make_case(M=70, N=96, K=1536, g=256, seed=5, outlier_count=12,
                               outlier_factor=20.0)
    wide = torch.zeros(70, 1536 + 64, dtype=torch.bfloat16)
    wide[:, :1536] = case.x
    xg = wide.cuda()[:, :1536]
    assert xg.stride(0) == 1600
    q, s = sd.sdnq_rotquant_act(xg, 256)
    q_ref, s_ref = oracle.rotate_quantize(synthetic.bits(case.x), 256)
    assert_equal(q.cpu().numpy(), q_ref, "strided codes")
    assert_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32), "strided scales")
    qw, sw = gpu_rotquant(case.W, 256, weight=True)
    qw_ref, sw_ref = oracle.rotate_quantize(synthetic.bits(case.W), 256)
    assert_equal(qw, qw_ref, "weight codes")
    assert_equal(sw.view(np.uint32), sw_ref.view(np.uint32), "weight scales")


def test_rotquant_empty_batch_is_a_noop():
    x = torch.zeros(0, 256, dtype=torch.bfloat16, device="cuda")
    q, s = sd.sdnq_rotquant_act(x, 256)
    assert q.shape == (0, 256) and s.shape == (0,)


# ------------------------------------------------------------------ int8 linear

def run_linear_case(case, with_acc=True, lora=False):
    xg = case.x.cuda()
    Wg = case.W.cuda()
    qW, sW = sd.sdnq_rotate_quant_weight(Wg, case.g)
    qx, sx = sd.sdnq_rotquant_act(xg, case.g)
    bias = case.bias.cuda() if case.bias is not None else None
    acc = torch.empty((case.M, case.N), dtype=torch.int32, device="cuda") if with_acc else None
    if lora:
        u = torch.empty((case.M, case.A.shape[1]), dtype=torch.bfloat16, device="cuda")
        out = sd.sdnq_int8_linear_lora(qx, sx, qW, sW, bias, xg, case.A.cuda(), case.B.cuda(),
                                       case.lora_scale, u_ws=u, acc_out=acc)
    else:
        u = None
        out = sd.sdnq_int8_linear(qx, sx, qW, sW, bias, acc_out=acc)
    torch.cuda.synchronize()
    res = {"qx": qx.cpu().numpy(), "sx": sx.cpu().numpy(), "qW": qW.cpu().numpy(),
           "sW": sW.cpu().numpy(), "out": bits_of(out)}
    if acc is not None:
        res["acc"] = acc.cpu().numpy()
    if u is not None:
        res["u"] = bits_of(u)
    return res


LINEAR_CASES = [
    (128, 256, 128, 128), (1, 1, 256, 256), (300, 520, 768, 256), (257, 8, 256, 64),
    (130, 300, 1040, 16), (129, 257, 4096, 128), (64, 1000, 512, 8), (512, 768, 3072, 256),
]


@pytest.mark.parametrize("M,N,K,g", LINEAR_CASES)
@pytest.mark.parametrize("bias", [False, True])
def test_linear_bit_exact_small(M, N, K, g, bias):
    case = synthetic.make_case(M=M, N=N, K=K, g=g, seed=M * 7 + N, outlier_count=K // 64,
                               outlier_factor=30.0, bias_std=0.01 if bias else None)
    got = run_linear_case(case)
    ref = oracle.linear(synthetic.bits(case.x),
                        *oracle.rotate_quantize(synthetic.bits(case.W), g), g,
                        bias_bits=synthetic.bits(case.bias) if bias else None)
    assert_equal(got["qx"], ref["qx"], "qx")
    assert_equal(got["sx"].view(np.uint32), ref["sx"].view(np.uint32), "sx")
    assert_equal(got["acc"], ref["acc"], "int32 accumulators")
    assert_equal(got["out"], ref["out"], "bf16 outputs")


def test_linear_empty_batch_is_a_noop():
    qx = torch.zeros(0, 256, dtype=torch.int8, device="cuda")
    sx = torch.zeros(0, dtype=torch.float32, device="cuda")
    qW = torch.zeros(64, 256, dtype=torch.int8, device="cuda")
    sW = torch.zeros(64, dtype=torch.float32, device="cuda")
    out = sd.sdnq_int8_linear(qx, sx, qW, sW)
    assert out.shape == (0, 64)


def test_linear_extreme_codes_max_accumulator():
    """Every code +-127 at K = 131072 (the largest accepted K): |acc| = 127^2 K < 2^31."""
    M, N, K = 3, 40, 131072
    qx = torch.full((M, K), -127, dtype=torch.int8, device="cuda")
    qx[1] = 127
    qx[2, ::2] = 127
    qW = torch.full((N, K), -127, dtype=torch.int8, device="cuda")
    qW[5] = 127
    sx = torch.ones(M, dtype=torch.float32, device="cuda")
    sW = torch.ones(N, dtype=torch.float32, device="cuda")
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    out = sd.sdnq_int8_linear(qx, sx, qW, sW, acc_out=acc)
    ref = oracle.gemm_s8(qx.cpu().numpy(), qW.cpu().numpy())
    assert_equal(acc.cpu().numpy(), ref, "extreme accumulators")
    ref_out = oracle.dequant_epilogue(ref, np.ones(M, np.float32), np.ones(N, np.float32))
    assert_equal(bits_of(out), ref_out, "extreme outputs")


# ------------------------------------------------------------------ LoRA

@pytest.mark.parametrize("M,N,K,rank", [(128, 128, 256, 64), (300, 264, 512, 16),
                                        (200, 520, 1024, 80), (129, 136, 768, 256)])
def test_lora_within_one_ulp(M, N, K, rank):
    case = synthetic.make_case(M=M, N=N, K=K, g=256, seed=rank + M, outlier_count=K // 100,
                               outlier_factor=30.0, bias_std=0.01, lora_rank=rank,
                               lora_scale=0.75)
    got = run_linear_case(case, lora=True)
    ref = oracle.linear(synthetic.bits(case.x), *oracle.rotate_quantize(synthetic.bits(case.W), 256),
                        256, bias_bits=synthetic.bits(case.bias), A_bits=synthetic.bits(case.A),
                        B_bits=synthetic.bits(case.B), lora_scale=0.75)
    assert_equal(got["acc"], ref["acc"], "int32 accumulators (LoRA kernel)")
    check_lora_tolerance(case, got["u"], got["out"], ref, 0.75)


@pytest.mark.parametrize("M,N,K,rank,g", [
    (200, 64, 64, 16, 64),      # one k-block: a down-projection stage half used
    (300, 64, 192, 32, 64),     # three k-blocks: a full stage, then a half one
    (9000, 64, 512, 64, 256),   # 71 row blocks of the down-projection
    (20000, 32, 256, 48, 256),  # 157 row blocks: more than one CTA per SM over the launch
])
def test_lora_few_k_blocks_and_many_row_blocks(M, N, K, rank, g):
    """The down-projection u = x A streams two 64-column k-blocks of x per pipeline stage,
    one 128-row block per CTA: an odd number of k-blocks and launches of more row blocks
    than SMs stay within the fp32 accumulation bound of the oracle's u and output, and
    repeating the call gives the same bits."""
    case = synthetic.make_case(M=M, N=N, K=K, g=g, seed=M + K + rank, outlier_count=K // 64,
                               outlier_factor=30.0, bias_std=None, lora_rank=rank,
                               lora_scale=0.5)
    got = run_linear_case(case, lora=True)
    again = run_linear_case(case, lora=True)
    assert_equal(again["u"], got["u"], "repeat: u")
    assert_equal(again["out"], got["out"], "repeat: outputs")
    ref = oracle.linear(synthetic.bits(case.x), *oracle.rotate_quantize(synthetic.bits(case.W), g),
                        g, A_bits=synthetic.bits(case.A), B_bits=synthetic.bits(case.B),
                        lora_scale=0.5)
    assert_equal(got["acc"], ref["acc"], "int32 accumulators (LoRA kernel)")
    check_lora_tolerance(case, got["u"], got["out"], ref, 0.5)


@pytest.mark.parametrize("M,N,K,rank", [(300, 264, 512, 16), (4608, 1024, 3072, 64)])
def test_lora_halves_equal_the_whole_call(M, N, K, rank):
    """sdnq_lora_down then sdnq_int8_linear_lora_up give the bits of sdnq_int8_linear_lora
    (u and outputs), and u is within the fp32 accumulation bound of the oracle's."""
    case = synthetic.make_case(M=M, N=N, K=K, g=256, seed=M + rank, outlier_count=K // 100,
                               outlier_factor=30.0, bias_std=0.01, lora_rank=rank,
                               lora_scale=0.75)
    xg, A, B = case.x.cuda(), case.A.cuda(), case.B.cuda()
    qW, sW = sd.sdnq_rotate_quant_weight(case.W.cuda(), 256)
    qx, sx = sd.sdnq_rotquant_act(xg, 256)
    bias = case.bias.cuda()
    u_whole = torch.empty((M, rank), dtype=torch.bfloat16, device="cuda")
    whole = sd.sdnq_int8_linear_lora(qx, sx, qW, sW, bias, xg, A, B, 0.75, u_ws=u_whole)
    u = sd.sdnq_lora_down(xg, A)
    halves = sd.sdnq_int8_linear_lora_up(qx, sx, qW, sW, bias, u, B, 0.75)
    torch.cuda.synchronize()
    assert_equal(bits_of(u), bits_of(u_whole), "u")
    assert_equal(bits_of(halves), bits_of(whole), "outputs")
    ref = oracle.linear(synthetic.bits(case.x), *oracle.rotate_quantize(synthetic.bits(case.W), 256),
                        256, bias_bits=synthetic.bits(case.bias), A_bits=synthetic.bits(case.A),
                        B_bits=synthetic.bits(case.B), lora_scale=0.75)
    check_lora_tolerance(case, bits_of(u), bits_of(halves), ref, 0.75)


def lora_tolerances(x_bits, A_bits, B_bits, u_ref_bits, out_ref_bits, scale, rows=None):
    """Tolerance derived from the arithmetic (the adapter path accumulates in fp32, the
    oracle in fp64): one bf16 ulp of the result plus the fp32 accumulation bound
    2K * 2^-24 * sum|x A| for u, carried through u B for the output."""
    xv = bf16_val(x_bits).astype(np.float64)
    Av = np.abs(bf16_val(A_bits).astype(np.float64))
    Bv = np.abs(bf16_val(B_bits).astype(np.float64))
    K, r = Av.shape
    u_ref = bf16_val(u_ref_bits).astype(np.float64)
    tol_u = np.abs(u_ref) * 2.0 ** -7 + 2 * K * 2.0 ** -24 * (np.abs(xv) @ Av) + 1e-30
    out_ref = bf16_val(out_ref_bits).astype(np.float64)
    tol_out = (np.abs(out_ref) * 2.0 ** -7
               + abs(scale) * ((2 * tol_u) @ Bv + 2 * r * 2.0 ** -24 * (np.abs(u_ref) @ Bv))
               + 1e-30)
    return tol_u, tol_out


def check_lora_tolerance(case, u_bits, out_bits, ref, scale):
    tol_u, tol_out = lora_tolerances(synthetic.bits(case.x), synthetic.bits(case.A),
                                     synthetic.bits(case.B), ref["u"], ref["out"], scale)
    du = np.abs(bf16_val(u_bits).astype(np.float64) - bf16_val(ref["u"]).astype(np.float64))
    assert np.all(du <= tol_u), f"u outside the fp32-accumulation bound: {np.count_nonzero(du > tol_u)}"
    dout = np.abs(bf16_val(out_bits).astype(np.float64) - bf16_val(ref["out"]).astype(np.float64))
    assert np.all(dout <= tol_out), f"out outside the bound: {np.count_nonzero(dout > tol_out)}"
    # and nearly everywhere within one ulp
    within = (ulp_diff(out_bits, ref["out"]) <= 1).mean()
    assert within > 0.999, within


# ------------------------------------------------------------------ GELU

def test_gelu_bit_exact():
    rng = np.random.default_rng(0)
    vals = np.concatenate([rng.standard_normal(300_000) * 3, np.linspace(-14, 14, 40_001),
                           [0.0, -0.0, 1e-30, -1e-30, 50, -50, 3e38, -3e38, 1e-40, -1e-40]])
    n = (len(vals) // 8) * 8
    x = torch.from_numpy(vals[:n].astype(np.float32)).to(torch.bfloat16).view(-1, 8)
    out = sd.sdnq_gelu_bf16(x.cuda())
    torch.cuda.synchronize()
    assert_equal(bits_of(out), oracle.gelu_bf16(synthetic.bits(x)), "gelu")


def _finite_bf16_patterns():
    b = np.arange(65536, dtype=np.uint32)
    return b[((b >> 7) & 0xFF) != 0xFF].astype(np.uint16)  # all but NaN and Inf


def test_gelu_exhaustive_over_finite_bf16():
    pats = _finite_bf16_patterns()
    x = torch.from_numpy(pats.view(np.int16)).view(torch.bfloat16).reshape(-1, 8).cuda()
    out = sd.sdnq_gelu_bf16(x)
    torch.cuda.synchronize()
    assert_equal(bits_of(out).reshape(-1), oracle.gelu_bf16(pats), "gelu, every finite bf16 input")


@pytest.mark.parametrize("M", [3, 130])
def test_linear_gelu_epilogue_exhaustive_over_finite_bf16(M):
    """Zero codes make the pre-GELU value exactly the bias, so a bias holding every finite
    bf16 pattern drives the epilogue's GELU (its table and its closed-form ranges) through
    all of them; 3 rows run the single-SM kernel, 130 the CTA-pair kernel."""
    pats = _finite_bf16_patterns()
    N, K = len(pats), 16
    qx = torch.zeros((M, K), dtype=torch.int8, device="cuda")
    qW = torch.zeros((N, K), dtype=torch.int8, device="cuda")
    sx = torch.ones(M, dtype=torch.float32, device="cuda")
    sW = torch.ones(N, dtype=torch.float32, device="cuda")
    bias = torch.from_numpy(pats.view(np.int16)).view(torch.bfloat16).cuda()
    out = sd.sdnq_int8_linear_gelu(qx, sx, qW, sW, bias)
    torch.cuda.synchronize()
    want = oracle.gelu_bf16(oracle.dequant_epilogue(np.zeros((M, N), np.int32), np.ones(M, np.float32),
                                                    np.ones(N, np.float32), bias_bits=pats))
    assert_equal(bits_of(out), want, "fused GELU, every finite bf16 pre-activation")


def test_gelu_ragged_and_strided():
    x = (torch.randn(37, 133 + 11, generator=torch.Generator().manual_seed(3)) * 4).to(torch.bfloat16)
    wide = x.cuda()
    src = wide[:, :133]  # row stride 144, 133 columns: ragged tail
    assert src.stride(0) == 144
    out = sd.sdnq_gelu_bf16(src)
    assert_equal(bits_of(out), oracle.gelu_bf16(synthetic.bits(x[:, :133].contiguous())), "gelu ragged")


@pytest.mark.parametrize("gelu", [False, True])
def test_epilogue_rounds_twice_on_fma_sensitive_ties(gelu):
    """The de-quant epilogue rounds (float(acc) * t) and (v + bias) separately, as the oracle
    does; an accidental multiply-add contraction shows up on these inputs (diagonal)."""
    a1, a2, sx, sw, bias = fma_sensitive_epilogue_inputs()
    H, K = len(a1), 16
    qx = np.zeros((H, K), np.int8)
    qW = np.zeros((H, K), np.int8)
    qx[:, 0] = a1
    qW[:, 0] = a2
    acc = oracle.gemm_s8(qx, qW)
    want = oracle.dequant_epilogue(acc, sx, sw, bias_bits=bias)
    if gelu:
        want = oracle.gelu_bf16(want)
    fn = sd.sdnq_int8_linear_gelu if gelu else sd.sdnq_int8_linear
    out = fn(torch.from_numpy(qx).cuda(), torch.from_numpy(sx).cuda(), torch.from_numpy(qW).cuda(),
             torch.from_numpy(sw).cuda(), torch.from_numpy(bias.view(np.int16)).cuda().view(torch.bfloat16))
    torch.cuda.synchronize()
    got = bits_of(out)
    assert_equal(np.diagonal(got), np.diagonal(want), "tie-sensitive diagonal")
    assert_equal(got, want, "all outputs")


@pytest.mark.parametrize("M,N,K,g,w_std", [(128, 256, 256, 256, 0.02), (300, 520, 768, 256, 0.2),
                                            (257, 136, 1024, 128, 1.0), (513, 1000, 3840, 256, 0.015)])
def test_linear_gelu_epilogue_bit_exact(M, N, K, g, w_std):
    """GELU fused into the GEMM epilogue equals the oracle's linear followed by its GELU, and
    the library's own two-pass chain, bit for bit. The larger weight scales push outputs past
    |y| = 10 and near bf16 rounding boundaries, where the fp64 path decides."""
    case = synthetic.make_case(M=M, N=N, K=K, g=g, seed=M + N + K, dist="student_t",
                               w_std=w_std, bias_std=0.05)
    xg = case.x.cuda()
    qW, sW = sd.sdnq_rotate_quant_weight(case.W.cuda(), g)
    qx, sx = sd.sdnq_rotquant_act(xg, g)
    bias = case.bias.cuda()
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    fused = sd.sdnq_int8_linear_gelu(qx, sx, qW, sW, bias, acc_out=acc)
    two_pass = sd.sdnq_gelu_bf16(sd.sdnq_int8_linear(qx, sx, qW, sW, bias))
    torch.cuda.synchronize()
    ref = oracle.linear(synthetic.bits(case.x), *oracle.rotate_quantize(synthetic.bits(case.W), g),
                        g, bias_bits=synthetic.bits(case.bias))
    assert_equal(acc.cpu().numpy(), ref["acc"], "int32 accumulators (GELU kernel)")
    assert_equal(bits_of(fused), oracle.gelu_bf16(ref["out"]), "fused GELU outputs")
    assert_equal(bits_of(fused), bits_of(two_pass), "fused against two-pass GELU")


# ------------------------------------------------------------------ failure detection

def test_bounded_wait_reports_timeout_and_context_survives():
    assert sd.sdnq_device_status() == 0
    sd.sdnq_selftest_wait_timeout(2_000_000)  # 2 ms limit on a wait nothing can satisfy
    assert sd.sdnq_device_status() == sd._native.SDNQ_ERR_TIMEOUT
    assert sd.sdnq_device_status() == 0       # cleared
    x = torch.ones(2, 256, dtype=torch.bfloat16, device="cuda")
    q, s = sd.sdnq_rotquant_act(x, 256)       # the context is still usable
    assert int(q[0, 0]) == 127


def test_calls_follow_the_current_stream():
    case = synthetic.make_case(M=256, N=256, K=512, g=256, seed=11)
    side = torch.cuda.Stream()
    x = case.x.cuda()
    torch.cuda.synchronize()
    with torch.cuda.stream(side):
        q, s = sd.sdnq_rotquant_act(x, 256)
    side.synchronize()
    q_ref, _ = oracle.rotate_quantize(synthetic.bits(case.x), 256)
    assert_equal(q.cpu().numpy(), q_ref, "side-stream codes")
