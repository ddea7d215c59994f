"""Pins for the CPU oracle: each test checks the oracle against something other than
itself (closed forms, library routines, brute force, hand-derived worked examples), so
that a plausible slip in the oracle (a dropped term, a wrong sign or index, a transposed
operand, a wrong rounding rule) fails at least one test. No GPU is needed."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from hadamard_rotated_int8_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
GROUPS = [1, 2, 4, 8, 16, 32, 64, 128, 256]


def sylvester(g: int) -> np.ndarray:
    """Closed form H[i][j] = (-1)^popcount(i & j), as int64."""
    i = np.arange(g)[:, None]
    j = np.arange(g)[None, :]
    pc = np.vectorize(lambda v: bin(int(v)).count("1"))(i & j)
    return np.where(pc % 2 == 0, 1, -1).astype(np.int64)


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Library routine: torch's fp32 -> bf16 cast (round to nearest even)."""
    return synthetic.bits(torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16))


def bf16_value(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------- number formats

def test_f32_to_bf16_matches_torch_cast():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(200_000).astype(np.float32) * np.float32(1e3)
    # exact ties: low 16 bits 0x8000 with even and odd upper halves
    ties = (rng.integers(0, 2**31, 4096, dtype=np.uint32) & 0xffff0000) | 0x8000
    ties = ties.view(np.float32)
    ties = ties[np.isfinite(ties)]
    special = np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38, 3.3895e38, 1e-40, -1e-40,
                        np.inf, -np.inf], np.float32)
    for arr in (x, ties, special):
        assert np.array_equal(oracle.f32_to_bf16(arr), bf16_bits_from_f32(arr))


def _nearest_bf16_brute(d: float) -> int:
    """Brute force: try the candidate bf16 patterns around d and keep the nearest, ties to
    the even pattern."""
    f = np.float32(d)
    base = int(np.array([f], np.float32).view(np.uint32)[0] >> 16)
    cands = []
    for b in range(base - 2, base + 3):
        b &= 0xffff
        v = float(bf16_value(np.array([b]))[0])
        if math.isnan(v):
            continue
        cands.append((abs(v - d), b & 1, b, v))
    # the infinity is the right answer only past the overflow threshold
    cands.sort()
    return cands[0][2]


def test_f64_to_bf16_is_single_correct_rounding():
    rng = np.random.default_rng(1)
    vals = list(rng.standard_normal(3000) * 10.0 ** rng.integers(-40, 38, 3000))
    # double-rounding traps: just above a bf16 midpoint, within fp32 rounding distance
    for _ in range(500):
        b = int(rng.integers(0x0100, 0x7f00))
        lo = float(bf16_value(np.array([b]))[0])
        hi = float(bf16_value(np.array([b + 1]))[0])
        mid = (lo + hi) / 2
        vals += [mid, mid + (hi - lo) * 2.0 ** -20, mid - (hi - lo) * 2.0 ** -20]
    # bf16 subnormals (grid 2^-133)
    vals += list(rng.uniform(-2.0 ** -126, 2.0 ** -126, 500))
    vals += [0.0, -0.0, 2.0 ** -133, 2.0 ** -134, 3 * 2.0 ** -135]
    d = np.array(vals, np.float64)
    got = oracle.f64_to_bf16(d)
    for di, gi in zip(d, got):
        if di == 0.0:
            assert gi == (0x8000 if math.copysign(1, di) < 0 else 0)
            continue
        assert gi == _nearest_bf16_brute(float(di)), (di, hex(gi))


def test_f64_to_bf16_overflow_and_sign():
    big = np.array([3.4e38, -3.4e38, 1e300, -1e300, np.inf, -np.inf], np.float64)
    got = oracle.f64_to_bf16(big)
    assert list(got) == [0x7f80, 0xff80, 0x7f80, 0xff80, 0x7f80, 0xff80]


# ---------------------------------------------------------------- Walsh-Hadamard butterfly

@pytest.mark.parametrize("g", GROUPS)
def test_butterfly_matrix_is_sylvester_and_orthogonal(g):
    """Applying the oracle butterfly to the unit vectors reproduces the closed form
    H[i][j] = (-1)^popcount(i&j), and H H^T = g I."""
    eye = np.eye(g, dtype=np.float32)
    cols = oracle.fwht_f32(eye, g)  # row i = FWHT(e_i) = column i of H
    H = cols.T.astype(np.int64)
    assert np.array_equal(H, sylvester(g))
    assert np.array_equal(H @ H.T, g * np.eye(g, dtype=np.int64))


@pytest.mark.parametrize("g", GROUPS)
def test_butterfly_equals_dense_product_on_integers(g):
    """For integer inputs with |v| < 2^24/g every fp32 step is exact, so the butterfly must
    equal the dense integer product bit for bit (numpy int64 matmul)."""
    rng = np.random.default_rng(g)
    bound = (1 << 24) // g - 1
    rows, K = 7, 4 * g
    v = rng.integers(-bound, bound + 1, size=(rows, K))
    got = oracle.fwht_f32(v.astype(np.float32), g)
    H = sylvester(g)
    want = (v.reshape(rows, K // g, g) @ H.T).reshape(rows, K)
    assert np.array_equal(got.astype(np.int64), want)


@pytest.mark.parametrize("g", [8, 64, 256])
def test_butterfly_is_an_involution_up_to_g(g):
    rng = np.random.default_rng(100 + g)
    v = rng.integers(-1000, 1001, size=(3, 2 * g)).astype(np.float32)
    twice = oracle.fwht_f32(oracle.fwht_f32(v, g), g)
    assert np.array_equal(twice, g * v)


@pytest.mark.parametrize("g", [64, 128, 256])
def test_butterfly_fp32_error_within_textbook_bound(g):
    """Real-valued input: fp32 butterfly vs the exact (fp64 dense) product, within the
    standard bound log2(g) * u * sum|v| per output (u = 2^-24) + a small slack."""
    rng = np.random.default_rng(7 + g)
    v = rng.standard_normal((16, g)).astype(np.float32)
    got = oracle.fwht_f32(v, g).astype(np.float64)
    exact = v.astype(np.float64) @ sylvester(g).T.astype(np.float64)
    bound = (math.log2(g) * 2.0 ** -24 * 1.01) * np.abs(v).astype(np.float64).sum(1,
                                                                                 keepdims=True)
    assert np.all(np.abs(got - exact) <= bound)


@pytest.mark.parametrize("g", [64, 128, 256])
def test_rotation_cancels_in_the_product(g):
    """(x H)(W H)^T = g * x W^T: in exact integer arithmetic through the oracle's own
    fp32 butterfly, and in fp64 to ~1e-12 through its fp64 butterfly (normalised)."""
    rng = np.random.default_rng(11 + g)
    K = 2 * g
    x = rng.integers(-50, 51, size=(5, K))
    W = rng.integers(-50, 51, size=(6, K))
    zx = oracle.fwht_f32(x.astype(np.float32), g).astype(np.int64)
    zw = oracle.fwht_f32(W.astype(np.float32), g).astype(np.int64)
    assert np.array_equal(zx @ zw.T, g * (x @ W.T))
    xf = rng.standard_normal((5, K))
    Wf = rng.standard_normal((6, K))
    rx = oracle.fwht_f64(xf, g) / math.sqrt(g)
    rw = oracle.fwht_f64(Wf, g) / math.sqrt(g)
    ref = xf @ Wf.T
    assert np.max(np.abs(rx @ rw.T - ref)) <= 1e-12 * np.max(np.abs(ref)) * K


# ---------------------------------------------------------------- rotate + quantize

def _ties_even_nearest(t: np.float32) -> int:
    """Brute force over the whole grid [-127, 127]: nearest point, ties to the even one."""
    best = None
    for q in range(-127, 128):
        d = abs(float(t) - q)
        key = (d, q & 1)
        if best is None or key < best[0]:
            best = (key, q)
    return best[1]


@pytest.mark.parametrize("K", [8, 16, 32])
def test_codes_brute_force_g8(K):
    """g = 8, K <= 32, integer inputs (so the rotation z is exact): every code is the
    nearest grid point to the IEEE fp32 quotient z / fp32(amax/127), ties to even, and the
    scale is fp32(amax/127) * fp32(1/sqrt(8))."""
    rng = np.random.default_rng(K)
    rows = 40
    x = rng.integers(-200, 201, size=(rows, K)).astype(np.float32)
    x[3] = 0.0                       # zero row
    x[4, :] = 0.0
    x[4, 0] = 5.0                    # single spike -> flat rotation
    xb = bf16_bits_from_f32(x)
    assert np.array_equal(bf16_value(xb), x)  # integers < 256 are exact in bf16
    q, s = oracle.rotate_quantize(xb, 8)
    H = sylvester(8)
    z = (x.astype(np.int64).reshape(rows, K // 8, 8) @ H.T).reshape(rows, K)
    c8 = np.float32(1.0 / math.sqrt(8.0))
    for r in range(rows):
        amax = np.float32(np.abs(z[r]).max())
        sz = np.float32(amax / np.float32(127.0))
        if amax == 0:
            assert np.all(q[r] == 0) and s[r] == 0
            continue
        assert s[r] == np.float32(sz * c8)
        for k in range(K):
            t = np.float32(np.float32(z[r, k]) / sz)
            assert q[r, k] == _ties_even_nearest(t), (r, k, t)


def test_g1_is_textbook_per_row_absmax_int8():
    """g = 1 (no rotation) must be plain per-row absmax INT8: s = amax/127,
    q = round_half_even(x / s)."""
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((64, 96)) * 3).astype(np.float32)
    xb = bf16_bits_from_f32(x)
    xv = bf16_value(xb)
    q, s = oracle.rotate_quantize(xb, 1)
    amax = np.abs(xv).max(1)
    s_ref = (amax / np.float32(127)).astype(np.float32)
    q_ref = np.clip(np.round(xv / s_ref[:, None]), -127, 127).astype(np.int8)
    assert np.array_equal(s, s_ref)
    assert np.array_equal(q, q_ref)


@pytest.mark.parametrize("g", [8, 16, 32, 64, 128, 256])
def test_quantization_invariants(g):
    case = synthetic.make_case(M=33, N=8, K=1024, g=g, seed=g, outlier_count=10,
                               outlier_factor=25.0)
    xb = synthetic.bits(case.x)
    q, s = oracle.rotate_quantize(xb, g)
    z = oracle.fwht_f32(bf16_value(xb), g)
    c = np.float32(1.0 / math.sqrt(g))
    assert q.min() >= -127 and q.max() <= 127
    for r in range(q.shape[0]):
        amax = np.abs(z[r]).max()
        sz = np.float32(amax / np.float32(127))
        # the element(s) attaining the row absmax land on the top of the grid
        top = np.abs(z[r]) == amax
        assert np.all(np.abs(q[r][top]) == 127)
        # half-step bound (plus the fp32 rounding of the quotient)
        err = np.abs(z[r].astype(np.float64) - q[r].astype(np.float64) * float(sz))
        assert np.all(err <= float(sz) * (0.5 + 2.0 ** -16))
        assert s[r] == np.float32(sz * c)


@pytest.mark.parametrize("g", [64, 256])
def test_power_of_four_groups_equal_quantizing_the_normalised_rotation(g):
    """For g = 4^k the normaliser 1/sqrt(g) is a power of two, so folding it into the scale
    is the same as quantizing the normalised rotation z/sqrt(g) directly (the HSWQ page
    sizes its ConvRot groups in powers of 4)."""
    case = synthetic.make_case(M=20, N=8, K=2 * g, g=g, seed=3, outlier_count=3,
                               outlier_factor=30.0)
    xb = synthetic.bits(case.x)
    q, s = oracle.rotate_quantize(xb, g)
    zn32 = oracle.fwht_f32(bf16_value(xb), g) * np.float32(1 / math.sqrt(g))
    s_direct = (np.abs(zn32).max(1) / np.float32(127)).astype(np.float32)
    q_direct = np.clip(np.round(zn32 / s_direct[:, None]), -127, 127).astype(np.int8)
    assert np.array_equal(s, s_direct)
    assert np.array_equal(q, q_direct)


def test_golden_worked_rotquant():
    d = json.load(open(os.path.join(GOLDEN, "rotquant_g8_worked.json")))
    g = d["g"]
    for case in d["cases"]:
        x = np.array([case["x"]], np.float32)
        z = oracle.fwht_f32(x, g)
        assert np.array_equal(z[0], np.array(case["z"], np.float32))
        q, s = oracle.rotate_quantize(bf16_bits_from_f32(x), g)
        assert list(q[0]) == case["codes"]
        want_s = np.float32(np.float32(case["amax"]) / np.float32(127)) * np.float32(
            1 / math.sqrt(g))
        assert s[0] == np.float32(want_s)


def test_rows_are_independent_and_strided_input():
    case = synthetic.make_case(M=50, N=8, K=512, g=256, seed=9)
    xb = synthetic.bits(case.x)
    q_all, s_all = oracle.rotate_quantize(xb, 256)
    for r in (0, 17, 49):
        q1, s1 = oracle.rotate_quantize(xb[r:r + 1], 256, nthreads=1)
        assert np.array_equal(q1[0], q_all[r]) and s1[0] == s_all[r]


def test_reconstruction_quality_and_rotation_helps_outliers():
    """Quality report (not parity): dequantised rotated product vs fp64 x W^T. With outlier
    channels the Hadamard rotation lowers the max-token error against no rotation."""
    case = synthetic.make_case(M=64, N=96, K=1024, g=256, seed=21, outlier_frac=0.01,
                               outlier_factor=30.0)
    xb, wb = synthetic.bits(case.x), synthetic.bits(case.W)
    ref = bf16_value(xb).astype(np.float64) @ bf16_value(wb).astype(np.float64).T
    errs = {}
    for g in (1, 256):
        qx, sx = oracle.rotate_quantize(xb, g)
        qw, sw = oracle.rotate_quantize(wb, g)
        acc = oracle.gemm_s8(qx, qw).astype(np.float64)
        y = acc * sx[:, None].astype(np.float64) * sw[None, :].astype(np.float64)
        tok_err = np.abs(y - ref).max(1) / np.abs(ref).max(1)
        errs[g] = tok_err.max()
    assert errs[256] < 0.05
    assert errs[256] < errs[1]


# ---------------------------------------------------------------- GEMM and epilogue

@pytest.mark.parametrize("shape", [(1, 1, 16), (17, 33, 48), (64, 40, 1024)])
def test_gemm_matches_numpy_int64(shape):
    M, N, K = shape
    rng = np.random.default_rng(M * N)
    a = rng.integers(-127, 128, size=(M, K), dtype=np.int8)
    b = rng.integers(-127, 128, size=(N, K), dtype=np.int8)
    acc = oracle.gemm_s8(a, b)
    assert np.array_equal(acc.astype(np.int64), a.astype(np.int64) @ b.astype(np.int64).T)


def test_gemm_extreme_accumulator():
    K = 131072
    a = np.full((1, K), -127, np.int8)
    b = np.full((2, K), -127, np.int8)
    b[1] = 127
    acc = oracle.gemm_s8(a, b)
    assert acc[0, 0] == 127 * 127 * K and acc[0, 1] == -127 * 127 * K


def test_golden_worked_epilogue():
    d = json.load(open(os.path.join(GOLDEN, "linear_int8_worked.json")))
    qx = np.array(d["qx"], np.int8)
    qw = np.array(d["qw"], np.int8)
    acc = oracle.gemm_s8(qx, qw)
    assert acc.tolist() == d["acc"]
    out = oracle.dequant_epilogue(acc, np.array(d["sx"], np.float32),
                                  np.array(d["sw"], np.float32),
                                  bf16_bits_from_f32(np.array(d["bias"], np.float32)))
    assert bf16_value(out).tolist() == d["out"]


def test_epilogue_rounds_twice_not_fused():
    """The pages ask for the de-quant steps in fp32; the reading is one IEEE rounding per
    operation (no fused multiply-add). On inputs where that is visible after the bf16
    rounding, the oracle's outputs are those of the two roundings and not of the fma."""
    from tests.epilogue_ties import fma_sensitive_epilogue_inputs
    a1, a2, sx, sw, bias = fma_sensitive_epilogue_inputs(count=64)
    acc = (a1 * a2).astype(np.int32).reshape(8, 8)
    sx2 = np.ascontiguousarray(sx.reshape(8, 8))
    sw2 = np.ascontiguousarray(sw.reshape(8, 8))
    b2 = np.ascontiguousarray(bias.reshape(8, 8))
    for r in range(8):  # one output row per call: element (r, n) pairs sx2[r, n] with sw2[r, n]
        for n in range(8):
            out = oracle.dequant_epilogue(acc[r:r + 1, n:n + 1], sx2[r, n:n + 1], sw2[r, n:n + 1],
                                          b2[r, n:n + 1])
            t = np.float32(sx2[r, n]) * np.float32(sw2[r, n])
            v = np.float32(acc[r, n]) * t
            two = v + bf16_value(b2[r, n:n + 1])[0]
            fused = np.float32(np.float64(acc[r, n]) * np.float64(t) +
                               np.float64(bf16_value(b2[r, n:n + 1])[0]))
            assert bf16_bits_from_f32(np.array([two], np.float32))[0] != \
                bf16_bits_from_f32(np.array([fused], np.float32))[0]
            assert out[0, 0] == bf16_bits_from_f32(np.array([two], np.float32))[0]


def test_epilogue_within_one_ulp_of_fp64_and_op_order():
    """Against an fp64 recompute from the same codes and scales: every output within one
    bf16 ulp; the fp32 op order (s_x*s_w first, no fused multiply-add) is checked by a
    float32 numpy recompute that must match bit for bit."""
    rng = np.random.default_rng(3)
    # large enough that an fp32 op-order change shows up after the bf16 rounding
    M, N, K = 1024, 2048, 512
    acc = rng.integers(-2_000_000, 2_000_001, size=(M, N)).astype(np.int32)
    sx = (rng.random(M) * 0.05).astype(np.float32)
    sw = (rng.random(N) * 1e-4).astype(np.float32)
    bias = bf16_bits_from_f32(rng.standard_normal(N).astype(np.float32) * 0.01)
    L = (rng.standard_normal((M, N)) * 0.1).astype(np.float32)
    for use_bias, use_L in ((False, False), (True, False), (True, True)):
        out = oracle.dequant_epilogue(acc, sx, sw, bias if use_bias else None,
                                      L if use_L else None, 0.75)
        exact = acc.astype(np.float64) * sx[:, None].astype(np.float64) * sw[None, :]
        if use_bias:
            exact = exact + bf16_value(bias)[None, :].astype(np.float64)
        if use_L:
            exact = exact + 0.75 * L.astype(np.float64)
        got = bf16_value(out).astype(np.float64)
        # one bf16 ulp of the result, plus the fp32 rounding of the terms (which only
        # matters where bias and product nearly cancel)
        terms = np.abs(acc.astype(np.float64) * sx[:, None] * sw[None, :])
        if use_bias:
            terms = terms + np.abs(bf16_value(bias))[None, :]
        if use_L:
            terms = terms + 0.75 * np.abs(L)
        bound = np.abs(exact) * 2.0 ** -7 + terms * 2.0 ** -21
        assert np.all(np.abs(got - exact) <= bound)
        v = acc.astype(np.float32) * (sx[:, None] * sw[None, :])
        if use_bias:
            v = v + bf16_value(bias)[None, :]
        if use_L:
            v = v + np.float32(0.75) * L
        assert np.array_equal(out, bf16_bits_from_f32(v))


def test_zero_row_gives_bias_only():
    M, N, K = 3, 16, 256
    x = np.zeros((M, K), np.float32)
    x[1] = np.linspace(-1, 1, K, dtype=np.float32)
    rng = np.random.default_rng(0)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    bias = bf16_bits_from_f32(rng.standard_normal(N).astype(np.float32) * 0.01)
    qw, sw = oracle.rotate_quantize(bf16_bits_from_f32(W), 256)
    res = oracle.linear(bf16_bits_from_f32(x), qw, sw, 256, bias_bits=bias)
    assert res["sx"][0] == 0 and res["sx"][2] == 0
    assert np.array_equal(res["out"][0], bias) and np.array_equal(res["out"][2], bias)


# ---------------------------------------------------------------- LoRA and GELU

def test_lora_down_and_up_against_fp64_products():
    case = synthetic.make_case(M=37, N=70, K=320, g=64, seed=4, lora_rank=16,
                               outlier_count=3, outlier_factor=30.0)
    xb, Ab, Bb = (synthetic.bits(t) for t in (case.x, case.A, case.B))
    u = oracle.lora_down(xb, Ab)
    exact_u = bf16_value(xb).astype(np.float64) @ bf16_value(Ab).astype(np.float64)
    got_u = bf16_value(u).astype(np.float64)
    assert np.all(np.abs(got_u - exact_u) <= np.abs(exact_u) * 2.0 ** -8 + 1e-30)
    # u is the single rounding of the fp64 sum: equal to torch's rounding of it except at
    # double-rounding traps, which are rare
    via_torch = bf16_bits_from_f32(exact_u.astype(np.float32))
    assert (u == via_torch).mean() > 0.999
    L = oracle.lora_up(u, Bb)
    exact_L = got_u @ bf16_value(Bb).astype(np.float64)
    assert np.all(np.abs(L.astype(np.float64) - exact_L) <=
                  np.abs(exact_L) * 2.0 ** -23 + 1e-30)


def test_gelu_against_scipy_normal_cdf_and_special_values():
    """GELU(x) = x * Phi(x), with Phi from scipy's normal CDF (accurate in relative terms
    in the lower tail, where 1 + erf cancels)."""
    from scipy.special import ndtr
    rng = np.random.default_rng(8)
    x = np.concatenate([rng.standard_normal(20000) * 3, np.linspace(-12, 12, 2001),
                        [0.0, -0.0, 1e-30, -1e-30, 50.0, -50.0, 3e38, -3e38]])
    xb = bf16_bits_from_f32(x.astype(np.float32))
    xv = bf16_value(xb).astype(np.float64)
    got = bf16_value(oracle.gelu_bf16(xb)).astype(np.float64)
    ref = xv * ndtr(xv)
    ok = np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-37
    assert ok.all()
    g = oracle.gelu_bf16(bf16_bits_from_f32(np.array([0.0, 50.0, -50.0, 2.0], np.float32)))
    assert g[0] == 0 and bf16_value(g[1:2])[0] == 50.0
    assert g[2] == 0x8000  # -50 * Phi(-50) underflows to -0
    assert bf16_value(g[3:4])[0] == np.float32(1.953125)  # 2*Phi(2)=1.9545 -> bf16 1.953125


# ---------------------------------------------------------------- input gradient (backward)

def _exact_grad_case(g, M=6, N=48, groups=2, seed=0):
    """Inputs on which every step of the input-gradient path is exact: codes Q with +-127 in
    every row, power-of-two row scales S and column scales sw, dy = Q S / sw (exact in bf16:
    |Q| < 128 has at most 7 significant bits), weight codes in [-7, 7] so that the butterfly
    of the accumulators stays below 2^24."""
    rng = np.random.default_rng(seed)
    K = g * groups
    Q = rng.integers(-127, 128, size=(M, N))
    Q[np.arange(M), rng.integers(0, N, M)] = 127 * rng.choice([-1, 1], M)
    e_row = rng.integers(3, 9, M)                       # S = 2^-e_row
    e_col = rng.integers(2, 7, N)                       # sw = 2^-e_col
    sw = np.ldexp(1.0, -e_col).astype(np.float32)
    dy = np.ldexp(Q.astype(np.float64), (e_col[None, :] - e_row[:, None]))
    dyb = bf16_bits_from_f32(dy.astype(np.float32))
    assert np.array_equal(bf16_value(dyb).astype(np.float64), dy)
    qw = rng.integers(-7, 8, size=(N, K)).astype(np.int8)
    return Q, e_row, sw, dyb, qw


@pytest.mark.parametrize("g", [8, 64, 128, 256])
def test_grad_input_exact_case_against_explicit_hadamard(g):
    """dx = ((dy * sw) qw) H_g / sqrt(g) with the explicit Sylvester matrix, in exact integer
    arithmetic, rounded once to bf16; the oracle's codes and scales are the constructed ones."""
    Q, e_row, sw, dyb, qw = _exact_grad_case(g, seed=g)
    res = oracle.grad_input(dyb, qw, sw, g)
    assert np.array_equal(res["qg"], Q.astype(np.int8))
    assert np.array_equal(res["sg"], np.ldexp(1.0, -e_row).astype(np.float32))
    M, K = Q.shape[0], qw.shape[1]
    acc = Q.astype(np.int64) @ qw.astype(np.int64)
    H = sylvester(g)
    rot = (acc.reshape(M, K // g, g) @ H).reshape(M, K)       # H symmetric
    assert np.abs(rot).max() < 2 ** 24
    if g in (64, 256):
        exact = np.ldexp(rot.astype(np.float64), -e_row[:, None]) / math.sqrt(g)
        assert np.array_equal(res["dx"], oracle.f64_to_bf16(exact))
    else:
        # 1/sqrt(g) is not a power of two: the oracle rounds z * fp32(1/sqrt(g)) in fp32
        c_g = np.float32(1.0 / math.sqrt(g))
        z = np.ldexp(rot.astype(np.float64), -e_row[:, None]).astype(np.float32)
        assert np.array_equal(res["dx"], bf16_bits_from_f32(z * c_g))


def test_colscale_quantize_with_unit_scales_is_textbook_per_row_int8():
    """sw = 1 reduces the backward quantizer to plain per-row absmax int8 (the g = 1 case of
    the forward quantizer, itself pinned against the textbook formula)."""
    rng = np.random.default_rng(11)
    dyb = bf16_bits_from_f32((rng.standard_normal((37, 200)) * 0.01).astype(np.float32))
    q, s = oracle.colscale_quantize(dyb, np.ones(200, np.float32))
    q1, s1 = oracle.rotate_quantize(dyb, 1)
    assert np.array_equal(q, q1) and np.array_equal(s, s1)


def test_colscale_quantize_brute_force_codes():
    """Every code is the nearest grid point to fp32(fp32(dy * sw) / fp32(amax / 127)), ties to
    even, over rows that include a zero row."""
    rng = np.random.default_rng(12)
    dy = (rng.standard_normal((12, 24)) * 0.3).astype(np.float32)
    dy[5] = 0.0
    dyb = bf16_bits_from_f32(dy)
    sw = (rng.random(24) * 0.01 + 1e-4).astype(np.float32)
    q, s = oracle.colscale_quantize(dyb, sw)
    c = (bf16_value(dyb) * sw[None, :]).astype(np.float32)
    for r in range(12):
        amax = np.float32(np.abs(c[r]).max())
        if amax == 0:
            assert s[r] == 0 and np.all(q[r] == 0)
            continue
        sz = np.float32(amax / np.float32(127.0))
        assert s[r] == sz
        for n in range(24):
            assert q[r, n] == _ties_even_nearest(np.float32(c[r, n] / sz))


def test_gemm_nn_matches_numpy_int64():
    rng = np.random.default_rng(13)
    a = rng.integers(-127, 128, size=(9, 70), dtype=np.int8)
    b = rng.integers(-127, 128, size=(70, 33), dtype=np.int8)
    assert np.array_equal(oracle.gemm_s8_nn(a, b).astype(np.int64),
                          a.astype(np.int64) @ b.astype(np.int64))


@pytest.mark.parametrize("g", [64, 256])
def test_grad_input_is_the_chain_rule_of_the_dequantized_layer(g):
    """Against fp64 dy W_hat, with W_hat = diag(sw) qw H_g / sqrt(g) the weight the layer
    holds: the error is bounded by the int8 quantization of dy * sw (half a step per
    element, carried through |qw H|/sqrt(g)), plus one bf16 ulp and fp32 rounding."""
    rng = np.random.default_rng(g)
    M, N, K = 16, 96, 2 * g
    case = synthetic.make_case(M=N, N=1, K=K, g=g, seed=g)
    qw, sw = oracle.rotate_quantize(synthetic.bits(case.x), g)   # a weight's codes
    dyb = bf16_bits_from_f32((rng.standard_normal((M, N)) * 0.05).astype(np.float32))
    res = oracle.grad_input(dyb, qw, sw, g)
    H = sylvester(g).astype(np.float64) / math.sqrt(g)
    Hb = np.kron(np.eye(K // g), H)
    w_hat = (sw.astype(np.float64)[:, None] * qw.astype(np.float64)) @ Hb
    ref = bf16_value(dyb).astype(np.float64) @ w_hat
    got = bf16_value(res["dx"]).astype(np.float64)
    qstep = res["sg"].astype(np.float64)[:, None] / 2.0
    spread = np.abs(qw.astype(np.float64) @ Hb).sum(0)[None, :]
    bound = qstep * spread + np.abs(ref) * 2.0 ** -7 + 2.0 ** -20 * np.abs(got) * g + 1e-30
    assert np.all(np.abs(got - ref) <= bound)


def test_grad_input_zero_gradient_row():
    rng = np.random.default_rng(14)
    dy = (rng.standard_normal((4, 32)) * 0.1).astype(np.float32)
    dy[2] = 0.0
    qw = rng.integers(-127, 128, size=(32, 256), dtype=np.int8)
    res = oracle.grad_input(bf16_bits_from_f32(dy), qw, np.full(32, 0.01, np.float32), 256)
    assert res["sg"][2] == 0 and np.all(res["qg"][2] == 0)
    assert np.all(bf16_value(res["dx"][2]) == 0)


# ---------------------------------------------------------------- FP8 (e4m3) variant

def _torch_e4m3(x):
    """Library routine: torch's fp32 -> float8_e4m3fn cast (round to nearest even)."""
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_encode_matches_torch_cast_in_range():
    rng = np.random.default_rng(21)
    x = np.concatenate([rng.standard_normal(100_000) * 30, rng.standard_normal(20_000) * 0.01,
                        (rng.random(20_000) - 0.5) * 927.0]).astype(np.float32)
    x = x[np.abs(x) < 464.0]                     # torch gives NaN beyond; we saturate
    # exact ties: midpoints between neighbouring codes
    codes = np.arange(0, 126, dtype=np.uint8)
    lo, hi = oracle.e4m3_decode(codes[:-1]), oracle.e4m3_decode(codes[1:])
    mids = ((lo.astype(np.float64) + hi) / 2).astype(np.float32)
    for arr in (x, mids, -mids):
        assert np.array_equal(oracle.e4m3_encode(arr), _torch_e4m3(arr))


def test_e4m3_decode_matches_torch_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_decode(codes)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    finite = ~np.isnan(want)
    assert np.array_equal(np.isnan(got), ~finite)
    assert np.array_equal(got[finite], want[finite])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9


def test_e4m3_encode_brute_force_nearest_ties_even_and_saturation():
    rng = np.random.default_rng(22)
    table = oracle.e4m3_decode(np.arange(256, dtype=np.uint8)).astype(np.float64)
    finite = np.array([c for c in range(256) if not np.isnan(table[c])])
    x = np.concatenate([rng.standard_normal(3000) * 20, rng.standard_normal(1000) * 0.005,
                        [448.0, 460.0, 463.9, 500.0, 1e30, -1e30, 0.0]]).astype(np.float32)
    got = oracle.e4m3_encode(x)
    for v, c in zip(x.astype(np.float64), got):
        if abs(v) >= 448.0:
            assert table[c] == np.sign(v) * 448.0
            continue
        d = np.abs(table[finite] - v)
        best = finite[d == d.min()]
        if len(best) > 1:  # a tie (or +-0): the even code, sign of v
            best = [b for b in best if b % 2 == 0 and (np.signbit(table[b]) == np.signbit(v)
                                                        or table[b] != 0)]
        assert table[c] == table[best[0]], (v, c, best)


def test_fp8_gemm_matches_numpy_fp64():
    rng = np.random.default_rng(23)
    a = rng.integers(0, 256, size=(17, 96), dtype=np.uint8)
    b = rng.integers(0, 256, size=(9, 96), dtype=np.uint8)
    a[(a & 0x7F) == 0x7F] = 0   # no NaN codes
    b[(b & 0x7F) == 0x7F] = 0
    got = oracle.gemm_fp8(a, b)
    da = oracle.e4m3_decode(a).astype(np.float64)
    db = oracle.e4m3_decode(b).astype(np.float64)
    assert np.array_equal(got, (da @ db.T).astype(np.float32))


def test_fp8_epilogue_equals_int8_epilogue_on_integral_accumulators():
    rng = np.random.default_rng(24)
    acc = rng.integers(-2_000_000, 2_000_001, size=(64, 80)).astype(np.int32)
    sx = (rng.random(64) * 0.05).astype(np.float32)
    sw = (rng.random(80) * 1e-4).astype(np.float32)
    bias = bf16_bits_from_f32(rng.standard_normal(80).astype(np.float32) * 0.01)
    assert np.array_equal(oracle.dequant_epilogue_f32(acc.astype(np.float32), sx, sw, bias),
                          oracle.dequant_epilogue(acc, sx, sw, bias))


@pytest.mark.parametrize("g", [8, 64, 256])
def test_rotate_quantize_fp8_brute_force(g):
    """Integer inputs (exact rotation): codes are e4m3 of the IEEE fp32 quotient
    z / fp32(amax / 448), the scale is fp32(amax/448) * fp32(1/sqrt g), amax maps to +-448,
    and a zero row gives s = 0 and +0 codes."""
    rng = np.random.default_rng(g + 5)
    rows, K = 12, 2 * g
    x = rng.integers(-200, 201, size=(rows, K)).astype(np.float32)
    x[3] = 0.0
    xb = bf16_bits_from_f32(x)
    q, s = oracle.rotate_quantize_fp8(xb, g)
    H = sylvester(g)
    z = (x.astype(np.int64).reshape(rows, K // g, g) @ H.T).reshape(rows, K)
    cg = np.float32(1.0 / math.sqrt(g))
    for r in range(rows):
        amax = np.float32(np.abs(z[r]).max())
        if amax == 0:
            assert s[r] == 0 and np.all(q[r] == 0)
            continue
        sz = np.float32(amax / np.float32(448.0))
        assert s[r] == np.float32(sz * cg)
        t = (z[r].astype(np.float32) / sz).astype(np.float32)
        assert np.array_equal(q[r], _torch_e4m3(np.clip(t, -448, 448)))
        assert np.abs(oracle.e4m3_decode(q[r])).max() == 448.0


def test_fp8_rotated_linear_tracks_the_exact_product():
    """Quality (not parity): the FP8 rotated linear stays close to the fp64 product, and the
    rotation helps on outlier inputs as it does for int8."""
    case = synthetic.make_case(M=64, N=96, K=1024, g=256, seed=25, outlier_count=10,
                               outlier_factor=40.0)
    xv = bf16_value(synthetic.bits(case.x)).astype(np.float64)
    wv = bf16_value(synthetic.bits(case.W)).astype(np.float64)
    ref = xv @ wv.T
    errs = {}
    for g in (1, 256):
        qw, sw = oracle.rotate_quantize_fp8(synthetic.bits(case.W), g)
        res = oracle.linear_fp8(synthetic.bits(case.x), qw, sw, g)
        errs[g] = np.abs(bf16_value(res["out"]) - ref).max()
    assert errs[256] < 0.08 * np.abs(ref).max()
    assert errs[256] < errs[1]


# ---------------------------------------------------------------- int8 QK attention

def _attn_inputs(B, Lq, Lk, H, D, seed, scale_q=1.0):
    gen = torch.Generator().manual_seed(seed)
    q = (torch.randn(B, Lq, H, D, generator=gen) * scale_q).to(torch.bfloat16)
    k = torch.randn(B, Lk, H, D, generator=gen).to(torch.bfloat16)
    v = torch.randn(B, Lk, H, D, generator=gen).to(torch.bfloat16)
    return q, k, v


def test_attn_prep_without_smoothing_is_the_linear_quantizer():
    """With smooth_k off, Q and K codes and scales are those of the (pinned) row quantizer of
    the linear path applied to the token-head rows, with the group capped at D."""
    q, k, _ = _attn_inputs(2, 40, 56, 3, 64, seed=1)
    res = oracle.attn_prep(synthetic.bits(q), synthetic.bits(k), 256, smooth_k=False)
    qc, qs = oracle.rotate_quantize(synthetic.bits(q).reshape(-1, 64), 64)
    kc, ks = oracle.rotate_quantize(synthetic.bits(k).reshape(-1, 64), 64)
    assert np.array_equal(res["qq"].reshape(-1, 64), qc)
    assert np.array_equal(res["kq"].reshape(-1, 64), kc)
    assert np.array_equal(res["sq"], qs.reshape(2, 40, 3).transpose(0, 2, 1))
    assert np.array_equal(res["sk"], ks.reshape(2, 56, 3).transpose(0, 2, 1))
    assert np.all(res["mu"] == 0)


def test_attn_smooth_k_subtracts_the_exact_channel_mean():
    """Integer K built so that every channel mean is an integer: mu is that mean, and the K
    codes are the row quantizer's codes of the integer rows K - mu."""
    rng = np.random.default_rng(2)
    B, Lk, H, D = 1, 64, 2, 128
    k = rng.integers(-60, 61, size=(B, Lk, H, D)).astype(np.float64)
    shift = rng.integers(-20, 21, size=(B, 1, H, D))
    k = k - k.mean(axis=1, keepdims=True).round() + shift   # means are exactly `shift` +- 0
    k[:, -1] += (Lk * shift[:, 0] - k.sum(axis=1))          # force sum == Lk * shift
    kb = bf16_bits_from_f32(k.astype(np.float32))
    assert np.array_equal(bf16_value(kb), k.astype(np.float32))
    q = np.zeros((B, 8, H, D), np.float32)
    res = oracle.attn_prep(bf16_bits_from_f32(q), kb, 128, smooth_k=True)
    assert np.array_equal(res["mu"], shift[:, 0].astype(np.float32))
    centred = (k - shift).astype(np.float32)
    kc, ks = oracle.rotate_quantize(bf16_bits_from_f32(centred).reshape(-1, D), 128)
    assert np.array_equal(res["kq"].reshape(-1, D), kc)


def test_attn_logits_are_dequantized_products():
    q, k, _ = _attn_inputs(1, 33, 70, 2, 128, seed=3)
    res = oracle.attention(synthetic.bits(q), synthetic.bits(k), synthetic.bits(k), 256)
    acc = np.einsum("bihd,bjhd->bhij", res["qq"].astype(np.int64), res["kq"].astype(np.int64))
    scale = np.float32(1.0 / np.sqrt(128.0))
    ref = (acc * res["sq"][..., None].astype(np.float64) * res["sk"][:, :, None, :] * scale)
    assert np.all(np.abs(res["logits"] - ref) <= 3 * 2.0 ** -24 * np.abs(ref) + 1e-30)


def test_attn_softmax_pv_matches_torch_fp64():
    """softmax(logits) V against torch's fp64 softmax and matmul: within one bf16 rounding."""
    rng = np.random.default_rng(4)
    B, H, Lq, Lk, D = 2, 3, 17, 45, 64
    logits = (rng.standard_normal((B, H, Lq, Lk)) * 3).astype(np.float32)
    v = torch.randn(B, Lk, H, D, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    got = bf16_value(oracle.attn_softmax_pv(logits, synthetic.bits(v))).astype(np.float64)
    p = torch.softmax(torch.from_numpy(logits).double(), dim=-1)
    ref = torch.einsum("bhij,bjhd->bihd", p, v.double()).numpy()
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-300)


@pytest.mark.parametrize("smooth", [False, True])
def test_attn_tracks_sdpa(smooth):
    """Quality: the int8-QK attention stays close to fp64 SDPA, with or without smoothing."""
    q, k, v = _attn_inputs(1, 64, 128, 2, 128, seed=6)
    res = oracle.attention(synthetic.bits(q), synthetic.bits(k), synthetic.bits(v), 256,
                           smooth_k=smooth)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double().transpose(1, 2), k.double().transpose(1, 2), v.double().transpose(1, 2)
    ).transpose(1, 2).numpy()
    got = bf16_value(res["o"]).astype(np.float64)
    assert np.abs(got - ref).max() < 0.03
