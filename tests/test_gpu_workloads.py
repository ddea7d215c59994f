"""GPU parity at the full DiT workload sizes, in the launch configuration the benchmark times.
Every int8 code and fp32 scale is compared in full (the oracle's rotation is cheap); the
matmul outputs are compared on sampled rows (all columns) and sampled columns (all rows),
which the oracle computes from its own codes."""
import numpy as np
import pytest
import torch

import oracle
import hadamard_rotated_int8_b200 as sd
from hadamard_rotated_int8_b200 import _build, synthetic
from tests.test_gpu_parity import assert_equal, bf16_val, bits_of, lora_tolerances, ulp_diff

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    _build.build()
    oracle.build()
    yield
    torch.cuda.synchronize()
    assert sd.sdnq_device_status() == 0


def sample(n, k, seed, must=()):
    rng = np.random.default_rng(seed)
    picks = set(int(i) for i in must if 0 <= i < n)
    picks |= set(int(i) for i in rng.choice(n, size=min(k, n), replace=False))
    return np.array(sorted(picks))


def check_linear(case, name, seed):
    g = case.g
    xg, Wg = case.x.cuda(), case.W.cuda()
    qW, sW = sd.sdnq_rotate_quant_weight(Wg, g)
    qx, sx = sd.sdnq_rotquant_act(xg, g)
    bias = case.bias.cuda() if case.bias is not None else None
    lora = case.A is not None
    if lora:
        u = torch.empty((case.M, case.A.shape[1]), dtype=torch.bfloat16, device="cuda")
        out = sd.sdnq_int8_linear_lora(qx, sx, qW, sW, bias, xg, case.A.cuda(), case.B.cuda(),
                                       case.lora_scale, u_ws=u)
    else:
        out = sd.sdnq_int8_linear(qx, sx, qW, sW, bias)
    torch.cuda.synchronize()

    xb, Wb = synthetic.bits(case.x), synthetic.bits(case.W)
    bb = synthetic.bits(case.bias) if case.bias is not None else None
    qx_r, sx_r = oracle.rotate_quantize(xb, g)
    qW_r, sW_r = oracle.rotate_quantize(Wb, g)
    assert_equal(qx.cpu().numpy(), qx_r, f"{name}: activation codes")
    assert_equal(sx.cpu().numpy().view(np.uint32), sx_r.view(np.uint32), f"{name}: token scales")
    assert_equal(qW.cpu().numpy(), qW_r, f"{name}: weight codes")
    assert_equal(sW.cpu().numpy().view(np.uint32), sW_r.view(np.uint32), f"{name}: row scales")

    out_b = bits_of(out)
    rows = sample(case.M, 12, seed, must=(0, 127, 128, case.M - 1))
    cols = sample(case.N, 6, seed + 1, must=(0, 255, 256, case.N - 1))
    L_rows = L_cols = None
    if lora:
        Ab, Bb = synthetic.bits(case.A), synthetic.bits(case.B)
        Bc = np.ascontiguousarray(Bb[:, cols])
        u_rows = oracle.lora_down(xb[rows], Ab)
        L_rows = oracle.lora_up(u_rows, Bb)
        u_all = oracle.lora_down(xb, Ab)
        L_cols = oracle.lora_up(u_all, Bc)
    acc_rows = oracle.gemm_s8(qx_r[rows], qW_r)
    ref_rows = oracle.dequant_epilogue(acc_rows, sx_r[rows], sW_r, bb, L_rows, case.lora_scale)
    acc_cols = oracle.gemm_s8(qx_r, np.ascontiguousarray(qW_r[cols]))
    ref_cols = oracle.dequant_epilogue(acc_cols, sx_r, sW_r[cols],
                                       bb[cols] if bb is not None else None, L_cols,
                                       case.lora_scale)
    if lora:
        u_b = bits_of(u)
        tol_u, tol_rows = lora_tolerances(xb[rows], Ab, Bb, u_rows, ref_rows, case.lora_scale)
        _, tol_cols = lora_tolerances(xb, Ab, Bc, u_all, ref_cols, case.lora_scale)
        du = np.abs(bf16_val(u_b[rows]).astype(np.float64) - bf16_val(u_rows))
        assert np.all(du <= tol_u), f"{name}: u outside the fp32-accumulation bound"
        for got, ref, tol, what in ((out_b[rows], ref_rows, tol_rows, "rows"),
                                    (out_b[:, cols], ref_cols, tol_cols, "cols")):
            d = np.abs(bf16_val(got).astype(np.float64) - bf16_val(ref))
            assert np.all(d <= tol), f"{name}: {what} outside the bound"
            assert (ulp_diff(got, ref) <= 1).mean() > 0.999, f"{name}: {what}"
    else:
        assert_equal(out_b[rows], ref_rows, f"{name}: sampled rows")
        assert_equal(out_b[:, cols], ref_cols, f"{name}: sampled columns")


@pytest.mark.parametrize("name,g", [
    ("tiny_256", 256),
    ("dit_attn_4096x3072x3072", 256),
    ("peft_lora_8192x12288x3072_r64", 256),
    ("quarot_16384x4096x4096", 64),
    ("quarot_16384x4096x4096", 128),
    ("quarot_16384x4096x4096", 256),
])
def test_workload_parity(name, g):
    case = synthetic.workload(name, g=g)
    check_linear(case, f"{name} g={g}", seed=g)


def test_dit_mlp_chain_parity():
    """Up projection -> GELU -> per-token requantisation -> down projection, on the MLP
    workload; the oracle runs the same chain from x for sampled tokens, and the fused
    up-projection + GELU equals the two-pass chain on every element."""
    case = synthetic.workload("dit_mlp_4608x3840x10240")
    g = case.g
    W_down = case.extra["W_down"]
    xg = case.x.cuda()
    qWu, sWu = sd.sdnq_rotate_quant_weight(case.W.cuda(), g)
    qWd, sWd = sd.sdnq_rotate_quant_weight(W_down.cuda(), g)
    qx, sx = sd.sdnq_rotquant_act(xg, g)
    up = sd.sdnq_int8_linear(qx, sx, qWu, sWu)
    h = sd.sdnq_gelu_bf16(up)
    h_fused = sd.sdnq_int8_linear_gelu(qx, sx, qWu, sWu)  # the step's fused up-projection
    qh, sh = sd.sdnq_rotquant_act(h, g)
    down = sd.sdnq_int8_linear(qh, sh, qWd, sWd)
    torch.cuda.synchronize()

    rows = sample(case.M, 10, 3, must=(0, case.M - 1))
    xb = synthetic.bits(case.x)
    qx_r, sx_r = oracle.rotate_quantize(xb[rows], g)
    qWu_r, sWu_r = oracle.rotate_quantize(synthetic.bits(case.W), g)
    qWd_r, sWd_r = oracle.rotate_quantize(synthetic.bits(W_down), g)
    up_r = oracle.dequant_epilogue(oracle.gemm_s8(qx_r, qWu_r), sx_r, sWu_r)
    h_r = oracle.gelu_bf16(up_r)
    qh_r, sh_r = oracle.rotate_quantize(h_r, g)
    down_r = oracle.dequant_epilogue(oracle.gemm_s8(qh_r, qWd_r), sh_r, sWd_r)
    assert_equal(bits_of(up)[rows], up_r, "up projection")
    assert_equal(bits_of(h)[rows], h_r, "gelu")
    assert_equal(bits_of(h_fused), bits_of(h), "GELU fused into the up-projection epilogue")
    assert_equal(qh.cpu().numpy()[rows], qh_r, "requantised codes")
    assert_equal(sh.cpu().numpy()[rows].view(np.uint32), sh_r.view(np.uint32), "requantised scales")
    assert_equal(bits_of(down)[rows], down_r, "down projection")
