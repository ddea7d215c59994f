"""Full-size GPU parity cases: every element of every output against the CPU oracle.

Each case runs one of the DiT-shaped workloads at its full size, in the launch configuration
a real call (and the benchmark) uses, and compares every int8 code, every fp32 scale, every
int32 accumulator and every bf16 output with the oracle, which computes the whole problem
from the same seeded bf16 inputs on its own. Exact where the arithmetic is pinned (codes,
scales, accumulators, outputs without LoRA); within the stated bound where the tensor cores
accumulate floating point in their own order (the LoRA adapter, the FP8 accumulators,
attention).

``tests/test_gpu_fullsize.py`` runs each case in a child process of its own
(``python -m tests.fullsize_cases <case>``), so that a sticky CUDA fault in one case cannot
fail the others. The child prints one JSON line of observations (for LoRA: the largest ulp
distance and how many outputs sit at one ulp) and exits 0 if every check passed.

Test infrastructure: it imports the oracle, which the product never does.
"""
from __future__ import annotations

import json
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import oracle  # noqa: E402
import hadamard_rotated_int8_b200 as sd  # noqa: E402
from hadamard_rotated_int8_b200 import _build, _native, synthetic  # noqa: E402
from tests.test_gpu_parity import (assert_equal, bf16_val, bits_of,  # noqa: E402
                                   lora_tolerances, ulp_diff)


def _u32(a):
    return np.asarray(a).view(np.uint32)


def _acc(M, N):
    return torch.empty((M, N), dtype=torch.int32, device="cuda")


def _ulp_report(got_bits, ref_bits):
    d = ulp_diff(got_bits, ref_bits)
    return {"max_ulp": int(d.max()) if d.size else 0, "at_1_ulp": int(np.count_nonzero(d == 1)),
            "above_1_ulp": int(np.count_nonzero(d > 1)), "n": int(d.size)}


# ------------------------------------------------------------------ linear workloads

def linear(name: str, g: int):
    """Two launches (rotate+quantize, then the GEMM with its epilogue; with LoRA the
    down-projection kernel and the GEMM with the second accumulator), and for the base layer
    also the one-launch kernel and the library's automatic choice."""
    case = synthetic.workload(name, g=g)
    M, N, K = case.M, case.N, case.K
    lora = case.A is not None
    xg = case.x.cuda()
    qW, sW = sd.sdnq_rotate_quant_weight(case.W.cuda(), g)
    qx, sx = sd.sdnq_rotquant_act(xg, g)
    bias = case.bias.cuda() if case.bias is not None else None
    acc = _acc(M, N)
    if lora:
        u = torch.empty((M, case.A.shape[1]), dtype=torch.bfloat16, device="cuda")
        out = sd.sdnq_int8_linear_lora(qx, sx, qW, sW, bias, xg, case.A.cuda(), case.B.cuda(),
                                       case.lora_scale, u_ws=u, acc_out=acc)
    else:
        out = sd.sdnq_int8_linear(qx, sx, qW, sW, bias, acc_out=acc)
    torch.cuda.synchronize()
    got = {"qx": qx.cpu().numpy(), "sx": sx.cpu().numpy(), "qW": qW.cpu().numpy(),
           "sW": sW.cpu().numpy(), "acc": acc.cpu().numpy(), "out": bits_of(out)}
    if lora:
        got["u"] = bits_of(u)
    fused = {}
    if not lora:
        for policy, tag in ((_native.FUSE_ALWAYS, "one"), (_native.FUSE_AUTO, "auto")):
            qx_f = torch.empty_like(qx)
            sx_f = torch.empty_like(sx)
            acc_f = _acc(M, N)
            out_f = sd.sdnq_int8_linear_fused(xg, g, qW, sW, bias, qx_ws=qx_f, sx_ws=sx_f,
                                              acc_out=acc_f, policy=policy)
            torch.cuda.synchronize()
            fused[tag] = {"qx": qx_f.cpu().numpy(), "sx": sx_f.cpu().numpy(),
                          "acc": acc_f.cpu().numpy(), "out": bits_of(out_f)}
    assert sd.sdnq_device_status() == 0
    del out, acc, qx, qW, xg
    torch.cuda.empty_cache()

    xb, Wb = synthetic.bits(case.x), synthetic.bits(case.W)
    bb = synthetic.bits(case.bias) if case.bias is not None else None
    qx_r, sx_r = oracle.rotate_quantize(xb, g)
    qW_r, sW_r = oracle.rotate_quantize(Wb, g)
    acc_r = oracle.gemm_s8(qx_r, qW_r)
    L = u_r = None
    if lora:
        Ab, Bb = synthetic.bits(case.A), synthetic.bits(case.B)
        u_r = oracle.lora_down(xb, Ab)
        L = oracle.lora_up(u_r, Bb)
    out_r = oracle.dequant_epilogue(acc_r, sx_r, sW_r, bb, L, case.lora_scale)

    assert_equal(got["qW"], qW_r, "weight codes")
    assert_equal(_u32(got["sW"]), _u32(sW_r), "weight row scales")
    assert_equal(got["qx"], qx_r, "activation codes")
    assert_equal(_u32(got["sx"]), _u32(sx_r), "token scales")
    assert_equal(got["acc"], acc_r, "int32 accumulators")
    report = {"elements": int(out_r.size)}
    if lora:
        tol_u, tol_out = lora_tolerances(xb, Ab, Bb, u_r, out_r, case.lora_scale)
        du = np.abs(bf16_val(got["u"]).astype(np.float64) - bf16_val(u_r))
        assert np.all(du <= tol_u), f"u: {np.count_nonzero(du > tol_u)} outside the bound"
        dout = np.abs(bf16_val(got["out"]).astype(np.float64) - bf16_val(out_r))
        assert np.all(dout <= tol_out), \
            f"outputs: {np.count_nonzero(dout > tol_out)} outside the bound"
        report["u"] = _ulp_report(got["u"], u_r)
        report["out"] = _ulp_report(got["out"], out_r)
        # Outputs further than one bf16 ulp from the oracle are those where the sum
        # acc * t + bias + lora_scale * L cancels: the fp32 accumulation-order difference of
        # the adapter terms (bounded above) is then more than an ulp of the small result.
        # Every output is within the bound; at most 2 in 10^4 may sit beyond one ulp (the
        # full PEFT workload shows 0.8 in 10^4). The report gives, for those outputs, the
        # largest ratio of |result| to the magnitude of its int8 term (small: cancellation).
        d = ulp_diff(got["out"], out_r)
        far = d > 1
        assert far.mean() <= 2e-4, f"LoRA outputs: {report['out']}"
        if far.any():
            rows, cols = np.nonzero(far)
            term = (np.abs(acc_r[rows, cols].astype(np.float64)) * sx_r[rows].astype(np.float64)
                    * sW_r[cols].astype(np.float64))
            res = np.abs(bf16_val(out_r[rows, cols]).astype(np.float64))
            report["out"]["far_max_result_over_int8_term"] = float((res / np.maximum(term, 1e-30)).max())
            report["out"]["far_median_result_over_int8_term"] = float(np.median(res / np.maximum(term, 1e-30)))
    else:
        assert_equal(got["out"], out_r, "bf16 outputs")
        for tag, f in fused.items():
            assert_equal(f["qx"], qx_r, f"{tag}-launch path: activation codes")
            assert_equal(_u32(f["sx"]), _u32(sx_r), f"{tag}-launch path: token scales")
            assert_equal(f["acc"], acc_r, f"{tag}-launch path: int32 accumulators")
            assert_equal(f["out"], out_r, f"{tag}-launch path: bf16 outputs")
        report["auto_one_launch"] = bool(sd.sdnq_int8_linear_fused_plan(M, N, K))
    return report


# ------------------------------------------------------------------ the MLP pair

def mlp():
    """Up-projection with GELU in its epilogue, per-token requantisation of the hidden layer,
    down-projection (the benchmark's step), plus the unfused up-projection and the standalone
    GELU kernel; every element against the oracle's chain from x."""
    case = synthetic.workload("dit_mlp_4608x3840x10240")
    g, M, N, K = case.g, case.M, case.N, case.K
    Wd = case.extra["W_down"]
    xg = case.x.cuda()
    qWu, sWu = sd.sdnq_rotate_quant_weight(case.W.cuda(), g)
    qWd, sWd = sd.sdnq_rotate_quant_weight(Wd.cuda(), g)
    qx, sx = sd.sdnq_rotquant_act(xg, g)
    acc_up = _acc(M, N)
    h = sd.sdnq_int8_linear_gelu(qx, sx, qWu, sWu, acc_out=acc_up)
    qh, sh = sd.sdnq_rotquant_act(h, g)
    acc_dn = _acc(M, K)
    down = sd.sdnq_int8_linear(qh, sh, qWd, sWd, acc_out=acc_dn)
    up_plain = sd.sdnq_int8_linear(qx, sx, qWu, sWu)
    h_two_pass = sd.sdnq_gelu_bf16(up_plain)
    torch.cuda.synchronize()
    assert sd.sdnq_device_status() == 0
    got = {"qx": qx.cpu().numpy(), "sx": sx.cpu().numpy(), "acc_up": acc_up.cpu().numpy(),
           "h": bits_of(h), "qh": qh.cpu().numpy(), "sh": sh.cpu().numpy(),
           "acc_dn": acc_dn.cpu().numpy(), "down": bits_of(down), "up": bits_of(up_plain),
           "h2": bits_of(h_two_pass), "qWu": qWu.cpu().numpy(), "sWu": sWu.cpu().numpy(),
           "qWd": qWd.cpu().numpy(), "sWd": sWd.cpu().numpy()}
    del h, qh, down, up_plain, h_two_pass, acc_up, acc_dn
    torch.cuda.empty_cache()

    xb = synthetic.bits(case.x)
    qWu_r, sWu_r = oracle.rotate_quantize(synthetic.bits(case.W), g)
    qWd_r, sWd_r = oracle.rotate_quantize(synthetic.bits(Wd), g)
    qx_r, sx_r = oracle.rotate_quantize(xb, g)
    acc_up_r = oracle.gemm_s8(qx_r, qWu_r)
    up_r = oracle.dequant_epilogue(acc_up_r, sx_r, sWu_r)
    h_r = oracle.gelu_bf16(up_r)
    qh_r, sh_r = oracle.rotate_quantize(h_r, g)
    acc_dn_r = oracle.gemm_s8(qh_r, qWd_r)
    down_r = oracle.dequant_epilogue(acc_dn_r, sh_r, sWd_r)

    assert_equal(got["qWu"], qWu_r, "up weight codes")
    assert_equal(_u32(got["sWu"]), _u32(sWu_r), "up weight scales")
    assert_equal(got["qWd"], qWd_r, "down weight codes")
    assert_equal(_u32(got["sWd"]), _u32(sWd_r), "down weight scales")
    assert_equal(got["qx"], qx_r, "activation codes")
    assert_equal(_u32(got["sx"]), _u32(sx_r), "token scales")
    assert_equal(got["acc_up"], acc_up_r, "up-projection int32 accumulators")
    assert_equal(got["up"], up_r, "up-projection bf16 outputs (plain epilogue)")
    assert_equal(got["h"], h_r, "GELU-epilogue outputs")
    assert_equal(got["h2"], h_r, "standalone GELU outputs")
    assert_equal(got["qh"], qh_r, "hidden-layer codes")
    assert_equal(_u32(got["sh"]), _u32(sh_r), "hidden-layer scales")
    assert_equal(got["acc_dn"], acc_dn_r, "down-projection int32 accumulators")
    assert_equal(got["down"], down_r, "down-projection bf16 outputs")
    return {"elements_up": int(up_r.size), "elements_down": int(down_r.size)}


# ------------------------------------------------------------------ input gradient

def grad(name: str):
    from tests.test_gpu_grad import oracle_ref, run_gpu
    case = synthetic.workload(name)
    got = run_gpu(case.x, case.W, case.g, case.N)
    assert sd.sdnq_device_status() == 0
    ref = oracle_ref(case.x, case.W, case.g, case.N)
    assert_equal(got["qg"], ref["qg"], "codes of dy * sW")
    assert_equal(_u32(got["sg"]), _u32(ref["sg"]), "scales of dy * sW")
    assert_equal(got["acc"], ref["acc"], "int32 accumulators")
    assert_equal(got["dx"], ref["dx"], "bf16 dx")
    return {"elements": int(ref["dx"].size)}


# ------------------------------------------------------------------ FP8

def fp8(name: str):
    from tests.test_gpu_fp8 import check_against_oracle, run_fp8
    case = synthetic.workload(name)
    got = run_fp8(case)
    assert sd.sdnq_device_status() == 0
    err, bound = check_against_oracle(case, got)
    return {"elements": int(got["out"].size),
            "max_acc_err_over_bound": float((err / np.maximum(bound, 1e-300)).max())}


# ------------------------------------------------------------------ attention

def attention():
    """The Flux.1 joint attention (B 1, 4608 tokens, 24 heads of 128) on the GPU; the oracle
    recomputes two whole heads (first and last) from their own slices of q, k and v: key
    means, every query and key code and scale, and every output row of those heads."""
    from tests.test_gpu_attention import run_gpu
    case = synthetic.workload("attn_flux_b1_l4608_h24_d128")
    q, k, v = case.x, case.W, case.extra["v"]
    got = run_gpu(q, k, v, case.g, True)
    assert sd.sdnq_device_status() == 0
    heads = [0, q.shape[2] - 1]
    sl = lambda t: synthetic.bits(t[:, :, heads, :].contiguous())  # noqa: E731
    ref = oracle.attention(sl(q), sl(k), sl(v), case.g, smooth_k=True)
    assert_equal(got["mu"][:, heads], ref["mu"], "key means")
    assert_equal(got["kq"][:, :, heads], ref["kq"], "key codes")
    assert_equal(_u32(got["sk"][:, heads]), _u32(ref["sk"]), "key scales")
    assert_equal(got["qq"][:, :, heads], ref["qq"], "query codes")
    assert_equal(_u32(got["sq"][:, heads]), _u32(ref["sq"]), "query scales")
    absv = sl(v.abs())
    S = bf16_val(oracle.attn_softmax_pv(ref["logits"], absv)).astype(np.float64) * (1 + 2.0 ** -7)
    o_ref = bf16_val(ref["o"]).astype(np.float64)
    o_got = bf16_val(np.ascontiguousarray(got["o"][:, :, heads])).astype(np.float64)
    Lk = k.shape[1]
    bound = 2.0 ** -8 * np.abs(o_ref) + (2.0 ** -8 + 2 * Lk * 2.0 ** -24 + 2.0 ** -16) * S + 1e-30
    err = np.abs(o_got - o_ref)
    assert np.all(err <= bound), float((err / bound).max())
    return {"heads": heads, "rows_per_head": int(q.shape[1]),
            "max_err_over_bound": float((err / bound).max()),
            "exact": float((o_got == o_ref).mean())}


CASES = {
    "tiny_256": lambda: linear("tiny_256", 256),
    "dit_attn_4096x3072x3072": lambda: linear("dit_attn_4096x3072x3072", 256),
    "peft_lora_8192x12288x3072_r64": lambda: linear("peft_lora_8192x12288x3072_r64", 256),
    "quarot_16384x4096x4096_g64": lambda: linear("quarot_16384x4096x4096", 64),
    "quarot_16384x4096x4096_g128": lambda: linear("quarot_16384x4096x4096", 128),
    "quarot_16384x4096x4096_g256": lambda: linear("quarot_16384x4096x4096", 256),
    "dit_mlp_4608x3840x10240": mlp,
    "grad_dit_attn_4096x3072x3072": lambda: grad("grad_dit_attn_4096x3072x3072"),
    "grad_peft_8192x12288x3072": lambda: grad("grad_peft_8192x12288x3072"),
    "fp8_dit_attn_4096x3072x3072": lambda: fp8("fp8_dit_attn_4096x3072x3072"),
    "fp8_quarot_16384x4096x4096": lambda: fp8("fp8_quarot_16384x4096x4096"),
    "attn_flux_b1_l4608_h24_d128": attention,
}


def main(argv):
    name = argv[1]
    _build.build()
    oracle.build()
    torch.cuda.set_device(0)
    t0 = time.time()
    report = CASES[name]()
    report.update({"case": name, "seconds": round(time.time() - t0, 1)})
    print("REPORT " + json.dumps(report), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main(sys.argv))
