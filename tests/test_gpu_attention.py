"""GPU parity of the Hadamard-rotated int8-QK attention against the oracle.

Bit-exact: the smooth_k key means, the int8 codes and fp32 scales of Q and K (same fp32
arithmetic on both sides). Outputs: the oracle takes the softmax and PV in fp64 from its fp32
logits; the GPU forms base-2 logits (acc * s_k) * (s_q * scale * log2 e) (within a few fp32
ulps of the oracle's, which moves a probability by about |logit| 2^-22), takes ex2.approx
(2^-22), rounds P to bf16 for the PV product and accumulates in fp32. So per element
|o - o_ref| <= 2^-8 |o_ref| + (2^-8 + 2 Lk 2^-24 + 2^-16) S, with
S = sum_j p_ij |v_j| / sum_j p_ij (one bf16 rounding of P and of o, the fp32 sums over Lk
keys, the logit and exponential differences), S computed by the oracle with |v| in place of
v. Every input is seeded."""
import numpy as np
import pytest
import torch

import oracle
import hadamard_rotated_int8_b200 as sd
from hadamard_rotated_int8_b200 import _build, _native, synthetic
from tests.test_gpu_parity import assert_equal, bf16_val, bits_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    _build.build()
    oracle.build()
    torch.cuda.init()
    yield
    assert sd.sdnq_device_status() == 0


def qkv(B, Lq, Lk, H, seed, k_offset=0.0):
    gen = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Lq, H, 128, generator=gen)
    k = torch.randn(B, Lk, H, 128, generator=gen) + k_offset * torch.randn(1, 1, H, 128, generator=gen)
    v = torch.randn(B, Lk, H, 128, generator=gen)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def run_gpu(q, k, v, g, smooth):
    B, Lq, H, D = q.shape
    Lk = k.shape[1]
    total, off = _native.attention_workspace(B, Lq, Lk, H, D)
    ws = torch.empty(total, dtype=torch.uint8, device="cuda")
    o = sd.sdnq_attention_int8qk(q.cuda(), k.cuda(), v.cuda(), g, smooth_k=smooth, ws=ws)
    torch.cuda.synchronize()
    w = ws.cpu().numpy()

    def view(i, dtype, shape):
        n = int(np.prod(shape)) * np.dtype(dtype).itemsize
        return w[off[i]:off[i] + n].view(dtype).reshape(shape)
    lqp, lkp = (Lq + 127) // 128 * 128, (Lk + 127) // 128 * 128
    return {"o": bits_of(o), "qq": view(0, np.int8, (B, Lq, H, D)),
            "kq": view(1, np.int8, (B, Lk, H, D)),
            "sq": np.ascontiguousarray(view(2, np.float32, (B, H, lqp))[:, :, :Lq]),
            "sk": np.ascontiguousarray(view(3, np.float32, (B, H, lkp))[:, :, :Lk]),
            "mu": view(4, np.float32, (B, H, D))}


def check(q, k, v, g, smooth, rows=None):
    got = run_gpu(q, k, v, g, smooth)
    qb, kb, vb = synthetic.bits(q), synthetic.bits(k), synthetic.bits(v)
    if rows is not None:
        qb = np.ascontiguousarray(qb[:, rows])
    ref = oracle.attention(qb, kb, vb, g, smooth_k=smooth)
    sel = slice(None) if rows is None else rows
    assert_equal(got["mu"], ref["mu"], "key means")
    assert_equal(got["kq"], ref["kq"], "key codes")
    assert_equal(got["sk"].view(np.uint32), ref["sk"].view(np.uint32), "key scales")
    assert_equal(got["qq"][:, sel], ref["qq"], "query codes")
    assert_equal(got["sq"][:, :, sel].view(np.uint32), ref["sq"].view(np.uint32), "query scales")
    absv = synthetic.bits(v.abs())
    S = bf16_val(oracle.attn_softmax_pv(ref["logits"], absv)).astype(np.float64) * (1 + 2.0 ** -7)
    o_ref = bf16_val(ref["o"]).astype(np.float64)
    o_got = bf16_val(got["o"][:, sel]).astype(np.float64)
    Lk = k.shape[1]
    bound = 2.0 ** -8 * np.abs(o_ref) + (2.0 ** -8 + 2 * Lk * 2.0 ** -24 + 2.0 ** -16) * S + 1e-30
    err = np.abs(o_got - o_ref)
    assert np.all(err <= bound), float((err / bound).max())
    return err, bound


@pytest.mark.parametrize("B,Lq,Lk,H,g,smooth", [
    (1, 128, 128, 1, 256, True), (2, 200, 333, 3, 256, True), (1, 77, 1000, 2, 64, True),
    (2, 256, 129, 2, 128, False), (1, 1, 5, 4, 8, True), (1, 300, 4096, 1, 256, True),
])
def test_attention_parity(B, Lq, Lk, H, g, smooth):
    q, k, v = qkv(B, Lq, Lk, H, seed=B * 1000 + Lq + Lk + g, k_offset=3.0)
    check(q, k, v, g, smooth)


def test_attention_flux_shape_sampled_rows():
    """B = 1, 4608 joint tokens, 24 heads of 128 (Flux.1): every code and scale, outputs of
    sampled query rows of every head."""
    q, k, v = qkv(1, 4608, 4608, 24, seed=11, k_offset=3.0)
    rng = np.random.default_rng(12)
    rows = np.unique(np.concatenate([[0, 4607], rng.choice(4608, 10, replace=False)]))
    check(q, k, v, 256, True, rows=rows)


def test_split_calls_equal_the_composed_call():
    q, k, v = qkv(2, 150, 260, 3, seed=21, k_offset=2.0)
    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    ws = sd._native.sdnq_attention_prep(qg, kg, 128)
    o_split = sd._native.sdnq_attention_core(vg, 150, ws)
    o = sd.sdnq_attention_int8qk(qg, kg, vg, 128)
    torch.cuda.synchronize()
    assert_equal(bits_of(o_split), bits_of(o), "split against composed")


def wide_qkv(seed, sign):
    """Keys whose norms alternate 1x / 8x inside every block, queries (anti-)aligned with a
    shared key direction: logits of several hundred in base 2 and a key-scale range of about
    8x per block."""
    gen = torch.Generator().manual_seed(seed)
    B, Lq, Lk, H = 1, 96, 520, 2
    amp = torch.where(torch.arange(Lk) % 2 == 0, 1.0, 8.0).reshape(1, Lk, 1, 1)
    base = torch.randn(1, 1, H, 128, generator=gen)
    k = (0.5 * base + torch.randn(B, Lk, H, 128, generator=gen)) * amp
    q = sign * 6.0 * base + torch.randn(B, Lq, H, 128, generator=gen)
    v = torch.randn(B, Lk, H, 128, generator=gen)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


@pytest.mark.parametrize("sign,smooth", [(1.0, True), (1.0, False), (-1.0, False)])
def test_attention_wide_logits(sign, smooth):
    """Logits of several hundred (base 2), positive and negative row maxima, a ragged last key
    block, workspace left uninitialised: outputs within the same bound."""
    q, k, v = wide_qkv(31 + int(sign), sign)
    check(q, k, v, 256, smooth)

