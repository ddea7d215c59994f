"""Inputs on which the de-quant epilogue's rounding structure is visible.

The epilogue rounds twice: v = fp32(float(acc) * t), then fp32(v + bias). A fused
multiply-add rounds once, and on most inputs the two agree after the final bf16 rounding.
These inputs are the exceptions, so a test on them tells two roundings from one."""
import numpy as np


def fma_sensitive_epilogue_inputs(count=256, seed=5):
    """`count` tuples (a1, a2, sx, sw, bias_bits), acc = a1 * a2 (int8 codes), t = fp32(sx *
    sw), for which the two roundings v = fp32(acc * t), fp32(v + bias) give a different bf16
    output than one fused multiply-add would: the bias cancels most of v, so that the sum is
    exact and sits on a bf16 rounding tie. Found by a seeded search on the host (numpy)."""
    f = np.float32
    rng = np.random.default_rng(seed)

    def to_bf16_bits(a):
        u = np.asarray(a, f).view(np.uint32).astype(np.uint64)
        return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)

    picks = []
    while sum(len(p[0]) for p in picks) < count:
        n = 2_000_000
        a1 = rng.integers(-127, 128, n)
        a2 = rng.integers(-127, 128, n)
        sx = rng.uniform(1e-3, 1e-1, n).astype(f)
        sw = rng.uniform(1e-4, 1e-2, n).astype(f)
        t = (sx * sw).astype(f)
        v = ((a1 * a2).astype(f) * t).astype(f)
        bias = to_bf16_bits((-v * rng.uniform(0.3, 0.95, n)).astype(f))
        biasf = (bias.astype(np.uint32) << 16).view(f)
        two = (v + biasf).astype(f)
        fused = ((a1 * a2).astype(np.float64) * t.astype(np.float64) + biasf).astype(f)
        hit = to_bf16_bits(two) != to_bf16_bits(fused)
        picks.append((a1[hit], a2[hit], sx[hit], sw[hit], bias[hit]))
    a1, a2, sx, sw, bias = (np.concatenate(c)[:count] for c in zip(*picks))
    return a1, a2, sx, sw, bias
