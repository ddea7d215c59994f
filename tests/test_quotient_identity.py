"""The division-free quotient the quantizer kernels use for the row scale (CPU only).

s_z = RN(amax / D), D = 127 (int8 grid) or 448 (e4m3 grid), is computed on the GPU as
q0 = RN(amax * y), r = RN(amax - q0 * D), s_z = RN(q0 + r * y) with y = RN(1 / D) (Markstein's
correction; P. Markstein, IBM J. Res. Dev. 34(1), 1990). This checks, for every fp32 input
of two whole binades, that r is exact and that s_z is the IEEE quotient. Scaling by a power
of two scales every step exactly while the intermediates stay normal, so these binades stand
for all inputs the kernels send down this path (amax >= 2^-100); smaller maxima use the IEEE
division. The GPU parity tests compare the scales themselves with the oracle.
"""
import numpy as np
import pytest

Y_BITS = {127: 0x3C010204, 448: 0x3B124925}


@pytest.mark.parametrize("D", [127, 448])
@pytest.mark.parametrize("exponent", [0, 1])
def test_division_free_quotient_is_the_ieee_quotient(D, exponent):
    y = np.array([Y_BITS[D]], dtype=np.uint32).view(np.float32)[0]
    assert y == np.float32(1) / np.float32(D)          # y = RN(1 / D)
    mant = np.arange(1 << 23, dtype=np.uint32)
    a = ((np.uint32(127 + exponent) << 23) | mant).view(np.float32)
    q0 = a * y                                         # fp32 product, one rounding
    r64 = a.astype(np.float64) - q0.astype(np.float64) * D   # exact (both terms < 2^53 apart)
    r = r64.astype(np.float32)
    assert np.array_equal(r.astype(np.float64), r64), "residual not exact in fp32"
    # q0 + r * y: r * y is exact in fp64; the fp64 sum is within 2^-53 of the exact value,
    # so its fp32 rounding is the exact value's unless it sits on an fp32 midpoint
    s64 = q0.astype(np.float64) + r.astype(np.float64) * np.float64(y)
    ref64 = a.astype(np.float64) / D

    def midpointish(x64):
        x32 = x64.astype(np.float32)
        ulp = np.spacing(np.abs(x32)).astype(np.float64)
        return np.abs(np.abs((x64 - x32.astype(np.float64)) / ulp) - 0.5) < 1e-6

    assert not midpointish(s64).any() and not midpointish(ref64).any()
    assert np.array_equal(s64.astype(np.float32), ref64.astype(np.float32))
