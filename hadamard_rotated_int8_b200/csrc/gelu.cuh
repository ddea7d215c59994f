// GELU between the up and down projections of a DiT MLP, bf16 -> bf16, exact-erf form
// GELU(x) = x * Phi(x) = 0.5 * x * erfc(-x / sqrt(2)), rounded once to bf16.
//
// Fast path in fp32 with CUDA's erfcf. Its relative error against the exact value is at
// most about (x^2 + 6.5) * 2^-23 (argument rounding of x/sqrt(2), amplified by the
// logarithmic slope of erfc, which is at most 2a^2 + 2 for a = -x/sqrt(2); erfcf's own
// 4 ulp; one final product). The kernel widens that to a margin of (x^2 + 16) * 2^-22 and
// keeps the fp32 result only when the whole interval value +- margin rounds to one bf16
// value: then that value is the correctly rounded bf16 of the exact GELU. Otherwise (a value
// near a bf16 rounding boundary, or |x| > 10 where fp32 underflows) it recomputes in fp64
// and rounds the fp64 value to bf16 directly, with a single rounding.
#pragma once

#include <cuda_bf16.h>

#include "device.cuh"

namespace sdnq {

// binary64 -> bf16, round to nearest even, one rounding (bf16 keeps 1 + 7 significand bits).
__device__ __forceinline__ uint32_t f64_to_bf16_bits(double d)
{
    if (isnan(d))
        return 0x7fc0u;
    const uint32_t sign = signbit(d) ? 0x8000u : 0u;
    const double a = fabs(d);
    if (isinf(a))
        return sign | 0x7f80u;
    double r;
    if (a < 0x1p-126) {
        r = rint(a * 0x1p133) * 0x1p-133;  // bf16 subnormal grid 2^-133
    } else {
        unsigned long long u = static_cast<unsigned long long>(__double_as_longlong(a));
        u += (1ull << 44) - 1ull + ((u >> 45) & 1ull);
        u &= ~((1ull << 45) - 1ull);
        r = __longlong_as_double(static_cast<long long>(u));
    }
    const float f = __double2float_rn(r);  // exact, or +inf past the range
    return sign | (__float_as_uint(f) >> 16);
}

__device__ __forceinline__ uint32_t f32_to_bf16_bits_rn(float f)
{
    return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(f)));
}

// fp64 evaluation, rounded once to bf16: the rare inputs the fp32 path cannot decide
__device__ __noinline__ uint32_t gelu_bf16_bits_fp64(uint32_t xb)
{
    const double xd = static_cast<double>(__uint_as_float(xb << 16));
    const double y = 0.5 * xd * erfc(-xd * 0.70710678118654752440);
    return f64_to_bf16_bits(y);
}

__device__ __forceinline__ uint32_t gelu_bf16_bits(uint32_t xb)
{
    const float x = __uint_as_float(xb << 16);
    if (fabsf(x) <= 10.0f) {
        const float a = __fmul_rn(x, -0.70710678118654752440f);
        const float e = erfcf(a);
        const float v = __fmul_rn(__fmul_rn(0.5f, x), e);
        const float margin = __fmul_rn(fabsf(v), __fmul_rn(__fadd_rn(__fmul_rn(x, x), 16.0f), 0x1p-22f));
        const uint32_t lo = f32_to_bf16_bits_rn(__fsub_rn(v, margin));
        const uint32_t hi = f32_to_bf16_bits_rn(__fadd_rn(v, margin));
        if (lo == hi)
            return lo;
    }
    return gelu_bf16_bits_fp64(xb);
}

// ---- table form, for bf16 inputs produced inside another kernel (the GEMM epilogue) ----
// A bf16 -> bf16 function has only 65536 inputs, and outside |x| in [2^-10, 16) the correctly
// rounded GELU has a closed form:
//   * |x| < 2^-10 (normal): GELU(x) = x/2 + x^2/sqrt(2 pi) + O(x^4) differs from x/2 (a bf16
//     value) by a relative 0.8|x| < 2^-10.3, less than half a bf16 ulp (>= 2^-9 relative,
//     also just below a binade boundary), so the result is x/2, exactly;
//   * x >= 16: 1 - Phi(16) ~ 6e-58, the result is x; x <= -16: |GELU(x)| < 1e-56, far
//     below half the smallest bf16 subnormal, the result is -0;
//   * +-0: +-0.
// The 3584 inputs in between (both signs, biased exponents 117..130, all 128 mantissas) go
// through a table built with gelu_bf16_bits. Below 2^-125 (subnormal and the smallest normal
// binade) Phi(x) rounds to 0.5 even in fp64, so the result is x/2 rounded half to even on
// the subnormal grid; +Inf gives +Inf, -Inf and NaN give NaN (0x7fc0).
constexpr int kGeluLutExpLo = 117;                    // 2^-10
constexpr int kGeluLutExpHi = 130;                    // [8, 16)
constexpr int kGeluLutHalf = (kGeluLutExpHi - kGeluLutExpLo + 1) * 128;
constexpr int kGeluLutEntries = 2 * kGeluLutHalf;     // 3584
constexpr int kGeluLutBytes = 2 * kGeluLutEntries;    // 7168

// bf16 input pattern of table entry i
__device__ __forceinline__ uint32_t gelu_lut_input(int i)
{
    const uint32_t sign = i >= kGeluLutHalf ? 1u : 0u;
    const uint32_t r = static_cast<uint32_t>(i) - sign * kGeluLutHalf;
    return (sign << 15) | ((kGeluLutExpLo + (r >> 7)) << 7) | (r & 127u);
}


// The table, built once per device by gelu_lut_build_kernel (the library launches it, and
// waits for it, on the first call that needs it), then copied into each GEMM CTA's shared
// memory. Keeping the exact evaluation out of the GEMM kernels keeps their register
// allocation to what the epilogue needs.
__device__ __align__(16) uint16_t g_gelu_lut[kGeluLutEntries];

__global__ void gelu_lut_build_kernel()
{
    const int i = static_cast<int>(blockIdx.x * blockDim.x + threadIdx.x);
    if (i < kGeluLutEntries)
        g_gelu_lut[i] = static_cast<uint16_t>(gelu_bf16_bits(gelu_lut_input(i)));
}

// Copies the table into shared memory with `nthreads` threads of index `t` (16 bytes each);
// the caller synchronises those threads before the first lookup.
__device__ __forceinline__ void gelu_lut_load(uint16_t *lut, int t, int nthreads)
{
    const uint4 *src = reinterpret_cast<const uint4 *>(g_gelu_lut);
    uint4 *dst = reinterpret_cast<uint4 *>(lut);
    for (int i = t; i < kGeluLutBytes / 16; i += nthreads)
        dst[i] = src[i];
}


// Table-form GELU of the 16 bf16 patterns packed in w[8] (two per word), in place; `lut`
// is the table in shared memory. The hot path is only the index, one table load and an
// out-of-table flag per value, all independent so that the loads are in flight together;
// the closed forms of the other inputs (tiny and subnormal: x/2 rounded half to even;
// |x| >= 16: x or -0; zero; Inf, NaN) run only for a group of 16 that holds such a value.
__device__ __forceinline__ void gelu_bf16x16_lut(uint32_t *w, const uint16_t *lut)
{
    constexpr uint32_t kLo = static_cast<uint32_t>(kGeluLutExpLo) << 7;   // first magnitude
    uint32_t r[16];
    bool out = false;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const uint32_t b = (k & 1) ? (w[k >> 1] >> 16) : (w[k >> 1] & 0xffffu);
        const uint32_t d = (b & 0x7fffu) - kLo;            // offset inside the table's half
        const bool in_tab = d < static_cast<uint32_t>(kGeluLutHalf);
        const uint32_t i = d + (b >> 15) * static_cast<uint32_t>(kGeluLutHalf);
        r[k] = lut[in_tab ? i : 0u];
        out |= !in_tab;
    }
    if (out) {
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const uint32_t b = (k & 1) ? (w[k >> 1] >> 16) : (w[k >> 1] & 0xffffu);
            const uint32_t e = (b >> 7) & 0xffu;
            const uint32_t sign = b >> 15;
            if (e - kGeluLutExpLo <= static_cast<uint32_t>(kGeluLutExpHi - kGeluLutExpLo))
                continue;   // in the table
            if (e == 255u) {           // +Inf -> +Inf; -Inf (-inf * 0) and NaN -> NaN
                r[k] = ((b & 127u) != 0u || sign) ? 0x7fc0u : 0x7f80u;
            } else if (e < 2u) {
                // |x| < 2^-125: Phi(x) is 0.5 to far below the precision, GELU(x) = x / 2
                // rounded half to even on the subnormal grid (n * 2^-133, n = b & 0x7fff)
                const uint32_t n = b & 0x7fffu, h = n >> 1;
                r[k] = (b & 0x8000u) | (h + (n & h & 1u));
            } else {   // x >= 16 -> x, x <= -16 -> -0, tiny normal -> x/2
                r[k] = e > kGeluLutExpHi ? (sign ? 0x8000u : b) : b - 0x80u;
            }
        }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k)
        w[k] = r[2 * k] | (r[2 * k + 1] << 16);
}

struct GeluParams {
    const uint16_t *in;
    uint16_t *out;
    int64_t M, N, ld_in, ld_out;
    int64_t vecs_per_row;  // ceil(N / 8)
};

__global__ void __launch_bounds__(256) gelu_kernel(const GeluParams p)
{
    const int64_t total = p.M * p.vecs_per_row;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t row = i / p.vecs_per_row;
        const int64_t col = (i - row * p.vecs_per_row) * 8;
        const uint16_t *src = p.in + row * p.ld_in + col;
        uint16_t *dst = p.out + row * p.ld_out + col;
        if (col + 8 <= p.N) {
            const uint4 r = *reinterpret_cast<const uint4 *>(src);
            const uint32_t w[4] = {r.x, r.y, r.z, r.w};
            uint32_t o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                o[j] = gelu_bf16_bits(w[j] & 0xffffu) | (gelu_bf16_bits(w[j] >> 16) << 16);
            st_v4(dst, o[0], o[1], o[2], o[3]);
        } else {
            for (int64_t j = 0; col + j < p.N; ++j)
                dst[j] = static_cast<uint16_t>(gelu_bf16_bits(src[j]));
        }
    }
}

} // namespace sdnq
