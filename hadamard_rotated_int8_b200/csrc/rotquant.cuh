// Fused online rotate + quantize: per row (token or weight row), a block-diagonal
// Walsh-Hadamard butterfly over groups of G columns, the full-row absmax, the fp32 scale and
// round-half-to-even int8 codes, in one pass over HBM. With G = 1 and a column multiplier
// (COLSCALE) the same kernels quantize dy * sW per token for the input gradient of the frozen
// base (no rotation on that operand); with FP8 they write e4m3 codes on the +-448 grid.
// The kernels let the next kernel in the stream launch at once (griddepcontrol), which waits
// for their completion before it reads their codes and scales.
//
// Sources: "SDNQ: SD.Next Quantization Engine" README (Hadamard rotations on both the
// quantized weights and the quantized matmul; row-wise scales, FP32 de-quant); "ConvRot /
// Hadamard SDNQ" (group 256 = ConvRot, smaller = QuaRot-style); "Hybrid-Sensitivity-
// Weighted-Quantization" README, Rigorous grid / pack simulation (rotate, then absmax onto
// the symmetric int8 grid).
//
// Work mapping. A row is cut into chunks of 1024 elements; one warp owns one chunk at a
// time. Lane l = (hi2, lo3) with lo3 = l & 7 and hi2 = l >> 3; the lane holds four 16-byte
// vectors v = 0..3, each of 8 consecutive bf16. Element index inside the chunk:
//     e = hi2*256 + v*64 + lo3*8 + i          (i = 0..7 inside the vector)
// so for a fixed v the warp's 32 loads cover four fully used 128-byte lines. For a
// 256-group the butterfly bits map as: b0..b2 = i (in registers), b3..b5 = lo3 (lane
// shuffles), b6..b7 = v (in registers): three of the eight stages need a shuffle.
// Smaller groups use a prefix of the same bit order.
//
// Exactness. The butterfly runs its stages in ascending order h = 1, 2, ..., G/2, each
// element one IEEE fp32 add or subtract (packed two at a time with the f32x2 instructions,
// which round each lane like the scalar ones). A shuffle stage computes fma(self, +-1,
// partner), the single rounding of partner +- self. The codes use the exact IEEE quotient
// z / s_z (see quant8), so they are those of round_half_even(fp32(z / s_z)).
#pragma once

#include "device.cuh"

namespace sdnq {

struct RotquantParams {  // shared by both rotate+quantize kernels
    const uint16_t *x;   // [M, K] bf16 patterns, row stride ldx
    int64_t ldx;
    int8_t *q;           // [M, K] dense
    float *s;            // [M]
    int64_t M;
    int32_t K;
    int32_t nchunks;     // ceil(K / 1024)
    int32_t wpr;         // warps per row
    int32_t rpc;         // rows per CTA
    float c_g;           // fp32(1/sqrt(G)); 1 without rotation
    const float *colscale;  // [K] column multipliers, or nullptr
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4 r, float (&f)[8])
{
    f[0] = __uint_as_float(r.x << 16);
    f[1] = __uint_as_float(r.x & 0xffff0000u);
    f[2] = __uint_as_float(r.y << 16);
    f[3] = __uint_as_float(r.y & 0xffff0000u);
    f[4] = __uint_as_float(r.z << 16);
    f[5] = __uint_as_float(r.z & 0xffff0000u);
    f[6] = __uint_as_float(r.w << 16);
    f[7] = __uint_as_float(r.w & 0xffff0000u);
}

// Butterfly pair (a, b) -> (a + b, a - b) on two adjacent pairs at once.
__device__ __forceinline__ void bfly2(float &a0, float &a1, float &b0, float &b1)
{
    float s0, s1, d0, d1;
    add2(s0, s1, a0, a1, b0, b1);
    sub2(d0, d1, a0, a1, b0, b1);
    a0 = s0; a1 = s1; b0 = d0; b1 = d1;
}

// Unnormalised butterfly of the G-groups held by one warp (one chunk, 32 values per lane).
template <int G>
__device__ __forceinline__ void chunk_butterfly(float (&v)[4][8], uint32_t lane)
{
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        // stage h = 1: the two halves of each loaded 32-bit word
        if (G > 1) {
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                const float a = v[t][i], b = v[t][i + 1];
                v[t][i] = __fadd_rn(a, b);
                v[t][i + 1] = __fsub_rn(a, b);
            }
        }
        // stage h = 2: (0,1)+-(2,3), (4,5)+-(6,7)
        if (G > 2) {
            bfly2(v[t][0], v[t][1], v[t][2], v[t][3]);
            bfly2(v[t][4], v[t][5], v[t][6], v[t][7]);
        }
        // stage h = 4: (0,1)+-(4,5), (2,3)+-(6,7)
        if (G > 4) {
            bfly2(v[t][0], v[t][1], v[t][4], v[t][5]);
            bfly2(v[t][2], v[t][3], v[t][6], v[t][7]);
        }
    }
    // stages h = 8, 16, 32: across lanes lo3 ^ 1, ^ 2, ^ 4; fma(self, +-1, partner)
#pragma unroll
    for (int sb = 0; sb < 3; ++sb) {
        if (G > (8 << sb)) {
            const float sgn = ((lane >> sb) & 1u) ? -1.0f : 1.0f;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
#pragma unroll
                for (int i = 0; i < 8; i += 2) {
                    const float p0 = __shfl_xor_sync(0xffffffffu, v[t][i], 1 << sb);
                    const float p1 = __shfl_xor_sync(0xffffffffu, v[t][i + 1], 1 << sb);
                    fma2(v[t][i], v[t][i + 1], v[t][i], v[t][i + 1], sgn, sgn, p0, p1);
                }
            }
        }
    }
    // stages h = 64, 128: across the lane's vectors (v ^ 1, v ^ 2)
#pragma unroll
    for (int vb = 1; vb <= 2; vb <<= 1) {
        if (G > (32 << vb)) {
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                if ((t & vb) == 0) {
#pragma unroll
                    for (int i = 0; i < 8; i += 2)
                        bfly2(v[t][i], v[t][i + 1], v[t + vb][i], v[t + vb][i + 1]);
                }
            }
        }
    }
}

__device__ __forceinline__ void load_chunk(const uint16_t *xr, int32_t K, int32_t c, bool ok,
                                           uint32_t lane, float (&v)[4][8])
{
    const int32_t base = c * 1024 + static_cast<int32_t>(lane >> 3) * 256 +
                         static_cast<int32_t>(lane & 7u) * 8;
    uint4 raw[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int32_t e = base + t * 64;
        raw[t] = make_uint4(0u, 0u, 0u, 0u);
        if (ok && e < K)
            raw[t] = ld_nc_v4(xr + e);
    }
#pragma unroll
    for (int t = 0; t < 4; ++t)
        bf16x8_to_f32(raw[t], v[t]);
}

// The column multipliers of the lane's 32 values of chunk c (0 past the row end).
__device__ __forceinline__ void load_colscale(float (&m)[4][8], const float *cs, int32_t K,
                                              int32_t c, uint32_t lane)
{
    const int32_t base = c * 1024 + static_cast<int32_t>(lane >> 3) * 256 +
                         static_cast<int32_t>(lane & 7u) * 8;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int32_t e = base + t * 64;
        uint4 a = make_uint4(0u, 0u, 0u, 0u), b = make_uint4(0u, 0u, 0u, 0u);
        if (e < K) {
            a = ld_nc_v4(cs + e);
            b = ld_nc_v4(cs + e + 4);
        }
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
            m[t][i] = __uint_as_float(w[i]);
    }
}

// v *= m elementwise (one fp32 rounding each; the products feed no addition, so the pairs
// cannot be merged into a multiply-add).
__device__ __forceinline__ void mul_colscale(float (&v)[4][8], const float (&m)[4][8])
{
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
        for (int i = 0; i < 8; i += 2)
            mul2(v[t][i], v[t][i + 1], v[t][i], v[t][i + 1], m[t][i], m[t][i + 1]);
}

// v *= colscale[column] for the lane's 32 values of chunk c.
__device__ __forceinline__ void apply_colscale(float (&v)[4][8], const float *cs, int32_t K,
                                               int32_t c, uint32_t lane)
{
    const int32_t base = c * 1024 + static_cast<int32_t>(lane >> 3) * 256 +
                         static_cast<int32_t>(lane & 7u) * 8;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int32_t e = base + t * 64;
        uint4 a = make_uint4(0u, 0u, 0u, 0u), b = make_uint4(0u, 0u, 0u, 0u);
        if (e < K) {
            a = ld_nc_v4(cs + e);
            b = ld_nc_v4(cs + e + 4);
        }
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 8; i += 2)
            mul2(v[t][i], v[t][i + 1], v[t][i], v[t][i + 1], __uint_as_float(w[i]),
                 __uint_as_float(w[i + 1]));
    }
}

__device__ __forceinline__ float chunk_absmax(const float (&v)[4][8])
{
    float m = 0.0f;
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
        for (int i = 0; i < 8; ++i)
            m = fmaxf(m, fabsf(v[t][i]));
    return m;
}

__device__ __forceinline__ uint32_t pack4(uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    return __byte_perm(__byte_perm(a, b, 0x0040u), __byte_perm(c, d, 0x0040u), 0x5410u);
}

// The exact path for one vector of 8 values: IEEE fp32 quotient, half-to-even, clamp.
__device__ __noinline__ uint2 quant8_exact(float z0, float z1, float z2, float z3, float z4,
                                           float z5, float z6, float z7, float s_z)
{
    const float z[8] = {z0, z1, z2, z3, z4, z5, z6, z7};
    uint32_t c[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float t = __fdiv_rn(z[i], s_z);
        const float r = fminf(fmaxf(rintf(t), -127.0f), 127.0f);
        c[i] = (t == t) ? static_cast<uint32_t>(__float2int_rn(r)) : 0u;
    }
    return make_uint2(pack4(c[0], c[1], c[2], c[3]), pack4(c[4], c[5], c[6], c[7]));
}

// Codes of one vector of 8 values. The IEEE quotient Q = RN(z / s_z) is obtained without a
// division by Markstein's correction (P. Markstein, "Computation of elementary functions on
// the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990): with y = RN(1/s_z) and
// q0 = RN(z * y), the residual r = z - q0 * s_z is exact in one fused multiply-add and
// RN(q0 + r * y) = RN(z / s_z). Q is then rounded half-to-even to an integer by adding
// 1.5 * 2^23 (|Q| <= 127.5, so the integer lands in the low mantissa bits). Needs s_z normal;
// otherwise (a row whose scale is subnormal) the IEEE division is used.
__device__ __forceinline__ uint2 quant8(const float (&z)[8], float s_z, float rcp, bool fast)
{
    if (!fast)  // warp-uniform: s_z is the row's scale
        return quant8_exact(z[0], z[1], z[2], z[3], z[4], z[5], z[6], z[7], s_z);
    constexpr float MAGIC = 12582912.0f;  // 1.5 * 2^23
    const float neg_s = -s_z;
    float f[8];
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        float q0, q1, r0, r1, c0, c1;
        mul2(q0, q1, z[i], z[i + 1], rcp, rcp);             // q = RN(z * y)
        fma2(r0, r1, q0, q1, neg_s, neg_s, z[i], z[i + 1]);  // r = z - q * s_z, exact
        fma2(c0, c1, r0, r1, rcp, rcp, q0, q1);              // Q = RN(q + r * y)
        add2(f[i], f[i + 1], c0, c1, MAGIC, MAGIC);          // M + rne(Q)
    }
    // the low byte of f is the code in two's complement
    return make_uint2(pack4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                            __float_as_uint(f[3])),
                      pack4(__float_as_uint(f[4]), __float_as_uint(f[5]), __float_as_uint(f[6]),
                            __float_as_uint(f[7])));
}

// The row scale s_z = RN(amax / D) for the grid's largest code D (127 for int8, 448 for
// e4m3), without a division: with y = RN(1 / D) and q0 = RN(amax * y), the residual
// amax - q0 * D is exact in one fused multiply-add and RN(q0 + r * y) is the IEEE quotient
// (Markstein's correction, as in quant8; checked on every fp32 input of two binades, which
// covers all inputs whose intermediates stay normal). Tiny maxima take the IEEE division.
template <int D>
__device__ __forceinline__ float div_by_grid(float amax)
{
    static_assert(D == 127 || D == 448, "the int8 and e4m3 grids");
    if (!(amax >= 0x1p-100f))
        return __fdiv_rn(amax, static_cast<float>(D));
    // RN(1 / D): 0x3c010204 for 127, 0x3b124925 for 448
    const float y = __uint_as_float(D == 127 ? 0x3c010204u : 0x3b124925u);
    const float q0 = __fmul_rn(amax, y);
    const float r = __fmaf_rn(-q0, static_cast<float>(D), amax);
    return __fmaf_rn(r, y, q0);
}

// e4m3 codes of two fp32 values (round to nearest even, saturating at +-448), low byte = lo
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi)
{
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
    return d;
}

__device__ __noinline__ uint2 quant8_e4m3_exact(float z0, float z1, float z2, float z3, float z4,
                                                float z5, float z6, float z7, float s_z)
{
    const float t[8] = {__fdiv_rn(z0, s_z), __fdiv_rn(z1, s_z), __fdiv_rn(z2, s_z),
                        __fdiv_rn(z3, s_z), __fdiv_rn(z4, s_z), __fdiv_rn(z5, s_z),
                        __fdiv_rn(z6, s_z), __fdiv_rn(z7, s_z)};
    return make_uint2(e4m3x2(t[0], t[1]) | (e4m3x2(t[2], t[3]) << 16),
                      e4m3x2(t[4], t[5]) | (e4m3x2(t[6], t[7]) << 16));
}

// e4m3 codes of one vector of 8 values: the IEEE quotient RN(z / s_z) by the same Markstein
// correction as quant8, then one rounding to e4m3.
__device__ __forceinline__ uint2 quant8_e4m3(const float (&z)[8], float s_z, float rcp, bool fast)
{
    if (!fast)
        return quant8_e4m3_exact(z[0], z[1], z[2], z[3], z[4], z[5], z[6], z[7], s_z);
    const float neg_s = -s_z;
    float c[8];
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        float q0, q1, r0, r1;
        mul2(q0, q1, z[i], z[i + 1], rcp, rcp);
        fma2(r0, r1, q0, q1, neg_s, neg_s, z[i], z[i + 1]);
        fma2(c[i], c[i + 1], r0, r1, rcp, rcp, q0, q1);
    }
    return make_uint2(e4m3x2(c[0], c[1]) | (e4m3x2(c[2], c[3]) << 16),
                      e4m3x2(c[4], c[5]) | (e4m3x2(c[6], c[7]) << 16));
}

template <bool FP8 = false>
__device__ __forceinline__ void quant_store_chunk(const float (&v)[4][8], int8_t *qr, int32_t K,
                                                  int32_t c, bool ok, uint32_t lane, float s_z,
                                                  bool zero)
{
    const bool fast = s_z >= 0x1p-126f;
    const float rcp = __frcp_rn(s_z);
    const int32_t base = c * 1024 + static_cast<int32_t>(lane >> 3) * 256 +
                         static_cast<int32_t>(lane & 7u) * 8;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int32_t e = base + t * 64;
        uint2 w = make_uint2(0u, 0u);
        if (!zero)  // warp-uniform: the whole warp works on one row
            w = FP8 ? quant8_e4m3(v[t], s_z, rcp, fast) : quant8(v[t], s_z, rcp, fast);
        if (ok && e < K)
            st_v2(qr + e, w.x, w.y);
    }
}

__device__ __forceinline__ void load_raw(const uint16_t *xr, int32_t K, int32_t c, bool ok,
                                         uint32_t lane, uint4 (&raw)[4])
{
    const int32_t base = c * 1024 + static_cast<int32_t>(lane >> 3) * 256 +
                         static_cast<int32_t>(lane & 7u) * 8;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int32_t e = base + t * 64;
        raw[t] = make_uint4(0u, 0u, 0u, 0u);
        if (ok && e < K)
            raw[t] = ld_nc_v4(xr + e);
    }
}

// The persistent loop below run by `nw` warps inside another kernel (the fused activation
// quantizer of the int8 GEMM): warp w of the group is `warp`, the group synchronises on named
// barrier `bar_id` (32 * nw threads) and exchanges row maxima through s_amax[2][nw] in shared
// memory. Warps beyond wpr * rpc only take part in the barriers. Rows are published per
// 128-row block: ready[b] counts wpr per stored row of block b (a row group never straddles
// a block, since rpc divides 128). One lane of the group's last warp adds a whole row group
// with release semantics once the next barrier shows every warp past its stores, so that one
// thread, not every warp, waits on the release.
template <int G>
__device__ __forceinline__ void rotquant_worker_rows(const RotquantParams &p, int32_t warp,
                                                     int32_t nw, uint32_t bar_id, float *s_amax,
                                                     uint32_t *ready)
{
    const uint32_t lane = lane_id();
    const int32_t r_local = warp / p.wpr;
    const int32_t wr = warp - r_local * p.wpr;
    const bool active = r_local < p.rpc;
    const bool has_chunk = active && wr < p.nchunks;
    const int64_t n_groups = (p.M + p.rpc - 1) / p.rpc;
    const bool signaller = warp == nw - 1 && lane == 0;
    auto publish = [&](int64_t group) {
        const int64_t r0 = group * p.rpc;
        const int64_t rows = p.M - r0 < p.rpc ? p.M - r0 : p.rpc;
        red_add_release_gpu(ready + (r0 >> 7), static_cast<uint32_t>(rows * p.wpr));
    };

    int64_t rg = blockIdx.x;
    int64_t prev = -1;  // row group stored in the previous iteration, not yet published
    uint4 raw[4];
    {
        const int64_t row = rg * p.rpc + r_local;
        const bool ok = rg < n_groups && row < p.M && has_chunk;
        load_raw(p.x + (ok ? row : 0) * p.ldx, p.K, wr, ok, lane, raw);
    }
    for (int parity = 0; rg < n_groups; rg += gridDim.x, parity ^= 1) {
        const int64_t row = rg * p.rpc + r_local;
        const bool row_ok = active && row < p.M;
        float v[4][8];
#pragma unroll
        for (int t = 0; t < 4; ++t)
            bf16x8_to_f32(raw[t], v[t]);
        {
            const int64_t nrg = rg + gridDim.x;
            const int64_t nrow = nrg * p.rpc + r_local;
            const bool ok = nrg < n_groups && nrow < p.M && has_chunk;
            load_raw(p.x + (ok ? nrow : 0) * p.ldx, p.K, wr, ok, lane, raw);
        }
        chunk_butterfly<G>(v, lane);
        float amax = chunk_absmax(v);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        if (lane == 0)
            s_amax[parity * nw + warp] = amax;
        asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(32 * nw) : "memory");
        if (signaller && prev >= 0)
            publish(prev);  // every warp is past the stores of row group `prev`
        amax = 0.0f;
        if (active)
            for (int32_t w = 0; w < p.wpr; ++w)
                amax = fmaxf(amax, s_amax[parity * nw + r_local * p.wpr + w]);
        const float s_z = __fdiv_rn(amax, 127.0f);
        const bool zero = !(amax > 0.0f);
        if (row_ok && wr == 0 && lane == 0)
            p.s[row] = zero ? 0.0f : __fmul_rn(s_z, p.c_g);
        int8_t *qr = p.q + (row_ok ? row : 0) * static_cast<int64_t>(p.K);
        quant_store_chunk(v, qr, p.K, wr, row_ok && has_chunk, lane, s_z, zero);
        prev = rg;
    }
    asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(32 * nw) : "memory");
    if (signaller && prev >= 0)
        publish(prev);
}

// Rows of at most 16 chunks (K <= 16384): each warp owns one chunk of a row, a CTA owns
// `rpc` rows at a time and walks row groups persistently, loading the next row group into
// registers while it rotates and quantizes the current one.
template <int G, bool COLSCALE, bool FP8 = false>
__global__ void __launch_bounds__(512) rotquant_persistent_kernel(const RotquantParams p)
{
    grid_dependents_launch();
    __shared__ float s_amax[2][32];
    const uint32_t lane = lane_id();
    const int32_t warp = static_cast<int32_t>(threadIdx.x >> 5);
    const int32_t r_local = warp / p.wpr;
    const int32_t wr = warp - r_local * p.wpr;   // this warp's chunk of the row
    const bool has_chunk = wr < p.nchunks;
    const int64_t n_groups = (p.M + p.rpc - 1) / p.rpc;

    // a warp keeps one chunk of every row it visits: its column multipliers stay in registers
    float cmul[COLSCALE ? 4 : 1][8];
    if constexpr (COLSCALE)
        load_colscale(cmul, p.colscale, p.K, has_chunk ? wr : p.nchunks, lane);  // zeros if none
    int64_t rg = blockIdx.x;
    uint4 raw[4];
    {
        const int64_t row = rg * p.rpc + r_local;
        const bool ok = rg < n_groups && row < p.M && has_chunk;
        load_raw(p.x + (ok ? row : 0) * p.ldx, p.K, wr, ok, lane, raw);
    }
    for (int parity = 0; rg < n_groups; rg += gridDim.x, parity ^= 1) {
        const int64_t row = rg * p.rpc + r_local;
        const bool row_ok = row < p.M;
        float v[4][8];
#pragma unroll
        for (int t = 0; t < 4; ++t)
            bf16x8_to_f32(raw[t], v[t]);
        {   // prefetch the next row group while this one is computed
            const int64_t nrg = rg + gridDim.x;
            const int64_t nrow = nrg * p.rpc + r_local;
            const bool ok = nrg < n_groups && nrow < p.M && has_chunk;
            load_raw(p.x + (ok ? nrow : 0) * p.ldx, p.K, wr, ok, lane, raw);
        }
        if constexpr (COLSCALE)
            mul_colscale(v, cmul);
        chunk_butterfly<G>(v, lane);
        float amax = chunk_absmax(v);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        if (lane == 0)
            s_amax[parity][warp] = amax;
        __syncthreads();  // one barrier per row group: s_amax is double-buffered
        amax = 0.0f;
        for (int32_t w = 0; w < p.wpr; ++w)
            amax = fmaxf(amax, s_amax[parity][r_local * p.wpr + w]);
        const float s_z = __fdiv_rn(amax, FP8 ? 448.0f : 127.0f);  // grid: +-127 or +-448
        const bool zero = !(amax > 0.0f);
        if (row_ok && wr == 0 && lane == 0)
            p.s[row] = zero ? 0.0f : __fmul_rn(s_z, p.c_g);
        int8_t *qr = p.q + (row_ok ? row : 0) * static_cast<int64_t>(p.K);
        quant_store_chunk<FP8>(v, qr, p.K, wr, row_ok && has_chunk, lane, s_z, zero);
    }
}

template <int G, bool COLSCALE, bool FP8 = false>
__global__ void __launch_bounds__(512) rotquant_kernel(const RotquantParams p)
{
    grid_dependents_launch();
    __shared__ float s_amax[32];
    const uint32_t lane = lane_id();
    const int32_t warp = static_cast<int32_t>(threadIdx.x >> 5);
    const int32_t r_local = warp / p.wpr;
    const int32_t wr = warp - r_local * p.wpr;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * p.rpc + r_local;
    const bool row_ok = row < p.M;
    const uint16_t *xr = p.x + (row_ok ? row : 0) * p.ldx;
    int8_t *qr = p.q + (row_ok ? row : 0) * static_cast<int64_t>(p.K);

    // chunks of this warp: wr, wr + wpr, ...
    const int32_t my_chunks = (wr < p.nchunks) ? (p.nchunks - 1 - wr) / p.wpr + 1 : 0;
    const bool single = my_chunks <= 1;

    float v[4][8];
    float amax = 0.0f;
    if (single) {
        load_chunk(xr, p.K, wr, row_ok && my_chunks == 1, lane, v);
        if (COLSCALE && my_chunks == 1)
            apply_colscale(v, p.colscale, p.K, wr, lane);
        chunk_butterfly<G>(v, lane);
        amax = chunk_absmax(v);
    } else {
        // long rows: first pass for the absmax only; the second pass recomputes the
        // rotation (the row is then read from L2)
        for (int32_t j = 0; j < my_chunks; ++j) {
            load_chunk(xr, p.K, wr + j * p.wpr, row_ok, lane, v);
            if (COLSCALE)
                apply_colscale(v, p.colscale, p.K, wr + j * p.wpr, lane);
            chunk_butterfly<G>(v, lane);
            amax = fmaxf(amax, chunk_absmax(v));
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (lane == 0)
        s_amax[warp] = amax;
    __syncthreads();
    amax = 0.0f;
    for (int32_t w = 0; w < p.wpr; ++w)
        amax = fmaxf(amax, s_amax[r_local * p.wpr + w]);

    const float s_z = __fdiv_rn(amax, FP8 ? 448.0f : 127.0f);
    const bool zero = !(amax > 0.0f);
    if (row_ok && wr == 0 && lane == 0)
        p.s[row] = zero ? 0.0f : __fmul_rn(s_z, p.c_g);

    if (single) {
        quant_store_chunk<FP8>(v, qr, p.K, wr, row_ok && my_chunks == 1, lane, s_z, zero);
    } else {
        for (int32_t j = 0; j < my_chunks; ++j) {
            load_chunk(xr, p.K, wr + j * p.wpr, row_ok, lane, v);
            if (COLSCALE)
                apply_colscale(v, p.colscale, p.K, wr + j * p.wpr, lane);
            chunk_butterfly<G>(v, lane);
            quant_store_chunk<FP8>(v, qr, p.K, wr + j * p.wpr, row_ok, lane, s_z, zero);
        }
    }
}

// ---------------------------------------------------------------------------------------
// Run-per-lane rotate + quantize (rows up to 32768 elements).
//
// Each lane owns one run of 64 consecutive elements of a row, loaded as four 32-byte pieces
// (one full sector each), so that the butterfly stages h = 1 .. 32 run in its registers.
// For groups of 128 and 256 the remaining stages (h = 64, 128) cross the runs of a group,
// which sit on the group's G / 64 neighbouring lanes: the lanes swap their values through a
// padded shared-memory buffer (one store and one load of 16 bytes per 4 values) so that
// each lane then holds, for every run of its group, one contiguous piece of 64 / (G / 64)
// elements, and those stages run in registers too. The buffer keeps owner o's slot s (four
// fp32 values) at 16-byte unit o * 17 + Pc * (s % spp) + s / spp, with Pc = G / 64 lanes per
// group and spp = 16 / Pc slots per piece: both the stores (fixed s, consecutive owners) and
// the loads (fixed run and slot, consecutive lanes) hit eight different bank groups per
// quarter warp, and both are a lane base plus a compile-time offset.
//
// A block holds `rows` rows of runs per iteration (slot = row_local * rpr + run for its
// threads), walks the row blocks persistently and loads the next block's runs into
// registers while it rotates and quantizes the current one. The row maximum combines the
// lanes of a row inside each warp (segmented shuffle), then across warps with one shared
// atomic max per warp segment and one block barrier per iteration; the three row-maximum
// buffers rotate so that resetting one never races with the iterations around it.
struct RotquantRunParams {
    const uint16_t *x;   // [M, K] bf16 patterns, row stride ldx
    int64_t ldx;
    int8_t *q;           // [M, K] dense
    float *s;            // [M]
    int64_t M;
    int32_t K;
    int32_t rpr;         // runs of 64 elements per row, ceil(K / 64)
    int32_t rows;        // rows per block iteration
    float c_g;           // fp32(1 / sqrt(G))
};

__device__ __forceinline__ void ld_nc_v8(const void *ptr, uint32_t *r)
{
    asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "l"(ptr));
}

__device__ __forceinline__ void ld_nc_v4_l1(const void *ptr, uint32_t *r)
{
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "l"(ptr));
}

// The lane's run of 64 elements (4 pieces of 16; a piece past the row end reads zeros).
// V8: one 32-byte load per piece (row start 32-byte aligned); otherwise two 16-byte loads
// through L1, so that the second half of each sector is served from there.
template <bool V8>
__device__ __forceinline__ void load_run(const uint16_t *xr, int32_t e0, int32_t K, bool ok,
                                         uint32_t (&raw)[32])
{
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int32_t e = e0 + 16 * t;
        if (ok && e < K) {
            if constexpr (V8) {
                ld_nc_v8(xr + e, raw + 8 * t);
            } else {
                ld_nc_v4_l1(xr + e, raw + 8 * t);
                ld_nc_v4_l1(xr + e + 8, raw + 8 * t + 4);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                raw[8 * t + i] = 0u;
        }
    }
}

// fmax of m and the magnitudes of a and b, one three-input maximum
__device__ __forceinline__ float max3_abs(float m, float a, float b)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(m), "f"(fabsf(a)), "f"(fabsf(b)));
    return d;
}

// Butterfly stages h = 1 .. min(G, 64) / 2 over the run's 64 consecutive values. Stage 1
// pairs the two halves of each register pair (scalar); the later stages pair registers
// pairwise (f32x2, two lanes of IEEE fp32 per instruction).
template <int G>
__device__ __forceinline__ void run_butterfly(float (&v)[64])
{
    if (G > 1) {
#pragma unroll
        for (int i = 0; i < 64; i += 2) {
            const float a = v[i], b = v[i + 1];
            v[i] = __fadd_rn(a, b);
            v[i + 1] = __fsub_rn(a, b);
        }
    }
#pragma unroll
    for (int h = 2; h < 64 && h < G; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 64; i += 2)
            if ((i & h) == 0)
                bfly2(v[i], v[i + 1], v[i + h], v[i + h + 1]);
    }
}

template <int G, bool FP8, bool V8>
__global__ void __launch_bounds__(512) rotquant_run_kernel(const RotquantRunParams p)
{
    grid_dependents_launch();
    constexpr int PC = G >= 128 ? G / 64 : 1;   // lanes (runs) per group in the transposed stages
    constexpr int PIECE = 64 / PC;              // elements of each run a lane holds afterwards
    extern __shared__ __align__(16) uint8_t rq_smem[];
    const int32_t nwarps = static_cast<int32_t>(blockDim.x >> 5);
    uint32_t *s_max = reinterpret_cast<uint32_t *>(rq_smem + (G >= 128 ? nwarps * 32 * 272 : 0));
    const uint32_t lane = lane_id();
    const int32_t warp = static_cast<int32_t>(threadIdx.x >> 5);
    const int32_t slot = static_cast<int32_t>(threadIdx.x);
    const int32_t row_local = slot / p.rpr;
    const int32_t run = slot - row_local * p.rpr;
    const bool active = row_local < p.rows;
    const int32_t e0 = run * 64;
    const int64_t n_blocks = (p.M + p.rows - 1) / p.rows;

    // segmented maximum over the lanes of this lane's row inside the warp: step d takes
    // lane + d's value when that lane holds the same row
    const int32_t row_end = (row_local + 1) * p.rpr;   // first slot of the next row
    const bool seg_first = active && (lane == 0u || run == 0);
    for (int32_t i = slot; i < 3 * p.rows; i += static_cast<int32_t>(blockDim.x))
        s_max[i] = 0u;
    __syncthreads();

    // transposition buffer of this warp (groups of 128 and 256)
    const uint32_t tbuf = smem_u32(rq_smem) + static_cast<uint32_t>(warp) * (32u * 272u);
    const uint32_t t_wr = tbuf + lane * 272u;                          // owner = lane
    const uint32_t t_rd = tbuf + ((lane / PC) * PC * 17u + lane % PC) * 16u;
    const int32_t p_in_group = static_cast<int32_t>(lane % PC);
    const int32_t group_run0 = run - p_in_group;                       // first run of the group

    int64_t rb = blockIdx.x;
    uint32_t raw[32];
    {
        const int64_t row = rb * p.rows + row_local;
        const bool ok = rb < n_blocks && active && row < p.M;
        load_run<V8>(p.x + (ok ? row : 0) * p.ldx, e0, p.K, ok, raw);
    }
    for (int it = 0; rb < n_blocks; rb += gridDim.x, ++it) {
        const int64_t row = rb * p.rows + row_local;
        const bool row_ok = active && row < p.M;
        float v[64];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            v[2 * i] = __uint_as_float(raw[i] << 16);
            v[2 * i + 1] = __uint_as_float(raw[i] & 0xffff0000u);
        }
        {   // the next row block's runs, while this one is computed
            const int64_t nrb = rb + gridDim.x;
            const int64_t nrow = nrb * p.rows + row_local;
            const bool ok = nrb < n_blocks && active && nrow < p.M;
            load_run<V8>(p.x + (ok ? nrow : 0) * p.ldx, e0, p.K, ok, raw);
        }
        run_butterfly<G>(v);
        if constexpr (G >= 128) {
            // to the transposed layout: owner `lane` stores its 16 slots of four values
            constexpr int SPP = 16 / PC;
#pragma unroll
            for (int sl = 0; sl < 16; ++sl)
                sts_v4(t_wr + static_cast<uint32_t>(PC * (sl % SPP) + sl / SPP) * 16u,
                       __float_as_uint(v[4 * sl]), __float_as_uint(v[4 * sl + 1]),
                       __float_as_uint(v[4 * sl + 2]), __float_as_uint(v[4 * sl + 3]));
            __syncwarp();
            // v[j * PIECE + i] = element p_in_group * PIECE + i of run j of the group
#pragma unroll
            for (int j = 0; j < PC; ++j)
#pragma unroll
                for (int k = 0; k < SPP; ++k) {
                    const float4 f = lds_v4(t_rd + static_cast<uint32_t>(j * 17 + PC * k) * 16u);
                    v[j * PIECE + 4 * k] = f.x;
                    v[j * PIECE + 4 * k + 1] = f.y;
                    v[j * PIECE + 4 * k + 2] = f.z;
                    v[j * PIECE + 4 * k + 3] = f.w;
                }
            // stage h = 64 across runs j, j + 1; h = 128 across runs j, j + 2
#pragma unroll
            for (int d = 1; d < PC; d <<= 1)
#pragma unroll
                for (int j = 0; j < PC; ++j)
                    if ((j & d) == 0)
#pragma unroll
                        for (int i = 0; i < PIECE; i += 2)
                            bfly2(v[j * PIECE + i], v[j * PIECE + i + 1], v[(j + d) * PIECE + i],
                                  v[(j + d) * PIECE + i + 1]);
        }
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 64; i += 2)
            amax = max3_abs(amax, v[i], v[i + 1]);
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const float o = __shfl_down_sync(0xffffffffu, amax, d);
            if (static_cast<int32_t>(lane) + d < 32 && slot + d < row_end)
                amax = fmaxf(amax, o);
        }
        uint32_t *mx = s_max + (it % 3) * p.rows;
        if (seg_first)
            atomicMax(mx + row_local, __float_as_uint(amax));   // amax >= 0: bits order as values
        __syncthreads();
        if (slot < p.rows)
            s_max[((it + 2) % 3) * p.rows + slot] = 0u;          // the buffer of iteration it + 2
        amax = active ? __uint_as_float(mx[row_local]) : 0.0f;
        const float s_z = div_by_grid<FP8 ? 448 : 127>(amax);
        const bool zero = !(amax > 0.0f);
        if (row_ok && run == 0)
            p.s[row] = zero ? 0.0f : __fmul_rn(s_z, p.c_g);
        const bool fast = s_z >= 0x1p-126f;
        const float rcp = __frcp_rn(s_z);
        int8_t *qr = p.q + (row_ok ? row : 0) * static_cast<int64_t>(p.K);
        // codes of 16 consecutive values -> one 16-byte store
        auto store16 = [&](const float *z, int32_t e) {
            uint2 a = make_uint2(0u, 0u), b = make_uint2(0u, 0u);
            if (!zero) {
                const float za[8] = {z[0], z[1], z[2], z[3], z[4], z[5], z[6], z[7]};
                const float zb[8] = {z[8], z[9], z[10], z[11], z[12], z[13], z[14], z[15]};
                a = FP8 ? quant8_e4m3(za, s_z, rcp, fast) : quant8(za, s_z, rcp, fast);
                b = FP8 ? quant8_e4m3(zb, s_z, rcp, fast) : quant8(zb, s_z, rcp, fast);
            }
            if (row_ok && e < p.K)
                st_v4(qr + e, a.x, a.y, b.x, b.y);
        };
        if constexpr (G >= 128) {
#pragma unroll
            for (int j = 0; j < PC; ++j)
#pragma unroll
                for (int i = 0; i < PIECE; i += 16)
                    store16(v + j * PIECE + i, (group_run0 + j) * 64 + p_in_group * PIECE + i);
        } else {
#pragma unroll
            for (int t = 0; t < 4; ++t)
                store16(v + 16 * t, e0 + 16 * t);
        }
    }
}

} // namespace sdnq
