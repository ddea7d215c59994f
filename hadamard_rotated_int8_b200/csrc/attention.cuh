// Attention with a Hadamard-rotated int8 QK^T and a bf16 PV, on the 5th-generation tensor
// cores. Sources: "SDNQ: SD.Next Quantization Engine" README, SDNQ attention (an SDPA
// replacement with an int8 QK matmul, smooth_k, use_hadamard and hadamard_group_size, the PV
// matmul left unquantized); "ConvRot / Hadamard SDNQ" (group 256 = ConvRot).
//
// Q, K, V are [B][L][H][D] bf16 (D = 128): token-head rows of D contiguous values.
//   1. attn_ksum_kernel + attn_kmean_kernel: mu[b][h][d] = fp32(sum_j K[b][j][h][d] / Lk),
//      the sum in fp64 (smooth_k; subtracting mu from every key leaves the softmax unchanged).
//   2. attn_rowquant_kernel: Q rows, and K rows minus mu, rotated by the butterfly over groups
//      of min(g, D) and quantized per row to int8 as in the linear path (codes, scale
//      s = fp32(amax/127) * fp32(1/sqrt(G))); scales stored [B][H][L].
//   3. attn_kernel: one CTA per (b, h, 256 queries) = two 128-query tiles.
//      - warp 0 loads both Q tiles once, then rings of K codes, key scales and V through TMA;
//      - warp 1 issues S_t(j) = Q_t K_j^T (tcgen05 kind::i8, int32 in TMEM) and
//        O_t += P_t(j) V_j (kind::f16, bf16 P and V, fp32 O in TMEM) for both tiles;
//      - warps 2..5 (tile 0) and 6..9 (tile 1), one thread per query row, form base-2 logits
//        (acc * s_k) * (s_q * scale * log2 e) (a few fp32 roundings away from the oracle's
//        order), run an online softmax with ex2.approx (rescaling O and the row sum only when
//        the row maximum grows by more than 2^8, so P stays below 256), write P_t(j) as bf16
//        into a 128-byte-swizzled K-major tile, and finally write O / l as bf16. The two tiles
//        take turns at the exponentials.
// Every wait is bounded as in the GEMM kernel.
#pragma once

#include <cuda_bf16.h>

#include "device.cuh"
#include "rotquant.cuh"

namespace sdnq {

constexpr int kAttnD = 128;
constexpr int kAttnBlock = 128;        // queries per tile (two tiles per CTA) and keys per step
constexpr int kAttnSumSplits = 32;     // key splits of the channel sums

// ---------------------------------------------------------------- smooth_k channel means

// partial[(bh * splits + split) * D + d] = sum over this split's keys of K[b][j][h][d] (fp64)
__global__ void __launch_bounds__(256) attn_ksum_kernel(const uint16_t *k, int32_t Lk, int32_t H,
                                                        double *partial)
{
    grid_dependents_launch();
    grid_dependency_wait();   // launched programmatically: nothing is read or written before
    const int32_t bh = blockIdx.x, split = blockIdx.y;
    const int32_t b = bh / H, h = bh % H;
    const int32_t d8 = (threadIdx.x & 15) * 8;   // 16 threads cover the 128 channels
    const int32_t lane_row = threadIdx.x >> 4;   // 16 keys per pass
    const int32_t per = (Lk + kAttnSumSplits - 1) / kAttnSumSplits;
    const int32_t j0 = split * per, j1 = j0 + per < Lk ? j0 + per : Lk;
    // three keys in flight per thread (the fp64 sums of bf16 values are exact, so the order
    // of the additions does not matter)
    double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int32_t j = j0 + lane_row; j < j1; j += 48) {
        uint4 r[3];
#pragma unroll
        for (int u = 0; u < 3; ++u)
            r[u] = j + 16 * u < j1
                       ? ld_nc_v4(k + ((static_cast<int64_t>(b) * Lk + j + 16 * u) * H + h) * kAttnD + d8)
                       : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int u = 0; u < 3; ++u) {
            const uint32_t w[4] = {r[u].x, r[u].y, r[u].z, r[u].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                acc[2 * i] += static_cast<double>(__uint_as_float(w[i] << 16));
                acc[2 * i + 1] += static_cast<double>(__uint_as_float(w[i] & 0xffff0000u));
            }
        }
    }
    __shared__ double red[16][kAttnD];
#pragma unroll
    for (int i = 0; i < 8; ++i)
        red[lane_row][d8 + i] = acc[i];
    __syncthreads();
    if (threadIdx.x < kAttnD) {
        double s = 0.0;
        for (int r = 0; r < 16; ++r)
            s += red[r][threadIdx.x];
        partial[(static_cast<int64_t>(bh) * kAttnSumSplits + split) * kAttnD + threadIdx.x] = s;
    }
}

// mu[bh][d] = fp32(sum of the splits / Lk). The fp64 sums of bf16 values are exact when a
// channel spans less than 2^45 in magnitude, so the split order does not matter.
__global__ void attn_kmean_kernel(const double *partial, int32_t Lk, float *mu)
{
    grid_dependents_launch();
    grid_dependency_wait();
    const int32_t bh = blockIdx.x, d = threadIdx.x;
    double part[kAttnSumSplits];   // all loads in flight, then the sum
#pragma unroll
    for (int i = 0; i < kAttnSumSplits; ++i)
        part[i] = partial[(static_cast<int64_t>(bh) * kAttnSumSplits + i) * kAttnD + d];
    double s = 0.0;
#pragma unroll
    for (int i = 0; i < kAttnSumSplits; ++i)
        s += part[i];
    mu[static_cast<int64_t>(bh) * kAttnD + d] = static_cast<float>(s / static_cast<double>(Lk));
}

// ---------------------------------------------------------------- Q / K row quantizer

struct AttnQuantParams {
    const uint16_t *x;     // [B][L][H][D] bf16
    const float *mu;       // [B][H][D] or nullptr (queries)
    int8_t *q;             // [B][L][H][D]
    float *s;              // [B][H][ls]
    int64_t rows;          // B * L * H (below 2^31)
    int32_t L, H;
    int32_t ls;            // scale row stride: L rounded up to a multiple of 128
    float c_g;
};

// One warp per 1024-element chunk = 8 consecutive token-head rows of 128; the butterfly over
// groups of G <= 128 never crosses a row. Lane (hi2, lo3) holds rows 2 hi2 (t = 0, 1) and
// 2 hi2 + 1 (t = 2, 3) of the chunk; a row's maximum combines its 8 lanes by shuffles.
template <int G>
__global__ void __launch_bounds__(256, 4) attn_rowquant_kernel(const AttnQuantParams p)
{
    grid_dependents_launch();
    grid_dependency_wait();
    const uint32_t lane = lane_id();
    const int64_t nchunks = (p.rows + 7) / 8;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t c = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
         c < nchunks; c += warps) {
        const int64_t row0 = c * 8 + 2 * static_cast<int64_t>(lane >> 3);
        const int64_t base = c * 1024 + static_cast<int64_t>(lane >> 3) * 256 +
                             static_cast<int64_t>(lane & 7u) * 8;
        // (b, l, h) of the lane's two rows, in 32-bit arithmetic (rows < 2^31), once
        const uint32_t H = static_cast<uint32_t>(p.H), L = static_cast<uint32_t>(p.L);
        uint32_t hr[2], lr[2], br[2];
        {
            const uint32_t r0 = static_cast<uint32_t>(row0), t0 = r0 / H;
            hr[0] = r0 - t0 * H;
            br[0] = t0 / L;
            lr[0] = t0 - br[0] * L;
            hr[1] = hr[0] + 1u, lr[1] = lr[0], br[1] = br[0];
            if (hr[1] == H) {
                hr[1] = 0u;
                if (++lr[1] == L)
                    lr[1] = 0u, ++br[1];
            }
        }
        float v[4][8];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int64_t row = row0 + (t >> 1);
            uint4 r = make_uint4(0u, 0u, 0u, 0u);
            if (row < p.rows)
                r = ld_nc_v4(p.x + base + t * 64);
            bf16x8_to_f32(r, v[t]);
            if (p.mu != nullptr && row < p.rows) {
                const int64_t bh = static_cast<int64_t>(br[t >> 1]) * H + hr[t >> 1];
                const int32_t d = (t & 1) * 64 + static_cast<int32_t>(lane & 7u) * 8;
                const float *m = p.mu + bh * kAttnD + d;
                const uint4 a = ld_nc_v4(m), bb = ld_nc_v4(m + 4);
                const uint32_t w[8] = {a.x, a.y, a.z, a.w, bb.x, bb.y, bb.z, bb.w};
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    v[t][i] = __fsub_rn(v[t][i], __uint_as_float(w[i]));
            }
        }
        chunk_butterfly<G>(v, lane);
        float m0 = 0.0f, m1 = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            m0 = fmaxf(m0, fmaxf(fabsf(v[0][i]), fabsf(v[1][i])));
            m1 = fmaxf(m1, fmaxf(fabsf(v[2][i]), fabsf(v[3][i])));
        }
#pragma unroll
        for (int off = 1; off < 8; off <<= 1) {
            m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, off));
            m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, off));
        }
        const float amax[2] = {m0, m1};
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            const int64_t row = row0 + rr;
            const float s_z = __fdiv_rn(amax[rr], 127.0f);
            const bool zero = !(amax[rr] > 0.0f);
            const bool fast = s_z >= 0x1p-126f;
            const float rcp = __frcp_rn(s_z);
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                const int t = 2 * rr + tt;
                uint2 w = make_uint2(0u, 0u);
                if (!zero)
                    w = quant8(v[t], s_z, rcp, fast);
                if (row < p.rows)
                    st_v2(p.q + base + t * 64, w.x, w.y);
            }
            if (row < p.rows && (lane & 7u) == 0u) {
                const int64_t bh = static_cast<int64_t>(br[rr]) * H + hr[rr];
                p.s[bh * p.ls + lr[rr]] = zero ? 0.0f : __fmul_rn(s_z, p.c_g);
            }
        }
    }
}

// ---------------------------------------------------------------- the attention kernel

// 2^x in one MUFU instruction (relative error about 2^-22; 0 for x = -inf)
__device__ __forceinline__ float ex2_approx(float x)
{
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// max(a, b, c) in one instruction (sm_100)
__device__ __forceinline__ float max3f(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

struct AttnParams {
    const float *sq;       // [B][H][Lq_pad] query scales (rows padded to 128)
    const float *sk;       // [B][H][Lk_pad] key scales
    uint16_t *o;           // [B][Lq][H][D] bf16
    int32_t B, Lq, Lk, H;
    int32_t q_blocks;      // ceil(Lq / 256): pairs of 128-query tiles
    int32_t lq_pad, lk_pad;  // Lq, Lk rounded up to 128
    float scale;           // softmax scale applied to the logits (fp32)
    uint64_t timeout_ns;
};

// ---------------------------------------------------------------- the attention kernel
//
// One CTA per (b, h, 256 queries) = two 128-query tiles sharing every K / V block. Warps 2..5
// run the softmax of tile 0 and warps 6..9 that of tile 1, one thread per query row (all 128
// key columns of a block in registers, so the row maximum and sum need no exchange). Each SM
// sub-partition holds one warp of each tile; the two tiles run out of phase, so one tile's
// softmax covers the other's waits on S and PV. TMEM: S_0, S_1, O_0, O_1 (128 columns each).
// The MMA warp issues S_t(j+1) as soon as tile t has read S_t(j), and PV_t(j) once tile t
// has written P_t(j); a tile overwrites its P tile once PV_t(j-1) is done.
struct AttnConfig {
    static constexpr int THREADS = 320;                   // loader, MMA, 2 x 4 softmax warps
    static constexpr int NK = 3, NV = 2, NSK = 2;         // K, V, key-scale stages
    static constexpr int Q_OFF = 0;                       // 2 x int8 [128 x 128]
    static constexpr int K_OFF = 32768;                   // NK x int8 [128 x 128]
    static constexpr int V_OFF = K_OFF + NK * 16384;      // NV x bf16 [128 x 128]
    static constexpr int P_OFF = V_OFF + NV * 32768;      // 2 x bf16 [128 x 128], K-major
    static constexpr int SK_OFF = P_OFF + 2 * 32768;      // NSK x 128 fp32
    static constexpr int BAR_OFF = SK_OFF + NSK * 512;
    // barriers: q_full, k_full[NK], k_empty[NK], v_full[NV], v_empty[NV], sk_full[NSK],
    // sk_empty[NSK], then per tile s_full, s_empty, p_full, pv_done, turn, and drain
    static constexpr int NBARS = 1 + 2 * NK + 2 * NV + 2 * NSK + 10 + 1;
    static constexpr int SMEM_BYTES = 1024 + BAR_OFF + NBARS * 8 + 16;
    static constexpr int TMEM_COLS = 512;
    static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
};

__global__ void __launch_bounds__(AttnConfig::THREADS, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const AttnParams p)
{
    using C = AttnConfig;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw_addr);
    const uint32_t bar0 = base + C::BAR_OFF;
    constexpr int NK = C::NK, NV = C::NV, NSK = C::NSK;
    const uint32_t q_full = bar0;
    auto k_full = [&](int s) { return bar0 + 8u * (1 + s); };
    auto k_empty = [&](int s) { return bar0 + 8u * (1 + NK + s); };
    auto v_full = [&](int s) { return bar0 + 8u * (1 + 2 * NK + s); };
    auto v_empty = [&](int s) { return bar0 + 8u * (1 + 2 * NK + NV + s); };
    auto sk_full = [&](int s) { return bar0 + 8u * (1 + 2 * NK + 2 * NV + s); };
    auto sk_empty = [&](int s) { return bar0 + 8u * (1 + 2 * NK + 2 * NV + NSK + s); };
    constexpr int TB = 1 + 2 * NK + 2 * NV + 2 * NSK;
    // per tile t, one phase per key block: S_t(j) written / read, P_t(j) written / read by PV
    auto s_full = [&](int t) { return bar0 + 8u * (TB + t); };
    auto s_empty = [&](int t) { return bar0 + 8u * (TB + 2 + t); };
    auto p_full = [&](int t) { return bar0 + 8u * (TB + 4 + t); };
    auto pv_done = [&](int t) { return bar0 + 8u * (TB + 6 + t); };
    // turn(t): tile t may run its exponentials (the tiles alternate on the MUFU pipe)
    auto turn = [&](int t) { return bar0 + 8u * (TB + 8 + t); };
    const uint32_t drain_bar = bar0 + 8u * (TB + 10);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::BAR_OFF + C::NBARS * 8);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_holder + 1);
    float *sk_smem = reinterpret_cast<float *>(smem + C::SK_OFF);

    const uint32_t warp = threadIdx.x >> 5;
    const uint32_t lane = lane_id();
    const int32_t qp = static_cast<int32_t>(blockIdx.x) % p.q_blocks;   // pair of query tiles
    const int32_t bh = static_cast<int32_t>(blockIdx.x) / p.q_blocks;
    const int32_t b = bh / p.H, h = bh % p.H;
    const int32_t q0 = qp * 2 * kAttnBlock;
    const int32_t nkv = (p.Lk + kAttnBlock - 1) / kAttnBlock;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < NK; ++s) {
            mbar_init(k_full(s), 1);
            mbar_init(k_empty(s), 1);
        }
        for (int s = 0; s < NV; ++s) {
            mbar_init(v_full(s), 1);
            mbar_init(v_empty(s), 1);
        }
        for (int s = 0; s < NSK; ++s) {
            mbar_init(sk_full(s), 1);
            mbar_init(sk_empty(s), 8);   // both tiles' warps read the key scales
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(s_full(t), 1);
            mbar_init(s_empty(t), 4);
            mbar_init(p_full(t), 4);
            mbar_init(pv_done(t), 1);
            mbar_init(turn(t), 4);
        }
        mbar_init(drain_bar, 1);
        *abort = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_holder;
    // the prologue may overlap the preparation (programmatic launch); its codes and scales
    // are read from here on
    grid_dependency_wait();

    if (warp == 0) {
        // ------------------------------------------------------------ loads
        if (lane == 0) {
            // both Q tiles (rows past Lq read as zeros)
            mbar_arrive_expect_tx(q_full, 32768);
            tma_load_3d(base + C::Q_OFF, &tmQ, q_full, h * kAttnD, q0, b);
            tma_load_3d(base + C::Q_OFF + 16384, &tmQ, q_full, h * kAttnD, q0 + kAttnBlock, b);
            int nk = 0, nsk = 0, nv = 0;   // copies issued per ring
            for (int j = 0; j < nkv; ++j) {
                const int32_t j0 = j * kAttnBlock;
                const int ks = j % NK, ss = j % NSK, vs = j % NV;
                if (!mbar_wait_bounded(k_empty(ks), (static_cast<uint32_t>(j / NK) & 1u) ^ 1u, abort,
                                       p.timeout_ns))
                    break;
                mbar_arrive_expect_tx(k_full(ks), 16384);
                tma_load_3d(base + C::K_OFF + ks * 16384, &tmK, k_full(ks), h * kAttnD, j0, b);
                ++nk;
                if (!mbar_wait_bounded(sk_empty(ss), (static_cast<uint32_t>(j / NSK) & 1u) ^ 1u,
                                       abort, p.timeout_ns))
                    break;
                mbar_arrive_expect_tx(sk_full(ss), 512);
                bulk_load_1d(smem_u32(sk_smem + ss * kAttnBlock),
                             p.sk + static_cast<int64_t>(bh) * p.lk_pad + j0, 512, sk_full(ss));
                ++nsk;
                if (!mbar_wait_bounded(v_empty(vs), (static_cast<uint32_t>(j / NV) & 1u) ^ 1u, abort,
                                       p.timeout_ns))
                    break;
                mbar_arrive_expect_tx(v_full(vs), 32768);
                tma_load_3d(base + C::V_OFF + vs * 32768, &tmV, v_full(vs), h * kAttnD, j0, b);
                tma_load_3d(base + C::V_OFF + vs * 32768 + 16384, &tmV, v_full(vs), h * kAttnD + 64,
                            j0, b);
                ++nv;
            }
            volatile int no_abort = 0;
            mbar_wait_bounded(q_full, 0u, &no_abort, p.timeout_ns);
            for (int j = nk - NK < 0 ? 0 : nk - NK; j < nk; ++j)
                mbar_wait_bounded(k_full(j % NK), static_cast<uint32_t>(j / NK) & 1u, &no_abort,
                                  p.timeout_ns);
            for (int j = nsk - NSK < 0 ? 0 : nsk - NSK; j < nsk; ++j)
                mbar_wait_bounded(sk_full(j % NSK), static_cast<uint32_t>(j / NSK) & 1u, &no_abort,
                                  p.timeout_ns);
            for (int j = nv - NV < 0 ? 0 : nv - NV; j < nv; ++j)
                mbar_wait_bounded(v_full(j % NV), static_cast<uint32_t>(j / NV) & 1u, &no_abort,
                                  p.timeout_ns);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issue
        if (lane == 0) {
            constexpr uint32_t IDESC_S = idesc_s8_s32(128, 128);
            constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 128, true);
            auto issue_s = [&](int t, int j) {
                // S_t(j) = Q_t K_j^T into TMEM columns [128 t, 128 t + 128)
                const uint32_t sq_addr = base + C::Q_OFF + t * 16384;
                const uint32_t sk_addr = base + C::K_OFF + (j % NK) * 16384;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_s8(tmem_base + t * 128, kmajor_desc(sq_addr + 32 * k),
                           kmajor_desc(sk_addr + 32 * k), IDESC_S, k != 0 ? 1u : 0u);
                tc_commit(s_full(t));
            };
            auto issue_pv = [&](int t, int j) {
                // O_t (+)= P_t(j) V_j: A = P_t, K-major bf16 in two 64-column atoms; B = V, N-major
                const uint32_t sp = base + C::P_OFF + t * 32768;
                const uint32_t sv = base + C::V_OFF + (j % NV) * 32768;
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_f16(tmem_base + 256 + t * 128, kmajor_desc(sp + (k >> 2) * 16384 + (k & 3) * 32),
                            mnmajor_desc(sv + 2048 * k, 16384), IDESC_PV, (j | k) != 0 ? 1u : 0u);
                tc_commit(pv_done(t));
            };
            bool ok = mbar_wait_bounded(q_full, 0u, abort, p.timeout_ns) &&
                      mbar_wait_bounded(k_full(0), 0u, abort, p.timeout_ns);
            if (ok) {
                tc_fence_after_sync();
                issue_s(0, 0);
                issue_s(1, 0);
                tc_commit(k_empty(0));
            }
            for (int j = 0; ok && j < nkv; ++j) {
                const uint32_t ph = static_cast<uint32_t>(j) & 1u;
                if (j + 1 < nkv) {
                    const int kn = (j + 1) % NK;
                    if (!mbar_wait_bounded(k_full(kn), static_cast<uint32_t>((j + 1) / NK) & 1u, abort,
                                           p.timeout_ns)) {
                        ok = false;
                        break;
                    }
#pragma unroll 1
                    for (int t = 0; t < 2; ++t) {
                        if (!mbar_wait_bounded(s_empty(t), ph, abort, p.timeout_ns)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after_sync();
                        issue_s(t, j + 1);
                    }
                    if (!ok)
                        break;
                    tc_commit(k_empty(kn));
                }
                if (!mbar_wait_bounded(v_full(j % NV), static_cast<uint32_t>(j / NV) & 1u, abort,
                                       p.timeout_ns)) {
                    ok = false;
                    break;
                }
#pragma unroll 1
                for (int t = 0; t < 2; ++t) {
                    if (!mbar_wait_bounded(p_full(t), ph, abort, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    issue_pv(t, j);
                }
                if (!ok)
                    break;
                tc_commit(v_empty(j % NV));
            }
            tc_commit(drain_bar);
            volatile int no_abort = 0;
            mbar_wait_bounded(drain_bar, 0u, &no_abort, p.timeout_ns);
        }
    } else {
        // ------------------------------------------------------------ softmax (warps 2..9)
        const uint32_t tile = (warp - 2u) >> 2;
        const uint32_t quad = warp & 3u;
        const int32_t r = static_cast<int32_t>(quad * 32u + lane);   // row in the tile
        const int32_t qrow = q0 + static_cast<int32_t>(tile) * kAttnBlock + r;
        const bool row_ok = qrow < p.Lq;
        const float sqr = row_ok ? p.sq[static_cast<int64_t>(bh) * p.lq_pad + qrow] : 0.0f;
        // logit * log2(e) = (acc * s_k) * row_f with row_f = s_q * scale * log2 e >= 0, applied
        // in the exponent's fused multiply-add; rounding is monotone, so the row maximum of
        // the logits is row_f times that of acc * s_k. The floor keeps a zero row (or scale)
        // finite against the padded keys' -inf (its logits stay 0 to within 2^-100).
        const float row_f = fmaxf(sqr * p.scale * 1.4426950408889634f, 0x1p-126f);
        const uint32_t t_lane = tmem_base + ((quad * 32u) << 16);
        const uint32_t s_col = tile * 128u, o_col = 256u + tile * 128u;
        float m_used = -INFINITY;  // base-2 maximum the exponentials are taken against
        float l_sum = 0.0f;        // the row sum
        bool ok = true;
        for (int j = 0; ok && j < nkv; ++j) {
            const uint32_t ph = static_cast<uint32_t>(j) & 1u;
            const int ss = j % NSK;
            bool got = mbar_wait_bounded(s_full(tile), ph, abort, p.timeout_ns) &&
                       mbar_wait_bounded(sk_full(ss), static_cast<uint32_t>(j / NSK) & 1u, abort,
                                         p.timeout_ns);
            if (!__all_sync(0xffffffffu, got)) {
                ok = false;
                break;
            }
            tc_fence_after_sync();
            // fp32(acc) without the conversion pipe: |acc| <= 127 * 127 * 128 < 2^22, so the
            // bits of acc + 0x4B400000 are the float 1.5 * 2^23 + acc, and subtracting
            // 1.5 * 2^23 (below, exact) leaves acc
            float y[128];
            {
                uint32_t a[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    tmem_ld_32x32b_x32(t_lane + s_col + c * 32, a[c]);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        y[c * 32 + i] = __uint_as_float(a[c][i] + 0x4B400000u);
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(s_empty(tile));
            const float4 *skb = reinterpret_cast<const float4 *>(sk_smem + ss * kAttnBlock);
#pragma unroll
            for (int c4 = 0; c4 < 32; ++c4) {
                const float4 k4 = skb[c4];   // same address across the warp: a broadcast
                float f0, f1, f2, f3;
                sub2(f0, f1, y[4 * c4], y[4 * c4 + 1], 12582912.0f, 12582912.0f);
                sub2(f2, f3, y[4 * c4 + 2], y[4 * c4 + 3], 12582912.0f, 12582912.0f);
                mul2(y[4 * c4], y[4 * c4 + 1], f0, f1, k4.x, k4.y);          // acc * s_k
                mul2(y[4 * c4 + 2], y[4 * c4 + 3], f2, f3, k4.z, k4.w);
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(sk_empty(ss));   // the stage's key scales are read
            const int32_t j0 = j * kAttnBlock;
            if (j0 + kAttnBlock > p.Lk) {    // the ragged last block (uniform)
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (j0 + c >= p.Lk)
                        y[c] = -INFINITY;
            }
            // 4 independent chains, chain i over the columns i + 4k (k = 0..31)
            float mx[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                mx[i] = y[i];
#pragma unroll
                for (int k = 1; k + 1 < 32; k += 2)
                    mx[i] = max3f(mx[i], y[i + 4 * k], y[i + 4 * k + 4]);
                mx[i] = fmaxf(mx[i], y[i + 124]);
            }
            const float mb = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * row_f;
            // P_t(j-1) has left the P tile, and O_t is stable, once PV_t(j-1) is done
            if (j >= 1) {
                got = mbar_wait_bounded(pv_done(tile), ph ^ 1u, abort, p.timeout_ns);
                if (!__all_sync(0xffffffffu, got)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
            }
            // rescale O and l only when the maximum grows by more than 8 (p stays <= 256); O is
            // rescaled after P is written (the logits are dead then), before PV_t(j) can start
            const bool grow = mb > m_used + 8.0f;
            const bool any_grow = __any_sync(0xffffffffu, grow);
            float alpha = 1.0f;
            if (any_grow) {
                const float m_new = grow ? mb : m_used;
                alpha = grow && m_used != -INFINITY ? ex2_approx(m_used - m_new) : (grow ? 0.0f : 1.0f);
                l_sum *= alpha;
                m_used = m_new;
            }
            // the tiles take turns at the exponentials: tile 0 runs block j after tile 1 ran
            // block j - 1, tile 1 runs block j after tile 0 ran block j (the first wait of tile 0
            // passes at once); the other tile's scaling and maximum overlap this tile's
            got = mbar_wait_bounded(turn(tile), tile == 0 ? ph ^ 1u : ph, abort, p.timeout_ns);
            if (!__all_sync(0xffffffffu, got)) {
                ok = false;
                break;
            }
            // P = 2^(y - m), bf16, into the tile's swizzled K-major P: two 64-column atoms,
            // row r of an atom = 8 chunks of 16 bytes, chunk index XOR r mod 8
            const uint32_t prow = base + C::P_OFF + tile * 32768u + static_cast<uint32_t>(r) * 128u;
            const float neg_m = -m_used;
            float ls[8] = {0, 0, 0, 0, 0, 0, 0, 0};  // 8 independent partial sums
#pragma unroll
            for (int ch = 0; ch < 16; ++ch) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float d0, d1;   // (acc * s_k) * row_f - m in one rounding
                    fma2(d0, d1, y[ch * 8 + 2 * e], y[ch * 8 + 2 * e + 1], row_f, row_f, neg_m, neg_m);
                    const float p0 = ex2_approx(d0);
                    const float p1 = ex2_approx(d1);
                    add2(ls[2 * e], ls[2 * e + 1], ls[2 * e], ls[2 * e + 1], p0, p1);
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                    w[e] = *reinterpret_cast<const uint32_t *>(&h2);
                }
                const uint32_t c16 = static_cast<uint32_t>(ch & 7) ^ (static_cast<uint32_t>(r) & 7u);
                sts_v4(prow + static_cast<uint32_t>(ch >> 3) * 16384u + (c16 << 4), w[0], w[1], w[2],
                       w[3]);
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(turn(tile ^ 1u));
            l_sum += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
            if (any_grow && j >= 1) {
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t a[32];
                    tmem_ld_32x32b_x32(t_lane + o_col + c * 32, a);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        a[i] = __float_as_uint(__uint_as_float(a[i]) * alpha);
                    tmem_st_32x32b_x32(t_lane + o_col + c * 32, a);
                }
                tmem_st_wait();
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(p_full(tile));
        }
        // O / l as bf16
        const bool fin = ok && mbar_wait_bounded(pv_done(tile), static_cast<uint32_t>(nkv - 1) & 1u,
                                                 abort, p.timeout_ns);
        if (__all_sync(0xffffffffu, fin)) {
            tc_fence_after_sync();
            const float inv = 1.0f / l_sum;
            uint16_t *orow = p.o + ((static_cast<int64_t>(b) * p.Lq + qrow) * p.H + h) * kAttnD;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t a[32];
                tmem_ld_32x32b_x32(t_lane + o_col + c * 32, a);
                tmem_ld_wait();
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(a[2 * i]) * inv,
                                                                    __uint_as_float(a[2 * i + 1]) * inv);
                    w[i] = *reinterpret_cast<const uint32_t *>(&h2);
                }
                if (row_ok) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        st_v4(orow + c * 32 + q * 8, w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
                }
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

} // namespace sdnq
