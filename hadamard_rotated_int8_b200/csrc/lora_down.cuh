// LoRA down-projection u = bf16(x A) on the tensor cores (tcgen05.mma kind::f16, bf16
// operands, fp32 accumulators in TMEM), x the unrotated bf16 layer input [M, K] and
// A [K, rank] bf16. Source: "ConvRot / Hadamard SDNQ", PEFT Behavior (the adapters stay
// trainable in bf16 beside the int8 base).
//
// One CTA per 128-row block of x. A k-block is 64 columns of x (128 bytes, one 128-byte
// swizzled K-major row per x row) and 64 rows of A, loaded as rank/64 boxes of [64 rank x
// 64 k], which is the MN-major layout the MMA reads for its B operand. A pipeline stage
// holds two k-blocks, so each x row is read in 256-byte runs (measured: 14.7 us against
// 17.1 us with one k-block per stage at 4608 x 3072, rank 64; 4 k-blocks: 15.0 us).
//   warp 0: TMA producer   warp 1: TMEM alloc + MMA issuer   warps 2..5: epilogue
#pragma once

#include <cuda_bf16.h>

#include "device.cuh"

namespace sdnq {

struct LoraDownParams {
    uint16_t *u;        // [M, rank] bf16 out
    int32_t M, K, rank;
    int32_t num_kb;     // ceil(K / 64)
    uint64_t timeout_ns;
};

#ifndef SDNQ_LORA_DOWN_KPS
#define SDNQ_LORA_DOWN_KPS 2
#endif

template <int RANK_PAD>  // rank rounded up to a multiple of 64 (64..256)
struct LoraDownConfig {
    static constexpr int KPS = SDNQ_LORA_DOWN_KPS;         // k-blocks per stage
    static constexpr int X_KB = 128 * 128;                 // 128 rows x 64 bf16
    static constexpr int A_KB = (RANK_PAD / 64) * 8192;    // boxes of 64 x 64 bf16
    static constexpr int KB_BYTES = X_KB + A_KB;
    static constexpr int X_BYTES = KPS * X_KB;
    static constexpr int A_BYTES = KPS * A_KB;
    static constexpr int STAGE_BYTES = X_BYTES + A_BYTES;
    // as many stages as fit 192 KB (8 at rank 64): the kernel streams x and has one CTA per
    // 128 rows, so the bytes each CTA keeps in flight set its bandwidth
    static constexpr int STAGES = (196608 / STAGE_BYTES) < 8 ? (196608 / STAGE_BYTES) : 8;
    static constexpr int TMEM_COLS = RANK_PAD < 32 ? 32 : RANK_PAD;  // power of two >= 32
    static constexpr int BAR_BYTES = (2 * STAGES + 2) * 8;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES + 16;
};

template <int RANK_PAD>
__global__ void __launch_bounds__(192, 1)
    lora_down_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmA,
                     const LoraDownParams p)
{
    using C = LoraDownConfig<RANK_PAD>;
    static_assert(RANK_PAD == 64 || RANK_PAD == 128 || RANK_PAD == 256, "rank tile");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw_addr);
    const uint32_t bar0 = base + C::STAGES * C::STAGE_BYTES;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
    const uint32_t done_bar = bar0 + 8u * (2 * C::STAGES);
    uint32_t *tmem_holder =
        reinterpret_cast<uint32_t *>(smem + C::STAGES * C::STAGE_BYTES + C::BAR_BYTES);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const uint32_t warp = threadIdx.x >> 5;
    const uint32_t lane = lane_id();
    const int m0 = blockIdx.x * 128;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(done_bar, 1);
        *abort = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmX);
        prefetch_tensormap(&tmA);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_holder;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            bool ok = true;
            for (int kb0 = 0; kb0 < p.num_kb; kb0 += C::KPS) {
                if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                const int nkb = p.num_kb - kb0 < C::KPS ? p.num_kb - kb0 : C::KPS;
                const uint32_t sx_ = base + stage * C::STAGE_BYTES;
                const uint32_t sa = sx_ + C::X_BYTES;
                mbar_arrive_expect_tx(full_bar(stage), static_cast<uint32_t>(nkb * C::KB_BYTES));
                for (int i = 0; i < nkb; ++i)
                    tma_load_2d(sx_ + i * C::X_KB, &tmX, full_bar(stage), (kb0 + i) * 64, m0);
                for (int i = 0; i < nkb; ++i)
#pragma unroll
                    for (int j = 0; j < RANK_PAD / 64; ++j)
                        tma_load_2d(sa + i * C::A_KB + j * 8192, &tmA, full_bar(stage), 64 * j,
                                    (kb0 + i) * 64);
                ++issued;
                if (++stage == C::STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) {
                const int n = issued < C::STAGES ? issued : C::STAGES;
                int s = stage;
                uint32_t ph = phase;
                for (int i = 0; i < n; ++i) {
                    if (--s < 0) {
                        s = C::STAGES - 1;
                        ph ^= 1u;
                    }
                    volatile int no_abort = 0;
                    mbar_wait_bounded(full_bar(s), ph, &no_abort, p.timeout_ns);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(128, p.rank, true);
            int stage = 0;
            uint32_t phase = 0;
            for (int kb0 = 0; kb0 < p.num_kb; kb0 += C::KPS) {
                if (!mbar_wait_bounded(full_bar(stage), phase, abort, p.timeout_ns))
                    break;
                tc_fence_after_sync();
                const int nkb = p.num_kb - kb0 < C::KPS ? p.num_kb - kb0 : C::KPS;
                for (int i = 0; i < nkb; ++i) {
                    const uint32_t sx_ = base + stage * C::STAGE_BYTES + i * C::X_KB;
                    const uint32_t sa = base + stage * C::STAGE_BYTES + C::X_BYTES + i * C::A_KB;
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_f16(tmem_base, kmajor_desc(sx_ + 32 * k), mnmajor_desc(sa + 2048 * k, 8192),
                                idesc, ((kb0 + i) | k) != 0 ? 1u : 0u);
                }
                tc_commit(empty_bar(stage));
                if (++stage == C::STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            tc_commit(done_bar);  // also drains every MMA issued
        }
    } else {
        const uint32_t quad = warp & 3u;
        const int m = m0 + static_cast<int>(quad * 32u + lane);
        const bool row_ok = m < p.M;
        const bool ready = mbar_wait_bounded(done_bar, 0u, abort, p.timeout_ns);
        if (__all_sync(0xffffffffu, ready)) {  // warp-uniform: tcgen05.ld needs convergence
            tc_fence_after_sync();
            const uint32_t t_row = tmem_base + ((quad * 32u) << 16);
            uint16_t *urow = p.u + static_cast<int64_t>(row_ok ? m : 0) * p.rank;
#pragma unroll 1
            for (int c = 0; c < p.rank; c += 16) {
                uint32_t r[16];
                tmem_ld_32x32b_x16(t_row + c, r);
                tmem_ld_wait();
                if (!row_ok)
                    continue;
                uint32_t w[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(r[2 * j])));
                    const uint32_t hi =
                        __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(r[2 * j + 1])));
                    w[j] = lo | (hi << 16);
                }
                st_v4(urow + c, w[0], w[1], w[2], w[3]);
                st_v4(urow + c + 8, w[4], w[5], w[6], w[7]);
            }
        }
    }

    // MMAs must be complete before TMEM is freed: the epilogue waited on done_bar; on an
    // abort, wait for it here (bounded) as well.
    if (warp == 1 && lane == 0 && *abort) {
        volatile int no_abort = 0;
        mbar_wait_bounded(done_bar, 0u, &no_abort, p.timeout_ns);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

} // namespace sdnq
