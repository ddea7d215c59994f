// The int8 (or e4m3) linear on CTA pairs: one tcgen05 MMA spans the tensor cores of two SMs
// (cta_group::2). A pair computes a 256 x 256 output tile: each CTA loads its own 128 rows
// of the activation codes and its own 128 rows of the weight codes (the tile's columns are
// split between the CTAs), so every SM streams 32 KB of operands per 128-byte K step where a
// single-SM 128 x 256 tile streams 48 KB, for the same tensor-core work per SM. Each CTA's
// tensor memory receives its 128 rows of the int32 (fp32 for e4m3) accumulators, and its own
// epilogue warps apply the same fp32 de-quant epilogue (and the GELU table) as the single-SM
// kernel, so outputs are bit for bit the same. With LORA the pair also accumulates the
// adapter term L = u B (bf16 operands, fp32, kind::f16) in a second 256-column accumulator
// after the int8 K loop, as the single-SM kernel does; the int32 and fp32 accumulators then
// fill the 512 columns, so there is one buffer. Its epilogue copies the int32 columns to
// registers and hands them back at once (tempty[0]), so the next tile's int8 K loop runs
// while the outputs of this one are formed; the adapter columns go back (tempty[1]) before
// the next tile's adapter MMAs. With GRAD_G the pair computes the input gradient: the weight
// codes are read N-major (each CTA one 128 x 128 box of its columns per k-block) and each
// CTA runs the single-SM kernel's inverse-rotation epilogue on its 128 x 256 tile.
//
// Sources: as the single-SM kernel ("SDNQ: SD.Next Quantization Engine" README, INT8
// quantized matmul and dequantize_fp32; "ConvRot / Hadamard SDNQ").
//
// Roles (320 threads per CTA; 576 with GELU; 608 with the activation quantizer inside):
//   warp 0      TMA producer of this CTA's halves. The loads of both CTAs complete on rank
//               0's full barrier (the cta_group::2 form of the tensor copy), whose
//               expected byte count rank 0 sets for both halves.
//   warp 1      both CTAs allocate the same tensor-memory columns; rank 0 issues the
//               pair's MMAs once a stage is full.
//   warps 2..   epilogue of this CTA's 128 rows (8 warps; 16 with GELU); they
//               release the accumulator buffer with a remote arrive on rank 0's
//               tensor-empty barrier (one arrival per epilogue warp of both CTAs).
//   then, with the activation quantizer inside (plain linear only): 8 warps that rotate and
//               quantize rows of x into the A operand, publishing 128-row blocks through
//               global counters, and one scale warp that waits (bounded) for this CTA's
//               block of each tile and copies its row scales to shared memory for the
//               producer and the epilogue. Tiles then run columns-fastest.
// The MMA completion (tcgen05.commit, multicast to both CTAs) frees each stage in both CTAs
// and announces each finished accumulator buffer to both epilogues. Every wait is bounded.
// A producer that gives up drains its own copies: rank 0 by waiting (bounded) on its full
// barriers; rank 1, whose copies complete on rank 0's barriers, by a bounded sleep far
// longer than a copy takes, before the final cluster barrier (until which rank 0's barriers
// stay valid).
#pragma once

#include "gemm.cuh"

#ifndef SDNQ_WIDE_EPI_WARPS
#define SDNQ_WIDE_EPI_WARPS 16
#endif
#ifndef SDNQ_LORA_EPI_WARPS
#define SDNQ_LORA_EPI_WARPS 8
#endif
#ifndef SDNQ_PAIR_KPS
#define SDNQ_PAIR_KPS 2
#endif

namespace sdnq {

template <bool GELU, bool LORA = false, bool FUSE = false>
struct PairConfig {
    static constexpr int BM = 128;                       // rows per CTA (256 per pair)
    static constexpr int BN = 256;                       // columns per pair tile
    static constexpr int BK = 128;                       // bytes of K per k-block (one TMA box)
    // k-blocks per pipeline stage: two halve the stage barriers and MMA commits per byte of
    // K (each stage costs the tensor pipe a little; measured with the loads removed: 148 us
    // against 163 us on 8192 x 12288 x 3072)
    static constexpr int KPS = SDNQ_PAIR_KPS;
    static constexpr int A_KB = BM * BK;                 // 16 KB per k-block
    static constexpr int B_KB = (BN / 2) * BK;           // this CTA's 128 columns: 16 KB
    static constexpr int A_BYTES = KPS * A_KB;
    static constexpr int B_BYTES = KPS * B_KB;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int ACC_COLS = LORA ? 2 * BN : BN;  // int32 (+ fp32 LoRA) columns per buffer
    static constexpr int NBUF = LORA ? 1 : 2;
    static constexpr int TMEM_COLS = NBUF * ACC_COLS;    // 512
    // four epilogue warps per TMEM lane quarter for the GELU table lookups (integer-heavy);
    // two for the plain epilogue and for LoRA, whose warps hold a row's fp32 partials for
    // their 128 columns in registers (168 per thread at 10 warps per CTA)
    static constexpr int EPI_WARPS = GELU ? SDNQ_WIDE_EPI_WARPS : LORA ? SDNQ_LORA_EPI_WARPS : 8;
    // with the activation quantizer inside: 8 quantizer warps and one scale warp more
    static constexpr int QUANT_WARPS = FUSE ? SDNQ_FUSED_QUANT_WARPS : 0;
    static constexpr int THREADS = 64 + 32 * EPI_WARPS + (FUSE ? 32 * (QUANT_WARPS + 1) : 0);
    static constexpr int EPI_COLS = BN / (EPI_WARPS / 4);
    // output staging per epilogue warp: a 32 x 32 bf16 block; with GELU (16 warps and the
    // table) a 32 x 16 block, so that three stages of two k-blocks still fit
    static constexpr int OUT_COLS = GELU ? 16 : 32;
    static constexpr int STAGE_OUT_BYTES = 32 * OUT_COLS * 2;
    static constexpr int LUT_BYTES = GELU ? kGeluLutBytes : 0;
    static constexpr int SCALE_BYTES = EPI_COLS * 8;
    static constexpr int FIXED = EPI_WARPS * (STAGE_OUT_BYTES + SCALE_BYTES) + LUT_BYTES +
                                 (FUSE ? 2 * 128 * 4 + 2 * SDNQ_FUSED_QUANT_WARPS * 4 + 32 : 0);
    static constexpr int STAGES = (232448 - 1024 - 512 - FIXED) / STAGE_BYTES > 6
                                      ? 6 : (232448 - 1024 - 512 - FIXED) / STAGE_BYTES;
    static constexpr int OUT_OFF = STAGES * STAGE_BYTES;
    static constexpr int SCALE_OFF = OUT_OFF + EPI_WARPS * STAGE_OUT_BYTES;
    static constexpr int LUT_OFF = SCALE_OFF + EPI_WARPS * SCALE_BYTES;
    static constexpr int SX_OFF = LUT_OFF + LUT_BYTES;     // fused: row scales per buffer
    static constexpr int SX_BYTES = FUSE ? 2 * 128 * 4 : 0;
    static constexpr int AMAX_OFF = SX_OFF + SX_BYTES;     // fused: quantizer row maxima
    static constexpr int AMAX_BYTES = FUSE ? 2 * QUANT_WARPS * 4 : 0;
    static constexpr int BAR_OFF = AMAX_OFF + AMAX_BYTES;
    // full[S], empty[S], tfull[2], tempty[2], drain, sxfull[2], sxempty[2]; then tmem base +
    // abort flag
    // full barriers per stage: one per k-block, so that a k-block's MMAs start as soon as its
    // own copies have landed (1-3% on the plain and LoRA kernels); one per stage with GELU
    // (measured: 128.8 against 124.8 us on the MLP up-projection with one per k-block)
    static constexpr int NFB = GELU ? 1 : KPS;
    static constexpr int BAR_BYTES = (2 * STAGES + 9 + (NFB - 1) * STAGES) * 8;
    static constexpr int SMEM_BYTES = 1024 + BAR_OFF + BAR_BYTES + 16;
    static_assert(STAGES >= 3, "pipeline depth");
    static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
};

// One 16-column output block: 8 packed bf16 pairs of this thread's row go through the warp's
// unswizzled 32 x 32-byte staging buffer to a TMA store of the warp's 32 x 16 block at
// (column nc, row mrow0); rows >= M and columns >= N fall outside the tensor and are dropped.
__device__ __forceinline__ void store_block16(const uint32_t *ob, uint32_t s_out, uint32_t lane,
                                              const CUtensorMap *tmO, int nc, int mrow0)
{
    if (lane == 0)
        bulk_wait_read_all();  // the previous block has left the staging buffer
    __syncwarp();
    const uint32_t row_addr = s_out + lane * 32u;
    sts_v4(row_addr, ob[0], ob[1], ob[2], ob[3]);
    sts_v4(row_addr + 16u, ob[4], ob[5], ob[6], ob[7]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d(tmO, s_out, nc, mrow0);
        bulk_commit_group();
    }
}

// The first fp32 steps of the de-quant epilogue for two adjacent columns: t = sx * sw (f32x2),
// v = fp32(acc) * t, then + bias; the products that feed an add as scalar intrinsics, the
// same steps as the single-SM epilogue.
template <bool FP8>
__device__ __forceinline__ void dequant_pair(uint32_t acc0, uint32_t acc1, float sxm, float w0,
                                             float w1, float b0, float b1, bool has_bias,
                                             float &v0, float &v1)
{
    float t0, t1;
    mul2(t0, t1, sxm, sxm, w0, w1);
    const float a0 = FP8 ? __uint_as_float(acc0) : __int2float_rn(static_cast<int>(acc0));
    const float a1 = FP8 ? __uint_as_float(acc1) : __int2float_rn(static_cast<int>(acc1));
    v0 = __fmul_rn(a0, t0);
    v1 = __fmul_rn(a1, t1);
    if (has_bias) {
        v0 = __fadd_rn(v0, b0);
        v1 = __fadd_rn(v1, b1);
    }
}

// LoRA epilogue of one warp (one TMEM lane quarter, EPI_COLS columns of the tile). The int32
// columns are copied to registers with one wait and released at once through rank 0's
// tempty[0]: the pair's next int8 K loop then runs while this warp de-quantizes, reads the
// adapter columns, adds lora_scale * L and stores the bf16 outputs; tempty[1] releases the
// adapter columns for the next tile's adapter MMAs. The arithmetic and its order are those
// of the one-pass epilogue, so outputs are unchanged.
template <class C>
__device__ __forceinline__ void lora_epilogue(uint32_t t_row, int col_base, int n0, int m0,
                                              uint32_t quad, uint32_t lane, float sxm,
                                              bool row_ok, int m, uint32_t s_sw,
                                              uint32_t s_bias, uint32_t s_out,
                                              const CUtensorMap *tmO, const GemmParams &p,
                                              uint32_t leader_tempty0)
{
    constexpr int NCH = C::EPI_COLS / 16;
    const bool has_bias = p.bias != nullptr;
    uint32_t acc[NCH][16];
#pragma unroll
    for (int k = 0; k < NCH; ++k)
        if (n0 + col_base + 16 * k < p.N)   // warp-uniform
            tmem_ld_32x32b_x16(t_row + col_base + 16 * k, acc[k]);
    tmem_ld_wait();
    tc_fence_before_sync();
    __syncwarp();
    if (lane == 0)
        mbar_arrive_remote(leader_tempty0);
    if (p.acc_out != nullptr && row_ok) {
        int32_t *arow = p.acc_out + static_cast<int64_t>(m) * p.N;
#pragma unroll
        for (int k = 0; k < NCH; ++k)
#pragma unroll
            for (int j = 0; j < 16; ++j)
                if (n0 + col_base + 16 * k + j < p.N)
                    arow[n0 + col_base + 16 * k + j] = static_cast<int32_t>(acc[k][j]);
    }
    // fp32(acc) * t + bias, in place
#pragma unroll
    for (int k = 0; k < NCH; ++k) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 w = lds_v4(s_sw + 4 * (16 * k + 4 * q));
            const float4 b = lds_v4(s_bias + 4 * (16 * k + 4 * q));
            const float wv[4] = {w.x, w.y, w.z, w.w};
            const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int j = 4 * q + 2 * h;
                float v0, v1;
                dequant_pair<false>(acc[k][j], acc[k][j + 1], sxm, wv[2 * h], wv[2 * h + 1],
                                    bv[2 * h], bv[2 * h + 1], has_bias, v0, v1);
                acc[k][j] = __float_as_uint(v0);
                acc[k][j + 1] = __float_as_uint(v1);
            }
        }
    }
#pragma unroll
    for (int c = 0; c < C::EPI_COLS; c += 32) {
        const int cc = col_base + c;
        const int nc = n0 + cc;
        if (nc < p.N) {   // warp-uniform
            uint32_t ob[16];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int k = c / 16 + hh;
                uint32_t l[16];
                tmem_ld_32x32b_x16(t_row + C::BN + cc + 16 * hh, l);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; j += 2) {
                    const float v0 = __fadd_rn(__uint_as_float(acc[k][j]),
                                               __fmul_rn(p.lora_scale, __uint_as_float(l[j])));
                    const float v1 = __fadd_rn(__uint_as_float(acc[k][j + 1]),
                                               __fmul_rn(p.lora_scale, __uint_as_float(l[j + 1])));
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(v0, v1);
                    ob[(16 * hh + j) >> 1] = *reinterpret_cast<const uint32_t *>(&h2);
                }
            }
            store_block(ob, s_out, lane, tmO, nc, m0 + static_cast<int>(quad * 32u));
        }
    }
    tc_fence_before_sync();
    __syncwarp();
    if (lane == 0)
        mbar_arrive_remote(leader_tempty0 + 8u);
}

template <bool GELU, bool FP8, bool LORA, int FUSE_G = 0, int GRAD_G = 0>
__global__ void __launch_bounds__(PairConfig<GELU, LORA, (FUSE_G > 0)>::THREADS, 1)
    gemm_s8_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmU,
                        const __grid_constant__ CUtensorMap tmL,
                        const __grid_constant__ CUtensorMap tmO, const GemmParams p)
{
    using C = PairConfig<GELU, LORA, (FUSE_G > 0)>;
    static_assert(!LORA || (!GELU && !FP8), "the adapter term rides on the plain int8 linear");
    static_assert(FUSE_G == 0 || (!LORA && !GELU && !FP8),
                  "the activation quantizer inside: the plain int8 linear");
    static_assert(GRAD_G == 0 || (!LORA && !GELU && !FP8 && FUSE_G == 0 &&
                                  (GRAD_G & (GRAD_G - 1)) == 0 && GRAD_G <= 256),
                  "the input gradient: the int8 product with the inverse-rotation epilogue");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw_addr);
    const uint32_t bar0 = base + C::BAR_OFF;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
    auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * C::STAGES + b); };
    auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * C::STAGES + 2 + b); };
    const uint32_t drain_bar = bar0 + 8u * (2 * C::STAGES + 4);
    auto sxfull_bar = [&](int b) { return bar0 + 8u * (2 * C::STAGES + 5 + b); };
    auto sxempty_bar = [&](int b) { return bar0 + 8u * (2 * C::STAGES + 7 + b); };
    // full barrier of k-block i of stage s (i = 0 is full_bar(s))
    auto kfull_bar = [&](int s, int i) {
        return i == 0 ? full_bar(s) : bar0 + 8u * (2 * C::STAGES + 9 + (i - 1) * C::STAGES + s);
    };
    float *sx_smem = reinterpret_cast<float *>(smem + C::SX_OFF);     // [2][128], fused only
    float *amax_smem = reinterpret_cast<float *>(smem + C::AMAX_OFF); // fused only
    // tile -> (pair-row block, column block): rows fastest; columns fastest with the
    // quantizer inside, whose 128-row blocks become ready in order
    auto tile_mb = [&](int tile) { return FUSE_G > 0 ? tile / p.num_n_blocks : tile % p.num_m_blocks; };
    auto tile_nb = [&](int tile) { return FUSE_G > 0 ? tile % p.num_n_blocks : tile / p.num_m_blocks; };
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::BAR_OFF + C::BAR_BYTES);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const uint32_t warp = threadIdx.x >> 5;
    const uint32_t lane = lane_id();
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0u;
    const int pair = static_cast<int>(cluster_id_x());
    const int npairs = static_cast<int>(nclusters_x());

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            for (int i = 0; i < C::NFB; ++i)
                mbar_init(kfull_bar(s, i), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < C::NBUF; ++b)
            mbar_init(tfull_bar(b), 1);
        // with LoRA: tempty[0] releases the int32 columns, tempty[1] the adapter columns
        for (int b = 0; b < (LORA ? 2 : C::NBUF); ++b)
            mbar_init(tempty_bar(b), 2 * C::EPI_WARPS);
        mbar_init(drain_bar, 1);
        if (FUSE_G > 0)
            for (int b = 0; b < C::NBUF; ++b) {
                mbar_init(sxfull_bar(b), 1);
                mbar_init(sxempty_bar(b), C::EPI_WARPS);
            }
        *abort = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        prefetch_tensormap(&tmO);
        if (LORA) {
            prefetch_tensormap(&tmU);
            prefetch_tensormap(&tmL);
        }
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_holder), C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    // both CTAs' barriers are initialised and their tensor memory allocated before any
    // remote arrive or multicast commit reaches them
    tc_fence_before_sync();
    cluster_sync_all();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_holder;
    grid_dependency_wait();

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            bool ok = true;
            const uint32_t leader_bar0 = mapa_shared(bar0, 0u);   // rank 0's barriers
            int local = 0;
            for (int tile = pair; ok && tile < p.num_tiles; tile += npairs, ++local) {
                const int m0 = tile_mb(tile) * 2 * C::BM + static_cast<int>(rank) * C::BM;
                const int nr0 = tile_nb(tile) * C::BN + static_cast<int>(rank) * (C::BN / 2);
                if constexpr (FUSE_G > 0) {
                    // the scale warp has seen this CTA's 128 activation rows published; order
                    // that before the tensor copies read them
                    const int buf = local % C::NBUF;
                    const uint32_t use = static_cast<uint32_t>(local / C::NBUF);
                    if (!mbar_wait_bounded(sxfull_bar(buf), use & 1u, abort, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    fence_proxy_async_global();
                }
                const int kstages = (p.num_kb + C::KPS - 1) / C::KPS;
                const int steps = kstages + (LORA ? p.lora_chunks : 0);
                for (int st = 0; st < steps; ++st) {
                    if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    const uint32_t sa = base + stage * C::STAGE_BYTES;
                    const uint32_t sb = sa + C::A_BYTES;
                    // rank 0's full barrier of k-block i of this stage
                    auto kfb = [&](int i) { return leader_bar0 + (kfull_bar(stage, i) - bar0); };
                    const uint32_t fb = kfb(0);
                    if (!LORA || st < kstages) {
                        // k-blocks kb0 .. kb0 + nkb - 1 of this CTA's A rows and B columns,
                        // each completing on its own barrier; a k-block past the end of K
                        // completes its barrier without copies (rank 0's plain arrive)
                        const int kb0 = st * C::KPS;
                        const int nkb = p.num_kb - kb0 < C::KPS ? p.num_kb - kb0 : C::KPS;
                        for (int i = 0; i < C::KPS; ++i) {
                            const int fi = C::NFB > 1 ? i : 0;   // this k-block's barrier
                            if (i < nkb) {
                                if (leader && (C::NFB > 1 || i == 0))
                                    mbar_arrive_expect_tx(
                                        kfull_bar(stage, fi),
                                        static_cast<uint32_t>(2 * (C::NFB > 1 ? 1 : nkb) * (C::A_KB + C::B_KB)));
                                tma_load_2d_pair(sa + i * C::A_KB, &tmA, kfb(fi), (kb0 + i) * C::BK, m0);
                                if constexpr (GRAD_G > 0)   // qW rows = contraction, N-major columns
                                    tma_load_2d_pair(sb + i * C::B_KB, &tmB, kfb(fi), nr0, (kb0 + i) * C::BK);
                                else
                                    tma_load_2d_pair(sb + i * C::B_KB, &tmB, kfb(fi), (kb0 + i) * C::BK, nr0);
                            } else if (leader && C::NFB > 1) {
                                mbar_arrive(kfull_bar(stage, i));
                            }
                        }
                    } else {
                        // LoRA chunk c: this CTA's U rows [128 x 64 rank] (K-major) into the A
                        // slot, its 128 columns of B [64 rank x 128] (N-major) as two 64-column
                        // boxes into the B slot (32 KB per CTA), on the stage's first barrier
                        if (leader) {
                            mbar_arrive_expect_tx(full_bar(stage),
                                                  static_cast<uint32_t>(2 * (C::A_KB + C::B_KB)));
                            for (int i = 1; i < C::NFB; ++i)
                                mbar_arrive(kfull_bar(stage, i));
                        }
                        const int c = st - kstages;
                        tma_load_2d_pair(sa, &tmU, fb, c * 64, m0);
                        tma_load_2d_pair(sb, &tmL, fb, nr0, c * 64);
                        tma_load_2d_pair(sb + 8192, &tmL, fb, nr0 + 64, c * 64);
                    }
                    ++issued;
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                if (leader) {
                    // drain: wait (bounded) for the copies of the last stages issued
                    const int n = issued < C::STAGES ? issued : C::STAGES;
                    int s = stage;
                    uint32_t ph = phase;
                    for (int i = 0; i < n; ++i) {
                        if (--s < 0) {
                            s = C::STAGES - 1;
                            ph ^= 1u;
                        }
                        for (int k = 0; k < C::NFB; ++k) {
                            volatile int no_abort = 0;
                            mbar_wait_bounded(kfull_bar(s, k), ph, &no_abort, p.timeout_ns);
                        }
                    }
                } else {
                    sleep_ns_bounded(1000000);   // 1 ms: this CTA's copies have landed
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // -------------------------------------------------------- MMA issuer (rank 0)
            constexpr uint32_t IDESC =
                FP8 ? idesc_e4m3_f32(256, C::BN) : idesc_s8_s32(256, C::BN, GRAD_G > 0);
            int stage = 0;
            uint32_t phase = 0;
            int local = 0;
            bool ok = true;
            for (int tile = pair; ok && tile < p.num_tiles; tile += npairs, ++local) {
                const int buf = local % C::NBUF;
                const uint32_t use = static_cast<uint32_t>(local / C::NBUF);
                if (!mbar_wait_bounded(tempty_bar(buf), (use & 1u) ^ 1u, abort, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_acc = tmem_base + buf * C::ACC_COLS;
                for (int kb0 = 0; ok && kb0 < p.num_kb; kb0 += C::KPS) {
                    const uint32_t sa = base + stage * C::STAGE_BYTES;
                    const uint32_t sb = sa + C::A_BYTES;
                    const int nkb = p.num_kb - kb0 < C::KPS ? p.num_kb - kb0 : C::KPS;
#pragma unroll
                    for (int i = 0; i < C::KPS; ++i) {
                        // each k-block's MMAs as soon as its own copies have landed (a block
                        // past the end of K has its barrier completed without copies)
                        if (i < C::NFB) {
                            if (!mbar_wait_bounded(kfull_bar(stage, i), phase, abort, p.timeout_ns)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after_sync();
                        }
                        if (i < nkb) {
#pragma unroll
                            for (int k = 0; k < C::BK / 32; ++k) {
                                const uint64_t da = kmajor_desc(sa + i * C::A_KB + 32 * k);
                                // the input gradient's N-major B: K = 32 rows of 128 bytes
                                const uint64_t db = GRAD_G > 0
                                                        ? mnmajor_desc(sb + i * C::B_KB + 4096 * k, 16384)
                                                        : kmajor_desc(sb + i * C::B_KB + 32 * k);
                                const uint32_t accum = ((kb0 + i) | k) != 0 ? 1u : 0u;
                                if constexpr (FP8)
                                    mma_f8_pair(d_acc, da, db, IDESC, accum);
                                else
                                    mma_s8_pair(d_acc, da, db, IDESC, accum);
                            }
                        }
                    }
                    tc_commit_pair(empty_bar(stage), 0x3);
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if constexpr (LORA) {
                    constexpr uint32_t IDESC_BF = idesc_bf16_f32(256, C::BN, true);
                    const uint32_t d_lora = d_acc + C::BN;
                    // the epilogues of both CTAs have read the previous tile's adapter columns
                    if (!mbar_wait_bounded(tempty_bar(1), (use & 1u) ^ 1u, abort, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    for (int c = 0; ok && c < p.lora_chunks; ++c) {
                        if (!mbar_wait_bounded(full_bar(stage), phase, abort, p.timeout_ns)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after_sync();
                        const uint32_t sa = base + stage * C::STAGE_BYTES;
                        const uint32_t sb = sa + C::A_BYTES;
                        // 4 MMAs of K = 16 rank rows: A advances 32 bytes along its swizzled
                        // rows, B (two 64-column atoms 8 KB apart) 16 rows = 2048 bytes
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            mma_f16_pair(d_lora, kmajor_desc(sa + 32 * k), mnmajor_desc(sb + 2048 * k, 8192),
                                         IDESC_BF, (c | k) != 0 ? 1u : 0u);
                        tc_commit_pair(empty_bar(stage), 0x3);
                        if (++stage == C::STAGES) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                }
                if (!ok)
                    break;
                tc_commit_pair(tfull_bar(buf), 0x3);
            }
            // drain: every MMA issued has completed before either CTA frees its tensor memory
            tc_commit_pair(drain_bar, 0x1);
            volatile int no_abort = 0;
            mbar_wait_bounded(drain_bar, 0u, &no_abort, p.timeout_ns);
        }
    } else if (FUSE_G > 0 && warp == 2 + C::EPI_WARPS + C::QUANT_WARPS) {
        // ------------------------------------------------------------ scale warp (fused)
        // Per tile of this CTA, ahead of the producer: wait (bounded, acquire) until this
        // CTA's 128 activation rows are published, count this CTA as one of the block's
        // readers (the last one clears the block's counters for the next launch), wait until
        // this CTA's epilogue has finished with the buffer's scales, copy the rows' scales to
        // shared memory and arrive on sxfull, which the producer and the epilogue wait for.
        if constexpr (FUSE_G > 0) {
            const int nb128 = (p.M + 127) / 128;
            int local = 0;
            for (int tile = pair; tile < p.num_tiles; tile += npairs, ++local) {
                const int m0 = tile_mb(tile) * 2 * C::BM + static_cast<int>(rank) * C::BM;
                const int b128 = m0 / 128;
                const int buf = local % C::NBUF;
                const uint32_t use = static_cast<uint32_t>(local / C::NBUF);
                const int rows = p.M - m0 < 128 ? (p.M - m0 > 0 ? p.M - m0 : 0) : 128;
                bool good = true;
                if (lane == 0) {
                    if (rows > 0) {
                        good = wait_count_bounded(p.sync + b128,
                                                  static_cast<uint32_t>(rows * p.rq.wpr), abort,
                                                  p.timeout_ns);
                        if (good) {
                            const uint32_t seen = atomicAdd(p.sync + nb128 + b128, 1u);
                            if (seen == static_cast<uint32_t>(p.num_n_blocks) - 1u) {
                                p.sync[b128] = 0u;
                                p.sync[nb128 + b128] = 0u;
                            }
                        }
                    }
                    if (good)
                        good = mbar_wait_bounded(sxempty_bar(buf), (use & 1u) ^ 1u, abort,
                                                 p.timeout_ns);
                }
                if (__shfl_sync(0xffffffffu, good ? 1 : 0, 0) == 0)
                    break;
                for (int i = static_cast<int>(lane); i < 128; i += 32)
                    sx_smem[buf * 128 + i] = m0 + i < p.M ? p.rq.s[m0 + i] : 0.0f;
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(sxfull_bar(buf));
            }
        }
    } else if (FUSE_G > 0 && warp >= 2 + C::EPI_WARPS) {
        // ------------------------------------------------------------ activation quantizer
        // rows of x -> rotated int8 codes (the A operand) and their scales, published per
        // 128-row block for the scale warps of every CTA
        if constexpr (FUSE_G > 0)
            rotquant_worker_rows<FUSE_G>(p.rq, static_cast<int32_t>(warp) - 2 - C::EPI_WARPS,
                                         C::QUANT_WARPS, 6u, amax_smem, p.sync);
    } else {
        // ------------------------------------------------------------ epilogue (warps 2..9)
        const uint32_t quad = warp & 3u;
        const uint32_t ew = warp - 2u;
        const int col_base = static_cast<int>(ew >> 2) * C::EPI_COLS;
        const int row_in_tile = static_cast<int>(quad * 32u + lane);
        const uint32_t s_out = base + C::OUT_OFF + ew * C::STAGE_OUT_BYTES;
        const uint32_t s_sw = base + C::SCALE_OFF + ew * C::SCALE_BYTES;
        const uint32_t s_bias = s_sw + C::EPI_COLS * 4;
        const bool has_bias = p.bias != nullptr;
        const uint32_t leader_tempty0 = mapa_shared(tempty_bar(0), 0u);
        uint16_t *lut = reinterpret_cast<uint16_t *>(smem + C::LUT_OFF);
        if constexpr (GELU) {
            gelu_lut_load(lut, static_cast<int>(ew * 32u + lane), 32 * C::EPI_WARPS);
            bar_sync_or(1, 32 * C::EPI_WARPS, false);
        }
        int local = 0;
        for (int tile = pair; tile < p.num_tiles; tile += npairs, ++local) {
            const int buf = local % C::NBUF;
            const uint32_t use = static_cast<uint32_t>(local / C::NBUF);
            const int m0 = tile_mb(tile) * 2 * C::BM + static_cast<int>(rank) * C::BM;
            const int n0 = tile_nb(tile) * C::BN;
            const int nw = n0 + col_base;
#pragma unroll
            for (int j = static_cast<int>(lane) * 4; GRAD_G == 0 && j < C::EPI_COLS; j += 128) {
                float w4[4], b4[4];
                if (nw + j + 4 <= p.N) {
                    const float4 f = __ldg(reinterpret_cast<const float4 *>(p.sw + nw + j));
                    w4[0] = f.x; w4[1] = f.y; w4[2] = f.z; w4[3] = f.w;
                    if (has_bias) {
                        const uint2 bb = __ldg(reinterpret_cast<const uint2 *>(p.bias + nw + j));
                        b4[0] = bf16_bits_to_float(bb.x & 0xffffu);
                        b4[1] = bf16_bits_to_float(bb.x >> 16);
                        b4[2] = bf16_bits_to_float(bb.y & 0xffffu);
                        b4[3] = bf16_bits_to_float(bb.y >> 16);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const bool ok = nw + j + e < p.N;
                        w4[e] = ok ? __ldg(p.sw + nw + j + e) : 0.0f;
                        b4[e] = (ok && has_bias) ? bf16_bits_to_float(__ldg(p.bias + nw + j + e)) : 0.0f;
                    }
                }
                if (!has_bias)
                    b4[0] = b4[1] = b4[2] = b4[3] = 0.0f;
                sts_v4(s_sw + 4 * j, __float_as_uint(w4[0]), __float_as_uint(w4[1]),
                       __float_as_uint(w4[2]), __float_as_uint(w4[3]));
                sts_v4(s_bias + 4 * j, __float_as_uint(b4[0]), __float_as_uint(b4[1]),
                       __float_as_uint(b4[2]), __float_as_uint(b4[3]));
            }
            __syncwarp();
            const int m = m0 + row_in_tile;
            const bool row_ok = m < p.M;
            // the row's scale is read before the accumulator wait (written by an earlier
            // launch, visible since the dependency wait)
            float sxm = (FUSE_G == 0 && row_ok) ? p.sx[m] : 0.0f;
            const bool ready = mbar_wait_bounded(tfull_bar(buf), use & 1u, abort, p.timeout_ns);
            if constexpr (GRAD_G > 0) {
                // the two warps of a lane quarter leave together: they meet at named
                // barriers inside the tile
                if (bar_sync_or(2u + quad, 64, !__all_sync(0xffffffffu, ready)))
                    break;
            } else {
                if (!__all_sync(0xffffffffu, ready))
                    break;
            }
            tc_fence_after_sync();
            if constexpr (FUSE_G > 0) {
                // the row scales the scale warp copied once the rows were published
                const bool got = mbar_wait_bounded(sxfull_bar(buf), use & 1u, abort, p.timeout_ns);
                if (!__all_sync(0xffffffffu, got))
                    break;
                sxm = row_ok ? sx_smem[buf * 128 + row_in_tile] : 0.0f;
            }
            const uint32_t t_row = tmem_base + ((quad * 32u) << 16) + buf * C::ACC_COLS;
            if constexpr (LORA) {
                lora_epilogue<C>(t_row, col_base, n0, m0, quad, lane, sxm, row_ok, m, s_sw, s_bias,
                                 s_out, &tmO, p, leader_tempty0);
            } else if constexpr (GRAD_G > 0) {
                // the same per-CTA tile (128 rows x 256 columns) as the single-SM kernel
                int32_t *acc_row = (p.acc_out != nullptr && row_ok)
                                       ? p.acc_out + static_cast<int64_t>(m) * p.N : nullptr;
                grad_epilogue_tile<GRAD_G>(t_row, static_cast<int>(ew >> 2), n0, p.N,
                                           m0 + static_cast<int>(quad * 32u), sxm, p.c_g, lane,
                                           2u + quad, s_out, &tmO, acc_row);
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive_remote(leader_tempty0 + 8u * buf);
            } else {
#pragma unroll 1
                for (int c = 0; c < C::EPI_COLS; c += 32) {
                    const int cc = col_base + c;
                    const int nc = n0 + cc;
                    if (nc >= p.N)
                        break;  // warp-uniform
                    uint32_t acc[32];
                    tmem_ld_32x32b_x32(t_row + cc, acc);
                    tmem_ld_wait();
                    uint32_t ob[16];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 w = lds_v4(s_sw + 4 * (c + 4 * q));
                        const float4 b = lds_v4(s_bias + 4 * (c + 4 * q));
                        const float wv[4] = {w.x, w.y, w.z, w.w};
                        const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int j = 4 * q + 2 * h;
                            // the same fp32 steps as the single-SM epilogue: t in f32x2, the
                            // products that feed an add as scalar intrinsics
                            float t0, t1;
                            mul2(t0, t1, sxm, sxm, wv[2 * h], wv[2 * h + 1]);
                            const float a0 = FP8 ? __uint_as_float(acc[j]) : __int2float_rn(static_cast<int>(acc[j]));
                            const float a1 = FP8 ? __uint_as_float(acc[j + 1])
                                                 : __int2float_rn(static_cast<int>(acc[j + 1]));
                            float v0 = __fmul_rn(a0, t0);
                            float v1 = __fmul_rn(a1, t1);
                            if (has_bias) {
                                v0 = __fadd_rn(v0, bv[2 * h]);
                                v1 = __fadd_rn(v1, bv[2 * h + 1]);
                            }
                            const __nv_bfloat162 h2 = __floats2bfloat162_rn(v0, v1);
                            ob[j >> 1] = *reinterpret_cast<const uint32_t *>(&h2);
                        }
                    }
                    if constexpr (GELU) {
                        gelu_bf16x16_lut(ob, lut);
                        gelu_bf16x16_lut(ob + 8, lut);
                        store_block16(ob, s_out, lane, &tmO, nc, m0 + static_cast<int>(quad * 32u));
                        store_block16(ob + 8, s_out, lane, &tmO, nc + 16, m0 + static_cast<int>(quad * 32u));
                    } else {
                        store_block(ob, s_out, lane, &tmO, nc, m0 + static_cast<int>(quad * 32u));
                    }
                    if (p.acc_out != nullptr && row_ok) {
                        int32_t *arow = p.acc_out + static_cast<int64_t>(m) * p.N;
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (nc + j < p.N)
                                arow[nc + j] = static_cast<int32_t>(acc[j]);
                    }
                }
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive_remote(leader_tempty0 + 8u * buf);
                    if (FUSE_G > 0)
                        mbar_arrive(sxempty_bar(buf));
                }
            }
        }
        if (lane == 0)
            bulk_wait_all();
    }

    // neither CTA frees its tensor memory or shared memory while the pair's MMAs may still
    // use them: rank 0's MMA warp has drained every MMA before it arrives here
    tc_fence_before_sync();
    __syncthreads();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    }
}

} // namespace sdnq
