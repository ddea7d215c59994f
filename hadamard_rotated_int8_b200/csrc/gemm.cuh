// INT8 x INT8 -> INT32 matmul on the 5th-generation tensor cores (tcgen05.mma kind::i8,
// accumulators in tensor memory), fed by TMA through a shared-memory ring, with the fp32
// de-quant epilogue fused: out = bf16(float(acc) * (sx[m] * sw[n]) + bias[n]
// [+ lora_scale * L[m][n]]), where L = u B is a second, bf16 x bf16 -> fp32 tensor-core
// accumulator (the PEFT adapter beside the frozen int8 base). With GELU the epilogue
// then applies the exact-erf GELU to that bf16 value and rounds once more to bf16, which is
// bit for bit the separate GELU pass of a DiT MLP's up-projection output.
//
// Sources: "SDNQ: SD.Next Quantization Engine" README, feature list (INT8 quantized matmul)
// and SDNQConfig (dequantize_fp32: FP32 scales and FP32 de-quant steps); "ConvRot / Hadamard
// SDNQ", PEFT Behavior (int8 frozen base, bf16 adapters).
//
// Shape of the kernel (one CTA per SM, persistent over output tiles):
//   warp 0      TMA producer (one lane): A tile [128 x 128 B], B tile [BN x 128 B] per stage
//   warp 1      TMEM allocator and MMA issuer (one lane): 4 MMAs of K = 32 per stage
//   warps 2..9  epilogue: TMEM -> registers -> scales, bias, LoRA -> bf16 -> global. A warp
//               may only read the TMEM lanes 32*(warp % 4) .. +31, so two warps share each
//               lane quarter and split the tile's columns in halves.
// Two accumulator buffers in TMEM let the epilogue of tile i overlap the MMAs of tile i+1
// (one buffer when a tile's accumulators fill all 512 columns, as with LoRA at N = 256).
// Operand tiles use the 128-byte swizzle written by TMA and read by the MMA descriptors.
// Further modes: the input gradient (N-major B, an inverse-butterfly epilogue), FP8 operands
// (kind::f8f6f4, fp32 accumulators) and the activation quantizer inside the kernel (extra
// warps that quantize x into the A operand and publish rows to the producers).
// Launched programmatically: the prologue may overlap the kernel before it in the stream,
// and every thread waits (griddepcontrol.wait) before it touches global memory.
//
// Every wait is bounded (mbar_wait_bounded): on timeout the CTA raises its abort flag and
// the device error word, each role leaves its loop, in-flight copies and MMAs are drained
// with bounded waits, and TMEM is freed before the CTA exits.
#pragma once

#include <cuda_bf16.h>

#include "device.cuh"
#include "gelu.cuh"
#include "rotquant.cuh"

#ifndef SDNQ_FUSED_QUANT_WARPS
#define SDNQ_FUSED_QUANT_WARPS 8
#endif

namespace sdnq {

struct GemmParams {
    const float *sx;          // [M]
    const float *sw;          // [N]
    const uint16_t *bias;     // [N] bf16 or nullptr
    uint16_t *out;            // [M, ldo] bf16
    int64_t ldo;
    int32_t *acc_out;         // [M, N] int32 or nullptr
    int32_t M, N, K;
    int32_t num_kb;           // ceil(K / 128)
    int32_t num_m_blocks;     // ceil(M / 128)
    int32_t num_tiles;
    int32_t lora_chunks;      // ceil(rank / 64); 0 without LoRA
    float lora_scale;
    float c_g;                // input-gradient mode: fp32(1/sqrt(g))
    uint64_t timeout_ns;
    // fused activation quantizer: rq quantizes x into the A operand (rq.q) and its scales
    // (rq.s, = sx); sync holds 2 * num_m_blocks counters, zero on entry and on exit
    RotquantParams rq;
    uint32_t *sync;
    int32_t num_n_blocks;
};

template <int BN, bool LORA, bool GELU = false, bool FUSE = false>
struct GemmConfig {
    static constexpr int BM = 128;
    static constexpr int BK = 128;                     // bytes of K per stage (int8)
    static constexpr int A_BYTES = BM * BK;            // 16 KB
    static constexpr int B_BYTES = BN * BK;            // 16 or 32 KB
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES = (BN == 256) ? 4 : 6;
    static constexpr int ACC_COLS = LORA ? 2 * BN : BN;   // TMEM columns per buffer
    static constexpr int NBUF = 512 / ACC_COLS >= 2 ? 2 : 1;  // accumulator buffers
    static constexpr int TMEM_COLS = NBUF * ACC_COLS;
    static constexpr int QUANT_WARPS = FUSE ? SDNQ_FUSED_QUANT_WARPS : 0;  // fused quantizer
    static constexpr int THREADS = 320 + 32 * (FUSE ? QUANT_WARPS + 1 : 0);  // 2 + 8 (+ 8 + 1) warps
    static constexpr int EPI_WARPS = 8;
    static constexpr int EPI_COLS = BN / 2;           // columns per epilogue warp
    // per epilogue warp: an output staging block [32 rows x 32 bf16] written with the
    // 64-byte swizzle for the TMA store, and its columns' scales and bias as fp32
    static constexpr int STAGE_OUT_BYTES = 32 * 64;
    static constexpr int OUT_OFF = STAGES * STAGE_BYTES;
    static constexpr int SCALE_OFF = OUT_OFF + EPI_WARPS * STAGE_OUT_BYTES;
    static constexpr int SCALE_BYTES = EPI_COLS * 8;  // sw[EPI_COLS], bias[EPI_COLS]
    static constexpr int LUT_OFF = SCALE_OFF + EPI_WARPS * SCALE_BYTES;  // GELU table
    static constexpr int LUT_BYTES = GELU ? kGeluLutBytes : 0;
    static constexpr int SX_OFF = LUT_OFF + LUT_BYTES;    // fused: row scales per buffer
    static constexpr int SX_BYTES = FUSE ? 2 * 128 * 4 : 0;
    static constexpr int AMAX_OFF = SX_OFF + SX_BYTES;     // fused: quantizer row maxima
    static constexpr int AMAX_BYTES = FUSE ? 2 * QUANT_WARPS * 4 : 0;
    static constexpr int BAR_OFF = AMAX_OFF + AMAX_BYTES;
    // barriers: full[S], empty[S], tfull[2], tempty[2], drain, sxfull[2]; then tmem base +
    // abort flag
    static constexpr int BAR_BYTES = (2 * STAGES + 7) * 8;
    static constexpr int SMEM_BYTES = 1024 /*align slack*/ + BAR_OFF + BAR_BYTES + 16;
    static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
    static_assert(TMEM_COLS <= 512, "tensor memory holds 512 columns");
    static_assert(BN % 32 == 0 && BN >= 64 && BN <= 256, "tile width");
};

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) { return __uint_as_float(b << 16); }

// One output block: 16 packed bf16 pairs (32 columns) of this thread's row go through the
// warp's 64-byte-swizzled staging buffer to a TMA store of the warp's 32 x 32 block at
// (column nc, row mrow0); rows >= M and columns >= N fall outside the tensor and are dropped.
__device__ __forceinline__ void store_block(const uint32_t (&ob)[16], uint32_t s_out, uint32_t lane,
                                            const CUtensorMap *tmO, int nc, int mrow0)
{
    if (lane == 0)
        bulk_wait_read_all();  // the previous block has left the staging buffer
    __syncwarp();
    const uint32_t row_addr = s_out + lane * 64u;
#pragma unroll
    for (int q = 0; q < 4; ++q)
        sts_v4(row_addr + ((static_cast<uint32_t>(q) ^ ((lane >> 1) & 3u)) << 4), ob[4 * q],
               ob[4 * q + 1], ob[4 * q + 2], ob[4 * q + 3]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d(tmO, s_out, nc, mrow0);
        bulk_commit_group();
    }
}

// ---- input-gradient epilogue: dx = bf16(FWHT_G(fp32(acc) * s_g) * fp32(1/sqrt(G))) ----

// Butterfly stages h = 1 .. GA/2 over 32 consecutive columns held in registers. Stage 1 adds
// products, so it uses scalar adds (an f32x2 add fed by a product may be merged with it
// into a multiply-add); the later stages add sums and use f32x2 pairs.
template <int GA>
__device__ __forceinline__ void butterfly32(float (&v)[32])
{
    if (GA > 1) {
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
            const float a = v[i], b = v[i + 1];
            v[i] = __fadd_rn(a, b);
            v[i + 1] = __fsub_rn(a, b);
        }
    }
#pragma unroll
    for (int h = 2; h < GA; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
            if ((i & h) == 0) {
                float s0, s1, d0, d1;
                add2(s0, s1, v[i], v[i + 1], v[i + h], v[i + h + 1]);
                sub2(d0, d1, v[i], v[i + 1], v[i + h], v[i + h + 1]);
                v[i] = s0; v[i + 1] = s1; v[i + h] = d0; v[i + h + 1] = d1;
            }
        }
    }
}

__device__ __forceinline__ void pack_scaled_bf16(const float (&z)[32], float c_g, uint32_t (&ob)[16])
{
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
        float a, b;
        mul2(a, b, z[i], z[i + 1], c_g, c_g);  // feeds no add
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(a, b);
        ob[i >> 1] = *reinterpret_cast<const uint32_t *>(&h2);
    }
}

// One 128 x 256 accumulator tile; this warp owns TMEM lanes 32*quad.. (one row per thread)
// and, in passes 1 and 3, the columns [128*half, 128*half + 128). Groups of G columns never
// straddle tiles (G divides 256) and never straddle N (N % G == 0).
//   pass 1: v = fp32(acc) * s_g and the stages h < 32 inside each 32-column load (for
//           G <= 32 that is the whole transform and the block goes straight out);
//   pass 2: stages h = 32 .. G/2 across the 32-column blocks, 4 columns of every block at a
//           time, the warp pair splitting the columns; results go back to TMEM;
//   pass 3: times 1/sqrt(G), bf16, TMA store.
// Passes exchange columns with the partner warp through TMEM: each ends with wait::st and a
// barrier of the pair (named barrier `pair_bar`, 64 threads).
template <int G>
__device__ __forceinline__ void grad_epilogue_tile(uint32_t t_row, int half, int n0, int N,
                                                   int mrow0, float sg, float c_g, uint32_t lane,
                                                   uint32_t pair_bar, uint32_t s_out,
                                                   const CUtensorMap *tmO, int32_t *acc_row)
{
    constexpr int GA = G < 32 ? G : 32;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
        const int cc = half * 128 + c * 32;
        if (n0 + cc >= N)
            break;  // warp-uniform
        uint32_t a[32];
        tmem_ld_32x32b_x32(t_row + cc, a);
        tmem_ld_wait();
        if (acc_row != nullptr) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (n0 + cc + j < N)
                    acc_row[n0 + cc + j] = static_cast<int32_t>(a[j]);
        }
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i)
            v[i] = __fmul_rn(__int2float_rn(static_cast<int>(a[i])), sg);
        butterfly32<GA>(v);
        if constexpr (G <= 32) {
            uint32_t ob[16];
            pack_scaled_bf16(v, c_g, ob);
            store_block(ob, s_out, lane, tmO, n0 + cc, mrow0);
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
                a[i] = __float_as_uint(v[i]);
            tmem_st_32x32b_x32(t_row + cc, a);
        }
    }
    if constexpr (G > 32) {
        tmem_st_wait();
        tc_fence_before_sync();
        bar_sync_or(pair_bar, 64, false);
        tc_fence_after_sync();
#pragma unroll 1
        for (int jb = 0; jb < 4; ++jb) {
            const int j0 = half * 16 + jb * 4;
            uint32_t r[8][4];
#pragma unroll
            for (int c = 0; c < 8; ++c)
                tmem_ld_32x32b_x4(t_row + c * 32 + j0, r[c]);
            tmem_ld_wait();
            float w[8][4];
#pragma unroll
            for (int c = 0; c < 8; ++c)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    w[c][j] = __uint_as_float(r[c][j]);
#pragma unroll
            for (int d = 1; 32 * d < G; d <<= 1) {
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    if ((c & d) == 0) {
#pragma unroll
                        for (int j = 0; j < 4; j += 2) {
                            float s0, s1, d0, d1;
                            add2(s0, s1, w[c][j], w[c][j + 1], w[c + d][j], w[c + d][j + 1]);
                            sub2(d0, d1, w[c][j], w[c][j + 1], w[c + d][j], w[c + d][j + 1]);
                            w[c][j] = s0; w[c][j + 1] = s1; w[c + d][j] = d0; w[c + d][j + 1] = d1;
                        }
                    }
                }
            }
#pragma unroll
            for (int c = 0; c < 8; ++c) {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    r[c][j] = __float_as_uint(w[c][j]);
                tmem_st_32x32b_x4(t_row + c * 32 + j0, r[c]);
            }
        }
        tmem_st_wait();
        tc_fence_before_sync();
        bar_sync_or(pair_bar, 64, false);
        tc_fence_after_sync();
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            const int cc = half * 128 + c * 32;
            if (n0 + cc >= N)
                break;
            uint32_t a[32];
            tmem_ld_32x32b_x32(t_row + cc, a);
            tmem_ld_wait();
            float z[32];
#pragma unroll
            for (int i = 0; i < 32; ++i)
                z[i] = __uint_as_float(a[i]);
            uint32_t ob[16];
            pack_scaled_bf16(z, c_g, ob);
            store_block(ob, s_out, lane, tmO, n0 + cc, mrow0);
        }
    }
}

template <int BN, bool LORA, bool GELU, int GRAD_G, int FUSE_G, bool FP8 = false>
__global__ void __launch_bounds__(GemmConfig<BN, LORA, GELU, (FUSE_G > 0)>::THREADS, 1)
    gemm_s8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmL,
                   const __grid_constant__ CUtensorMap tmO, const GemmParams p)
{
    using C = GemmConfig<BN, LORA, GELU, (FUSE_G > 0)>;
    static_assert(FUSE_G == 0 || (BN == 256 && !LORA && !GELU && GRAD_G == 0),
                  "fused activation quantizer: plain forward tiles of 256 columns");
    static_assert(!FP8 || (!LORA && !GELU && GRAD_G == 0 && FUSE_G == 0),
                  "e4m3 operands: the plain forward kernel");
    static_assert(GRAD_G == 0 || (BN == 256 && !LORA && !GELU && (GRAD_G & (GRAD_G - 1)) == 0 &&
                                  GRAD_G <= 256),
                  "input-gradient mode: plain tiles of 256 columns, G divides 256");
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment for the 128-byte swizzle atoms
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
    float *sx_smem = reinterpret_cast<float *>(smem + C::SX_OFF);     // [2][128], fused only
    float *amax_smem = reinterpret_cast<float *>(smem + C::AMAX_OFF); // [2][8], fused only
    // tile -> (m block, n block): m fastest; n fastest with the fused quantizer, whose row
    // blocks become ready in order
    auto tile_mb = [&](int tile) { return FUSE_G > 0 ? tile / p.num_n_blocks : tile % p.num_m_blocks; };
    auto tile_nb = [&](int tile) { return FUSE_G > 0 ? tile % p.num_n_blocks : tile / p.num_m_blocks; };
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::BAR_OFF + C::BAR_BYTES);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const uint32_t warp = threadIdx.x >> 5;
    const uint32_t lane = lane_id();

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < C::NBUF; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), C::EPI_WARPS);
        }
        mbar_init(drain_bar, 1);
        if (FUSE_G > 0)
            for (int b = 0; b < C::NBUF; ++b)
                mbar_init(sxfull_bar(b), 1);
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
        tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_holder;
    // the prologue above may overlap the previous kernel (programmatic launch); from here on
    // the codes, scales and LoRA terms it wrote are read
    grid_dependency_wait();

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            bool ok = true;
            int local = 0;
            for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x, ++local) {
                const int m0 = tile_mb(tile) * C::BM;
                const int n0 = tile_nb(tile) * BN;
                if constexpr (FUSE_G > 0) {
                    // the scale warp has seen the tile's activation rows published (and copied
                    // their scales); order that before the TMA engine reads the rows
                    const int buf = local % C::NBUF;
                    const uint32_t use = static_cast<uint32_t>(local / C::NBUF);
                    if (!mbar_wait_bounded(sxfull_bar(buf), use & 1u, abort, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    fence_proxy_async_global();
                }
                const int steps = p.num_kb + (LORA ? p.lora_chunks : 0);
                for (int kb = 0; kb < steps; ++kb) {
                    if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    const uint32_t sa = base + stage * C::STAGE_BYTES;
                    const uint32_t sb = sa + C::A_BYTES;
                    if (!LORA || kb < p.num_kb) {
                        mbar_arrive_expect_tx(full_bar(stage), C::STAGE_BYTES);
                        tma_load_2d(sa, &tmA, full_bar(stage), kb * C::BK, m0);
                        if constexpr (GRAD_G > 0) {
                            // B = qW rows kb*128.. (the contraction) x columns n0.. (N-major),
                            // as two 128-column boxes
                            tma_load_2d(sb, &tmB, full_bar(stage), n0, kb * C::BK);
                            tma_load_2d(sb + 16384, &tmB, full_bar(stage), n0 + 128, kb * C::BK);
                        } else {
                            tma_load_2d(sb, &tmB, full_bar(stage), kb * C::BK, n0);
                        }
                    } else {
                        // LoRA chunk c: U [128 x 64] bf16 (K-major) into the A slot and
                        // B [64 x BN] bf16 (N-major) as BN/64 boxes into the B slot
                        const int c = kb - p.num_kb;
                        mbar_arrive_expect_tx(full_bar(stage), 128 * 128 + BN * 128);
                        tma_load_2d(sa, &tmU, full_bar(stage), c * 64, m0);
#pragma unroll
                        for (int j = 0; j < BN / 64; ++j)
                            tma_load_2d(sb + j * 8192, &tmL, full_bar(stage), n0 + 64 * j, c * 64);
                    }
                    ++issued;
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                // drain: wait (bounded) for the copies of the last stages issued
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
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC_I8 = FP8 ? idesc_e4m3_f32(128, BN) : idesc_s8_s32(128, BN, GRAD_G > 0);
            constexpr uint32_t IDESC_BF = idesc_bf16_f32(128, BN, true);
            int stage = 0;
            uint32_t phase = 0;
            int local = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x, ++local) {
                const int buf = local % C::NBUF;
                const uint32_t use = static_cast<uint32_t>(local / C::NBUF);
                if (!mbar_wait_bounded(tempty_bar(buf), (use & 1u) ^ 1u, abort, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_acc = tmem_base + buf * C::ACC_COLS;
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    if (!mbar_wait_bounded(full_bar(stage), phase, abort, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t sa = base + stage * C::STAGE_BYTES;
                    const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
                    for (int k = 0; k < C::BK / 32; ++k) {
                        // K = 32 per MMA: 32 bytes along A's swizzled rows; for the N-major B
                        // of the input gradient, 32 K-rows of 128 bytes = 4096 bytes
                        const uint64_t bdesc = GRAD_G > 0 ? mnmajor_desc(sb + 4096 * k, 16384)
                                                          : kmajor_desc(sb + 32 * k);
                        if constexpr (FP8)
                            mma_f8(d_acc, kmajor_desc(sa + 32 * k), bdesc, IDESC_I8,
                                   (kb | k) != 0 ? 1u : 0u);
                        else
                            mma_s8(d_acc, kmajor_desc(sa + 32 * k), bdesc, IDESC_I8,
                                   (kb | k) != 0 ? 1u : 0u);
                    }
                    tc_commit(empty_bar(stage));
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (LORA) {
                    const uint32_t d_lora = d_acc + BN;
                    for (int c = 0; ok && c < p.lora_chunks; ++c) {
                        if (!mbar_wait_bounded(full_bar(stage), phase, abort, p.timeout_ns)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after_sync();
                        const uint32_t sa = base + stage * C::STAGE_BYTES;
                        const uint32_t sb = sa + C::A_BYTES;
                        // 4 MMAs of K = 16 rows of rank each: A advances 32 bytes along its
                        // swizzled K-major rows, B advances 16 K-rows = 2048 bytes
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            mma_f16(d_lora, kmajor_desc(sa + 32 * k), mnmajor_desc(sb + 2048 * k, 8192),
                                    IDESC_BF, (c | k) != 0 ? 1u : 0u);
                        tc_commit(empty_bar(stage));
                        if (++stage == C::STAGES) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                }
                if (!ok)
                    break;
                tc_commit(tfull_bar(buf));
            }
            // drain: every MMA this thread issued has completed before TMEM is freed
            tc_commit(drain_bar);
            volatile int no_abort = 0;
            mbar_wait_bounded(drain_bar, 0u, &no_abort, p.timeout_ns);
        }
    } else if (FUSE_G > 0 && warp == 10 + C::QUANT_WARPS) {
        // ------------------------------------------------------------ scale warp (fused)
        // Per tile of this CTA, ahead of the producer: wait (bounded, acquire) until the
        // tile's 128 activation rows are published, count this CTA as one of the block's
        // readers (the last one clears the block's counters for the next launch), wait until
        // the epilogue has released the buffer's scales, copy the rows' scales to shared
        // memory and arrive on sxfull, which both the producer and the epilogue wait for.
        if constexpr (FUSE_G > 0) {
            int local = 0;
            for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++local) {
                const int mb = tile_mb(tile);
                const int m0 = mb * C::BM;
                const int buf = local % C::NBUF;
                const uint32_t use = static_cast<uint32_t>(local / C::NBUF);
                const uint32_t rows = static_cast<uint32_t>(p.M - m0 < 128 ? p.M - m0 : 128);
                bool good = true;
                if (lane == 0) {
                    good = wait_count_bounded(p.sync + mb, rows * static_cast<uint32_t>(p.rq.wpr),
                                              abort, p.timeout_ns);
                    if (good) {
                        const uint32_t seen = atomicAdd(p.sync + p.num_m_blocks + mb, 1u);
                        if (seen == static_cast<uint32_t>(p.num_n_blocks) - 1u) {
                            p.sync[mb] = 0u;
                            p.sync[p.num_m_blocks + mb] = 0u;
                        }
                        good = mbar_wait_bounded(tempty_bar(buf), (use & 1u) ^ 1u, abort,
                                                 p.timeout_ns);
                    }
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
    } else if (FUSE_G > 0 && warp >= 10) {
        // ------------------------------------------------------------ activation quantizer
        // (warps 10..17): rows of x -> rotated int8 codes (the A operand) and their scales,
        // published per 128-row block for the scale warps of every CTA
        if constexpr (FUSE_G > 0)
            rotquant_worker_rows<FUSE_G>(p.rq, static_cast<int32_t>(warp) - 10, C::QUANT_WARPS, 6u,
                                         amax_smem, p.sync);
    } else {
        // ------------------------------------------------------------ epilogue (warps 2..9)
        const uint32_t quad = warp & 3u;  // TMEM lanes this warp may access: 32*quad ..
        const uint32_t ew = warp - 2u;    // epilogue warp index 0..7
        const int col_base = static_cast<int>(ew >> 2) * C::EPI_COLS;
        const int row_in_tile = static_cast<int>(quad * 32u + lane);
        const uint32_t s_out = base + C::OUT_OFF + ew * C::STAGE_OUT_BYTES;
        const uint32_t s_sw = base + C::SCALE_OFF + ew * C::SCALE_BYTES;
        const uint32_t s_bias = s_sw + C::EPI_COLS * 4;
        const bool has_bias = p.bias != nullptr;
        uint16_t *lut = reinterpret_cast<uint16_t *>(smem + C::LUT_OFF);
        if constexpr (GELU) {
            // the GELU table (built once per device), while the first tile's operands load
            gelu_lut_load(lut, static_cast<int>(ew * 32u + lane), 32 * C::EPI_WARPS);
            bar_sync_or(1, 32 * C::EPI_WARPS, false);  // epilogue warps only
        }
        int local = 0;
        for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++local) {
            const int buf = local % C::NBUF;
            const uint32_t use = static_cast<uint32_t>(local / C::NBUF);
            const int m0 = tile_mb(tile) * C::BM;
            const int n0 = tile_nb(tile) * BN;
            const int nw = n0 + col_base;     // first column of this warp
            // this warp's column scales and bias -> shared memory (fp32), before the wait
            // on the accumulator so that their latency overlaps the MMAs
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
            // warp-uniform decision: tcgen05.ld below needs the whole warp converged
            const bool ready = mbar_wait_bounded(tfull_bar(buf), use & 1u, abort, p.timeout_ns);
            if constexpr (GRAD_G > 0) {
                // the warp pair leaves together: it meets at named barriers inside the tile
                if (bar_sync_or(2u + quad, 64, !__all_sync(0xffffffffu, ready)))
                    break;
            } else {
                if (!__all_sync(0xffffffffu, ready))
                    break;
            }
            tc_fence_after_sync();
            const int m = m0 + row_in_tile;
            const bool row_ok = m < p.M;
            float sxm;
            if constexpr (FUSE_G > 0) {
                // the row scales the producer copied once the rows were published
                const bool got = mbar_wait_bounded(sxfull_bar(buf), use & 1u, abort, p.timeout_ns);
                if (!__all_sync(0xffffffffu, got))
                    break;
                sxm = row_ok ? sx_smem[buf * 128 + row_in_tile] : 0.0f;
            } else {
                sxm = row_ok ? p.sx[m] : 0.0f;
            }
            const uint32_t t_row = tmem_base + ((quad * 32u) << 16) + buf * C::ACC_COLS;
            if constexpr (GRAD_G > 0) {
                int32_t *acc_row = (p.acc_out != nullptr && row_ok)
                                       ? p.acc_out + static_cast<int64_t>(m) * p.N : nullptr;
                grad_epilogue_tile<GRAD_G>(t_row, static_cast<int>(ew >> 2), n0, p.N,
                                           m0 + static_cast<int>(quad * 32u), sxm, p.c_g, lane,
                                           2u + quad, s_out, &tmO, acc_row);
            }
#pragma unroll 1
            for (int c = 0; GRAD_G == 0 && c < C::EPI_COLS; c += 32) {
                const int cc = col_base + c;   // column inside the tile
                const int nc = n0 + cc;
                if (nc >= p.N)
                    break;  // warp-uniform
                uint32_t acc[32];
                tmem_ld_32x32b_x32(t_row + cc, acc);
                uint32_t lacc[LORA ? 32 : 1];
                if constexpr (LORA)
                    tmem_ld_32x32b_x32(t_row + BN + cc, lacc);
                tmem_ld_wait();
                // v = float(acc) * (sx * sw) [+ bias] [+ lora_scale * L], each op one fp32 rounding
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
                        // t in f32x2; the products that feed an add are scalar __fmul_rn /
                        // __fadd_rn, never merged into a multiply-add (a mul.rn.f32x2
                        // followed by an add.rn.f32x2 was observed to execute as one fused
                        // multiply-add, which differs from two roundings on ties)
                        float t0, t1;
                        mul2(t0, t1, sxm, sxm, wv[2 * h], wv[2 * h + 1]);
                        // accumulator: int32 (int8 operands) or fp32 bits (e4m3 operands)
                        const float a0 = FP8 ? __uint_as_float(acc[j]) : __int2float_rn(static_cast<int>(acc[j]));
                        const float a1 = FP8 ? __uint_as_float(acc[j + 1])
                                             : __int2float_rn(static_cast<int>(acc[j + 1]));
                        float v0 = __fmul_rn(a0, t0);
                        float v1 = __fmul_rn(a1, t1);
                        if (has_bias) {
                            v0 = __fadd_rn(v0, bv[2 * h]);
                            v1 = __fadd_rn(v1, bv[2 * h + 1]);
                        }
                        if constexpr (LORA) {
                            v0 = __fadd_rn(v0, __fmul_rn(p.lora_scale, __uint_as_float(lacc[j])));
                            v1 = __fadd_rn(v1, __fmul_rn(p.lora_scale, __uint_as_float(lacc[j + 1])));
                        }
                        const __nv_bfloat162 h2 = __floats2bfloat162_rn(v0, v1);
                        ob[j >> 1] = *reinterpret_cast<const uint32_t *>(&h2);
                    }
                }
                if constexpr (GELU) {
                    gelu_bf16x16_lut(ob, lut);
                    gelu_bf16x16_lut(ob + 8, lut);
                }
                store_block(ob, s_out, lane, &tmO, nc, m0 + static_cast<int>(quad * 32u));
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
            if (lane == 0)
                mbar_arrive(tempty_bar(buf));
        }
        if (lane == 0)
            bulk_wait_all();  // every output block is in global memory before the CTA exits
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

} // namespace sdnq
