// libsdnq.so: the C ABI declared in include/sdnq.h. Host side: argument validation, TMA
// tensor-map encoding, launch configuration and the device error word. All arithmetic of the
// layer runs in the kernels included below.
#include <cfloat>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "sdnq.h"

#include "device.cuh"
#include "gelu.cuh"
#include "gemm.cuh"
#include "gemm_pair.cuh"
#include "attention.cuh"
#include "lora_down.cuh"
#include "rotquant.cuh"

#define SDNQ_API extern "C" __attribute__((visibility("default")))

// Every entry point that validates and launches work opens an NVTX range named after itself,
// so that a profiler's timeline attributes kernels to the call that launched them. Without a
// profiler attached the push and pop do nothing.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};
#define SDNQ_NVTX_RANGE() NvtxRange sdnq_nvtx_range_(__func__)

namespace sdnq {
namespace {

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // 2 s for any single wait

// Tile width of the LoRA GEMM: 128 keeps two TMEM accumulator buffers (int32 + fp32 per
// tile), 256 uses one.
#ifndef SDNQ_LORA_BN
#define SDNQ_LORA_BN 256
#endif

// ---------------------------------------------------------------- device checks

struct DeviceInfo {
    int checked = 0;
    int supported = 0;
    int sm_count = 0;
    int index = 0;    // CUDA device ordinal
};
DeviceInfo g_dev[64];
std::mutex g_dev_mutex;

sdnq_status current_device(DeviceInfo *out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return SDNQ_ERR_UNSUPPORTED;  // no usable CUDA device: no sm_100 to run on
    }
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    DeviceInfo &d = g_dev[dev];
    if (!d.checked) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return SDNQ_ERR_CUDA;
        }
        d.supported = (major == 10 && minor == 0) ? 1 : 0;
        d.sm_count = sms;
        d.index = dev;
        d.checked = 1;
    }
    *out = d;
    return d.supported ? SDNQ_OK : SDNQ_ERR_UNSUPPORTED;
}

// ---------------------------------------------------------------- tensor maps

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        cudaGetLastError();
    });
    return fn;
}

// 2-D row-major tensor [outer, inner] with a row stride in bytes and swizzled boxes.
bool make_tmap_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *ptr, uint64_t inner,
                  uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                  CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_stride_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(map, dtype, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- validation helpers

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }

// A value computed once per (device, key) and cached: kernel attributes and occupancy are
// properties of a kernel on one device, so each device gets its own entry. Lookups and the
// first computation hold a lock (host threads may call the library concurrently).
template <int NKEYS>
struct PerDeviceCache {
    int value[64][NKEYS] = {};   // 0 = not computed yet
    std::mutex mutex;
    template <typename F>
    int get(int dev, int key, F compute)
    {
        std::lock_guard<std::mutex> lock(mutex);
        int &v = value[dev][key];
        if (v == 0)
            v = compute();
        return v;
    }
};

// Sets a kernel's dynamic shared-memory limit on the given (current) device, once per
// device. Returns false if the runtime refused it.
template <typename Kernel>
bool smem_attr_once(PerDeviceCache<1> &cache, int dev, Kernel k, int bytes)
{
    return cache.get(dev, 0, [&] {
               return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           bytes) == cudaSuccess ? 1 : -1;
           }) == 1;
}

sdnq_status launch_status()
{
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SDNQ_OK : SDNQ_ERR_CUDA;
}

// Programmatic launch (the kernel may start while the previous one in the stream drains; it
// waits with griddepcontrol.wait before touching memory). Errors are left for launch_status.
template <typename... KArgs, typename... Args>
void launch_programmatic(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                         cudaStream_t cs, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = cs;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, kernel, args...);
}

// ---------------------------------------------------------------- rotate + quantize

sdnq_status validate_rotquant(const void *x, int64_t rows, int64_t K, int64_t ld, int32_t group,
                              const void *q, const void *s)
{
    if (rows != 0 && (!x || !q || !s))  // an empty batch may come with NULL buffers
        return SDNQ_ERR_NULL;
    if (rows < 0 || rows > INT32_MAX || K <= 0 || K > SDNQ_MAX_K || K % 16 != 0 || ld < K)
        return SDNQ_ERR_SHAPE;
    if (!is_pow2(group) || group < SDNQ_MIN_GROUP || group > SDNQ_MAX_GROUP)
        return SDNQ_ERR_UNSUPPORTED;
    if (K % group != 0)
        return SDNQ_ERR_SHAPE;
    if (ld % 8 != 0 || !aligned(x, 16) || !aligned(q, 16) || !aligned(s, 4))
        return SDNQ_ERR_ALIGN;
    return SDNQ_OK;
}

// Rows of at most 16 chunks go to the persistent, prefetching kernel (grid = resident
// CTAs); longer rows to the two-pass kernel with one CTA per row.
// Block shape of the run-per-lane kernel: `warps` warps hold `rows` = floor(32 warps / rpr)
// rows of rpr runs of 64 elements. Small blocks keep more of them resident per SM, so that
// one block's row barrier overlaps the others' work (measured: 2-warp blocks beat 4- and
// 8-warp ones on 16384 x 4096); the shape is the smallest warp count in 2..16 that leaves at
// most a tenth of the lanes idle, else the one that leaves the fewest. rows == 0 means the
// row is too long for the kernel (rpr > 512).
struct RunShape {
    int warps = 0;
    int rows = 0;
};

RunShape run_shape(int64_t rpr)
{
    RunShape best;
    double best_used = -1.0;
    for (int w = 2; w <= 16; ++w) {
        const int64_t rows = 32 * w / rpr;
        if (rows < 1)
            continue;
        const double used = static_cast<double>(rows * rpr) / (32.0 * w);
        if (used >= 0.9)
            return RunShape{w, static_cast<int>(rows)};
        if (used > best_used + 1e-9) {
            best.warps = w;
            best.rows = static_cast<int>(rows);
            best_used = used;
        }
    }
    return best;
}

constexpr int kRunTransposeBytesPerWarp = 32 * 272;   // 32 owners x 17 units of 16 bytes

template <int G, bool FP8, bool V8>
void launch_rotquant_run(const RotquantParams &rp, const RunShape &shape, const DeviceInfo &dev,
                         cudaStream_t st)
{
    constexpr auto kernel = rotquant_run_kernel<G, FP8, V8>;
    const int threads = 32 * shape.warps;
    auto smem_for = [](int warps, int rows) {
        return (G >= 128 ? warps * kRunTransposeBytesPerWarp : 0) + 3 * rows * 4;
    };
    static PerDeviceCache<1> smem_attr;
    static PerDeviceCache<17> per_sm;   // resident blocks per SM, by warps per block
    if (!smem_attr_once(smem_attr, dev.index, kernel, smem_for(16, 512)))
        return;   // the launch below is then skipped; launch_status reports the error
    const int n_sm = per_sm.get(dev.index, shape.warps, [&] {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads,
                                                          smem_for(shape.warps, 32 * shape.warps)) !=
                cudaSuccess ||
            n < 1) {
            cudaGetLastError();
            n = 1;
        }
        return n;
    });
    RotquantRunParams p;
    p.x = rp.x;
    p.ldx = rp.ldx;
    p.q = rp.q;
    p.s = rp.s;
    p.M = rp.M;
    p.K = rp.K;
    p.rpr = (rp.K + 63) / 64;
    p.rows = shape.rows;
    p.c_g = rp.c_g;
    const int64_t blocks = (rp.M + shape.rows - 1) / shape.rows;
    const int64_t resident = static_cast<int64_t>(n_sm) * dev.sm_count;
    const unsigned grid = static_cast<unsigned>(blocks < resident ? blocks : resident);
    kernel<<<grid, threads, smem_for(shape.warps, shape.rows), st>>>(p);
}

// Rows of up to 512 runs (K <= 32768) go to the run-per-lane kernel; the column-multiplier
// mode (the input gradient's quantizer) to the chunk-per-warp persistent kernel for rows of
// at most 16 chunks; longer rows to the two-pass kernel with one block per row.
template <int G, bool COLSCALE = false, bool FP8 = false>
void launch_rotquant_g(const RotquantParams &p, dim3 grid, dim3 block, const DeviceInfo &dev,
                       cudaStream_t st)
{
    if constexpr (!COLSCALE) {
        const RunShape shape = run_shape((p.K + 63) / 64);
        if (shape.rows > 0) {
            const bool v8 = (reinterpret_cast<uintptr_t>(p.x) % 32) == 0 && (p.ldx % 16) == 0;
            if (v8)
                launch_rotquant_run<G, FP8, true>(p, shape, dev, st);
            else
                launch_rotquant_run<G, FP8, false>(p, shape, dev, st);
            return;
        }
    }
    if (p.nchunks <= 16) {
        // resident CTAs per SM, by device and warps per CTA
        static PerDeviceCache<33> per_sm;
        const int warps = static_cast<int>(block.x / 32);
        const int n_sm = per_sm.get(dev.index, warps, [&] {
            int n = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                    &n, rotquant_persistent_kernel<G, COLSCALE, FP8>, block.x, 0) != cudaSuccess ||
                n < 1) {
                cudaGetLastError();
                n = 1;
            }
            return n;
        });
        const int64_t groups = grid.x;
        const int64_t resident = static_cast<int64_t>(n_sm) * dev.sm_count;
        const dim3 pgrid(static_cast<unsigned>(groups < resident ? groups : resident));
        rotquant_persistent_kernel<G, COLSCALE, FP8><<<pgrid, block, 0, st>>>(p);
    } else {
        rotquant_kernel<G, COLSCALE, FP8><<<grid, block, 0, st>>>(p);
    }
}

// Per-row int8 quantization of rows x [rows, K] (validated by the caller): rotated by the
// block-diagonal Hadamard of `group` columns, or (group 1) multiplied by colscale[K].
sdnq_status launch_rowquant(const uint16_t *x, int64_t rows, int64_t K, int64_t ld,
                            int32_t group, const float *colscale, int8_t *q, float *s,
                            const DeviceInfo &dev, cudaStream_t cs, bool fp8 = false)
{
    RotquantParams p;
    p.x = x;
    p.ldx = ld;
    p.q = q;
    p.s = s;
    p.M = rows;
    p.K = static_cast<int32_t>(K);
    p.nchunks = static_cast<int32_t>((K + 1023) / 1024);
    p.wpr = p.nchunks < 16 ? p.nchunks : 16;  // <= 512 threads per CTA
    p.rpc = p.wpr <= 8 ? 8 / p.wpr : 1;
    p.c_g = static_cast<float>(1.0 / std::sqrt(static_cast<double>(group)));
    p.colscale = colscale;
    const dim3 block(32 * p.wpr * p.rpc);
    const dim3 grid(static_cast<unsigned>((rows + p.rpc - 1) / p.rpc));
    cudaGetLastError();
    if (fp8) {
        switch (group) {
        case 8: launch_rotquant_g<8, false, true>(p, grid, block, dev, cs); break;
        case 16: launch_rotquant_g<16, false, true>(p, grid, block, dev, cs); break;
        case 32: launch_rotquant_g<32, false, true>(p, grid, block, dev, cs); break;
        case 64: launch_rotquant_g<64, false, true>(p, grid, block, dev, cs); break;
        case 128: launch_rotquant_g<128, false, true>(p, grid, block, dev, cs); break;
        default: launch_rotquant_g<256, false, true>(p, grid, block, dev, cs); break;
        }
        return launch_status();
    }
    switch (group) {
    case 1: launch_rotquant_g<1, true>(p, grid, block, dev, cs); break;
    case 8: launch_rotquant_g<8>(p, grid, block, dev, cs); break;
    case 16: launch_rotquant_g<16>(p, grid, block, dev, cs); break;
    case 32: launch_rotquant_g<32>(p, grid, block, dev, cs); break;
    case 64: launch_rotquant_g<64>(p, grid, block, dev, cs); break;
    case 128: launch_rotquant_g<128>(p, grid, block, dev, cs); break;
    default: launch_rotquant_g<256>(p, grid, block, dev, cs); break;
    }
    return launch_status();
}

sdnq_status run_rotquant(const uint16_t *x, int64_t rows, int64_t K, int64_t ld, int32_t group,
                         int8_t *q, float *s, void *stream)
{
    sdnq_status st = validate_rotquant(x, rows, K, ld, group, q, s);
    if (st != SDNQ_OK)
        return st;
    DeviceInfo dev;
    if ((st = current_device(&dev)) != SDNQ_OK)
        return st;
    if (rows == 0)
        return SDNQ_OK;
    return launch_rowquant(x, rows, K, ld, group, nullptr, q, s, dev,
                           static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------- int8 linear (+ LoRA)

sdnq_status validate_linear(const void *qx, const void *sx, const void *qW, const void *sW,
                            const void *bias, int64_t M, int64_t N, int64_t K, const void *out,
                            int64_t ldo, const void *acc_out)
{
    if (!qW || !sW || (M != 0 && (!qx || !sx || !out)))  // empty batch: NULL row buffers ok
        return SDNQ_ERR_NULL;
    if (M < 0 || M > INT32_MAX || N <= 0 || N > INT32_MAX || K < 16 || K > SDNQ_MAX_K ||
        K % 16 != 0 || ldo < N)
        return SDNQ_ERR_SHAPE;
    if (ldo % 8 != 0 || !aligned(qx, 16) || !aligned(qW, 16) || !aligned(out, 16) ||
        !aligned(sx, 4) || !aligned(sW, 16) || (bias && !aligned(bias, 16)) ||
        (acc_out && !aligned(acc_out, 16)))
        return SDNQ_ERR_ALIGN;
    return SDNQ_OK;
}

// GRAD_G > 0: the input gradient's NN product, out [M, N] = epilogue(A [M, K] x W [K, N]),
// with W = the weight codes qW [N_out = K rows, K_in = N columns] read N-major.
// FUSE_G > 0: the activation quantizer runs inside the kernel (p.rq, p.sync set by the
// caller); the grid is launched cooperatively so that every CTA is resident, because the
// producers of one CTA wait for rows that the quantizer warps of others publish.
template <int BN, bool LORA, bool GELU = false, int GRAD_G = 0, int FUSE_G = 0, bool FP8 = false>
sdnq_status launch_gemm(const DeviceInfo &dev, const int8_t *qx, const int8_t *qW,
                        const uint16_t *u, const uint16_t *B, int32_t rank, GemmParams p,
                        cudaStream_t cs)
{
    using C = GemmConfig<BN, LORA, GELU, (FUSE_G > 0)>;
    constexpr auto kernel = gemm_s8_kernel<BN, LORA, GELU, GRAD_G, FUSE_G, FP8>;
    CUtensorMap tmA, tmB, tmU, tmL, tmO;
    const bool b_ok = GRAD_G > 0
                          ? make_tmap_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, qW, p.N, p.K, p.N, 128, 128)
                          : make_tmap_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, qW, p.K, p.N, p.K, 128, BN);
    if (!make_tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, qx, p.K, p.M, p.K, 128, 128) || !b_ok ||
        !make_tmap_2d(&tmO, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.out, p.N, p.M, 2ull * p.ldo, 32, 32,
                      CU_TENSOR_MAP_SWIZZLE_64B))
        return SDNQ_ERR_CUDA;
    if (LORA) {
        if (!make_tmap_2d(&tmU, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, u, rank, p.M, 2ull * rank, 64, 128) ||
            !make_tmap_2d(&tmL, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, p.N, rank, 2ull * p.N, 64, 64))
            return SDNQ_ERR_CUDA;
    } else {
        tmU = tmA;
        tmL = tmA;
    }
    static PerDeviceCache<1> smem_attr;
    if (!smem_attr_once(smem_attr, dev.index, kernel, C::SMEM_BYTES))
        return SDNQ_ERR_CUDA;
    p.num_kb = (p.K + C::BK - 1) / C::BK;
    p.num_m_blocks = (p.M + C::BM - 1) / C::BM;
    p.num_n_blocks = (p.N + BN - 1) / BN;
    p.num_tiles = p.num_m_blocks * p.num_n_blocks;
    const int grid = p.num_tiles < dev.sm_count ? p.num_tiles : dev.sm_count;
    cudaGetLastError();
    if constexpr (FUSE_G > 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(grid));
        cfg.blockDim = dim3(C::THREADS);
        cfg.dynamicSmemBytes = C::SMEM_BYTES;
        cfg.stream = cs;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, kernel, tmA, tmB, tmU, tmL, tmO, p) != cudaSuccess) {
            cudaGetLastError();
            return SDNQ_ERR_CUDA;
        }
    } else {
        // programmatic launch: the prologue overlaps the tail of the kernel before it (the
        // quantizer), whose results the kernel reads only after griddepcontrol.wait
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(grid));
        cfg.blockDim = dim3(C::THREADS);
        cfg.dynamicSmemBytes = C::SMEM_BYTES;
        cfg.stream = cs;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, kernel, tmA, tmB, tmU, tmL, tmO, p) != cudaSuccess) {
            cudaGetLastError();
            return SDNQ_ERR_CUDA;
        }
    }
    return launch_status();
}

// The CTA-pair kernel (cta_group::2, 256 x 256 tiles) for the plain, GELU and e4m3 linears.
// A cluster of two CTAs per pair, launched programmatically like the single-SM kernel; the
// grid holds as many pairs as the device can keep resident at once (or fewer, one per
// tile), each walking the tiles persistently.
template <bool GELU, bool FP8, bool LORA = false, int FUSE_G = 0, int GRAD_G = 0>
sdnq_status launch_gemm_pair(const DeviceInfo &dev, const int8_t *qx, const int8_t *qW,
                             GemmParams p, cudaStream_t cs, const uint16_t *u = nullptr,
                             const uint16_t *B = nullptr, int32_t rank = 0)
{
    using C = PairConfig<GELU, LORA, (FUSE_G > 0)>;
    constexpr auto kernel = gemm_s8_pair_kernel<GELU, FP8, LORA, FUSE_G, GRAD_G>;
    CUtensorMap tmA, tmB, tmU, tmL, tmO;
    if (!make_tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, qx, p.K, p.M, p.K, 128, 128) ||
        !(GRAD_G > 0
              // the input gradient reads qW [contraction rows, output columns] N-major: boxes
              // of this CTA's 128 columns x 128 contraction rows
              ? make_tmap_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, qW, p.N, p.K, p.N, C::BN / 2, 128)
              : make_tmap_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, qW, p.K, p.N, p.K, 128, C::BN / 2)) ||
        !make_tmap_2d(&tmO, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.out, p.N, p.M, 2ull * p.ldo,
                      C::OUT_COLS, 32,
                      C::OUT_COLS == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE))
        return SDNQ_ERR_CUDA;
    if (LORA) {
        if (!make_tmap_2d(&tmU, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, u, rank, p.M, 2ull * rank, 64, 128) ||
            !make_tmap_2d(&tmL, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, p.N, rank, 2ull * p.N, 64, 64))
            return SDNQ_ERR_CUDA;
    } else {
        tmU = tmA;
        tmL = tmA;
    }
    static PerDeviceCache<1> smem_attr;
    if (!smem_attr_once(smem_attr, dev.index, kernel, C::SMEM_BYTES))
        return SDNQ_ERR_CUDA;
    p.num_kb = (p.K + C::BK - 1) / C::BK;
    p.num_m_blocks = (p.M + 2 * C::BM - 1) / (2 * C::BM);
    p.num_n_blocks = (p.N + C::BN - 1) / C::BN;
    p.num_tiles = p.num_m_blocks * p.num_n_blocks;

    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = cs;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    if constexpr (FUSE_G > 0) {
        // the producers wait for rows that other CTAs' quantizer warps publish: every CTA
        // must be resident at once
        attr[1].id = cudaLaunchAttributeCooperative;
        attr[1].val.cooperative = 1;
    } else {
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
    }
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    static PerDeviceCache<1> max_pairs;
    const int resident_pairs = max_pairs.get(dev.index, 0, [&] {
        cudaLaunchConfig_t q = cfg;
        q.gridDim = dim3(static_cast<unsigned>(dev.sm_count / 2 * 2));
        q.numAttrs = 1;   // the cluster shape alone
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kernel, &q) != cudaSuccess || n < 1) {
            cudaGetLastError();
            n = dev.sm_count / 2;
        }
        return n;
    });
    const int pairs = p.num_tiles < resident_pairs ? p.num_tiles : resident_pairs;
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
    cudaGetLastError();
    if (cudaLaunchKernelEx(&cfg, kernel, tmA, tmB, tmU, tmL, tmO, p) != cudaSuccess) {
        cudaGetLastError();
        return SDNQ_ERR_CUDA;
    }
    return launch_status();
}

// Rows per call at which the CTA-pair kernel takes over from the single-SM one (below it,
// half of every 256-row pair tile would be padding).
constexpr int64_t kPairMinRows = 129;

template <int RANK_PAD>
sdnq_status launch_lora_down(const DeviceInfo &dev, const uint16_t *x, int64_t ldx,
                             const uint16_t *A, int32_t rank, uint16_t *u, int32_t M, int32_t K,
                             cudaStream_t cs)
{
    using C = LoraDownConfig<RANK_PAD>;
    CUtensorMap tmX, tmA;
    if (!make_tmap_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, K, M, 2ull * ldx, 64, 128) ||
        !make_tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, rank, K, 2ull * rank, 64, 64))
        return SDNQ_ERR_CUDA;
    static PerDeviceCache<1> smem_attr;
    if (!smem_attr_once(smem_attr, dev.index, lora_down_kernel<RANK_PAD>, C::SMEM_BYTES))
        return SDNQ_ERR_CUDA;
    LoraDownParams p;
    p.u = u;
    p.M = M;
    p.K = K;
    p.rank = rank;
    p.num_kb = (K + 63) / 64;
    p.timeout_ns = kDefaultTimeoutNs;
    cudaGetLastError();
    lora_down_kernel<RANK_PAD><<<(M + 127) / 128, 192, C::SMEM_BYTES, cs>>>(tmX, tmA, p);
    return launch_status();
}

// The GELU table in device memory (g_gelu_lut), built once per device: the first call that
// needs it launches the build kernel on its stream and waits for it, so that later calls on
// any stream find it complete. A failed build is retried by the next call.
sdnq_status ensure_gelu_lut(const DeviceInfo &dev, cudaStream_t cs)
{
    static PerDeviceCache<1> built;
    const int ok = built.get(dev.index, 0, [&] {
        cudaGetLastError();
        gelu_lut_build_kernel<<<(kGeluLutEntries + 255) / 256, 256, 0, cs>>>();
        if (cudaGetLastError() != cudaSuccess || cudaStreamSynchronize(cs) != cudaSuccess) {
            cudaGetLastError();
            return 0;
        }
        return 1;
    });
    return ok == 1 ? SDNQ_OK : SDNQ_ERR_CUDA;
}

// The adapter's part of a linear call: none, the down-projection u = bf16(x A) followed by
// the GEMM with the term lora_scale * (u B), or that GEMM alone from a given u.
enum LoraMode { kNoLora = 0, kLoraFull = 1, kLoraUp = 2 };

// Arguments of the down-projection u [M, rank] = bf16(x [M, K] A [K, rank]).
sdnq_status validate_lora_down(const uint16_t *x, int64_t ldx, const uint16_t *A, int32_t rank,
                               int64_t M, int64_t K, const uint16_t *u)
{
    if (!A || (M != 0 && (!x || !u)))
        return SDNQ_ERR_NULL;
    if (M < 0 || M > INT32_MAX || K < 16 || K > SDNQ_MAX_K || K % 16 != 0 || ldx < K)
        return SDNQ_ERR_SHAPE;
    if (rank < 16 || rank > SDNQ_MAX_RANK || rank % 16 != 0)
        return SDNQ_ERR_UNSUPPORTED;
    if (ldx % 8 != 0 || !aligned(x, 16) || !aligned(A, 16) || !aligned(u, 16))
        return SDNQ_ERR_ALIGN;
    return SDNQ_OK;
}

sdnq_status run_lora_down(const DeviceInfo &dev, const uint16_t *x, int64_t ldx, const uint16_t *A,
                          int32_t rank, uint16_t *u, int64_t M, int64_t K, cudaStream_t cs)
{
    const int32_t Mi = static_cast<int32_t>(M), Ki = static_cast<int32_t>(K);
    if (rank <= 64)
        return launch_lora_down<64>(dev, x, ldx, A, rank, u, Mi, Ki, cs);
    if (rank <= 128)
        return launch_lora_down<128>(dev, x, ldx, A, rank, u, Mi, Ki, cs);
    return launch_lora_down<256>(dev, x, ldx, A, rank, u, Mi, Ki, cs);
}

sdnq_status run_linear(const int8_t *qx, const float *sx, const int8_t *qW, const float *sW,
                       const uint16_t *bias, const uint16_t *x, int64_t ldx, const uint16_t *A,
                       const uint16_t *B, int32_t rank, float lora_scale, uint16_t *u_ws,
                       int64_t M, int64_t N, int64_t K, uint16_t *out, int64_t ldo,
                       int32_t *acc_out, void *stream, LoraMode lora, bool gelu = false)
{
    sdnq_status st = validate_linear(qx, sx, qW, sW, bias, M, N, K, out, ldo, acc_out);
    if (st != SDNQ_OK)
        return st;
    if (lora != kNoLora) {
        if (!B || (M != 0 && !u_ws))
            return SDNQ_ERR_NULL;
        if (lora == kLoraFull && (st = validate_lora_down(x, ldx, A, rank, M, K, u_ws)) != SDNQ_OK)
            return st;
        if (rank < 16 || rank > SDNQ_MAX_RANK || rank % 16 != 0)
            return SDNQ_ERR_UNSUPPORTED;
        if (N % 8 != 0)
            return SDNQ_ERR_SHAPE;
        if (!aligned(B, 16) || !aligned(u_ws, 16))
            return SDNQ_ERR_ALIGN;
    }
    DeviceInfo dev;
    if ((st = current_device(&dev)) != SDNQ_OK)
        return st;
    if (M == 0)
        return SDNQ_OK;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    GemmParams p = {};
    p.sx = sx;
    p.sw = sW;
    p.bias = bias;
    p.out = out;
    p.ldo = ldo;
    p.acc_out = acc_out;
    p.M = static_cast<int32_t>(M);
    p.N = static_cast<int32_t>(N);
    p.K = static_cast<int32_t>(K);
    p.lora_chunks = 0;
    p.lora_scale = lora_scale;
    p.c_g = 1.0f;
    p.timeout_ns = kDefaultTimeoutNs;
    if (gelu && (st = ensure_gelu_lut(dev, cs)) != SDNQ_OK)
        return st;
    if (lora == kNoLora && M >= kPairMinRows)
        return gelu ? launch_gemm_pair<true, false>(dev, qx, qW, p, cs)
                    : launch_gemm_pair<false, false>(dev, qx, qW, p, cs);
    if (lora == kNoLora)
        return gelu ? launch_gemm<256, false, true>(dev, qx, qW, nullptr, nullptr, 0, p, cs)
                    : launch_gemm<256, false>(dev, qx, qW, nullptr, nullptr, 0, p, cs);
    if (lora == kLoraFull && (st = run_lora_down(dev, x, ldx, A, rank, u_ws, M, K, cs)) != SDNQ_OK)
        return st;
    p.lora_chunks = (rank + 63) / 64;
    if (M >= kPairMinRows)
        return launch_gemm_pair<false, false, true>(dev, qx, qW, p, cs, u_ws, B, rank);
    return launch_gemm<SDNQ_LORA_BN, true>(dev, qx, qW, u_ws, B, rank, p, cs);
}

// ---------------------------------------------------------------- fused activation path

// the quantizer warps hold at most this many 1024-element chunks of a row
constexpr int kFusedMaxChunks = SDNQ_FUSED_QUANT_WARPS;

// Whether sdnq_int8_linear_fused takes one launch. The one-launch kernel overlaps the
// quantizer with the GEMM. It pays off once the GEMM has at least three waves of 128 x 256
// tiles (with fewer, its first wave needs most rows before it can start), N >= 3584 (the
// quantizer's share of the work shrinks with N) and K < 2 N (long rows delay the first
// published row block); otherwise the two launches, the GEMM's prologue overlapping the
// quantizer's tail, are as fast or faster (measured on 10 shapes from 4096 x 3072 x 3072 to
// 8192 x 12288 x 3072, one-launch kernel on CTA pairs). Rows longer than the quantizer warps
// can hold take the two launches.
bool fused_one_launch(const DeviceInfo &dev, int64_t M, int64_t N, int64_t K, int32_t policy)
{
    const int64_t nchunks = (K + 1023) / 1024;
    const int64_t tiles = ((M + 127) / 128) * ((N + 255) / 256);
    const bool auto_one = tiles >= 3ll * dev.sm_count && N >= 3584 && K < 2 * N;
    return nchunks <= kFusedMaxChunks &&
           (policy == SDNQ_FUSE_ALWAYS || (policy == SDNQ_FUSE_AUTO && auto_one));
}

// Above 128 rows the one-launch path runs on CTA pairs; if the device refuses that launch
// (a cooperative launch of clusters), the single-SM one-launch kernel runs instead, and the
// refusal is remembered for the device.
template <int G>
sdnq_status launch_linear_fused_g(const DeviceInfo &dev, GemmParams p, const int8_t *qW,
                                  cudaStream_t cs)
{
    static PerDeviceCache<1> pair_refused;
    if (p.M >= kPairMinRows && pair_refused.get(dev.index, 0, [] { return 2; }) == 2) {
        const sdnq_status st = launch_gemm_pair<false, false, false, G>(dev, p.rq.q, qW, p, cs);
        if (st == SDNQ_OK)
            return st;
        {
            std::lock_guard<std::mutex> lock(pair_refused.mutex);
            pair_refused.value[dev.index][0] = 1;
        }
    }
    return launch_gemm<256, false, false, 0, G>(dev, p.rq.q, qW, nullptr, nullptr, 0, p, cs);
}

sdnq_status run_linear_fused(const uint16_t *x, int64_t ldx, int32_t group, const int8_t *qW,
                             const float *sW, const uint16_t *bias, int64_t M, int64_t N,
                             int64_t K, int8_t *qx_ws, float *sx_ws, uint32_t *sync_ws,
                             uint16_t *out, int64_t ldo, int32_t *acc_out, int32_t policy,
                             void *stream)
{
    if (policy < SDNQ_FUSE_AUTO || policy > SDNQ_FUSE_NEVER)
        return SDNQ_ERR_UNSUPPORTED;
    sdnq_status st = validate_rotquant(x, M, K, ldx, group, qx_ws, sx_ws);
    if (st == SDNQ_OK)
        st = validate_linear(qx_ws, sx_ws, qW, sW, bias, M, N, K, out, ldo, acc_out);
    if (st != SDNQ_OK)
        return st;
    if (M != 0 && !sync_ws)
        return SDNQ_ERR_NULL;
    if (!aligned(sync_ws, 4))
        return SDNQ_ERR_ALIGN;
    DeviceInfo dev;
    if ((st = current_device(&dev)) != SDNQ_OK)
        return st;
    if (M == 0)
        return SDNQ_OK;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const int32_t nchunks = static_cast<int32_t>((K + 1023) / 1024);
    const bool fuse = fused_one_launch(dev, M, N, K, policy);
    if (!fuse) {
        // the two launches (same results)
        if ((st = launch_rowquant(x, M, K, ldx, group, nullptr, qx_ws, sx_ws, dev, cs)) != SDNQ_OK)
            return st;
        return run_linear(qx_ws, sx_ws, qW, sW, bias, nullptr, 0, nullptr, nullptr, 0, 0.0f,
                          nullptr, M, N, K, out, ldo, acc_out, stream, kNoLora);
    }
    GemmParams p = {};
    p.sx = sx_ws;
    p.sw = sW;
    p.bias = bias;
    p.out = out;
    p.ldo = ldo;
    p.acc_out = acc_out;
    p.M = static_cast<int32_t>(M);
    p.N = static_cast<int32_t>(N);
    p.K = static_cast<int32_t>(K);
    p.lora_chunks = 0;
    p.lora_scale = 0.0f;
    p.c_g = 1.0f;
    p.timeout_ns = kDefaultTimeoutNs;
    p.sync = sync_ws;
    RotquantParams &q = p.rq;
    q.x = x;
    q.ldx = ldx;
    q.q = qx_ws;
    q.s = sx_ws;
    q.M = M;
    q.K = static_cast<int32_t>(K);
    q.nchunks = nchunks;
    q.wpr = nchunks;
    q.rpc = 1;  // rows per group: a power of two (so a group never straddles a 128-row block)
    while (2 * q.rpc * nchunks <= SDNQ_FUSED_QUANT_WARPS)
        q.rpc *= 2;
    q.c_g = static_cast<float>(1.0 / std::sqrt(static_cast<double>(group)));
    q.colscale = nullptr;
    switch (group) {
    case 8: return launch_linear_fused_g<8>(dev, p, qW, cs);
    case 16: return launch_linear_fused_g<16>(dev, p, qW, cs);
    case 32: return launch_linear_fused_g<32>(dev, p, qW, cs);
    case 64: return launch_linear_fused_g<64>(dev, p, qW, cs);
    case 128: return launch_linear_fused_g<128>(dev, p, qW, cs);
    default: return launch_linear_fused_g<256>(dev, p, qW, cs);
    }
}

// ---------------------------------------------------------------- input gradient

// dx = dy W_hat through the frozen rotated base, in two launches: q_g, s_g = per-token int8
// of dy * sW, then the NN int8 product q_g qW with the row scale, inverse rotation and
// 1/sqrt(g) in the epilogue.
sdnq_status validate_grad_quant(const void *dy, int64_t lddy, const void *sW, int64_t M,
                                int64_t N, const void *qg, const void *sg)
{
    if (!sW || (M != 0 && (!dy || !qg || !sg)))
        return SDNQ_ERR_NULL;
    if (M < 0 || M > INT32_MAX || N < 16 || N > SDNQ_MAX_K || N % 16 != 0 || lddy < N)
        return SDNQ_ERR_SHAPE;
    if (lddy % 8 != 0 || !aligned(dy, 16) || !aligned(sW, 16) || !aligned(qg, 16) ||
        !aligned(sg, 4))
        return SDNQ_ERR_ALIGN;
    return SDNQ_OK;
}

sdnq_status validate_grad_gemm(const void *qg, const void *sg, const void *qW, int64_t M,
                               int64_t N, int64_t K, int32_t group, const void *dx,
                               int64_t lddx, const void *acc_out)
{
    if (!qW || (M != 0 && (!qg || !sg || !dx)))
        return SDNQ_ERR_NULL;
    if (M < 0 || M > INT32_MAX || N < 16 || N > SDNQ_MAX_K || N % 16 != 0 || K < 16 ||
        K > INT32_MAX || K % 16 != 0 || lddx < K)
        return SDNQ_ERR_SHAPE;
    if (!is_pow2(group) || group < SDNQ_MIN_GROUP || group > SDNQ_MAX_GROUP)
        return SDNQ_ERR_UNSUPPORTED;
    if (K % group != 0)
        return SDNQ_ERR_SHAPE;
    if (lddx % 8 != 0 || !aligned(qg, 16) || !aligned(sg, 4) || !aligned(qW, 16) ||
        !aligned(dx, 16) || (acc_out && !aligned(acc_out, 16)))
        return SDNQ_ERR_ALIGN;
    return SDNQ_OK;
}

sdnq_status launch_grad_gemm(const DeviceInfo &dev, const int8_t *qg, const float *sg,
                             const int8_t *qW, int64_t M, int64_t N, int64_t K, int32_t group,
                             uint16_t *dx, int64_t lddx, int32_t *acc_out, cudaStream_t cs)
{
    GemmParams p = {};
    p.sx = sg;
    p.sw = nullptr;    // not read in this mode
    p.bias = nullptr;
    p.out = dx;
    p.ldo = lddx;
    p.acc_out = acc_out;
    p.M = static_cast<int32_t>(M);
    p.N = static_cast<int32_t>(K);   // output columns: the layer's input features
    p.K = static_cast<int32_t>(N);   // contraction: the layer's output features
    p.lora_chunks = 0;
    p.lora_scale = 0.0f;
    p.c_g = static_cast<float>(1.0 / std::sqrt(static_cast<double>(group)));
    p.timeout_ns = kDefaultTimeoutNs;
    if (M >= kPairMinRows) {
        switch (group) {
        case 8: return launch_gemm_pair<false, false, false, 0, 8>(dev, qg, qW, p, cs);
        case 16: return launch_gemm_pair<false, false, false, 0, 16>(dev, qg, qW, p, cs);
        case 32: return launch_gemm_pair<false, false, false, 0, 32>(dev, qg, qW, p, cs);
        case 64: return launch_gemm_pair<false, false, false, 0, 64>(dev, qg, qW, p, cs);
        case 128: return launch_gemm_pair<false, false, false, 0, 128>(dev, qg, qW, p, cs);
        default: return launch_gemm_pair<false, false, false, 0, 256>(dev, qg, qW, p, cs);
        }
    }
    switch (group) {
    case 8: return launch_gemm<256, false, false, 8>(dev, qg, qW, nullptr, nullptr, 0, p, cs);
    case 16: return launch_gemm<256, false, false, 16>(dev, qg, qW, nullptr, nullptr, 0, p, cs);
    case 32: return launch_gemm<256, false, false, 32>(dev, qg, qW, nullptr, nullptr, 0, p, cs);
    case 64: return launch_gemm<256, false, false, 64>(dev, qg, qW, nullptr, nullptr, 0, p, cs);
    case 128: return launch_gemm<256, false, false, 128>(dev, qg, qW, nullptr, nullptr, 0, p, cs);
    default: return launch_gemm<256, false, false, 256>(dev, qg, qW, nullptr, nullptr, 0, p, cs);
    }
}

sdnq_status run_grad_quant(const uint16_t *dy, int64_t lddy, const float *sW, int64_t M,
                           int64_t N, int8_t *qg, float *sg, void *stream)
{
    sdnq_status st = validate_grad_quant(dy, lddy, sW, M, N, qg, sg);
    if (st != SDNQ_OK)
        return st;
    DeviceInfo dev;
    if ((st = current_device(&dev)) != SDNQ_OK)
        return st;
    if (M == 0)
        return SDNQ_OK;
    return launch_rowquant(dy, M, N, lddy, 1, sW, qg, sg, dev, static_cast<cudaStream_t>(stream));
}

sdnq_status run_grad_gemm(const int8_t *qg, const float *sg, const int8_t *qW, int64_t M,
                          int64_t N, int64_t K, int32_t group, uint16_t *dx, int64_t lddx,
                          int32_t *acc_out, void *stream)
{
    sdnq_status st = validate_grad_gemm(qg, sg, qW, M, N, K, group, dx, lddx, acc_out);
    if (st != SDNQ_OK)
        return st;
    DeviceInfo dev;
    if ((st = current_device(&dev)) != SDNQ_OK)
        return st;
    if (M == 0)
        return SDNQ_OK;
    return launch_grad_gemm(dev, qg, sg, qW, M, N, K, group, dx, lddx, acc_out,
                            static_cast<cudaStream_t>(stream));
}

sdnq_status run_grad_input(const uint16_t *dy, int64_t lddy, const int8_t *qW, const float *sW,
                           int64_t M, int64_t N, int64_t K, int32_t group, int8_t *qg_ws,
                           float *sg_ws, uint16_t *dx, int64_t lddx, int32_t *acc_out,
                           void *stream)
{
    sdnq_status st = validate_grad_quant(dy, lddy, sW, M, N, qg_ws, sg_ws);
    if (st == SDNQ_OK)
        st = validate_grad_gemm(qg_ws, sg_ws, qW, M, N, K, group, dx, lddx, acc_out);
    if (st != SDNQ_OK)
        return st;
    DeviceInfo dev;
    if ((st = current_device(&dev)) != SDNQ_OK)
        return st;
    if (M == 0)
        return SDNQ_OK;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if ((st = launch_rowquant(dy, M, N, lddy, 1, sW, qg_ws, sg_ws, dev, cs)) != SDNQ_OK)
        return st;
    return launch_grad_gemm(dev, qg_ws, sg_ws, qW, M, N, K, group, dx, lddx, acc_out, cs);
}

// ---------------------------------------------------------------- FP8 (e4m3) variant

sdnq_status run_rotquant_fp8(const uint16_t *x, int64_t rows, int64_t K, int64_t ld,
                             int32_t group, uint8_t *q, float *s, void *stream)
{
    sdnq_status st = validate_rotquant(x, rows, K, ld, group, q, s);
    if (st != SDNQ_OK)
        return st;
    DeviceInfo dev;
    if ((st = current_device(&dev)) != SDNQ_OK)
        return st;
    if (rows == 0)
        return SDNQ_OK;
    return launch_rowquant(x, rows, K, ld, group, nullptr, reinterpret_cast<int8_t *>(q), s, dev,
                           static_cast<cudaStream_t>(stream), true);
}

sdnq_status run_fp8_linear(const uint8_t *qx, const float *sx, const uint8_t *qW, const float *sW,
                           const uint16_t *bias, int64_t M, int64_t N, int64_t K, uint16_t *out,
                           int64_t ldo, float *acc_out, void *stream)
{
    sdnq_status st = validate_linear(qx, sx, qW, sW, bias, M, N, K, out, ldo, acc_out);
    if (st != SDNQ_OK)
        return st;
    DeviceInfo dev;
    if ((st = current_device(&dev)) != SDNQ_OK)
        return st;
    if (M == 0)
        return SDNQ_OK;
    GemmParams p = {};
    p.sx = sx;
    p.sw = sW;
    p.bias = bias;
    p.out = out;
    p.ldo = ldo;
    p.acc_out = reinterpret_cast<int32_t *>(acc_out);  // fp32 bits
    p.M = static_cast<int32_t>(M);
    p.N = static_cast<int32_t>(N);
    p.K = static_cast<int32_t>(K);
    p.c_g = 1.0f;
    p.timeout_ns = kDefaultTimeoutNs;
    if (M >= kPairMinRows)
        return launch_gemm_pair<false, true>(dev, reinterpret_cast<const int8_t *>(qx),
                                             reinterpret_cast<const int8_t *>(qW), p,
                                             static_cast<cudaStream_t>(stream));
    return launch_gemm<256, false, false, 0, 0, true>(
        dev, reinterpret_cast<const int8_t *>(qx), reinterpret_cast<const int8_t *>(qW), nullptr,
        nullptr, 0, p, static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------- int8-QK attention

bool make_tmap_3d(CUtensorMap *map, CUtensorMapDataType dtype, const void *ptr, uint64_t d0,
                  uint64_t d1, uint64_t d2, uint64_t stride1_bytes, uint64_t stride2_bytes,
                  uint32_t box0, uint32_t box1)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
    const cuuint32_t box[3] = {box0, box1, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(map, dtype, 3, const_cast<void *>(ptr), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// workspace: qq, kq (int8 codes), sq, sk (fp32 scales), mu (fp32 means), partial (fp64 sums)
int64_t attn_workspace(int64_t B, int64_t Lq, int64_t Lk, int64_t H, int64_t D, int64_t *off)
{
    auto up = [](int64_t v) { return (v + 255) / 256 * 256; };
    int64_t o[6];
    o[0] = 0;
    o[1] = o[0] + up(B * Lq * H * D);
    const int64_t lq_pad = (Lq + 127) / 128 * 128, lk_pad = (Lk + 127) / 128 * 128;
    o[2] = o[1] + up(B * Lk * H * D);
    o[3] = o[2] + up(4 * B * H * lq_pad);
    o[4] = o[3] + up(4 * B * H * lk_pad);
    o[5] = o[4] + up(4 * B * H * D);
    const int64_t total = o[5] + up(8 * B * H * kAttnSumSplits * D);
    if (off)
        for (int i = 0; i < 6; ++i)
            off[i] = o[i];
    return total;
}

template <int G>
void launch_attn_rowquant(const AttnQuantParams &p, int sm_count, cudaStream_t cs)
{
    const int64_t chunks = (p.rows + 7) / 8;
    int64_t blocks = (chunks + 7) / 8;  // 8 warps per block
    const int64_t cap = static_cast<int64_t>(sm_count) * 8;
    if (blocks > cap)
        blocks = cap;
    launch_programmatic(attn_rowquant_kernel<G>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0,
                        cs, p);
}

sdnq_status validate_attention(const void *q, const void *k, const void *v, const void *o,
                               int64_t B, int64_t Lq, int64_t Lk, int64_t H, int64_t D,
                               int32_t group, const void *ws, int64_t ws_bytes, int64_t *off)
{
    if (!q || !k || !v || !o || !ws)
        return SDNQ_ERR_NULL;
    if (B <= 0 || Lq <= 0 || Lk <= 0 || H <= 0 || B * H > INT32_MAX || Lq > INT32_MAX ||
        Lk > INT32_MAX || (B * H) * ((Lq + 127) / 128) > INT32_MAX || B * H * Lq > INT32_MAX ||
        B * H * Lk > INT32_MAX)
        return SDNQ_ERR_SHAPE;
    if (D != kAttnD || !is_pow2(group) || group < SDNQ_MIN_GROUP || group > SDNQ_MAX_GROUP)
        return SDNQ_ERR_UNSUPPORTED;
    if (ws_bytes < attn_workspace(B, Lq, Lk, H, D, off))
        return SDNQ_ERR_SHAPE;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
        !aligned(ws, 256))
        return SDNQ_ERR_ALIGN;
    return SDNQ_OK;
}

// smooth_k means and the Q / K codes into the workspace
sdnq_status launch_attention_prep(const uint16_t *q, const uint16_t *k, int64_t B, int64_t Lq,
                                  int64_t Lk, int64_t H, int64_t D, int32_t group, int32_t smooth_k,
                                  uint8_t *w, const int64_t *off, const DeviceInfo &dev,
                                  cudaStream_t cs)
{
    int8_t *qq = reinterpret_cast<int8_t *>(w + off[0]);
    int8_t *kq = reinterpret_cast<int8_t *>(w + off[1]);
    float *sq = reinterpret_cast<float *>(w + off[2]);
    float *sk = reinterpret_cast<float *>(w + off[3]);
    float *mu = reinterpret_cast<float *>(w + off[4]);
    double *partial = reinterpret_cast<double *>(w + off[5]);
    cudaGetLastError();
    const int32_t bh = static_cast<int32_t>(B * H);
    if (smooth_k) {
        launch_programmatic(attn_ksum_kernel, dim3(bh, kAttnSumSplits), dim3(256), 0, cs, k,
                            static_cast<int32_t>(Lk), static_cast<int32_t>(H), partial);
        launch_programmatic(attn_kmean_kernel, dim3(bh), dim3(kAttnD), 0, cs,
                            static_cast<const double *>(partial), static_cast<int32_t>(Lk), mu);
    } else {
        cudaMemsetAsync(mu, 0, 4 * B * H * D, cs);
    }
    const int32_t ge = group < kAttnD ? group : kAttnD;
    AttnQuantParams pq = {};
    pq.c_g = static_cast<float>(1.0 / std::sqrt(static_cast<double>(ge)));
    pq.H = static_cast<int32_t>(H);
    for (int pass = 0; pass < 2; ++pass) {
        pq.x = pass == 0 ? q : k;
        pq.mu = pass == 0 ? nullptr : mu;
        pq.q = pass == 0 ? qq : kq;
        pq.s = pass == 0 ? sq : sk;
        pq.L = static_cast<int32_t>(pass == 0 ? Lq : Lk);
        pq.ls = (pq.L + 127) / 128 * 128;
        pq.rows = B * pq.L * H;
        switch (ge) {
        case 8: launch_attn_rowquant<8>(pq, dev.sm_count, cs); break;
        case 16: launch_attn_rowquant<16>(pq, dev.sm_count, cs); break;
        case 32: launch_attn_rowquant<32>(pq, dev.sm_count, cs); break;
        case 64: launch_attn_rowquant<64>(pq, dev.sm_count, cs); break;
        default: launch_attn_rowquant<128>(pq, dev.sm_count, cs); break;
        }
    }
    return launch_status();
}

// the attention kernel on prepared codes
sdnq_status launch_attention_core(const DeviceInfo &dev, const uint16_t *v, int64_t B, int64_t Lq,
                                  int64_t Lk, int64_t H, int64_t D, float scale, uint8_t *w,
                                  const int64_t *off, uint16_t *o, cudaStream_t cs)
{
    CUtensorMap tmQ, tmK, tmV;
    const uint64_t row = static_cast<uint64_t>(H * D);
    if (!make_tmap_3d(&tmQ, CU_TENSOR_MAP_DATA_TYPE_UINT8, w + off[0], row, Lq, B, row, row * Lq, 128,
                      128) ||
        !make_tmap_3d(&tmK, CU_TENSOR_MAP_DATA_TYPE_UINT8, w + off[1], row, Lk, B, row, row * Lk, 128,
                      128) ||
        !make_tmap_3d(&tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, v, row, Lk, B, 2 * row, 2 * row * Lk,
                      64, 128))
        return SDNQ_ERR_CUDA;
    static PerDeviceCache<1> smem_attr;
    if (!smem_attr_once(smem_attr, dev.index, attn_kernel, AttnConfig::SMEM_BYTES))
        return SDNQ_ERR_CUDA;
    AttnParams p = {};
    p.sq = reinterpret_cast<const float *>(w + off[2]);
    p.sk = reinterpret_cast<const float *>(w + off[3]);
    p.o = o;
    p.B = static_cast<int32_t>(B);
    p.Lq = static_cast<int32_t>(Lq);
    p.Lk = static_cast<int32_t>(Lk);
    p.H = static_cast<int32_t>(H);
    p.q_blocks = static_cast<int32_t>((Lq + 255) / 256);   // pairs of query tiles
    p.lq_pad = static_cast<int32_t>((Lq + 127) / 128 * 128);   // query-scale row stride
    p.lk_pad = static_cast<int32_t>((Lk + 127) / 128 * 128);
    p.scale = scale;
    p.timeout_ns = kDefaultTimeoutNs;
    cudaGetLastError();
    // programmatic launch: the prologue overlaps the end of the preparation
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(B * H * p.q_blocks));
    cfg.blockDim = dim3(AttnConfig::THREADS);
    cfg.dynamicSmemBytes = AttnConfig::SMEM_BYTES;
    cfg.stream = cs;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, attn_kernel, tmQ, tmK, tmV, p) != cudaSuccess) {
        cudaGetLastError();
        return SDNQ_ERR_CUDA;
    }
    return launch_status();
}

// which: 1 = prep, 2 = core, 3 = both
sdnq_status run_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t B,
                          int64_t Lq, int64_t Lk, int64_t H, int64_t D, int32_t group, float scale,
                          int32_t smooth_k, void *ws, int64_t ws_bytes, uint16_t *o, void *stream,
                          int which)
{
    int64_t off[6];
    // the parts check only the tensors they read (unused ones are passed as ws)
    sdnq_status st = validate_attention(q, k, v, o, B, Lq, Lk, H, D, group, ws, ws_bytes, off);
    if (st != SDNQ_OK)
        return st;
    if ((which & 2) && !(scale >= 0.0f && scale <= FLT_MAX))   // the softmax scale: finite, >= 0
        return SDNQ_ERR_UNSUPPORTED;
    DeviceInfo dev;
    if ((st = current_device(&dev)) != SDNQ_OK)
        return st;
    uint8_t *w = static_cast<uint8_t *>(ws);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if ((which & 1) &&
        (st = launch_attention_prep(q, k, B, Lq, Lk, H, D, group, smooth_k, w, off, dev, cs)) != SDNQ_OK)
        return st;
    if (which & 2)
        return launch_attention_core(dev, v, B, Lq, Lk, H, D, scale, w, off, o, cs);
    return SDNQ_OK;
}

// ---------------------------------------------------------------- self-test kernel

__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns)
{
    __shared__ alignas(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(smem_u32(&bar), 1);
        fence_mbar_init();
        // nothing ever arrives: phase 0 never completes, the bounded wait gives up
        mbar_wait_bounded(smem_u32(&bar), 0u, &abort_flag, limit_ns);
        mbar_arrive(smem_u32(&bar));  // leave the barrier consistent
    }
}

} // namespace
} // namespace sdnq

using namespace sdnq;

SDNQ_API sdnq_status sdnq_rotate_quant_weight(const uint16_t *W, int64_t N, int64_t K, int64_t ldw,
                                              int32_t group, int8_t *qW, float *sW, void *stream)
{
    SDNQ_NVTX_RANGE();
    return run_rotquant(W, N, K, ldw, group, qW, sW, stream);
}

SDNQ_API sdnq_status sdnq_rotquant_act(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                                       int32_t group, int8_t *qx, float *sx, void *stream)
{
    SDNQ_NVTX_RANGE();
    return run_rotquant(x, M, K, ldx, group, qx, sx, stream);
}

SDNQ_API sdnq_status sdnq_int8_linear(const int8_t *qx, const float *sx, const int8_t *qW,
                                      const float *sW, const uint16_t *bias, int64_t M, int64_t N,
                                      int64_t K, uint16_t *out, int64_t ldo, int32_t *acc_out,
                                      void *stream)
{
    SDNQ_NVTX_RANGE();
    return run_linear(qx, sx, qW, sW, bias, nullptr, 0, nullptr, nullptr, 0, 0.0f, nullptr, M, N, K,
                      out, ldo, acc_out, stream, kNoLora);
}

SDNQ_API sdnq_status sdnq_int8_linear_fused(const uint16_t *x, int64_t ldx, int32_t group,
                                            const int8_t *qW, const float *sW,
                                            const uint16_t *bias, int64_t M, int64_t N, int64_t K,
                                            int8_t *qx_ws, float *sx_ws, uint32_t *sync_ws,
                                            uint16_t *out, int64_t ldo, int32_t *acc_out,
                                            int32_t policy, void *stream)
{
    SDNQ_NVTX_RANGE();
    return run_linear_fused(x, ldx, group, qW, sW, bias, M, N, K, qx_ws, sx_ws, sync_ws, out, ldo,
                            acc_out, policy, stream);
}

SDNQ_API sdnq_status sdnq_rotquant_fp8(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                                       int32_t group, uint8_t *q, float *s, void *stream)
{
    SDNQ_NVTX_RANGE();
    return run_rotquant_fp8(x, M, K, ldx, group, q, s, stream);
}

SDNQ_API sdnq_status sdnq_fp8_linear(const uint8_t *qx, const float *sx, const uint8_t *qW,
                                     const float *sW, const uint16_t *bias, int64_t M, int64_t N,
                                     int64_t K, uint16_t *out, int64_t ldo, float *acc_out,
                                     void *stream)
{
    SDNQ_NVTX_RANGE();
    return run_fp8_linear(qx, sx, qW, sW, bias, M, N, K, out, ldo, acc_out, stream);
}

SDNQ_API int64_t sdnq_attention_workspace(int64_t B, int64_t Lq, int64_t Lk, int64_t H,
                                          int64_t D, int64_t *offsets)
{
    if (B <= 0 || Lq <= 0 || Lk <= 0 || H <= 0 || D <= 0)
        return -1;
    return attn_workspace(B, Lq, Lk, H, D, offsets);
}

SDNQ_API sdnq_status sdnq_attention_int8qk(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                           int64_t B, int64_t Lq, int64_t Lk, int64_t H, int64_t D,
                                           int32_t group, float scale, int32_t smooth_k, void *ws,
                                           int64_t ws_bytes, uint16_t *o, void *stream)
{
    SDNQ_NVTX_RANGE();
    return run_attention(q, k, v, B, Lq, Lk, H, D, group, scale, smooth_k, ws, ws_bytes, o, stream, 3);
}

SDNQ_API sdnq_status sdnq_attention_prep(const uint16_t *q, const uint16_t *k, int64_t B,
                                         int64_t Lq, int64_t Lk, int64_t H, int64_t D,
                                         int32_t group, int32_t smooth_k, void *ws,
                                         int64_t ws_bytes, void *stream)
{
    SDNQ_NVTX_RANGE();
    // v and o are not touched by the preparation: the workspace stands in for them
    return run_attention(q, k, static_cast<const uint16_t *>(ws), B, Lq, Lk, H, D, group, 1.0f,
                         smooth_k, ws, ws_bytes, static_cast<uint16_t *>(ws), stream, 1);
}

SDNQ_API sdnq_status sdnq_attention_core(const uint16_t *v, int64_t B, int64_t Lq, int64_t Lk,
                                         int64_t H, int64_t D, float scale, void *ws,
                                         int64_t ws_bytes, uint16_t *o, void *stream)
{
    SDNQ_NVTX_RANGE();
    // q and k are not read by the attention kernel (their codes are in ws)
    return run_attention(static_cast<const uint16_t *>(ws), static_cast<const uint16_t *>(ws), v,
                         B, Lq, Lk, H, D, SDNQ_MAX_GROUP, scale, 0, ws, ws_bytes, o, stream, 2);
}

SDNQ_API sdnq_status sdnq_int8_linear_gelu(const int8_t *qx, const float *sx, const int8_t *qW,
                                           const float *sW, const uint16_t *bias, int64_t M,
                                           int64_t N, int64_t K, uint16_t *out, int64_t ldo,
                                           int32_t *acc_out, void *stream)
{
    SDNQ_NVTX_RANGE();
    return run_linear(qx, sx, qW, sW, bias, nullptr, 0, nullptr, nullptr, 0, 0.0f, nullptr, M, N, K,
                      out, ldo, acc_out, stream, kNoLora, true);
}

SDNQ_API sdnq_status sdnq_int8_linear_grad_input(const uint16_t *dy, int64_t lddy,
                                                 const int8_t *qW, const float *sW, int64_t M,
                                                 int64_t N, int64_t K, int32_t group,
                                                 int8_t *qg_ws, float *sg_ws, uint16_t *dx,
                                                 int64_t lddx, int32_t *acc_out, void *stream)
{
    SDNQ_NVTX_RANGE();
    return run_grad_input(dy, lddy, qW, sW, M, N, K, group, qg_ws, sg_ws, dx, lddx, acc_out,
                          stream);
}

SDNQ_API sdnq_status sdnq_quant_grad_output(const uint16_t *dy, int64_t lddy, const float *sW,
                                            int64_t M, int64_t N, int8_t *qg, float *sg,
                                            void *stream)
{
    SDNQ_NVTX_RANGE();
    return run_grad_quant(dy, lddy, sW, M, N, qg, sg, stream);
}

SDNQ_API sdnq_status sdnq_int8_grad_input_gemm(const int8_t *qg, const float *sg, const int8_t *qW,
                                               int64_t M, int64_t N, int64_t K, int32_t group,
                                               uint16_t *dx, int64_t lddx, int32_t *acc_out,
                                               void *stream)
{
    SDNQ_NVTX_RANGE();
    return run_grad_gemm(qg, sg, qW, M, N, K, group, dx, lddx, acc_out, stream);
}

SDNQ_API sdnq_status sdnq_int8_linear_lora(const int8_t *qx, const float *sx, const int8_t *qW,
                                           const float *sW, const uint16_t *bias, const uint16_t *x,
                                           int64_t ldx, const uint16_t *A, const uint16_t *B,
                                           int32_t rank, float lora_scale, uint16_t *u_ws,
                                           int64_t M, int64_t N, int64_t K, uint16_t *out,
                                           int64_t ldo, int32_t *acc_out, void *stream)
{
    SDNQ_NVTX_RANGE();
    return run_linear(qx, sx, qW, sW, bias, x, ldx, A, B, rank, lora_scale, u_ws, M, N, K, out, ldo,
                      acc_out, stream, kLoraFull);
}

SDNQ_API sdnq_status sdnq_lora_down(const uint16_t *x, int64_t ldx, const uint16_t *A,
                                    int32_t rank, int64_t M, int64_t K, uint16_t *u, void *stream)
{
    SDNQ_NVTX_RANGE();
    sdnq_status st = validate_lora_down(x, ldx, A, rank, M, K, u);
    if (st != SDNQ_OK)
        return st;
    DeviceInfo dev;
    if ((st = current_device(&dev)) != SDNQ_OK)
        return st;
    if (M == 0)
        return SDNQ_OK;
    return run_lora_down(dev, x, ldx, A, rank, u, M, K, static_cast<cudaStream_t>(stream));
}

SDNQ_API sdnq_status sdnq_int8_linear_lora_up(const int8_t *qx, const float *sx, const int8_t *qW,
                                              const float *sW, const uint16_t *bias,
                                              const uint16_t *u, const uint16_t *B, int32_t rank,
                                              float lora_scale, int64_t M, int64_t N, int64_t K,
                                              uint16_t *out, int64_t ldo, int32_t *acc_out,
                                              void *stream)
{
    SDNQ_NVTX_RANGE();
    return run_linear(qx, sx, qW, sW, bias, nullptr, 0, nullptr, B, rank, lora_scale,
                      const_cast<uint16_t *>(u), M, N, K, out, ldo, acc_out, stream, kLoraUp);
}

SDNQ_API sdnq_status sdnq_gelu_bf16(const uint16_t *in, int64_t M, int64_t N, int64_t ld_in,
                                    uint16_t *out, int64_t ld_out, void *stream)
{
    SDNQ_NVTX_RANGE();
    if (M != 0 && (!in || !out))
        return SDNQ_ERR_NULL;
    if (M < 0 || N <= 0 || ld_in < N || ld_out < N)
        return SDNQ_ERR_SHAPE;
    if (ld_in % 8 != 0 || ld_out % 8 != 0 || !aligned(in, 16) || !aligned(out, 16))
        return SDNQ_ERR_ALIGN;
    if (in == out && ld_in != ld_out)
        return SDNQ_ERR_SHAPE;
    DeviceInfo dev;
    sdnq_status st = current_device(&dev);
    if (st != SDNQ_OK)
        return st;
    if (M == 0)
        return SDNQ_OK;
    GeluParams p;
    p.in = in;
    p.out = out;
    p.M = M;
    p.N = N;
    p.ld_in = ld_in;
    p.ld_out = ld_out;
    p.vecs_per_row = (N + 7) / 8;
    const int64_t total = M * p.vecs_per_row;
    int64_t blocks = (total + 255) / 256;
    const int64_t cap = static_cast<int64_t>(dev.sm_count) * 16;
    if (blocks > cap)
        blocks = cap;
    cudaGetLastError();
    gelu_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
    return launch_status();
}

SDNQ_API sdnq_status sdnq_device_status(void *stream)
{
    SDNQ_NVTX_RANGE();
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return SDNQ_ERR_CUDA;
    }
    unsigned int word = 0;
    if (cudaMemcpyFromSymbol(&word, g_device_error, sizeof(word)) != cudaSuccess)
        return SDNQ_ERR_CUDA;
    if (word != kDevOk) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess)
            return SDNQ_ERR_CUDA;
        return SDNQ_ERR_TIMEOUT;
    }
    return SDNQ_OK;
}

SDNQ_API sdnq_status sdnq_selftest_wait_timeout(int64_t limit_ns, void *stream)
{
    SDNQ_NVTX_RANGE();
    if (limit_ns < 1000 || limit_ns > 10000000000ll)
        return SDNQ_ERR_SHAPE;
    DeviceInfo dev;
    sdnq_status st = current_device(&dev);
    if (st != SDNQ_OK)
        return st;
    cudaGetLastError();
    wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint64_t>(limit_ns));
    return launch_status();
}

SDNQ_API sdnq_status sdnq_int8_linear_fused_plan(int64_t M, int64_t N, int64_t K,
                                                 int32_t policy, int32_t *one_launch)
{
    if (!one_launch)
        return SDNQ_ERR_NULL;
    if (M < 0 || N < 1 || N > INT32_MAX || K < 16 || K % 16 != 0 || K > SDNQ_MAX_K)
        return SDNQ_ERR_SHAPE;
    if (policy < SDNQ_FUSE_AUTO || policy > SDNQ_FUSE_NEVER)
        return SDNQ_ERR_UNSUPPORTED;
    DeviceInfo dev;
    const sdnq_status st = current_device(&dev);
    if (st != SDNQ_OK)
        return st;
    *one_launch = fused_one_launch(dev, M, N, K, policy) ? 1 : 0;
    return SDNQ_OK;
}

SDNQ_API const char *sdnq_status_string(sdnq_status s)
{
    switch (s) {
    case SDNQ_OK: return "SDNQ_OK";
    case SDNQ_ERR_NULL: return "SDNQ_ERR_NULL: a required pointer is NULL";
    case SDNQ_ERR_SHAPE: return "SDNQ_ERR_SHAPE: a size is out of range or sizes are inconsistent";
    case SDNQ_ERR_ALIGN: return "SDNQ_ERR_ALIGN: a pointer or leading dimension breaks the 16-byte rule";
    case SDNQ_ERR_UNSUPPORTED: return "SDNQ_ERR_UNSUPPORTED: unsupported group/rank or device is not sm_100";
    case SDNQ_ERR_CUDA: return "SDNQ_ERR_CUDA: a CUDA runtime call or kernel launch failed";
    case SDNQ_ERR_TIMEOUT: return "SDNQ_ERR_TIMEOUT: a bounded wait inside a kernel gave up";
    }
    return "SDNQ_ERR_UNKNOWN";
}

SDNQ_API const char *sdnq_version(void) { return "sdnq-b200 0.1.0 sm_100a"; }

// The no-allocation LoRA variant (its own file; shares this translation unit).
#include "lora_noalloc.cu"
