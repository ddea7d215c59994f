// The LoRA linear without a caller-provided workspace.
//
// sdnq_int8_linear_lora needs a scratch buffer for u = bf16(x A) between its two kernels,
// and asks the caller for it (u_ws). Some callers cannot allocate one: their host framework
// owns every byte of device memory (a caching allocator or a fixed memory plan) and does not
// allow allocations from outside it, or they run where a cudaMalloc is not acceptable because
// it may synchronise the device and takes an unpredictable amount of time. For them this
// variant keeps u in a fixed array in the library's own device memory instead, so the call
// allocates nothing.
//
// This file is part of libsdnq.cu's translation unit (included at its end).

namespace sdnq {
namespace {

// u for the no-allocation variant: at most SDNQ_NOALLOC_MAX_U_ELEMS bf16 values (8 MiB),
// resident on every GPU that loads the library until the process exits.
static __device__ __align__(256) uint16_t g_noalloc_u[SDNQ_NOALLOC_MAX_U_ELEMS];

struct NoallocScratch {
    void *ptr[64] = {};
};
NoallocScratch g_noalloc_scratch;
std::mutex g_noalloc_mutex;

// Device address of g_noalloc_u on the current device, looked up once per device. In host
// code the array's name is only a host-side stand-in: a kernel must be given this address.
sdnq_status noalloc_scratch(void **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return SDNQ_ERR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_scratch.ptr[dev] == nullptr) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_u);
        if (e != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return SDNQ_ERR_CUDA;
        }
        g_noalloc_scratch.ptr[dev] = p;
    }
    *out = g_noalloc_scratch.ptr[dev];
    return SDNQ_OK;
}

} // namespace
} // namespace sdnq

SDNQ_API sdnq_status sdnq_int8_linear_lora_noalloc(const int8_t *qx, const float *sx,
                                                   const int8_t *qW, const float *sW,
                                                   const uint16_t *bias, const uint16_t *x,
                                                   int64_t ldx, const uint16_t *A,
                                                   const uint16_t *B, int32_t rank,
                                                   float lora_scale, int64_t M, int64_t N,
                                                   int64_t K, uint16_t *out, int64_t ldo,
                                                   int32_t *acc_out, void *stream)
{
    SDNQ_NVTX_RANGE();
    if (M < 0 || rank < 0)
        return SDNQ_ERR_SHAPE;
    // u would not fit the library's fixed scratch array (the division keeps the check free
    // of overflow for any M)
    if (rank > 0 && M > SDNQ_NOALLOC_MAX_U_ELEMS / rank)
        return SDNQ_ERR_SHAPE;
    DeviceInfo dev;
    sdnq_status st = current_device(&dev);
    if (st != SDNQ_OK)
        return st;
    void *u = nullptr;
    if ((st = sdnq::noalloc_scratch(&u)) != SDNQ_OK)
        return st;
    // u is written in full (rows < M) by the down-projection before the main kernel reads
    // it, and rows >= M are never read, so nothing has to be cleared between calls.
    return run_linear(qx, sx, qW, sW, bias, x, ldx, A, B, rank, lora_scale,
                      static_cast<uint16_t *>(u), M, N, K, out, ldo, acc_out, stream, kLoraFull);
}
