/*
 * sdnq.h -- C ABI of libsdnq.so: the Hadamard-rotated ("ConvRot") INT8 linear layer
 * on NVIDIA B200 (sm_100a).
 *
 * What it computes (sources are web pages on the method, cited by title and section):
 *  - "SDNQ: SD.Next Quantization Engine" README, feature list: Hadamard rotations apply on
 *    both the quantized weights and the quantized matmul; INT8 quantized matmul.
 *  - same README, SDNQConfig example: group_size = -1 is row-wise (one scale per output
 *    row); hadamard_group_size; dequantize_fp32 keeps the scales in FP32 and runs the
 *    de-quant steps in FP32.
 *  - "ConvRot / Hadamard SDNQ" (SimpleTuner), What The Options Do: group 256 is ConvRot,
 *    smaller groups are QuaRot-style; static full-row weight scales; the INT8 matmul path
 *    stays active. PEFT Behavior: the frozen base runs in int8 while LoRA adapters stay bf16.
 *  - "Hybrid-Sensitivity-Weighted-Quantization" README, Rigorous grid / pack simulation:
 *    ConvRot = Hadamard rotate, then channelwise absmax onto the symmetric INT8 grid.
 *
 * Exact definition (the readings where the pages are silent are stated here too):
 *  rotation   H_g = Sylvester Hadamard matrix in natural order, H[i][j] = (-1)^popcount(i&j),
 *             applied block-diagonally along K in groups of g, normalised by 1/sqrt(g).
 *             z = unnormalised butterfly of each group in fp32 with stages h = 1,2,..,g/2
 *             in ascending order, (a,b) -> (a+b, a-b), every step IEEE round-to-nearest-even.
 *  quantize   per row r: amax = max_k |z[r][k]| over the whole row; s_z = fp32(amax / 127);
 *             q[r][k] = clamp(round_half_even(fp32(z[r][k] / s_z)), -127, 127);
 *             stored scale s[r] = fp32(s_z * fp32(1/sqrt(g))). An all-zero row gives s = 0 and
 *             codes 0. So x_rot ~= s * q, with x_rot = x H_g / sqrt(g).
 *  matmul     acc[m][n] = sum_k qx[m][k] * qW[n][k] in int32 (exact for K <= 131072).
 *  epilogue   fp32: t = sx[m]*sW[n]; v = float(acc)*t; v = v + bias[n];
 *             (LoRA) v = v + lora_scale * L[m][n]; out = bf16_rne(v).
 *  LoRA       u = bf16_rne(x A) (fp32 accumulation), L = u B (fp32 accumulation), where x is
 *             the UNROTATED bf16 input: the adapter sits beside the frozen base layer.
 *
 * Conventions for every call:
 *  - Pointers are DEVICE pointers owned by the caller; the library allocates no device
 *    memory and keeps no per-call state. bf16 tensors are passed as their raw 16-bit
 *    patterns (uint16_t). Matrices are row-major; "ld" arguments are row strides in
 *    elements. When the row count of a call (M, or N for the weight call) is 0 the call
 *    is a no-op and the buffers that hold those rows may be NULL.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy default stream).
 *    The return value reports only argument validation and launch errors; nothing is
 *    launched when it is not SDNQ_OK, and outputs are then unspecified. Faults inside a
 *    kernel surface at the caller's next synchronisation.
 *  - Every bounded wait inside a kernel that gives up (default limit about 2 s) sets a
 *    device error word; sdnq_device_status() reads and clears it (SDNQ_ERR_TIMEOUT).
 *  - Only sm_100 devices are supported (SDNQ_ERR_UNSUPPORTED otherwise). There is no CPU
 *    and no other-architecture path.
 *  - The int8 GEMMs, the attention kernel and the attention preparation are launched with
 *    programmatic stream serialization. Such a kernel may start its prologue (barriers,
 *    tensor memory, descriptor prefetch) while the previous kernel in the stream drains. It
 *    reads or writes no global memory before that kernel has completed, so stream order
 *    holds for the caller's own kernels as well.
 */
#ifndef SDNQ_H
#define SDNQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SDNQ_OK = 0,
    SDNQ_ERR_NULL = 1,        /* a required pointer is NULL                               */
    SDNQ_ERR_SHAPE = 2,       /* a size is out of range or sizes are inconsistent          */
    SDNQ_ERR_ALIGN = 3,       /* a pointer or leading dimension breaks the 16-byte rule    */
    SDNQ_ERR_UNSUPPORTED = 4, /* group size or rank not supported, or device is not sm_100 */
    SDNQ_ERR_CUDA = 5,        /* a CUDA runtime call or a kernel launch failed             */
    SDNQ_ERR_TIMEOUT = 6      /* a bounded wait inside a kernel gave up                    */
} sdnq_status;

/* Largest K accepted by every call (int32 accumulators stay exact: 127*127*K < 2^31). */
#define SDNQ_MAX_K 131072
/* Supported Hadamard group sizes: powers of two in [SDNQ_MIN_GROUP, SDNQ_MAX_GROUP]. */
#define SDNQ_MIN_GROUP 8
#define SDNQ_MAX_GROUP 256
/* Supported LoRA ranks: multiples of 16 up to SDNQ_MAX_RANK. */
#define SDNQ_MAX_RANK 256

/*
 * Weight rotate + quantize (offline, once per weight): "ConvRot / Hadamard SDNQ", Quick
 * Setup and What The Options Do (sdnq_use_hadamard, sdnq_hadamard_group_size,
 * sdnq_group_size = -1 static full-row scales); "SDNQ: SD.Next Quantization Engine",
 * post-load quantization.
 *   W   [N, K] bf16, row stride ldw (>= K, multiple of 8), 16-byte aligned.
 *   qW  [N, K] int8 out, dense (row stride K), 16-byte aligned.
 *   sW  [N]    fp32 out, scale of row n of the normalised rotation.
 *   group: power of two, SDNQ_MIN_GROUP..SDNQ_MAX_GROUP; K % group == 0, K % 16 == 0,
 *   K <= SDNQ_MAX_K. N == 0 is a no-op.
 */
sdnq_status sdnq_rotate_quant_weight(const uint16_t *W, int64_t N, int64_t K, int64_t ldw,
                                     int32_t group, int8_t *qW, float *sW, void *stream);

/*
 * Online activation rotate + quantize, one dynamic scale per token: "SDNQ: SD.Next
 * Quantization Engine", feature list (Hadamard on the quantized matmul; INT8 matmul).
 * Same math as sdnq_rotate_quant_weight, applied to the rows (tokens) of x.
 *   x   [M, K] bf16, row stride ldx (>= K, multiple of 8), 16-byte aligned.
 *   qx  [M, K] int8 out, dense.   sx [M] fp32 out.   M == 0 is a no-op.
 */
sdnq_status sdnq_rotquant_act(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                              int32_t group, int8_t *qx, float *sx, void *stream);

/*
 * INT8 x INT8 -> INT32 matmul with the FP32 de-quant epilogue: "SDNQ: SD.Next Quantization
 * Engine", feature list (INT8 quantized matmul) and SDNQConfig (dequantize_fp32).
 *   qx [M, K] int8 dense, sx [M] fp32 (from sdnq_rotquant_act);
 *   qW [N, K] int8 dense, sW [N] fp32 (from sdnq_rotate_quant_weight), same group size.
 *   bias [N] bf16 or NULL. qx, qW, sW, bias and out are 16-byte aligned; sx 4-byte.
 *   out [M, N] bf16, row stride ldo (>= N, multiple of 8), 16-byte aligned.
 *   acc_out: NULL, or [M, N] int32 dense that also receives the raw accumulators (for
 *   parity checks; slower).
 *   K % 16 == 0, K <= SDNQ_MAX_K, N >= 1. M == 0 is a no-op.
 */
sdnq_status sdnq_int8_linear(const int8_t *qx, const float *sx, const int8_t *qW,
                             const float *sW, const uint16_t *bias, int64_t M, int64_t N,
                             int64_t K, uint16_t *out, int64_t ldo, int32_t *acc_out,
                             void *stream);

/*
 * The online path in one launch: sdnq_rotquant_act of x followed by sdnq_int8_linear, with
 * the activation rotate + quantize running inside the GEMM kernel on warps of its own (rows
 * are published per 128-row block; the tile loads wait for their block). Results are bit
 * for bit those of the two calls, which is also what the call runs when `policy` asks for it
 * or when the one launch does not pay off:
 *   policy SDNQ_FUSE_AUTO: one launch when the GEMM has at least three waves of 128 x 256
 *          tiles (ceil(M/128) * ceil(N/256) >= 3 * SM count), N >= 3584, K < 2 N and
 *          K <= 8192, else two;
 *   policy SDNQ_FUSE_ALWAYS: one launch whenever K <= 8192;  SDNQ_FUSE_NEVER: two launches.
 *   Above 128 rows the one launch runs on CTA pairs as a cooperative launch of two-CTA
 *   clusters (every CTA resident at once, since tile loads wait on rows that other CTAs
 *   quantize); if the device refuses that launch, the single-SM one-launch kernel runs
 *   instead (same bits) and the refusal is remembered for the device.
 *   x [M, K] bf16, row stride ldx; group as in sdnq_rotquant_act.
 *   qW, sW, bias, out, ldo, acc_out as in sdnq_int8_linear.
 *   qx_ws [M, K] int8 dense, sx_ws [M] fp32: caller-provided workspace for the activation
 *   codes and scales (they hold them afterwards).
 *   sync_ws: SDNQ_FUSED_SYNC_WORDS(M) uint32 counters, 4-byte aligned, which must be zero on
 *   entry; a call that returns SDNQ_OK with no device error leaves them zero again, so one
 *   zeroed buffer serves every later call on the same stream. Calls whose kernels overlap on
 *   the GPU need separate buffers. After a device timeout (sdnq_device_status) re-zero it.
 *   The two launches leave sync_ws untouched.
 *   The kernel is a cooperative launch (one CTA per SM, or one two-CTA cluster per two SMs,
 *   all resident at once); if the device can run neither form, the call returns
 *   SDNQ_ERR_CUDA.
 */
#define SDNQ_FUSED_SYNC_WORDS(M) (2 * (((M) + 127) / 128))
enum { SDNQ_FUSE_AUTO = 0, SDNQ_FUSE_ALWAYS = 1, SDNQ_FUSE_NEVER = 2 };
sdnq_status sdnq_int8_linear_fused(const uint16_t *x, int64_t ldx, int32_t group,
                                   const int8_t *qW, const float *sW, const uint16_t *bias,
                                   int64_t M, int64_t N, int64_t K, int8_t *qx_ws, float *sx_ws,
                                   uint32_t *sync_ws, uint16_t *out, int64_t ldo,
                                   int32_t *acc_out, int32_t policy, void *stream);

/*
 * The path sdnq_int8_linear_fused takes for these sizes and this policy on the current
 * device: *one_launch = 1 for the single kernel, 0 for the two launches (same results either
 * way). Nothing is launched and no pointer but one_launch is read, so a caller can label or
 * plan the path without restating the rule above.
 *   Errors: SDNQ_ERR_NULL (one_launch NULL), SDNQ_ERR_SHAPE (M < 0, N < 1, K < 16, K % 16,
 *   K > SDNQ_MAX_K), SDNQ_ERR_UNSUPPORTED (unknown policy or not an sm_100 device).
 */
sdnq_status sdnq_int8_linear_fused_plan(int64_t M, int64_t N, int64_t K, int32_t policy,
                                        int32_t *one_launch);

/*
 * sdnq_int8_linear with GELU fused into its epilogue, for the up-projection of a DiT MLP
 * whose output feeds the down-projection's rotate + quantize:
 *   out = gelu(bf16(float(acc) * (sx * sw) [+ bias])), GELU(y) = y * Phi(y) in the exact
 *   erf form, rounded once to bf16,
 * i.e. bit for bit sdnq_int8_linear followed by sdnq_gelu_bf16 on its output, without the
 * second pass over [M, N] in HBM. Arguments, layouts, alignment and errors are those of
 * sdnq_int8_linear; acc_out (if set) receives the raw accumulators.
 * The GELU values come from a 7 KB table that the library keeps in device memory: the first
 * call on a device builds it with a small kernel on `stream` and waits for that kernel (so
 * make the first call outside any stream capture); later calls only read it.
 */
sdnq_status sdnq_int8_linear_gelu(const int8_t *qx, const float *sx, const int8_t *qW,
                                  const float *sW, const uint16_t *bias, int64_t M, int64_t N,
                                  int64_t K, uint16_t *out, int64_t ldo, int32_t *acc_out,
                                  void *stream);

/*
 * Input gradient through the frozen rotated int8 base, for PEFT training where the base
 * layer is frozen and only its input needs a gradient ("ConvRot / Hadamard SDNQ", PEFT
 * Behavior; "SDNQ: SD.Next Quantization Engine", quantized training example: the quantized
 * matmul also runs on the backward pass). The layer holds W_hat = diag(sW) qW H_g / sqrt(g)
 * (H_g the block-diagonal Sylvester matrix, symmetric), so dx = dy W_hat is computed as:
 *   1. qg, sg = per-token int8 of c = fp32(dy) * sW[n] (sW varies along the contraction, so
 *      it is folded into dy): sg = fp32(amax_n |c| / 127), qg = rne(c / sg) clamped to
 *      [-127, 127]; an all-zero row gives sg = 0 and codes 0;
 *   2. acc[m][k] = sum_n qg[m][n] * qW[n][k] in int32 (tensor cores, qW read in place);
 *   3. dx = bf16( FWHT_g(fp32(acc) * sg[m]) * fp32(1/sqrt(g)) ), the butterfly in fp32
 *      with ascending stages per group of g columns.
 *   dy    [M, N] bf16, row stride lddy (>= N, multiple of 8), 16-byte aligned.
 *   qW    [N, K] int8 and sW [N] fp32 from sdnq_rotate_quant_weight with this `group`
 *         (16-byte aligned).
 *   qg_ws [M, N] int8 dense and sg_ws [M] fp32: caller-provided workspace; they hold qg and
 *         sg afterwards.
 *   dx    [M, K] bf16 out, row stride lddx (>= K, multiple of 8), 16-byte aligned.
 *   acc_out: NULL, or [M, K] int32 dense for the raw accumulators (parity checks).
 *   N % 16 == 0 (16..SDNQ_MAX_K), K % 16 == 0, K % group == 0. M == 0 is a no-op.
 */
sdnq_status sdnq_int8_linear_grad_input(const uint16_t *dy, int64_t lddy, const int8_t *qW,
                                        const float *sW, int64_t M, int64_t N, int64_t K,
                                        int32_t group, int8_t *qg_ws, float *sg_ws,
                                        uint16_t *dx, int64_t lddx, int32_t *acc_out,
                                        void *stream);

/*
 * Step 1 of sdnq_int8_linear_grad_input on its own: qg [M, N] int8 dense and sg [M] fp32,
 * the per-token int8 of fp32(dy) * sW. Arguments and rules as there.
 */
sdnq_status sdnq_quant_grad_output(const uint16_t *dy, int64_t lddy, const float *sW, int64_t M,
                                   int64_t N, int8_t *qg, float *sg, void *stream);

/*
 * Steps 2 and 3 of sdnq_int8_linear_grad_input on their own: dx [M, K] from qg, sg (step 1)
 * and the layer's codes qW [N, K] of this `group`. Arguments and rules as there.
 */
sdnq_status sdnq_int8_grad_input_gemm(const int8_t *qg, const float *sg, const int8_t *qW,
                                      int64_t M, int64_t N, int64_t K, int32_t group,
                                      uint16_t *dx, int64_t lddx, int32_t *acc_out,
                                      void *stream);

/*
 * As sdnq_int8_linear, plus the bf16 LoRA side term of PEFT training on a frozen int8
 * base ("ConvRot / Hadamard SDNQ", PEFT Behavior): out = bf16(v + lora_scale * (u B)),
 * u = bf16(x A).
 *   x  [M, K] bf16, the UNROTATED layer input, row stride ldx (multiple of 8).
 *   A  [K, rank] bf16 dense.   B [rank, N] bf16 dense (N % 8 == 0).
 *   rank: multiple of 16, 16..SDNQ_MAX_RANK.
 *   u_ws [M, rank] bf16: caller-provided workspace; holds u = bf16(x A) afterwards.
 */
sdnq_status sdnq_int8_linear_lora(const int8_t *qx, const float *sx, const int8_t *qW,
                                  const float *sW, const uint16_t *bias, const uint16_t *x,
                                  int64_t ldx, const uint16_t *A, const uint16_t *B,
                                  int32_t rank, float lora_scale, uint16_t *u_ws, int64_t M,
                                  int64_t N, int64_t K, uint16_t *out, int64_t ldo,
                                  int32_t *acc_out, void *stream);

/*
 * The two halves of sdnq_int8_linear_lora as calls of their own (same kernels, same bits):
 * the LoRA down-projection u = bf16(x A), and the int8 linear with the adapter term from a
 * given u, out = bf16(v + lora_scale * (u B)). A caller that keeps u (the adapter's weight
 * gradient dB = u^T dy reads it), or computes it on another stream, uses these.
 *
 * sdnq_lora_down: x [M, K] bf16, the UNROTATED layer input, row stride ldx (multiple of 8);
 *   A [K, rank] bf16 dense; u [M, rank] bf16 dense (output). K % 16 == 0, 16 <= K <=
 *   SDNQ_MAX_K; rank a multiple of 16, 16..SDNQ_MAX_RANK (else SDNQ_ERR_UNSUPPORTED);
 *   x, A, u 16-byte aligned. M == 0 is a no-op. u is rounded once from fp32 tensor-core
 *   sums (the order of the products is the tensor cores').
 * sdnq_int8_linear_lora_up: qx, sx, qW, sW, bias, M, N, K, out, ldo, acc_out as in
 *   sdnq_int8_linear; u [M, rank] bf16 dense as written by sdnq_lora_down (or any bf16
 *   values); B [rank, N] bf16 dense, N % 8 == 0; rank and alignment as above.
 */
sdnq_status sdnq_lora_down(const uint16_t *x, int64_t ldx, const uint16_t *A, int32_t rank,
                           int64_t M, int64_t K, uint16_t *u, void *stream);
sdnq_status sdnq_int8_linear_lora_up(const int8_t *qx, const float *sx, const int8_t *qW,
                                     const float *sW, const uint16_t *bias, const uint16_t *u,
                                     const uint16_t *B, int32_t rank, float lora_scale,
                                     int64_t M, int64_t N, int64_t K, uint16_t *out,
                                     int64_t ldo, int32_t *acc_out, void *stream);

/*
 * sdnq_int8_linear_lora without the caller-provided workspace. The pages have no
 * counterpart: this entry point is for callers that cannot allocate device memory for u_ws,
 * because their host framework owns all device memory (a caching allocator or a fixed
 * memory plan) and forbids allocations from outside it, or because a cudaMalloc, which may
 * synchronise the device and has unpredictable latency, is not acceptable where they run.
 * It allocates nothing: u = bf16(x A) lives in a fixed array inside the library, of
 * SDNQ_NOALLOC_MAX_U_ELEMS bf16 values (8 MiB), held on every GPU that loads the library
 * until the process exits. Arguments and results are those of sdnq_int8_linear_lora minus
 * u_ws; u itself is not returned.
 *   Limit: M * rank <= SDNQ_NOALLOC_MAX_U_ELEMS, else SDNQ_ERR_SHAPE and nothing is launched.
 *   The first call on each device looks up the array's device address (with that device
 *   current); make that first call before any stream capture.
 *   Every call uses the same array, which keeps the last call's u: calls whose kernels
 *   overlap on the GPU (different streams, or different host threads) race on it and must
 *   be serialised by the caller. Nothing in it needs clearing between calls.
 */
#define SDNQ_NOALLOC_MAX_U_ELEMS (1 << 22)
sdnq_status sdnq_int8_linear_lora_noalloc(const int8_t *qx, const float *sx, const int8_t *qW,
                                          const float *sW, const uint16_t *bias,
                                          const uint16_t *x, int64_t ldx, const uint16_t *A,
                                          const uint16_t *B, int32_t rank, float lora_scale,
                                          int64_t M, int64_t N, int64_t K, uint16_t *out,
                                          int64_t ldo, int32_t *acc_out, void *stream);

/*
 * FP8 (e4m3) variant of the rotated quantized matmul ("SDNQ: SD.Next Quantization Engine",
 * feature list and SDNQConfig: FP8 weights and FP8 quantized matmul beside INT8), same
 * rotation. e4m3 here is the "fn" format: bias 7, 3 mantissa bits, largest finite 448, no
 * infinities.
 *
 * sdnq_rotquant_fp8: rows of x (weights or activations) rotated as in sdnq_rotquant_act,
 * then s_z = fp32(amax / 448), codes = e4m3(fp32(z / s_z)) (round to nearest even,
 * saturating), stored scale s = fp32(s_z * fp32(1/sqrt(group))); an all-zero row gives s = 0
 * and +0 codes. Arguments, layouts and rules as sdnq_rotquant_act, codes as uint8.
 */
sdnq_status sdnq_rotquant_fp8(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                              int32_t group, uint8_t *q, float *s, void *stream);

/*
 * sdnq_fp8_linear: out = bf16(acc * (sx * sw) [+ bias]) with acc[m][n] = sum_k qx[m][k] *
 * qW[n][k] over e4m3 codes, accumulated in fp32 on the tensor cores (tcgen05 kind::f8f6f4;
 * the summation order is the hardware's, so acc matches an exact sum only to within fp32
 * accumulation error). Arguments, layouts and rules as sdnq_int8_linear; acc_out, if set, is
 * [M, N] fp32.
 */
sdnq_status sdnq_fp8_linear(const uint8_t *qx, const float *sx, const uint8_t *qW,
                            const float *sW, const uint16_t *bias, int64_t M, int64_t N,
                            int64_t K, uint16_t *out, int64_t ldo, float *acc_out, void *stream);

/*
 * Attention with a Hadamard-rotated int8 QK^T and a bf16 PV ("SDNQ: SD.Next Quantization
 * Engine", SDNQ attention: int8 QK matmul, smooth_k, use_hadamard, hadamard_group_size; PV
 * matmul unquantized). q [B, Lq, H, D], k and v [B, Lk, H, D], o [B, Lq, H, D], all bf16 and
 * dense (token-head rows of D contiguous values), 16-byte aligned; D must be 128.
 *   smooth_k != 0: mu[b][h][d] = fp32(sum_j k / Lk) (sum in fp64) is subtracted from every
 *   key in fp32 (the softmax is unchanged by it); else mu = 0.
 *   Q rows and K - mu rows are rotated by the butterfly over groups of min(group, D) and
 *   quantized per row exactly as sdnq_rotquant_act does; logits are
 *   fp32(fp32(fp32(acc) * fp32(s_q * s_k)) * scale), acc the int32 dot product of the codes;
 *   o = softmax(logits) v, with the probabilities rounded to bf16 for the PV product (fp32
 *   accumulation) and o rounded to bf16. scale: finite and >= 0 (else SDNQ_ERR_UNSUPPORTED);
 *   a usual scale is fp32(1/sqrt(D)).
 *   group: power of two, SDNQ_MIN_GROUP..SDNQ_MAX_GROUP (groups above D act as D).
 *   ws: caller workspace of sdnq_attention_workspace(...) bytes, 256-byte aligned. Afterwards
 *   it holds, at the offsets that function reports: [0] Q codes int8 [B, Lq, H, D], [1] K codes,
 *   [2] Q scales fp32 [B, H, Lq_pad], [3] K scales [B, H, Lk_pad] (L_pad = L rounded up to a
 *   multiple of 128; the padding is not written), [4] mu fp32 [B, H, D], [5] scratch.
 * Launches: (smooth_k) two for mu, two row quantizers, one attention kernel.
 */
int64_t sdnq_attention_workspace(int64_t B, int64_t Lq, int64_t Lk, int64_t H, int64_t D,
                                 int64_t *offsets /* [6] or NULL */);
sdnq_status sdnq_attention_int8qk(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                  int64_t B, int64_t Lq, int64_t Lk, int64_t H, int64_t D,
                                  int32_t group, float scale, int32_t smooth_k, void *ws,
                                  int64_t ws_bytes, uint16_t *o, void *stream);

/* The two halves of sdnq_attention_int8qk, same arguments and rules: the preparation
 * (smooth_k means, Q and K codes and scales into ws), and the attention kernel on a prepared
 * ws (o from the codes, the scales and v). */
sdnq_status sdnq_attention_prep(const uint16_t *q, const uint16_t *k, int64_t B, int64_t Lq,
                                int64_t Lk, int64_t H, int64_t D, int32_t group,
                                int32_t smooth_k, void *ws, int64_t ws_bytes, void *stream);
sdnq_status sdnq_attention_core(const uint16_t *v, int64_t B, int64_t Lq, int64_t Lk, int64_t H,
                                int64_t D, float scale, void *ws, int64_t ws_bytes, uint16_t *o,
                                void *stream);

/*
 * GELU between the up and down projections of a DiT MLP (exact erf form,
 * x * Phi(x), rounded once to bf16). Not on the pages; the MLP workload needs it.
 *   in [M, N] bf16 row stride ld_in; out [M, N] bf16 row stride ld_out (may alias in when
 *   ld_out == ld_in). Strides multiples of 8, pointers 16-byte aligned.
 */
sdnq_status sdnq_gelu_bf16(const uint16_t *in, int64_t M, int64_t N, int64_t ld_in,
                           uint16_t *out, int64_t ld_out, void *stream);

/*
 * Synchronises `stream`, then reads and clears the device error word that bounded waits
 * inside the kernels set when they give up. Returns SDNQ_OK, SDNQ_ERR_TIMEOUT, or
 * SDNQ_ERR_CUDA if the synchronisation itself failed.
 */
sdnq_status sdnq_device_status(void *stream);

/*
 * Self-test of the bounded-wait machinery: launches one small kernel whose wait can never
 * be satisfied (an mbarrier that nothing arrives on), with a limit of `limit_ns`
 * nanoseconds (1e3..1e10). The kernel gives up, records SDNQ_ERR_TIMEOUT in the device
 * error word and returns; no fault, trap or hang is involved.
 */
sdnq_status sdnq_selftest_wait_timeout(int64_t limit_ns, void *stream);

/* Human-readable name of a status code (static string, never NULL). */
const char *sdnq_status_string(sdnq_status s);

/* Library version string, e.g. "sdnq-b200 0.1.0 sm_100a". */
const char *sdnq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SDNQ_H */
