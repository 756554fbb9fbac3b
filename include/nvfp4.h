/*
 * nvfp4.h — C ABI of the B200 (sm_100a) NVFP4 linear-layer library.
 *
 * NVFP4 is two-level microblock quantization: an FP32 scale per tensor
 * (static or dynamic) and a scale per block of 16 elements computed
 * dynamically ("英伟达B200狂飙10.2倍！AI绘图告别龟速！", section
 * "NVFP4量化：在精度与速度之间寻得最佳平衡"; "Scaling NVFP4 Inference for
 * FLUX.2 on NVIDIA Blackwell Data Center GPUs", section "Key Questions
 * Answered").  Encoding used here: E2M1 elements (two per byte, the even
 * element in the low nibble) and unsigned E4M3 block scales.
 *
 * Quantization of a bf16 tensor X[rows, cols] (cols % 16 == 0), blocks of 16
 * contiguous elements along cols:
 *   S_enc = 2688 / amax        (1 if amax == 0, FLT_MAX if not finite)
 *   S_dec = 1 / S_enc
 *   per block b:  sf_b = E4M3_rn_satfinite((max|x| / 6) * S_enc)
 *                 q_i  = E2M1_rn_satfinite(x_i * (S_enc / sf_b)), 0 if sf_b == 0
 * Every fp32 step is one IEEE round-to-nearest-even operation, so results are
 * bit-reproducible.  A negative value that rounds to zero keeps its sign (-0).
 *
 * Scale-factor layout ("tiled SF"): pad128(rows) x pad4(cols/16) bytes in
 * 128-row x 4-block tiles of 512 bytes, tiles ordered row-block-major; in a
 * tile, (r, c) is at byte (r%32)*16 + ((r/32)%4)*4 + c%4.  Padding bytes are
 * written as 0.  This is the layout the tcgen05 block-scaled MMA consumes.
 *
 * GEMM: Y[m,n] = bf16_rn( a_s_dec * b_s_dec *
 *                sum_k e2m1(Aq[m,k]) sfA[m,k/16] e2m1(Bq[n,k]) sfB[n,k/16] )
 * with A = activations [M,K] and B = weights [N,K] (nn.Linear layout), fp32
 * accumulation in tensor memory.
 *
 * Conventions for every call below:
 *  - Pointers marked "device" are device memory owned by the caller; the
 *    library never allocates, frees or synchronises, and keeps no pointer
 *    after the call returns.  "host" pointers are host memory (pinned for
 *    truly asynchronous copies).
 *  - Work is enqueued on `stream` (NULL = legacy default stream) and runs
 *    asynchronously; results are valid after the stream is synchronised.
 *  - Argument errors are returned synchronously before anything is
 *    enqueued; launch errors are returned as NVFP4_ERR_LAUNCH.  Nothing
 *    aborts or throws across the ABI.  A kernel that gives up on a bounded
 *    wait records NVFP4_ERR_TIMEOUT in a device word read by
 *    nvfp4_device_error().
 *  - Device pointers must be 16-byte aligned (NVFP4_ERR_MISALIGNED).
 *  - An empty tensor (rows == 0) is valid input to every quantize call: no
 *    element is read or written, the arrays of the empty tensor may be NULL,
 *    and the per-tensor scalars are still written (amax 0, s_dec from the
 *    scale the call derives or is given).  GEMMs need M, N >= 1.
 *  - The device must be sm_100 (B200); otherwise NVFP4_ERR_UNSUPPORTED_DEVICE.
 *  - Inputs must be finite (no NaN/inf in X or W).
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream. */
typedef struct CUstream_st *nvfp4_stream_t;

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1,
    NVFP4_ERR_MISALIGNED = 2,
    NVFP4_ERR_UNSUPPORTED_DEVICE = 3,
    NVFP4_ERR_LAUNCH = 4,
    NVFP4_ERR_TIMEOUT = 5
} nvfp4_status;

/* Activation applied to the GEMM output inside a fused epilogue, before the
 * bf16 rounding.  The pages' GEMM kernels fuse consecutive operations into
 * the GEMM (xalabuda page, section "Квантование NVFP4 и оптимизация
 * вычислительных ядер"); in a DiT block the FFN up-projection is followed by
 * its activation, read here as the exact (erf) GELU, whose output is the
 * FFN down-projection's input. */
typedef enum {
    NVFP4_ACT_NONE = 0,
    NVFP4_ACT_GELU = 1 /* g(h) = 0.5 h (1 + erf(h / sqrt(2))) in fp32, erf by
                        * Abramowitz & Stegun 7.1.26 (|error| <= 1.5e-7) */
} nvfp4_activation;

/* Optional fused output quantization of the GEMM (the next layer's
 * activation quantize, done in the GEMM epilogue).  With h = alpha * acc in
 * fp32, Y = bf16_rn(h) (activation NONE) or bf16_rn(g(h)) (GELU); Y is then
 * quantized in blocks of 16 along N with the caller's S_enc (static, or the
 * previous call's amax via 2688/amax).  The bf16 output y_bf16 of
 * nvfp4_gemm, when given, is this same Y.  Requires N % 16 == 0.
 *   s_enc_y    device, 1 fp32, read
 *   yq         device, M*N/2 bytes, written (packed E2M1, row-major)
 *   ysf        device, nvfp4_sf_bytes(M, N) bytes, written (tiled SF, padding 0)
 *   amax_y     device, 1 fp32, overwritten with max|Y| over the bf16 Y
 *              (NULL = not computed)
 *   s_dec_y    device, 1 fp32, written with 1/S_enc (IEEE fp32 division), the
 *              decode scale a GEMM consuming (yq, ysf) needs (NULL = not
 *              written)
 *   activation an nvfp4_activation value; anything else is
 *              NVFP4_ERR_INVALID_ARG */
typedef struct {
    const float *s_enc_y;
    uint8_t *yq;
    uint8_t *ysf;
    float *amax_y;
    float *s_dec_y;
    int activation;
} nvfp4_fused_out;

/* Bytes of packed E2M1 data for a [rows, cols] tensor: rows * cols / 2. */
size_t nvfp4_packed_bytes(int64_t rows, int64_t cols);

/* Bytes of the tiled scale-factor buffer: pad128(rows) * pad4(cols / 16). */
size_t nvfp4_sf_bytes(int64_t rows, int64_t cols);

/* Static description of a status code (never NULL). */
const char *nvfp4_status_string(nvfp4_status status);

/* Per-tensor absolute maximum, the input of the dynamic per-tensor scale
 * (FP32 per-tensor scale "computed statically or dynamically": nmedialink
 * page above, NVFP4 section).
 *   x_bf16    device, numel bf16 values, read
 *   numel     >= 0 (0 writes amax = 0)
 *   amax_dev  device, 1 fp32, overwritten with max_i |x_i| */
nvfp4_status nvfp4_tensor_amax(const void *x_bf16, int64_t numel, float *amax_dev,
                               nvfp4_stream_t stream);

/* Dynamic NVFP4 quantization (per-16 block scales computed at run time:
 * nmedialink page above, NVFP4 section).  S_enc is derived on the device
 * from *amax_dev, so no host synchronisation is needed.
 *   x_bf16     device, [rows, cols] row-major bf16, read; cols % 16 == 0
 *   amax_dev   device, 1 fp32, read (normally from nvfp4_tensor_amax)
 *   q_out      device, rows*cols/2 bytes, written
 *   sf_out     device, nvfp4_sf_bytes(rows, cols) bytes, written (incl. padding)
 *   s_dec_out  device, 1 fp32, written with 1/S_enc (NULL = not written) */
nvfp4_status nvfp4_quantize(const void *x_bf16, int64_t rows, int64_t cols,
                            const float *amax_dev, uint8_t *q_out, uint8_t *sf_out,
                            float *s_dec_out, nvfp4_stream_t stream);

/* Static-scale variant: same as nvfp4_quantize but S_enc is given directly
 * (the per-tensor scale "computed statically": nmedialink page above).
 *   s_enc_dev  device, 1 fp32 > 0, read */
nvfp4_status nvfp4_quantize_with_scale(const void *x_bf16, int64_t rows, int64_t cols,
                                       const float *s_enc_dev, uint8_t *q_out,
                                       uint8_t *sf_out, float *s_dec_out,
                                       nvfp4_stream_t stream);

/* One-pass NVFP4 quantization with the tensor scale of an earlier tensor:
 * the per-tensor scale "static or dynamic" (nmedialink page above, NVFP4
 * section) read as dynamic but one call stale.  S_enc is derived on the
 * device from *amax_prev_dev exactly as nvfp4_quantize derives it from
 * *amax_dev, the tensor is read once (no amax pass before the quantize),
 * and this tensor's own amax is written for the next call.  Blocks whose
 * values outgrew the stale scale saturate (E4M3 448, E2M1 6).
 *   x_bf16, rows, cols, q_out, sf_out, s_dec_out  as for nvfp4_quantize
 *   amax_prev_dev  device, 1 fp32, read (an earlier call's amax_out, or any
 *                  amax the caller chooses for the first call)
 *   amax_out       device, 1 fp32, written with max|x| of this tensor; must
 *                  not alias amax_prev_dev (callers alternate two words) */
nvfp4_status nvfp4_quantize_one_pass(const void *x_bf16, int64_t rows, int64_t cols,
                                     const float *amax_prev_dev, uint8_t *q_out, uint8_t *sf_out,
                                     float *s_dec_out, float *amax_out, nvfp4_stream_t stream);

/* Bytes of device workspace needed by nvfp4_quantize_dynamic (32). */
size_t nvfp4_quantize_dynamic_workspace_bytes(void);

/* Dynamic NVFP4 quantization in one launch: the per-tensor amax, S_enc and
 * the per-16 block quantization of nvfp4_tensor_amax + nvfp4_quantize
 * (nmedialink page above, NVFP4 section: dynamic per-tensor and per-block
 * scales), with identical results.  A cooperative kernel reduces the amax,
 * crosses one grid barrier and quantizes; where a slice of the tensor per SM
 * fits in shared memory it stays there between the two phases, otherwise
 * the second read comes from L2 where the tensor fits.
 *   x_bf16, rows, cols, q_out, sf_out, s_dec_out  as for nvfp4_quantize
 *   amax_out   device, 1 fp32, written with max|x| (NULL = not written)
 *   workspace  device, nvfp4_quantize_dynamic_workspace_bytes() bytes,
 *              16-byte aligned, zero-filled once by the caller before its
 *              first use and then reused unchanged; calls that share a
 *              workspace must be ordered (same stream, or synchronised).
 *              After an NVFP4_ERR_TIMEOUT it must be zero-filled again. */
nvfp4_status nvfp4_quantize_dynamic(const void *x_bf16, int64_t rows, int64_t cols,
                                    uint8_t *q_out, uint8_t *sf_out, float *s_dec_out,
                                    float *amax_out, void *workspace, nvfp4_stream_t stream);

/* nvfp4_quantize_dynamic for callers that cannot allocate device memory: an
 * inference-engine plugin whose execute step may not allocate, a runtime
 * that owns all device memory through its own arena, or a latency-critical
 * loop that must avoid cudaMalloc/cudaFree because they can synchronise the
 * device.  No counterpart on the pages: it is the same computation with the
 * same results as nvfp4_quantize_dynamic, and allocates nothing.
 *   x_bf16, rows, cols, q_out, sf_out, s_dec_out, amax_out
 *              as for nvfp4_quantize_dynamic (the caller still provides every
 *              input and output)
 * Scratch: instead of a caller workspace the call uses a 256-byte array
 * inside the library (every GPU that loads the library holds it until the
 * process exits).  The call clears the part it needs on `stream` before
 * using it.  The scratch needed is 32 bytes for any tensor size; a call that
 * would need more than 256 bytes is refused with NVFP4_ERR_INVALID_ARG.
 * The first call on a device looks up the array's device address, so make
 * that first call before any stream capture.  All calls on a device share
 * the one array: calls that overlap on the GPU (on streams not ordered with
 * each other) race on it and give wrong results. */
nvfp4_status nvfp4_quantize_dynamic_noalloc(const void *x_bf16, int64_t rows, int64_t cols,
                                            uint8_t *q_out, uint8_t *sf_out, float *s_dec_out,
                                            float *amax_out, nvfp4_stream_t stream);

/* Block-scaled FP4 GEMM on tcgen05 tensor cores, Y = X . W^T (the NVFP4
 * linear layer whose weights are quantized once, "quantize_weights=True",
 * nmedialink page above, NVFP4 section).
 *   aq, asf, a_s_dec   device: activations [M,K] quantized (packed, tiled SF,
 *                      1 fp32 decode scale)
 *   bq, bsf, b_s_dec   device: weights [N,K] quantized likewise
 *   M >= 1, N >= 1 with N % 8 == 0, K >= 64 with K % 64 == 0
 *   y_bf16             device, [M,N] row-major bf16, written (NULL allowed
 *                      only when fused != NULL)
 *   fused              NULL, or the fused output quantization above */
nvfp4_status nvfp4_gemm(const uint8_t *aq, const uint8_t *asf, const float *a_s_dec,
                        const uint8_t *bq, const uint8_t *bsf, const float *b_s_dec,
                        int64_t M, int64_t N, int64_t K, void *y_bf16,
                        const nvfp4_fused_out *fused, nvfp4_stream_t stream);

/* Per-token activation scales (the per-tensor FP32 scale of the two-level
 * scheme taken per row, so an outlier token does not shrink every other
 * token's block scales).  The pages describe one FP32 scale over the whole
 * tensor (nmedialink page above, NVFP4 section); this is the finer-grained
 * variant of that level, with the same per-16 E4M3 block scales.  Row r is
 * quantized exactly as nvfp4_quantize would quantize the 1-row tensor X[r]
 * with its own amax (S_enc[r] = 2688 / amax(row r)); the codes and the tiled
 * scale layout are the usual ones (padding rows get zero scales).
 *   x_bf16, rows, cols, q_out, sf_out  as for nvfp4_quantize
 *   s_dec_rows  device, rows fp32, written with 1 / S_enc[r] (4-byte aligned)
 *   amax_rows   device, rows fp32, written with amax(row r), or NULL
 * One launch of independent warps (one per row), no grid-wide step. */
nvfp4_status nvfp4_quantize_rowwise(const void *x_bf16, int64_t rows, int64_t cols,
                                    uint8_t *q_out, uint8_t *sf_out, float *s_dec_rows,
                                    float *amax_rows, nvfp4_stream_t stream);

/* nvfp4_gemm with per-row decode scales for A (from nvfp4_quantize_rowwise):
 * Y[m,n] = bf16(S_dec,A[m] * S_dec,B * sum ...).  a_s_dec_rows holds M fp32
 * values; everything else as for nvfp4_gemm. */
nvfp4_status nvfp4_gemm_rowscale(const uint8_t *aq, const uint8_t *asf, const float *a_s_dec_rows,
                                 const uint8_t *bq, const uint8_t *bsf, const float *b_s_dec,
                                 int64_t M, int64_t N, int64_t K, void *y_bf16,
                                 const nvfp4_fused_out *fused, nvfp4_stream_t stream);

/* FP8 variant: the pages also run the DiT with an FP8 mode ("--variant
 * fp8r", xalabuda page, section "2. Запуск генерации изображения") without
 * describing its scaling; read here as E4M3 elements with one FP32 scale per
 * tensor: S_enc = 448 / amax (1 if amax == 0, FLT_MAX if not finite),
 * q = E4M3_rn_satfinite(x * S_enc) with the sign kept, S_dec = 1 / S_enc.
 *   x_bf16      device, [rows, cols] bf16 row-major, cols % 16 == 0
 *   amax_dev    device, 1 fp32, read (nvfp4_tensor_amax of x, or a static one)
 *   q_out       device, rows * cols bytes, written (E4M3 codes, row-major)
 *   s_dec_out   device, 1 fp32, written with 1 / S_enc */
nvfp4_status nvfp4_fp8_quantize(const void *x_bf16, int64_t rows, int64_t cols,
                                const float *amax_dev, uint8_t *q_out, float *s_dec_out,
                                nvfp4_stream_t stream);

/* FP8 GEMM on tcgen05 tensor cores (kind::f8f6f4, CTA pairs), Y = X . W^T
 * with Y[m,n] = bf16(S_dec,A * S_dec,B * sum_k e4m3(A[m,k]) e4m3(B[n,k])),
 * fp32 accumulation.  A [M,K] and B [N,K] E4M3 codes from nvfp4_fp8_quantize;
 * M > 128, N >= 256 with N % 8 == 0, K >= 32 with K % 32 == 0 (other shapes:
 * NVFP4_ERR_INVALID_ARG).  y_bf16 and fused as for nvfp4_gemm. */
nvfp4_status nvfp4_fp8_gemm(const uint8_t *a8, const float *a_s_dec, const uint8_t *b8,
                            const float *b_s_dec, int64_t M, int64_t N, int64_t K, void *y_bf16,
                            const nvfp4_fused_out *fused, nvfp4_stream_t stream);

/* Failure-detection self-test (no counterpart on the pages): launches one
 * warp that waits, through the same bounded mbarrier wait every kernel of
 * this library uses, on a barrier that is never completed.  After
 * timeout_us microseconds (1 .. 2000000) the wait gives up, the kernel
 * records NVFP4_ERR_TIMEOUT with detail NVFP4_SELFTEST_TAG in the device
 * error word and returns normally: nvfp4_device_error() then reports it, and
 * the context stays usable.  Faults, traps and hangs are never used. */
#define NVFP4_SELFTEST_TAG 90
nvfp4_status nvfp4_selftest_wait_timeout(int64_t timeout_us, nvfp4_stream_t stream);

/* Device buffers for nvfp4_linear_host (all caller-owned device memory):
 *   x      [M,K] bf16      xq  M*K/2 bytes      xsf  nvfp4_sf_bytes(M,K)
 *   amax   1 fp32          s_dec 1 fp32         y    [M,N] bf16
 *   dyn_ws workspace of nvfp4_quantize_dynamic (zero-filled once), or NULL
 *          to quantize with nvfp4_tensor_amax + nvfp4_quantize */
typedef struct {
    void *x;
    uint8_t *xq;
    uint8_t *xsf;
    float *amax;
    float *s_dec;
    void *y;
    void *dyn_ws;
} nvfp4_linear_workspace;

/* One NVFP4 linear layer from host memory: copies X host->device, runs
 * amax, dynamic quantize and the GEMM against pre-quantized weights, and
 * copies Y device->host, all enqueued on `stream` (the per-call activation
 * path of the pages' NVFP4 linear: dynamic activation quantization, static
 * weights).
 *   x_host_bf16   host, [M,K] bf16, read
 *   wq, wsf, w_s_dec  device, weights [N,K] quantized once
 *   y_host_bf16   host, [M,N] bf16, written once the stream completes */
nvfp4_status nvfp4_linear_host(const void *x_host_bf16, int64_t M, int64_t K,
                               const uint8_t *wq, const uint8_t *wsf,
                               const float *w_s_dec, int64_t N, void *y_host_bf16,
                               const nvfp4_linear_workspace *ws, nvfp4_stream_t stream);

/* Reads and clears the device-side error word of the current device
 * (synchronises the device).  *code_out = NVFP4_OK or NVFP4_ERR_TIMEOUT;
 * *detail_out (may be NULL) = which wait gave up (kernel-specific tag). */
nvfp4_status nvfp4_device_error(int *code_out, int *detail_out);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H */
