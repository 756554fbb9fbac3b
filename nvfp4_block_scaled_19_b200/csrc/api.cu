// C ABI of the NVFP4 linear-layer library (declared in include/nvfp4.h):
// argument checks, device check, TMA descriptor encoding and launches.
// The library never allocates device memory and never synchronises except in
// nvfp4_device_error().
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>

#include "api_checks.h"
#include "gemm.h"
#include "nvfp4.h"

namespace nvfp4 {
cudaError_t read_and_clear_device_error(int *code, int *detail);
}

namespace {

constexpr int kMaxDevices = 64;

// Per device: the SM count, published by a release store of `state` (0
// unknown, 1 supported, 2 unsupported), so host threads that make their first
// calls at the same time read either "unknown" or a complete entry.
struct DeviceInfo {
    std::atomic<int> state;
    std::atomic<int> num_sms;
};
DeviceInfo g_devices[kMaxDevices];

}  // namespace

namespace nvfp4 {

// The library ships one sm_100a image, so only compute capability 10.0 can
// run its kernels; any other device (other 10.x parts included) is refused
// up front instead of failing at launch.
nvfp4_status current_device(int *num_sms) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return NVFP4_ERR_UNSUPPORTED_DEVICE;
    }
    DeviceInfo &d = g_devices[dev];
    int state = d.state.load(std::memory_order_acquire);
    if (state == 0) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return NVFP4_ERR_UNSUPPORTED_DEVICE;
        }
        state = (major == 10 && minor == 0) ? 1 : 2;
        d.num_sms.store(sms, std::memory_order_relaxed);
        d.state.store(state, std::memory_order_release);
    }
    if (state != 1) return NVFP4_ERR_UNSUPPORTED_DEVICE;
    *num_sms = d.num_sms.load(std::memory_order_relaxed);
    return NVFP4_OK;
}

}  // namespace nvfp4

namespace {

using nvfp4::current_device;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

nvfp4_status from_cuda(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH; }

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    // Looked up once; atomic because host threads may make their first calls
    // at the same time (they all store the same entry point).
    static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> cached{nullptr};
    PFN_cuTensorMapEncodeTiled_v12000 fn = cached.load(std::memory_order_acquire);
    if (fn == nullptr) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess) {
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
            cached.store(fn, std::memory_order_release);
        } else {
            cudaGetLastError();
        }
    }
    return fn;
}

// 2-D byte tensor [rows, row_bytes] (row-major), 128-byte-swizzled boxes of
// box_rows x 128 bytes.
bool encode_operand_map(CUtensorMap *m, const void *base, uint64_t row_bytes, uint64_t rows,
                        uint32_t box_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (enc == nullptr) return false;
    cuuint64_t dims[2] = {row_bytes, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {128, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D bf16 tensor [rows, cols] (row-major) for TMA stores of 32-row x 64-column
// boxes (128 bytes per row, 128-byte swizzle); out-of-range rows and columns
// of a box are not written.
bool encode_output_map(CUtensorMap *m, void *base, uint64_t cols, uint64_t rows) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (enc == nullptr) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Tiled scale factors of a [rows, K] NVFP4 tensor as a 3-D byte tensor
// [ceil(rows / 128) blocks][K / 32 lines][256 bytes] (each 512-byte tile of
// 128 rows x 4 blocks is two lines), for boxes of 8 lines (one 256-element
// k-stage) x box_blocks row blocks.
bool encode_sf_map(CUtensorMap *m, const void *base, int64_t rows, int64_t K, uint32_t box_blocks) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (enc == nullptr) return false;
    const uint64_t lines = static_cast<uint64_t>(K / 32);
    cuuint64_t dims[3] = {256, lines, static_cast<uint64_t>((rows + 127) / 128)};
    cuuint64_t strides[2] = {256, 256 * lines};
    cuuint32_t box[3] = {256, 8, box_blocks};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

namespace nvfp4 {

nvfp4_status check_quantize_args(const void *x, int64_t rows, int64_t cols, const void *scale,
                                 const uint8_t *q, const uint8_t *sf) {
    if (rows < 0 || cols <= 0 || cols % 16 != 0) return NVFP4_ERR_INVALID_ARG;
    if (rows > (int64_t(1) << 40) / cols) return NVFP4_ERR_INVALID_ARG;
    if (scale == nullptr) return NVFP4_ERR_INVALID_ARG;
    // An empty tensor (rows == 0) has no elements to read or write: its
    // arrays may be NULL.
    if (rows > 0 && (x == nullptr || q == nullptr || sf == nullptr)) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(q) || !aligned16(sf)) return NVFP4_ERR_MISALIGNED;
    return NVFP4_OK;
}

}  // namespace nvfp4

namespace {

using nvfp4::check_quantize_args;

nvfp4_status quantize_impl(const void *x, int64_t rows, int64_t cols, const float *scale,
                           bool dynamic, uint8_t *q, uint8_t *sf, float *s_dec_out,
                           cudaStream_t stream) {
    nvfp4_status st = check_quantize_args(x, rows, cols, scale, q, sf);
    if (st != NVFP4_OK) return st;
    int sms = 0;
    st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    // rows == 0 still launches: the kernel writes s_dec_out from the scale.
    return from_cuda(
        nvfp4::launch_quantize(x, rows, cols, scale, dynamic, q, sf, s_dec_out, sms, stream));
}

}  // namespace

extern "C" {

size_t nvfp4_packed_bytes(int64_t rows, int64_t cols) {
    if (rows < 0 || cols < 0) return 0;
    return static_cast<size_t>(rows) * static_cast<size_t>(cols) / 2;
}

size_t nvfp4_sf_bytes(int64_t rows, int64_t cols) {
    if (rows < 0 || cols < 0) return 0;
    const int64_t kb = cols / 16;
    return static_cast<size_t>((rows + 127) / 128 * 128) * static_cast<size_t>((kb + 3) / 4 * 4);
}

const char *nvfp4_status_string(nvfp4_status s) {
    switch (s) {
        case NVFP4_OK: return "ok";
        case NVFP4_ERR_INVALID_ARG: return "invalid argument";
        case NVFP4_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case NVFP4_ERR_UNSUPPORTED_DEVICE: return "no sm_100 (B200) CUDA device";
        case NVFP4_ERR_LAUNCH: return "kernel launch or CUDA runtime error";
        case NVFP4_ERR_TIMEOUT: return "a device-side wait timed out";
    }
    return "unknown status";
}

nvfp4_status nvfp4_tensor_amax(const void *x_bf16, int64_t numel, float *amax_dev,
                               nvfp4_stream_t stream) {
    if (numel < 0 || amax_dev == nullptr || (numel > 0 && x_bf16 == nullptr))
        return NVFP4_ERR_INVALID_ARG;
    if (numel > 0 && !aligned16(x_bf16)) return NVFP4_ERR_MISALIGNED;
    if ((reinterpret_cast<uintptr_t>(amax_dev) & 3u) != 0) return NVFP4_ERR_MISALIGNED;
    int sms = 0;
    nvfp4_status st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    return from_cuda(nvfp4::launch_amax(x_bf16, numel, amax_dev, sms, stream));
}

nvfp4_status nvfp4_quantize(const void *x_bf16, int64_t rows, int64_t cols, const float *amax_dev,
                            uint8_t *q_out, uint8_t *sf_out, float *s_dec_out,
                            nvfp4_stream_t stream) {
    return quantize_impl(x_bf16, rows, cols, amax_dev, true, q_out, sf_out, s_dec_out, stream);
}

nvfp4_status nvfp4_quantize_with_scale(const void *x_bf16, int64_t rows, int64_t cols,
                                       const float *s_enc_dev, uint8_t *q_out, uint8_t *sf_out,
                                       float *s_dec_out, nvfp4_stream_t stream) {
    return quantize_impl(x_bf16, rows, cols, s_enc_dev, false, q_out, sf_out, s_dec_out, stream);
}

nvfp4_status nvfp4_quantize_one_pass(const void *x_bf16, int64_t rows, int64_t cols,
                                     const float *amax_prev_dev, uint8_t *q_out, uint8_t *sf_out,
                                     float *s_dec_out, float *amax_out, nvfp4_stream_t stream) {
    nvfp4_status st = check_quantize_args(x_bf16, rows, cols, amax_prev_dev, q_out, sf_out);
    if (st != NVFP4_OK) return st;
    if (amax_out == nullptr || amax_out == amax_prev_dev) return NVFP4_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(amax_out) & 3u) != 0) return NVFP4_ERR_MISALIGNED;
    int sms = 0;
    st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    return from_cuda(nvfp4::launch_quantize(x_bf16, rows, cols, amax_prev_dev, true, q_out, sf_out,
                                            s_dec_out, sms, stream, amax_out));
}

size_t nvfp4_quantize_dynamic_workspace_bytes(void) { return sizeof(nvfp4::DynWorkspace); }

nvfp4_status nvfp4_quantize_dynamic(const void *x_bf16, int64_t rows, int64_t cols, uint8_t *q_out,
                                    uint8_t *sf_out, float *s_dec_out, float *amax_out,
                                    void *workspace, nvfp4_stream_t stream) {
    nvfp4_status st = check_quantize_args(x_bf16, rows, cols, workspace, q_out, sf_out);
    if (st != NVFP4_OK) return st;
    if (!aligned16(workspace)) return NVFP4_ERR_MISALIGNED;
    int sms = 0;
    st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    nvfp4::DynWorkspace *ws = static_cast<nvfp4::DynWorkspace *>(workspace);
    cudaError_t e = nvfp4::launch_quantize_dynamic(x_bf16, rows, cols, q_out, sf_out, s_dec_out,
                                                   amax_out, ws, sms, stream);
    if (e == cudaErrorNotSupported) {
        cudaGetLastError();
        float *amax = amax_out != nullptr ? amax_out : &ws->fallback_amax;
        e = nvfp4::launch_amax(x_bf16, rows * cols, amax, sms, stream);
        if (e == cudaSuccess)
            e = nvfp4::launch_quantize(x_bf16, rows, cols, amax, true, q_out, sf_out, s_dec_out,
                                       sms, stream);
    }
    return from_cuda(e);
}

}  // extern "C"

namespace {

nvfp4_status gemm_impl(const uint8_t *aq, const uint8_t *asf, const float *a_s_dec,
                       const uint8_t *bq, const uint8_t *bsf, const float *b_s_dec, int64_t M,
                       int64_t N, int64_t K, void *y_bf16, const nvfp4_fused_out *fused,
                       bool a_row_scale, bool fp8, cudaStream_t stream) {
    if (M < 1 || N < 8 || N % 8 != 0) return NVFP4_ERR_INVALID_ARG;
    if (fp8 ? (K < 32 || K % 32 != 0 || M <= 128 || N < 256) : (K < 64 || K % 64 != 0))
        return NVFP4_ERR_INVALID_ARG;
    if (M > (int64_t(1) << 31) || N > (int64_t(1) << 31) || K > (int64_t(1) << 31))
        return NVFP4_ERR_INVALID_ARG;
    if (aq == nullptr || a_s_dec == nullptr || bq == nullptr || b_s_dec == nullptr ||
        (!fp8 && (asf == nullptr || bsf == nullptr)))
        return NVFP4_ERR_INVALID_ARG;
    if (y_bf16 == nullptr && fused == nullptr) return NVFP4_ERR_INVALID_ARG;
    if (fused != nullptr &&
        (N % 16 != 0 || fused->s_enc_y == nullptr || fused->yq == nullptr || fused->ysf == nullptr ||
         (fused->activation != NVFP4_ACT_NONE && fused->activation != NVFP4_ACT_GELU)))
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(aq) || !aligned16(bq) || (!fp8 && (!aligned16(asf) || !aligned16(bsf))) ||
        (y_bf16 != nullptr && !aligned16(y_bf16)))
        return NVFP4_ERR_MISALIGNED;
    if (fused != nullptr && (!aligned16(fused->yq) || !aligned16(fused->ysf)))
        return NVFP4_ERR_MISALIGNED;
    int sms = 0;
    nvfp4_status st = current_device(&sms);
    if (st != NVFP4_OK) return st;

    const nvfp4::GemmKind kind = nvfp4::gemm_kind(M, N);
    nvfp4::GemmMaps maps;
    std::memset(&maps, 0, sizeof(maps));
    const uint64_t row_bytes = static_cast<uint64_t>(fp8 ? K : K / 2);
    if (!encode_operand_map(&maps.a, aq, row_bytes, static_cast<uint64_t>(M), 128) ||
        !encode_operand_map(&maps.b, bq, row_bytes, static_cast<uint64_t>(N),
                            nvfp4::gemm_b_box_rows(kind)))
        return NVFP4_ERR_LAUNCH;
    if (y_bf16 != nullptr &&
        !encode_output_map(&maps.y, y_bf16, static_cast<uint64_t>(N), static_cast<uint64_t>(M)))
        return NVFP4_ERR_LAUNCH;
    if (!fp8 && (!encode_sf_map(&maps.sfa, asf, M, K, 1) ||
                 !encode_sf_map(&maps.sfb, bsf, N, K, kind == nvfp4::kGemm128 ? 1 : 2)))
        return NVFP4_ERR_LAUNCH;

    nvfp4::GemmParams p;
    p.a_s_dec = a_s_dec;
    p.b_s_dec = b_s_dec;
    p.y = static_cast<uint8_t *>(y_bf16);
    p.s_enc_y = fused ? fused->s_enc_y : nullptr;
    p.yq = fused ? fused->yq : nullptr;
    p.ysf = fused ? fused->ysf : nullptr;
    p.amax_y = fused ? fused->amax_y : nullptr;
    p.s_dec_y = fused ? fused->s_dec_y : nullptr;
    p.act = fused ? fused->activation : NVFP4_ACT_NONE;
    p.a_row_scale = a_row_scale ? 1 : 0;
    p.fp8 = fp8 ? 1 : 0;
    p.M = M;
    p.N = N;
    p.K = K;
    if (p.amax_y != nullptr) {
        cudaError_t e = cudaMemsetAsync(p.amax_y, 0, sizeof(float), stream);
        if (e != cudaSuccess) return NVFP4_ERR_LAUNCH;
    }
    return from_cuda(nvfp4::launch_gemm(maps, p, kind, sms, stream));
}

}  // namespace

extern "C" {

nvfp4_status nvfp4_gemm(const uint8_t *aq, const uint8_t *asf, const float *a_s_dec,
                        const uint8_t *bq, const uint8_t *bsf, const float *b_s_dec, int64_t M,
                        int64_t N, int64_t K, void *y_bf16, const nvfp4_fused_out *fused,
                        nvfp4_stream_t stream) {
    return gemm_impl(aq, asf, a_s_dec, bq, bsf, b_s_dec, M, N, K, y_bf16, fused, false, false,
                     stream);
}

nvfp4_status nvfp4_gemm_rowscale(const uint8_t *aq, const uint8_t *asf, const float *a_s_dec_rows,
                                 const uint8_t *bq, const uint8_t *bsf, const float *b_s_dec,
                                 int64_t M, int64_t N, int64_t K, void *y_bf16,
                                 const nvfp4_fused_out *fused, nvfp4_stream_t stream) {
    return gemm_impl(aq, asf, a_s_dec_rows, bq, bsf, b_s_dec, M, N, K, y_bf16, fused, true,
                     false, stream);
}

nvfp4_status nvfp4_fp8_quantize(const void *x_bf16, int64_t rows, int64_t cols,
                                const float *amax_dev, uint8_t *q_out, float *s_dec_out,
                                nvfp4_stream_t stream) {
    if (rows < 0 || cols <= 0 || cols % 16 != 0 || rows > (int64_t(1) << 40) / cols)
        return NVFP4_ERR_INVALID_ARG;
    if (amax_dev == nullptr || s_dec_out == nullptr) return NVFP4_ERR_INVALID_ARG;
    if (rows > 0 && (x_bf16 == nullptr || q_out == nullptr)) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(x_bf16) || !aligned16(q_out) ||
        (reinterpret_cast<uintptr_t>(amax_dev) & 3u) != 0 ||
        (reinterpret_cast<uintptr_t>(s_dec_out) & 3u) != 0)
        return NVFP4_ERR_MISALIGNED;
    int sms = 0;
    nvfp4_status st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    return from_cuda(
        nvfp4::launch_quantize_fp8(x_bf16, rows * cols, amax_dev, q_out, s_dec_out, sms, stream));
}

nvfp4_status nvfp4_fp8_gemm(const uint8_t *a8, const float *a_s_dec, const uint8_t *b8,
                            const float *b_s_dec, int64_t M, int64_t N, int64_t K, void *y_bf16,
                            const nvfp4_fused_out *fused, nvfp4_stream_t stream) {
    return gemm_impl(a8, nullptr, a_s_dec, b8, nullptr, b_s_dec, M, N, K, y_bf16, fused, false,
                     true, stream);
}

nvfp4_status nvfp4_quantize_rowwise(const void *x_bf16, int64_t rows, int64_t cols,
                                    uint8_t *q_out, uint8_t *sf_out, float *s_dec_rows,
                                    float *amax_rows, nvfp4_stream_t stream) {
    if (rows == 0 && cols > 0 && cols % 16 == 0) return NVFP4_OK;  // no rows, no scales
    nvfp4_status st = check_quantize_args(x_bf16, rows, cols, s_dec_rows, q_out, sf_out);
    if (st != NVFP4_OK) return st;
    if ((reinterpret_cast<uintptr_t>(s_dec_rows) & 3u) != 0 ||
        (reinterpret_cast<uintptr_t>(amax_rows) & 3u) != 0)
        return NVFP4_ERR_MISALIGNED;
    int sms = 0;
    st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    if (rows == 0) return NVFP4_OK;
    return from_cuda(nvfp4::launch_quantize_rowwise(x_bf16, rows, cols, q_out, sf_out, s_dec_rows,
                                                    amax_rows, stream));
}

nvfp4_status nvfp4_linear_host(const void *x_host_bf16, int64_t M, int64_t K, const uint8_t *wq,
                               const uint8_t *wsf, const float *w_s_dec, int64_t N,
                               void *y_host_bf16, const nvfp4_linear_workspace *ws,
                               nvfp4_stream_t stream) {
    if (x_host_bf16 == nullptr || y_host_bf16 == nullptr || ws == nullptr || ws->x == nullptr ||
        ws->xq == nullptr || ws->xsf == nullptr || ws->amax == nullptr || ws->s_dec == nullptr ||
        ws->y == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    if (M < 1 || K < 64 || K % 64 != 0 || N < 8 || N % 8 != 0) return NVFP4_ERR_INVALID_ARG;
    int sms = 0;
    nvfp4_status st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    const size_t xbytes = static_cast<size_t>(M) * static_cast<size_t>(K) * 2;
    const size_t ybytes = static_cast<size_t>(M) * static_cast<size_t>(N) * 2;
    if (cudaMemcpyAsync(ws->x, x_host_bf16, xbytes, cudaMemcpyHostToDevice, stream) != cudaSuccess)
        return NVFP4_ERR_LAUNCH;
    if (ws->dyn_ws != nullptr) {
        st = nvfp4_quantize_dynamic(ws->x, M, K, ws->xq, ws->xsf, ws->s_dec, ws->amax, ws->dyn_ws,
                                    stream);
    } else {
        st = nvfp4_tensor_amax(ws->x, M * K, ws->amax, stream);
        if (st == NVFP4_OK)
            st = nvfp4_quantize(ws->x, M, K, ws->amax, ws->xq, ws->xsf, ws->s_dec, stream);
    }
    if (st != NVFP4_OK) return st;
    st = nvfp4_gemm(ws->xq, ws->xsf, ws->s_dec, wq, wsf, w_s_dec, M, N, K, ws->y, nullptr, stream);
    if (st != NVFP4_OK) return st;
    if (cudaMemcpyAsync(y_host_bf16, ws->y, ybytes, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return NVFP4_ERR_LAUNCH;
    return NVFP4_OK;
}

nvfp4_status nvfp4_selftest_wait_timeout(int64_t timeout_us, nvfp4_stream_t stream) {
    if (timeout_us < 1 || timeout_us > 2000000) return NVFP4_ERR_INVALID_ARG;
    int sms = 0;
    nvfp4_status st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    return from_cuda(nvfp4::launch_selftest_wait_timeout(
        static_cast<uint64_t>(timeout_us) * 1000u, NVFP4_SELFTEST_TAG, stream));
}

nvfp4_status nvfp4_device_error(int *code_out, int *detail_out) {
    if (code_out == nullptr) return NVFP4_ERR_INVALID_ARG;
    int sms = 0;
    nvfp4_status st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    int code = 0, detail = 0;
    if (nvfp4::read_and_clear_device_error(&code, &detail) != cudaSuccess) return NVFP4_ERR_LAUNCH;
    *code_out = code;
    if (detail_out != nullptr) *detail_out = detail;
    return NVFP4_OK;
}

}  // extern "C"
