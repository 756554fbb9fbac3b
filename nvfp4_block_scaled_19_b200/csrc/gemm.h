// Host/device interface of the block-scaled FP4 GEMM kernel.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace nvfp4 {

struct GemmParams {
    const float *a_s_dec;   // 1 fp32
    const float *b_s_dec;   // 1 fp32
    uint8_t *y;             // bf16 [M,N] or null
    const float *s_enc_y;   // fused quantize: 1 fp32
    uint8_t *yq;            // fused quantize: packed [M, N/2] or null (= no fusion)
    uint8_t *ysf;           // fused quantize: tiled scales
    float *amax_y;          // fused quantize: 1 fp32 (pre-zeroed) or null
    float *s_dec_y;         // fused quantize: 1 fp32 written with 1/s_enc_y, or null
    int act;                // 0 none, 1 exact GELU on alpha * acc before the bf16 rounding
    int a_row_scale;        // 1: a_s_dec holds one decode scale per row of A (per token)
    int fp8;                // 1: A and B are E4M3 with per-tensor scales only (no asf/bsf)
    int64_t M, N, K;
};

// Device address of the library's error word (int[2]: code, tag) on the
// current device, for kernels outside the GEMM translation unit.
int *device_error_word();

// Kernel variant for a problem: 1-CTA 128x128 tiles, 1-CTA 128x256 tiles,
// or CTA pairs with 256x256 tiles.
enum GemmKind { kGemm128 = 1, kGemm256 = 2, kGemmPair = 3 };
GemmKind gemm_kind(int64_t M, int64_t N);

// Rows of the B (weight) TMA box for a kernel variant.
inline uint32_t gemm_b_box_rows(GemmKind k) { return k == kGemm256 ? 256u : 128u; }

// Tensor maps of one GEMM launch: A and B codes, Y (bf16, may be unused),
// and for the CTA-pair kernel the scale factors as 3-D byte tensors
// [128-row blocks][K / 32 lines][256 bytes] (a 512-byte scale tile is two
// lines), so one box brings a k-stage's scales of one or two row blocks.
struct GemmMaps {
    CUtensorMap a, b, y, sfa, sfb;
};

cudaError_t launch_gemm(const GemmMaps &maps, const GemmParams &p, GemmKind kind, int num_sms,
                        cudaStream_t stream);

cudaError_t launch_amax(const void *x, int64_t numel, float *amax, int num_sms,
                        cudaStream_t stream);

// amax_out (optional): also writes max |x| of this tensor (one pass).
cudaError_t launch_quantize(const void *x, int64_t rows, int64_t cols, const float *scale_in,
                            bool dynamic, uint8_t *q, uint8_t *sf, float *s_dec_out, int num_sms,
                            cudaStream_t stream, float *amax_out = nullptr);

// Workspace of the single-launch dynamic quantization (zero-initialised once
// by the caller; calls that share one must be stream-ordered).
struct DynWorkspace {
    // (barrier generation << 32) | amax bits of the launch that completed it;
    // one 64-bit word, so a CTA leaving the grid barrier reads both at once.
    unsigned long long state;
    unsigned count;         // CTAs arrived at the grid barrier (back to 0 after it)
    unsigned amax_acc;      // running amax bits of the current launch (back to 0 after it)
    float fallback_amax;    // used when rows are too wide for one resident grid
    unsigned pad[3];
};
static_assert(sizeof(DynWorkspace) == 32, "workspace size is part of the ABI");

cudaError_t launch_selftest_wait_timeout(uint64_t timeout_ns, int tag, cudaStream_t stream);

// FP8 variant: q = E4M3_rn_satfinite(x * 448 / amax), s_dec = amax / 448 (as
// 1 / S_enc), from a device amax.
cudaError_t launch_quantize_fp8(const void *x, int64_t numel, const float *amax, uint8_t *q,
                                float *s_dec_out, int num_sms, cudaStream_t stream);

cudaError_t launch_quantize_rowwise(const void *x, int64_t rows, int64_t cols, uint8_t *q,
                                    uint8_t *sf, float *s_dec_rows, float *amax_rows,
                                    cudaStream_t stream);

// Returns cudaErrorNotSupported when the rows are too wide for one
// cooperative grid (then use launch_amax + launch_quantize).
cudaError_t launch_quantize_dynamic(const void *x, int64_t rows, int64_t cols, uint8_t *q,
                                    uint8_t *sf, float *s_dec_out, float *amax_out,
                                    DynWorkspace *ws, int num_sms, cudaStream_t stream);

}  // namespace nvfp4
