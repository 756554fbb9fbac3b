// Per-tensor amax and NVFP4 block quantization kernels (HBM-bound).
//
// Two-level microblock scaling: an FP32 per-tensor scale computed from the
// tensor amax (dynamic) or given (static), and one E4M3 scale per block of 16
// contiguous elements computed at run time ("英伟达B200狂飙10.2倍！AI绘图告别
// 龟速！", section "NVFP4量化：在精度与速度之间寻得最佳平衡").
//
// amax: grid-stride 16-byte loads, packed 2x16-bit max on the bf16 bits,
//   warp-shuffle + shared-memory reduction, one atomicMax per CTA on the
//   float's bit pattern (valid for non-negative floats).
// quantize: two threads per 16-element block (8 elements = one 16-byte load
//   each), so a warp reads 512 contiguous bytes and writes 128 contiguous
//   bytes of packed codes; the pair exchanges its half-block maxima with one
//   shuffle; four consecutive block scales of a row are gathered with
//   shuffles into one 4-byte store in the 128x4-tiled layout.  The kernel also
//   writes the layout's zero padding (rows up to a multiple of 128, blocks up
//   to a multiple of 4), so the scale buffer needs no memset.
#include <cuda_runtime.h>

#include <cstdint>

#include "nvfp4_math.cuh"

namespace nvfp4 {

constexpr int kAmaxThreads = 256;

__global__ void __launch_bounds__(kAmaxThreads) amax_kernel(const uint4 *__restrict__ x,
                                                           int64_t nvec,
                                                           const uint16_t *__restrict__ tail,
                                                           int ntail, unsigned *__restrict__ out) {
    uint32_t m = 0;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    for (; i + 3 * stride < nvec; i += 4 * stride) {
        const uint4 a = __ldg(x + i);
        const uint4 b = __ldg(x + i + stride);
        const uint4 c = __ldg(x + i + 2 * stride);
        const uint4 d = __ldg(x + i + 3 * stride);
        m = max(m, max(max(absmax_bf16x8(a), absmax_bf16x8(b)),
                       max(absmax_bf16x8(c), absmax_bf16x8(d))));
    }
    for (; i < nvec; i += stride) m = max(m, absmax_bf16x8(__ldg(x + i)));
    if (blockIdx.x == 0 && static_cast<int>(threadIdx.x) < ntail)
        m = max(m, static_cast<uint32_t>(tail[threadIdx.x]) & 0x7FFFu);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    __shared__ uint32_t red[kAmaxThreads / 32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = m;
    __syncthreads();
    if (warp == 0) {
        m = lane < kAmaxThreads / 32 ? red[lane] : 0u;
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if (lane == 0 && m != 0) atomicMax(out, m << 16);
    }
}

constexpr int kQuantThreads = 128;  // 64 blocks of 16 elements per CTA row-slice
constexpr int kQuantRows = 4;       // rows per iteration (independent loads in flight)

// grid.x covers the padded block columns (2 threads each), grid.y strides rows.
template <bool kDynamic>
__global__ void __launch_bounds__(kQuantThreads) quantize_kernel(
    const uint16_t *__restrict__ x, int64_t rows, int64_t cols, const float *__restrict__ scale_in,
    uint8_t *__restrict__ q, uint8_t *__restrict__ sf, float *__restrict__ s_dec_out) {
    const float s_enc = kDynamic ? tensor_encode_scale(*scale_in) : *scale_in;
    if (s_dec_out != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0)
        *s_dec_out = __fdiv_rn(1.0f, s_enc);

    const int64_t kb = cols >> 4;
    const int64_t kb4 = (kb + 3) >> 2;  // scale tiles per 128-row block
    const int64_t kbp = kb4 << 2;       // padded blocks per row
    const int64_t rows_pad = (rows + 127) & ~int64_t(127);
    const int lane = threadIdx.x & 31;
    const int half = threadIdx.x & 1;
    const int64_t c = static_cast<int64_t>(blockIdx.x) * (kQuantThreads / 2) + (threadIdx.x >> 1);
    const bool col_ok = c < kb;
    const bool sf_writer = ((lane & 7) == 0) && c < kbp;  // c % 4 == 0 for these lanes
    const int64_t qrow = cols >> 1;

    for (int64_t r0 = static_cast<int64_t>(blockIdx.y) * kQuantRows; r0 < rows_pad;
         r0 += static_cast<int64_t>(gridDim.y) * kQuantRows) {
        uint4 v[kQuantRows];
#pragma unroll
        for (int u = 0; u < kQuantRows; ++u) {
            const int64_t r = r0 + u;
            v[u] = make_uint4(0u, 0u, 0u, 0u);
            if (r < rows && col_ok)
                v[u] = __ldg(reinterpret_cast<const uint4 *>(x + r * cols + c * 16 + half * 8));
        }
#pragma unroll
        for (int u = 0; u < kQuantRows; ++u) {
            const int64_t r = r0 + u;
            if (r >= rows_pad) break;  // uniform across the CTA
            const bool valid = r < rows && col_ok;
            uint32_t m = absmax_bf16x8(v[u]);
            m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
            const BlockScale bs = block_scale(__uint_as_float(m << 16), s_enc);
            const uint32_t sfc = valid ? bs.sf : 0u;
            if (valid) {
                const uint32_t codes = quantize_bf16x8(v[u], bs.inv);
                *reinterpret_cast<uint32_t *>(q + r * qrow + c * 8 + half * 4) = codes;
            }
            const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, sfc, 2);
            const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, sfc, 4);
            const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, sfc, 6);
            if (sf_writer)
                *reinterpret_cast<uint32_t *>(sf + sf_offset(r, c, kb4)) =
                    sfc | (s1 << 8) | (s2 << 16) | (s3 << 24);
        }
    }
}

cudaError_t launch_amax(const void *x, int64_t numel, float *amax, int num_sms,
                        cudaStream_t stream) {
    cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float), stream);
    if (e != cudaSuccess || numel == 0) return e;
    const int64_t nvec = numel / 8;
    const int ntail = static_cast<int>(numel - nvec * 8);
    int64_t blocks = (nvec + kAmaxThreads * 4 - 1) / (kAmaxThreads * 4);
    const int64_t cap = static_cast<int64_t>(num_sms) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    amax_kernel<<<static_cast<unsigned>(blocks), kAmaxThreads, 0, stream>>>(
        reinterpret_cast<const uint4 *>(x), nvec,
        reinterpret_cast<const uint16_t *>(x) + nvec * 8, ntail,
        reinterpret_cast<unsigned *>(amax));
    return cudaGetLastError();
}

cudaError_t launch_quantize(const void *x, int64_t rows, int64_t cols, const float *scale_in,
                            bool dynamic, uint8_t *q, uint8_t *sf, float *s_dec_out, int num_sms,
                            cudaStream_t stream) {
    const int64_t kbp = ((cols / 16 + 3) / 4) * 4;
    const int64_t rows_pad = (rows + 127) / 128 * 128;
    const int64_t gx = (kbp + kQuantThreads / 2 - 1) / (kQuantThreads / 2);
    const int64_t target = static_cast<int64_t>(num_sms) * 16;
    int64_t gy = (rows_pad + kQuantRows - 1) / kQuantRows;
    int64_t cap = target / gx;
    if (cap < 1) cap = 1;
    if (gy > cap) gy = cap;
    if (gy > 65535) gy = 65535;
    if (gx > 2147483647) return cudaErrorInvalidValue;
    dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
    const uint16_t *xp = reinterpret_cast<const uint16_t *>(x);
    if (dynamic)
        quantize_kernel<true><<<grid, kQuantThreads, 0, stream>>>(xp, rows, cols, scale_in, q, sf,
                                                                 s_dec_out);
    else
        quantize_kernel<false><<<grid, kQuantThreads, 0, stream>>>(xp, rows, cols, scale_in, q,
                                                                  sf, s_dec_out);
    return cudaGetLastError();
}

}  // namespace nvfp4
