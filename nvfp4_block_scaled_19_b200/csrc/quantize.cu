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
// quantize_dynamic: both in one cooperative launch.  Phase 1 reduces the
//   amax (one atomicMax per CTA into a per-launch word of a small workspace),
//   a bounded grid barrier publishes it, phase 2 quantizes.  Phase 2 walks the
//   rows in the opposite order to phase 1, so the part of the tensor phase 1
//   read last is still in L2 (all of it when the tensor fits in L2).
#include <cuda_runtime.h>

#include <cstdint>

#include "gemm.h"
#include "nvfp4_math.cuh"

namespace nvfp4 {

constexpr uint64_t kBarrierTimeoutNs = 2000000000ull;

constexpr int kAmaxThreads = 256;

// Persistent grid-stride amax: 32-byte loads, four in flight per thread.
__global__ void __launch_bounds__(kAmaxThreads, 3) amax_kernel(const uint8_t *__restrict__ x,
                                                              int64_t nvec32,
                                                              const uint16_t *__restrict__ tail,
                                                              int ntail, unsigned *__restrict__ out) {
    uint32_t m = 0;
    const bool a32 = (reinterpret_cast<uintptr_t>(x) & 31) == 0;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    for (; i + 3 * stride < nvec32; i += 4 * stride) {
        const BF16x16 a = ldg_32B(x + 32 * i, a32);
        const BF16x16 b = ldg_32B(x + 32 * (i + stride), a32);
        const BF16x16 c = ldg_32B(x + 32 * (i + 2 * stride), a32);
        const BF16x16 d = ldg_32B(x + 32 * (i + 3 * stride), a32);
        m = max(m, max(max(absmax_bf16x16(a), absmax_bf16x16(b)),
                       max(absmax_bf16x16(c), absmax_bf16x16(d))));
    }
    for (; i < nvec32; i += stride) m = max(m, absmax_bf16x16(ldg_32B(x + 32 * i, a32)));
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

constexpr int kSliceBlocks = 64;    // 16-element blocks (one per thread) per column slice
constexpr int kQuantThreads = 128;  // two row streams per CTA in the standalone kernel
constexpr int kQuantRows = 2;       // rows per group; the next group is loaded ahead

// Quantizes the rows of one "row stream": thread tx (0..63) of column slice
// bx handles block column c = 64*bx + tx (32 contiguous bytes per row); the
// stream takes row groups rs, rs + n_streams, ... of kQuantRows rows, visited
// in descending order when `descending`, with the next group's loads in
// flight while the current one is computed.  Covers the padded scale layout:
// rows up to a multiple of 128 and block columns up to a multiple of 4 get
// zero scales.  All 32 lanes of a warp share (bx, rs), so shuffles are uniform.
__device__ __forceinline__ void quantize_rows(const uint16_t *__restrict__ x, int64_t rows,
                                              int64_t cols, float s_enc, uint8_t *__restrict__ q,
                                              uint8_t *__restrict__ sf, int bx, int64_t rs,
                                              int64_t n_streams, int tx, bool descending) {
    const int64_t kb = cols >> 4;
    const int64_t kb4 = (kb + 3) >> 2;  // scale tiles per 128-row block
    const int64_t kbp = kb4 << 2;       // padded blocks per row
    const int64_t rows_pad = (rows + 127) & ~int64_t(127);
    const int64_t n_groups = (rows_pad + kQuantRows - 1) / kQuantRows;
    const int64_t c = static_cast<int64_t>(bx) * kSliceBlocks + tx;
    const bool col_ok = c < kb;
    const bool sf_writer = ((tx & 3) == 0) && c < kbp;  // c % 4 == 0 for these lanes
    const int64_t qrow = cols >> 1;
    const uint8_t *xb = reinterpret_cast<const uint8_t *>(x) + c * 32;
    const bool a32 = (reinterpret_cast<uintptr_t>(x) & 31) == 0;  // rows are 32-byte multiples

    auto row_of = [&](int64_t g) { return (descending ? (n_groups - 1 - g) : g) * kQuantRows; };
    auto load = [&](int64_t r0, BF16x16 (&v)[kQuantRows]) {
#pragma unroll
        for (int u = 0; u < kQuantRows; ++u) {
            const int64_t r = r0 + u;
            if (r < rows && col_ok) {
                v[u] = ldg_32B(xb + r * cols * 2, a32);
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) v[u].w[k] = 0u;
            }
        }
    };

    int64_t g = rs;
    if (g >= n_groups) return;
    BF16x16 cur[kQuantRows];
    load(row_of(g), cur);
    while (true) {
        const int64_t r0 = row_of(g);
        const int64_t g_next = g + n_streams;
        BF16x16 nxt[kQuantRows];
        if (g_next < n_groups) load(row_of(g_next), nxt);
#pragma unroll
        for (int u = 0; u < kQuantRows; ++u) {
            const int64_t r = r0 + u;
            if (r >= rows_pad) break;  // uniform across the warp
            const bool valid = r < rows && col_ok;
            const BlockScale bs = block_scale(__uint_as_float(absmax_bf16x16(cur[u]) << 16), s_enc);
            const uint32_t sfc = valid ? bs.sf : 0u;
            if (valid) {
                const uint4 lo = make_uint4(cur[u].w[0], cur[u].w[1], cur[u].w[2], cur[u].w[3]);
                const uint4 hi = make_uint4(cur[u].w[4], cur[u].w[5], cur[u].w[6], cur[u].w[7]);
                *reinterpret_cast<uint2 *>(q + r * qrow + c * 8) =
                    make_uint2(quantize_bf16x8(lo, bs.inv), quantize_bf16x8(hi, bs.inv));
            }
            const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, sfc, 1);
            const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, sfc, 2);
            const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, sfc, 3);
            if (sf_writer)
                *reinterpret_cast<uint32_t *>(sf + sf_offset(r, c, kb4)) =
                    sfc | (s1 << 8) | (s2 << 16) | (s3 << 24);
        }
        if (g_next >= n_groups) break;
        g = g_next;
#pragma unroll
        for (int u = 0; u < kQuantRows; ++u) cur[u] = nxt[u];
    }
}

// grid.x covers the padded block columns (64 per slice), grid.y x 2 row
// streams stride the rows.
template <bool kDynamic>
__global__ void __launch_bounds__(kQuantThreads) quantize_kernel(
    const uint16_t *__restrict__ x, int64_t rows, int64_t cols, const float *__restrict__ scale_in,
    uint8_t *__restrict__ q, uint8_t *__restrict__ sf, float *__restrict__ s_dec_out) {
    const float s_enc = kDynamic ? tensor_encode_scale(*scale_in) : *scale_in;
    if (s_dec_out != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0)
        *s_dec_out = __fdiv_rn(1.0f, s_enc);
    constexpr int kStreams = kQuantThreads / kSliceBlocks;
    quantize_rows(x, rows, cols, s_enc, q, sf, blockIdx.x,
                  static_cast<int64_t>(blockIdx.y) * kStreams + threadIdx.x / kSliceBlocks,
                  static_cast<int64_t>(gridDim.y) * kStreams, threadIdx.x % kSliceBlocks, false);
}

constexpr int kDynThreads = 512;  // 4 row streams x 128 threads

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_gpu(unsigned *p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Cooperative launch (8 row streams x 64 threads): every CTA is resident, so the grid barrier cannot
// deadlock; it is still bounded (error tag 7 on timeout).
__global__ void __launch_bounds__(kDynThreads) quantize_dynamic_kernel(
    const uint16_t *__restrict__ x, int64_t rows, int64_t cols, uint8_t *__restrict__ q,
    uint8_t *__restrict__ sf, float *__restrict__ s_dec_out, float *__restrict__ amax_out,
    DynWorkspace *ws, int *err, int gx) {
    __shared__ unsigned s_gen, s_amax;
    __shared__ int s_fail;
    __shared__ uint32_t red[kDynThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        s_gen = ld_acquire_gpu(&ws->gen);
        s_fail = 0;
    }
    __syncthreads();
    const unsigned gen = s_gen;
    // The next launch's amax word starts at zero; nobody reads it in this one.
    if (blockIdx.x == 0 && tid == 0) ws->amax_bits[(gen + 1) & 1] = 0u;

    // Phase 1: amax (32-byte loads, four in flight per thread).
    const uint8_t *xb = reinterpret_cast<const uint8_t *>(x);
    const bool a32 = (reinterpret_cast<uintptr_t>(x) & 31) == 0;
    const int64_t nvec32 = rows * cols / 16;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kDynThreads;
    int64_t i = static_cast<int64_t>(blockIdx.x) * kDynThreads + tid;
    uint32_t m = 0;
    for (; i + 3 * stride < nvec32; i += 4 * stride) {
        const BF16x16 a = ldg_32B(xb + 32 * i, a32);
        const BF16x16 b = ldg_32B(xb + 32 * (i + stride), a32);
        const BF16x16 c = ldg_32B(xb + 32 * (i + 2 * stride), a32);
        const BF16x16 d = ldg_32B(xb + 32 * (i + 3 * stride), a32);
        m = max(m, max(max(absmax_bf16x16(a), absmax_bf16x16(b)),
                       max(absmax_bf16x16(c), absmax_bf16x16(d))));
    }
    for (; i < nvec32; i += stride) m = max(m, absmax_bf16x16(ldg_32B(xb + 32 * i, a32)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    if (warp == 0) {
        m = lane < kDynThreads / 32 ? red[lane] : 0u;
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if (lane == 0) {
            if (m != 0) atomicMax(&ws->amax_bits[gen & 1], m << 16);
            __threadfence();
            // Grid barrier: the last CTA to arrive resets the count and
            // advances the generation; the others wait for that.
            const unsigned arrived = atomicAdd(&ws->count, 1u);
            if (arrived == gridDim.x - 1) {
                ws->count = 0u;
                __threadfence();
                st_release_gpu(&ws->gen, gen + 1);
            } else {
                const uint64_t t0 = globaltimer_ns();
                while (ld_acquire_gpu(&ws->gen) == gen) {
                    if (globaltimer_ns() - t0 > kBarrierTimeoutNs) {
                        s_fail = 1;
                        if (err != nullptr && atomicCAS(err, 0, 5) == 0) err[1] = 7;
                        break;
                    }
                    __nanosleep(64);
                }
            }
            s_amax = ld_acquire_gpu(&ws->amax_bits[gen & 1]);
        }
    }
    __syncthreads();
    if (s_fail) return;
    const float amax = __uint_as_float(s_amax);
    const float s_enc = tensor_encode_scale(amax);
    if (blockIdx.x == 0 && tid == 0) {
        if (s_dec_out != nullptr) *s_dec_out = __fdiv_rn(1.0f, s_enc);
        if (amax_out != nullptr) *amax_out = amax;
    }

    // Phase 2: quantize, rows descending.
    const int nby = static_cast<int>(gridDim.x) / gx;
    const int byc = static_cast<int>(blockIdx.x) / gx;
    if (byc >= nby) return;
    constexpr int kStreams = kDynThreads / kSliceBlocks;
    quantize_rows(x, rows, cols, s_enc, q, sf, static_cast<int>(blockIdx.x) % gx,
                  static_cast<int64_t>(byc) * kStreams + tid / kSliceBlocks,
                  static_cast<int64_t>(nby) * kStreams, tid % kSliceBlocks, true);
}

cudaError_t launch_amax(const void *x, int64_t numel, float *amax, int num_sms,
                        cudaStream_t stream) {
    cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float), stream);
    if (e != cudaSuccess || numel == 0) return e;
    const int64_t nvec32 = numel / 16;
    const int ntail = static_cast<int>(numel - nvec32 * 16);
    int64_t blocks = (nvec32 + kAmaxThreads - 1) / kAmaxThreads;
    const int64_t cap = static_cast<int64_t>(num_sms) * 3;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    amax_kernel<<<static_cast<unsigned>(blocks), kAmaxThreads, 0, stream>>>(
        reinterpret_cast<const uint8_t *>(x), nvec32,
        reinterpret_cast<const uint16_t *>(x) + nvec32 * 16, ntail,
        reinterpret_cast<unsigned *>(amax));
    return cudaGetLastError();
}

cudaError_t launch_quantize(const void *x, int64_t rows, int64_t cols, const float *scale_in,
                            bool dynamic, uint8_t *q, uint8_t *sf, float *s_dec_out, int num_sms,
                            cudaStream_t stream) {
    const int64_t kbp = ((cols / 16 + 3) / 4) * 4;
    const int64_t rows_pad = (rows + 127) / 128 * 128;
    const int64_t gx = (kbp + kSliceBlocks - 1) / kSliceBlocks;
    const int64_t streams_per_cta = kQuantThreads / kSliceBlocks;
    const int64_t target = static_cast<int64_t>(num_sms) * 16;
    const int64_t groups = (rows_pad + kQuantRows - 1) / kQuantRows;
    int64_t gy = (groups + streams_per_cta - 1) / streams_per_cta;
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

cudaError_t launch_quantize_dynamic(const void *x, int64_t rows, int64_t cols, uint8_t *q,
                                    uint8_t *sf, float *s_dec_out, float *amax_out,
                                    DynWorkspace *ws, int num_sms, cudaStream_t stream) {
    static int resident[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (resident[dev] == 0) {
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quantize_dynamic_kernel,
                                                          kDynThreads, 0);
        if (e != cudaSuccess || per_sm < 1) return e != cudaSuccess ? e : cudaErrorInvalidValue;
        resident[dev] = per_sm;
    }
    const int64_t kbp = ((cols / 16 + 3) / 4) * 4;
    int gx = static_cast<int>((kbp + kSliceBlocks - 1) / kSliceBlocks);
    int grid = num_sms * resident[dev];
    // Phase 2 needs at least one CTA per column slice; very wide rows use
    // several passes of the slices (not reached by DiT shapes).
    if (gx > grid) return cudaErrorNotSupported;
    grid = (grid / gx) * gx;
    int *err = device_error_word();
    const uint16_t *xp = reinterpret_cast<const uint16_t *>(x);
    void *args[] = {&xp, &rows, &cols, &q, &sf, &s_dec_out, &amax_out, &ws, &err, &gx};
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(quantize_dynamic_kernel),
                                       dim3(grid), dim3(kDynThreads), args, 0, stream);
}

}  // namespace nvfp4
