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
// quantize_dynamic: both in one launch of a grid that is resident all at
//   once.  Phase 1 reduces the amax (one atomicMax per CTA into a per-launch
//   word of a small workspace), a bounded grid barrier publishes it, phase 2
//   quantizes, walking the tensor in the opposite order to phase 1 so that
//   what phase 1 read last is still in L2 (all of it when the tensor fits).
//   Rows of a multiple of 64 elements (every DiT shape) take the resident
//   kernel when a slice per SM fits in shared memory (phase 2 then reads the
//   slice from there, see quantize_dynamic_resident_kernel), else the flat
//   kernel: the tensor is seen as one array of 16-element blocks, thread g owns
//   blocks g, g + S, g + 2S, g + 3S of each round (S = threads in the grid),
//   so every thread has four 32-byte loads in flight in both phases and a
//   warp's codes are one contiguous 256-byte store.  Other widths take the
//   row-stream kernel (quantize_rows).
#include <cuda_runtime.h>

#include <atomic>
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
__device__ __forceinline__ uint32_t quantize_rows(const uint16_t *__restrict__ x, int64_t rows,
                                              int64_t cols, float s_enc, const float *inv_tab,
                                              uint8_t *__restrict__ q, uint8_t *__restrict__ sf,
                                              int bx, int64_t rs, int64_t n_streams, int tx,
                                              bool descending) {
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

    uint32_t amax_bits = 0;  // running |x| maximum of this thread's blocks (bf16 bits)
    int64_t g = rs;
    if (g >= n_groups) return amax_bits;
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
            const uint32_t mb = absmax_bf16x16(cur[u]);  // 0 for padding (zero-filled)
            amax_bits = max(amax_bits, mb);
            const BlockScale bs = block_scale(__uint_as_float(mb << 16), s_enc, inv_tab);
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
    return amax_bits;
}

// grid.x covers the padded block columns (64 per slice), grid.y x 2 row
// streams stride the rows.
// amax_out (optional, zeroed by the launch): max |x| of this tensor, folded
// in with one atomicMax per warp on the float's bit pattern; the one-pass
// quantize with an earlier call's scale hands it to the next call.
template <bool kDynamic>
__global__ void __launch_bounds__(kQuantThreads) quantize_kernel(
    const uint16_t *__restrict__ x, int64_t rows, int64_t cols, const float *__restrict__ scale_in,
    uint8_t *__restrict__ q, uint8_t *__restrict__ sf, float *__restrict__ s_dec_out,
    unsigned *__restrict__ amax_out) {
    const float s_enc = kDynamic ? tensor_encode_scale(*scale_in) : *scale_in;
    if (s_dec_out != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0)
        *s_dec_out = __fdiv_rn(1.0f, s_enc);
    __shared__ float inv_tab[128];
    fill_inv_table(inv_tab, s_enc);
    __syncthreads();
    constexpr int kStreams = kQuantThreads / kSliceBlocks;
    uint32_t m = quantize_rows(x, rows, cols, s_enc, inv_tab, q, sf, blockIdx.x,
                               static_cast<int64_t>(blockIdx.y) * kStreams + threadIdx.x / kSliceBlocks,
                               static_cast<int64_t>(gridDim.y) * kStreams, threadIdx.x % kSliceBlocks,
                               false);
    if (amax_out != nullptr) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if ((threadIdx.x & 31) == 0 && m != 0) atomicMax(amax_out, m << 16);
    }
}

constexpr int kDynThreads = 512;  // 4 row streams x 128 threads

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ unsigned long long ld_acquire_gpu_u64(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// Relaxed load with no compiler barrier: issued early, consumed late.
__device__ __forceinline__ unsigned long long ld_relaxed_gpu_u64(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ void st_release_gpu_u64(unsigned long long *p, unsigned long long v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ unsigned atom_add_acq_rel_gpu(unsigned *p, unsigned v) {
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// Called by one thread per CTA with the CTA's amax bits (bf16 |x| pattern)
// and the generation it read from ws->state at kernel start.  Folds the bits
// into the launch's running amax, then waits (bounded) for every CTA.  The
// arrival is a release-acquire RMW on the counter; the last arrival reads the
// final amax, resets the counter and the running amax for the next launch,
// and publishes (gen + 1, amax) with one release store that the other CTAs
// poll, so leaving the barrier costs no further read.  Returns false (and
// records error tag 7) on timeout.
__device__ __forceinline__ bool grid_amax_barrier(DynWorkspace *ws, unsigned gen, uint32_t m,
                                                  int *err, unsigned *amax_bits_out) {
    if (m != 0) atomicMax(&ws->amax_acc, m << 16);
    const unsigned arrived = atom_add_acq_rel_gpu(&ws->count, 1u);
    if (arrived == gridDim.x - 1) {
        const unsigned a = *reinterpret_cast<volatile unsigned *>(&ws->amax_acc);
        ws->count = 0u;  // both resets are ordered before the release below
        ws->amax_acc = 0u;
        st_release_gpu_u64(&ws->state, (static_cast<unsigned long long>(gen + 1) << 32) | a);
        *amax_bits_out = a;
        return true;
    }
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        const unsigned long long st = ld_acquire_gpu_u64(&ws->state);
        if (static_cast<unsigned>(st >> 32) != gen) {
            *amax_bits_out = static_cast<unsigned>(st);
            return true;
        }
        if (globaltimer_ns() - t0 > kBarrierTimeoutNs) {
            if (err != nullptr && atomicCAS(err, 0, 5) == 0) err[1] = 7;
            return false;
        }
        __nanosleep(32);
    }
}

// L2 eviction-priority policies for loads (createpolicy): lines loaded with
// evict_last stay in L2 ahead of normal and evict_first lines.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// 32 bytes at p (16-byte aligned at least) with an L2 policy, bypassing L1.
__device__ __forceinline__ BF16x16 ldg_32B_policy(const uint8_t *p, bool aligned32, uint64_t pol) {
    BF16x16 v;
    if (aligned32) {
        asm volatile(
            "ld.global.nc.L1::no_allocate.L2::cache_hint.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7},"
            " [%8], %9;"
            : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3]), "=r"(v.w[4]), "=r"(v.w[5]),
              "=r"(v.w[6]), "=r"(v.w[7])
            : "l"(p), "l"(pol));
    } else {
        asm volatile(
            "ld.global.nc.L1::no_allocate.L2::cache_hint.v4.b32 {%0, %1, %2, %3}, [%4], %5;"
            : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3])
            : "l"(p), "l"(pol));
        asm volatile(
            "ld.global.nc.L1::no_allocate.L2::cache_hint.v4.b32 {%0, %1, %2, %3}, [%4], %5;"
            : "=r"(v.w[4]), "=r"(v.w[5]), "=r"(v.w[6]), "=r"(v.w[7])
            : "l"(p + 16), "l"(pol));
    }
    return v;
}

constexpr int kFlatThreads = 512;
constexpr int kFlatU = 4;  // 16-element blocks (32-byte loads) in flight per thread
// Input bytes the single-launch quantize keeps in L2 between its two passes
// (of the 126 MB L2, leaving room for the codes and scales it writes).
constexpr int64_t kFlatKeepBytes = int64_t(80) << 20;

// Flat dynamic quantization for cols % 64 == 0 (so 4 consecutive blocks never
// straddle a row and the scale layout has no column padding).  Block v of the
// tensor (row v / kb, block column v % kb) is the 32 bytes at x + 32 v; its
// codes are the 8 bytes at q + 8 v.  Idx is uint32_t when the block count and
// the grid's index range fit 32 bits (register pressure), else int64_t.
template <typename Idx>
__global__ void __launch_bounds__(kFlatThreads, 2) quantize_dynamic_flat_kernel(
    const uint8_t *__restrict__ x, int64_t rows, int64_t cols, uint8_t *__restrict__ q,
    uint8_t *__restrict__ sf, float *__restrict__ s_dec_out, float *__restrict__ amax_out,
    DynWorkspace *ws, int *err) {
    __shared__ unsigned s_amax;
    __shared__ int s_fail;
    __shared__ uint32_t red[kFlatThreads / 32];
    __shared__ float inv_tab[128];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // Only thread 0 needs the generation; its load overlaps phase 1's.  The
    // previous launch on this workspace has completed (stream order).
    const unsigned long long state0 = tid == 0 ? ld_relaxed_gpu_u64(&ws->state) : 0ull;

    const bool a32 = (reinterpret_cast<uintptr_t>(x) & 31) == 0;
    const Idx kb = static_cast<Idx>(cols >> 4);
    const Idx kb4 = kb >> 2;
    const Idx nvec = static_cast<Idx>(rows) * kb;  // a multiple of 4
    const Idx S = static_cast<Idx>(gridDim.x) * kFlatThreads;
    const Idx chunk = S * kFlatU;
    const Idx g = static_cast<Idx>(blockIdx.x) * kFlatThreads + tid;
    const Idx n_rounds = (nvec + chunk - 1) / chunk;

    // Phase 2 walks the rounds backwards, so the rounds phase 1 reads last are
    // the ones it re-reads first: phase 1 loads those (up to kFlatKeepBytes)
    // with an evict-last L2 policy so they are still in L2 for phase 2, which
    // re-reads them with evict-first so they do not stay pinned after the
    // kernel; every other load has the default policy.
    const Idx keep_rounds = static_cast<Idx>(kFlatKeepBytes / (32 * static_cast<int64_t>(chunk)));
    const uint64_t pol_keep = l2_policy_evict_last();
    const uint64_t pol_done = l2_policy_evict_first();
    auto load_round = [&](Idx rd, BF16x16 (&v)[kFlatU], int hint) {  // hint: 0 none, 1 keep, 2 done
#pragma unroll
        for (int u = 0; u < kFlatU; ++u) {
            const Idx idx = rd * chunk + u * S + g;
            const uint8_t *p = x + 32 * static_cast<int64_t>(idx);
            if (idx >= nvec) {
#pragma unroll
                for (int k = 0; k < 8; ++k) v[u].w[k] = 0u;
            } else if (hint == 0) {
                v[u] = ldg_32B(p, a32);
            } else {
                v[u] = ldg_32B_policy(p, a32, hint == 1 ? pol_keep : pol_done);
            }
        }
    };

    // Phase 1: amax.  v keeps the last round for phase 2.
    uint32_t m = 0;
    BF16x16 v[kFlatU];
    for (Idx rd = 0; rd < n_rounds; ++rd) {
        load_round(rd, v, rd + keep_rounds >= n_rounds ? 1 : 0);
#pragma unroll
        for (int u = 0; u < kFlatU; ++u) m = max(m, absmax_bf16x16(v[u]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    if (warp == 0) {
        m = lane < kFlatThreads / 32 ? red[lane] : 0u;
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if (lane == 0) {
            unsigned bits = 0;
            s_fail = grid_amax_barrier(ws, static_cast<unsigned>(state0 >> 32), m, err, &bits) ? 0 : 1;
            s_amax = bits;
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
    fill_inv_table(inv_tab, s_enc);
    __syncthreads();

    // Phase 2: quantize, rounds in reverse order (the last round straight
    // from the registers phase 1 left it in).  Validity is uniform over
    // each group of 4 lanes (nvec and every warp's first index are multiples
    // of 4), so the scale gather's shuffles see consistent neighbours.
    for (Idx rd = n_rounds; rd-- > 0;) {
        if (rd + 1 != n_rounds) load_round(rd, v, rd + keep_rounds >= n_rounds ? 2 : 0);
#pragma unroll
        for (int u = 0; u < kFlatU; ++u) {
            const Idx idx = rd * chunk + u * S + g;
            const bool valid = idx < nvec;
            const BlockScale bs =
                block_scale(__uint_as_float(absmax_bf16x16(v[u]) << 16), s_enc, inv_tab);
            if (valid) {
                const uint4 lo = make_uint4(v[u].w[0], v[u].w[1], v[u].w[2], v[u].w[3]);
                const uint4 hi = make_uint4(v[u].w[4], v[u].w[5], v[u].w[6], v[u].w[7]);
                *reinterpret_cast<uint2 *>(q + 8 * static_cast<int64_t>(idx)) =
                    make_uint2(quantize_bf16x8(lo, bs.inv), quantize_bf16x8(hi, bs.inv));
            }
            const uint32_t sfc = valid ? bs.sf : 0u;
            const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, sfc, 1);
            const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, sfc, 2);
            const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, sfc, 3);
            if (valid && (lane & 3) == 0) {
                const Idx r = idx / kb;
                const Idx c = idx - r * kb;
                *reinterpret_cast<uint32_t *>(sf + sf_offset(r, c, kb4)) =
                    sfc | (s1 << 8) | (s2 << 16) | (s3 << 24);
            }
        }
    }
    // Zero scales of the padding rows [rows, pad128(rows)).
    const Idx rows_i = static_cast<Idx>(rows);
    const Idx n_pad = (((rows_i + 127) & ~Idx(127)) - rows_i) * kb4;
    for (Idx i = g; i < n_pad; i += S) {
        const Idx pr = i / kb4;
        *reinterpret_cast<uint32_t *>(sf + sf_offset(rows_i + pr, 4 * (i - pr * kb4), kb4)) = 0u;
    }
}

// Row-stream variant (8 row streams x 64 threads) for widths that are not a
// multiple of 64.  The grid is resident all at once; the barrier is bounded.
__global__ void __launch_bounds__(kDynThreads) quantize_dynamic_kernel(
    const uint16_t *__restrict__ x, int64_t rows, int64_t cols, uint8_t *__restrict__ q,
    uint8_t *__restrict__ sf, float *__restrict__ s_dec_out, float *__restrict__ amax_out,
    DynWorkspace *ws, int *err, int gx) {
    __shared__ unsigned s_amax;
    __shared__ int s_fail;
    __shared__ uint32_t red[kDynThreads / 32];
    __shared__ float inv_tab[128];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const unsigned long long state0 = tid == 0 ? ld_relaxed_gpu_u64(&ws->state) : 0ull;

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
            unsigned bits = 0;
            s_fail = grid_amax_barrier(ws, static_cast<unsigned>(state0 >> 32), m, err, &bits) ? 0 : 1;
            s_amax = bits;
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
    fill_inv_table(inv_tab, s_enc);
    __syncthreads();

    // Phase 2: quantize, rows descending.
    const int nby = static_cast<int>(gridDim.x) / gx;
    const int byc = static_cast<int>(blockIdx.x) / gx;
    if (byc >= nby) return;
    constexpr int kStreams = kDynThreads / kSliceBlocks;
    quantize_rows(x, rows, cols, s_enc, inv_tab, q, sf, static_cast<int>(blockIdx.x) % gx,
                  static_cast<int64_t>(byc) * kStreams + tid / kSliceBlocks,
                  static_cast<int64_t>(nby) * kStreams, tid % kSliceBlocks, true);
}

constexpr int kRowWarps = 8;  // rows per CTA of the per-row kernel

// Per-token (per-row) tensor scales: row r is quantized as its own tensor,
// S_enc[r] = 2688 / amax(row r), with the usual per-16 block scales.  One warp
// per row: pass 1 reduces the row's amax (lane l takes blocks l, l+32, ...),
// pass 2 re-reads the row (from L1/L2) and quantizes; four block scales of
// the row are gathered with shuffles into one 4-byte store.  Warps of the
// padding rows [rows, pad128(rows)) write zero scale words.  No grid-wide
// step, so one launch of independent warps.
__global__ void __launch_bounds__(32 * kRowWarps) quantize_rowwise_kernel(
    const uint8_t *__restrict__ x, int64_t rows, int64_t cols, uint8_t *__restrict__ q,
    uint8_t *__restrict__ sf, float *__restrict__ s_dec_rows, float *__restrict__ amax_rows) {
    const int lane = threadIdx.x & 31;
    const int64_t r = static_cast<int64_t>(blockIdx.x) * kRowWarps + (threadIdx.x >> 5);
    const int64_t kb = cols >> 4;
    const int64_t kb4 = (kb + 3) >> 2;
    const int64_t kbp = kb4 << 2;
    const int64_t rows_pad = (rows + 127) & ~int64_t(127);
    if (r >= rows_pad) return;
    if (r >= rows) {
        for (int64_t c4 = lane; c4 < kb4; c4 += 32)
            *reinterpret_cast<uint32_t *>(sf + sf_offset(r, 4 * c4, kb4)) = 0u;
        return;
    }
    const uint8_t *xr = x + r * cols * 2;
    // Pass 1: row amax (16-byte loads that allocate in L1 for pass 2).
    uint32_t m = 0;
#pragma unroll 4
    for (int64_t c = lane; c < kb; c += 32) m = max(m, absmax_bf16x16(ldg_32B(xr + 32 * c, false)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    const float amax = __uint_as_float(m << 16);
    const float s_enc = tensor_encode_scale(amax);
    if (lane == 0) {
        s_dec_rows[r] = __fdiv_rn(1.0f, s_enc);
        if (amax_rows != nullptr) amax_rows[r] = amax;
    }
    // Pass 2: quantize.  All lanes run the same iterations (shuffles).
    uint8_t *qr = q + r * (cols >> 1);
    for (int64_t c0 = 0; c0 < kbp; c0 += 32) {
        const int64_t c = c0 + lane;
        const bool valid = c < kb;
        BF16x16 v;
        if (valid) {
            v = ldg_32B(xr + 32 * c, false);
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) v.w[k] = 0u;
        }
        const BlockScale bs = block_scale_direct(__uint_as_float(absmax_bf16x16(v) << 16), s_enc);
        if (valid) {
            const uint4 lo = make_uint4(v.w[0], v.w[1], v.w[2], v.w[3]);
            const uint4 hi = make_uint4(v.w[4], v.w[5], v.w[6], v.w[7]);
            *reinterpret_cast<uint2 *>(qr + 8 * c) =
                make_uint2(quantize_bf16x8(lo, bs.inv), quantize_bf16x8(hi, bs.inv));
        }
        const uint32_t sfc = valid ? bs.sf : 0u;
        const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, sfc, 1);
        const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, sfc, 2);
        const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, sfc, 3);
        if ((lane & 3) == 0 && c < kbp)
            *reinterpret_cast<uint32_t *>(sf + sf_offset(r, c, kb4)) =
                sfc | (s1 << 8) | (s2 << 16) | (s3 << 24);
    }
}

cudaError_t launch_quantize_rowwise(const void *x, int64_t rows, int64_t cols, uint8_t *q,
                                    uint8_t *sf, float *s_dec_rows, float *amax_rows,
                                    cudaStream_t stream) {
    const int64_t rows_pad = (rows + 127) / 128 * 128;
    const int64_t blocks = (rows_pad + kRowWarps - 1) / kRowWarps;
    if (blocks > 2147483647) return cudaErrorInvalidValue;
    quantize_rowwise_kernel<<<static_cast<unsigned>(blocks), 32 * kRowWarps, 0, stream>>>(
        reinterpret_cast<const uint8_t *>(x), rows, cols, q, sf, s_dec_rows, amax_rows);
    return cudaGetLastError();
}

// FP8 variant (E4M3 elements, one FP32 per-tensor scale, the pages' FP8 mode):
// S_enc = 448 / amax (1 if amax == 0, FLT_MAX if not finite), each element
// E4M3_rn_satfinite(x * S_enc) with its sign.  Grid-stride over groups of 8
// elements: one 16-byte load, four cvt.rn.satfinite.e4m3x2, one 8-byte store.
__global__ void __launch_bounds__(256) quantize_fp8_kernel(const uint4 *__restrict__ x,
                                                            int64_t n8, const float *__restrict__ amax,
                                                            uint2 *__restrict__ q,
                                                            float *__restrict__ s_dec_out) {
    const float a = *amax;
    float s_enc = 1.0f;
    if (a != 0.0f) {
        s_enc = __fdiv_rn(448.0f, a);
        if (!isfinite(s_enc)) s_enc = FLT_MAX;
    }
    if (blockIdx.x == 0 && threadIdx.x == 0 && s_dec_out != nullptr)
        *s_dec_out = __fdiv_rn(1.0f, s_enc);
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
         i += stride) {
        const uint4 v = __ldg(x + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t h[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float lo = __fmul_rn(bf16_lo(w[k]), s_enc);
            const float hi = __fmul_rn(bf16_hi(w[k]), s_enc);
            // cvt ... e4m3x2 d, a, b puts a in the upper byte: element 2k+1.
            asm("{\n\t.reg .b16 t;\n\t"
                "cvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\t"
                "cvt.u32.u16 %0, t;\n\t}\n"
                : "=r"(h[k])
                : "f"(hi), "f"(lo));
        }
        q[i] = make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
    }
}

cudaError_t launch_quantize_fp8(const void *x, int64_t numel, const float *amax, uint8_t *q,
                                float *s_dec_out, int num_sms, cudaStream_t stream) {
    const int64_t n8 = numel / 8;
    int64_t blocks = (n8 + 255) / 256;
    const int64_t cap = static_cast<int64_t>(num_sms) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    quantize_fp8_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        reinterpret_cast<const uint4 *>(x), n8, amax, reinterpret_cast<uint2 *>(q), s_dec_out);
    return cudaGetLastError();
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

// ------------------------------------------------------------------------
// One-pass block quantize with S_enc known before the pass (given, or derived
// from an amax the caller holds), for rows of a multiple of 64 elements: the
// flat layout of quantize_dynamic_flat_kernel's phase 2 without its amax
// phase and grid barrier.  Thread g of S quantizes blocks g, g+S, g+2S, g+3S
// of every round of 4S blocks, all four loads in flight; optionally folds
// max |x| into amax_out (zeroed by the launch) for a later call.
template <bool kDynamic, typename Idx>
__global__ void __launch_bounds__(kFlatThreads, 2) quantize_flat_kernel(
    const uint8_t *__restrict__ x, int64_t rows, int64_t cols, const float *__restrict__ scale_in,
    uint8_t *__restrict__ q, uint8_t *__restrict__ sf, float *__restrict__ s_dec_out,
    unsigned *__restrict__ amax_out) {
    __shared__ float inv_tab[128];
    const int tid = threadIdx.x, lane = tid & 31;
    const float s_enc = kDynamic ? tensor_encode_scale(*scale_in) : *scale_in;
    if (s_dec_out != nullptr && blockIdx.x == 0 && tid == 0) *s_dec_out = __fdiv_rn(1.0f, s_enc);
    fill_inv_table(inv_tab, s_enc);
    __syncthreads();

    const bool a32 = (reinterpret_cast<uintptr_t>(x) & 31) == 0;
    const Idx kb = static_cast<Idx>(cols >> 4);
    const Idx kb4 = kb >> 2;
    const Idx nvec = static_cast<Idx>(rows) * kb;  // a multiple of 4
    const Idx S = static_cast<Idx>(gridDim.x) * kFlatThreads;
    const Idx chunk = S * kFlatU;
    const Idx g = static_cast<Idx>(blockIdx.x) * kFlatThreads + tid;
    const Idx n_rounds = (nvec + chunk - 1) / chunk;
    uint32_t m = 0;
    for (Idx rd = 0; rd < n_rounds; ++rd) {
        BF16x16 v[kFlatU];
#pragma unroll
        for (int u = 0; u < kFlatU; ++u) {
            const Idx idx = rd * chunk + u * S + g;
            if (idx < nvec) {
                v[u] = ldg_32B(x + 32 * static_cast<int64_t>(idx), a32);
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) v[u].w[k] = 0u;
            }
        }
        // Validity is uniform over each group of 4 lanes (nvec, S and every
        // warp's first index are multiples of 4).
#pragma unroll
        for (int u = 0; u < kFlatU; ++u) {
            const Idx idx = rd * chunk + u * S + g;
            const bool valid = idx < nvec;
            const uint32_t mb = absmax_bf16x16(v[u]);
            m = max(m, mb);
            const BlockScale bs = block_scale(__uint_as_float(mb << 16), s_enc, inv_tab);
            if (valid) {
                const uint4 lo = make_uint4(v[u].w[0], v[u].w[1], v[u].w[2], v[u].w[3]);
                const uint4 hi = make_uint4(v[u].w[4], v[u].w[5], v[u].w[6], v[u].w[7]);
                *reinterpret_cast<uint2 *>(q + 8 * static_cast<int64_t>(idx)) =
                    make_uint2(quantize_bf16x8(lo, bs.inv), quantize_bf16x8(hi, bs.inv));
            }
            const uint32_t sfc = valid ? bs.sf : 0u;
            const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, sfc, 1);
            const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, sfc, 2);
            const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, sfc, 3);
            if (valid && (lane & 3) == 0) {
                const Idx r = idx / kb;
                const Idx c = idx - r * kb;
                *reinterpret_cast<uint32_t *>(sf + sf_offset(r, c, kb4)) =
                    sfc | (s1 << 8) | (s2 << 16) | (s3 << 24);
            }
        }
    }
    // Zero scales of the padding rows [rows, pad128(rows)).
    const Idx rows_i = static_cast<Idx>(rows);
    const Idx n_pad = (((rows_i + 127) & ~Idx(127)) - rows_i) * kb4;
    for (Idx i = g; i < n_pad; i += S) {
        const Idx pr = i / kb4;
        *reinterpret_cast<uint32_t *>(sf + sf_offset(rows_i + pr, 4 * (i - pr * kb4), kb4)) = 0u;
    }
    if (amax_out != nullptr) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if (lane == 0 && m != 0) atomicMax(amax_out, m << 16);
    }
}

cudaError_t launch_quantize(const void *x, int64_t rows, int64_t cols, const float *scale_in,
                            bool dynamic, uint8_t *q, uint8_t *sf, float *s_dec_out, int num_sms,
                            cudaStream_t stream, float *amax_out) {
    if (amax_out != nullptr) {
        const cudaError_t e = cudaMemsetAsync(amax_out, 0, sizeof(float), stream);
        if (e != cudaSuccess) return e;
    }
    unsigned *am = reinterpret_cast<unsigned *>(amax_out);
    if (cols % 64 == 0) {
        // Flat one-pass kernel: up to 2 CTAs per SM, at least ~one block per
        // thread; 32-bit indices where every index (blocks, padded scale
        // offsets, the last round's overshoot) stays below 2^31.
        const int64_t nvec = rows * (cols / 16);
        int64_t grid = (nvec + kFlatThreads - 1) / kFlatThreads;
        const int64_t cap = static_cast<int64_t>(num_sms) * 2;
        if (grid > cap) grid = cap;
        if (grid < 1) grid = 1;
        const int64_t span = grid * kFlatThreads * kFlatU;
        const int64_t sf_span = ((rows + 127) / 128 * 128) * (cols / 16);
        const uint8_t *xb = reinterpret_cast<const uint8_t *>(x);
        const unsigned gs = static_cast<unsigned>(grid);
        const bool narrow = nvec + span < (int64_t(1) << 31) && sf_span < (int64_t(1) << 31);
        if (dynamic) {
            if (narrow)
                quantize_flat_kernel<true, uint32_t><<<gs, kFlatThreads, 0, stream>>>(
                    xb, rows, cols, scale_in, q, sf, s_dec_out, am);
            else
                quantize_flat_kernel<true, int64_t><<<gs, kFlatThreads, 0, stream>>>(
                    xb, rows, cols, scale_in, q, sf, s_dec_out, am);
        } else {
            if (narrow)
                quantize_flat_kernel<false, uint32_t><<<gs, kFlatThreads, 0, stream>>>(
                    xb, rows, cols, scale_in, q, sf, s_dec_out, am);
            else
                quantize_flat_kernel<false, int64_t><<<gs, kFlatThreads, 0, stream>>>(
                    xb, rows, cols, scale_in, q, sf, s_dec_out, am);
        }
        return cudaGetLastError();
    }
    const int64_t kbp = ((cols / 16 + 3) / 4) * 4;
    const int64_t rows_pad = (rows + 127) / 128 * 128;
    const int64_t gx = (kbp + kSliceBlocks - 1) / kSliceBlocks;
    const int64_t streams_per_cta = kQuantThreads / kSliceBlocks;
    const int64_t target = static_cast<int64_t>(num_sms) * 16;
    const int64_t groups = (rows_pad + kQuantRows - 1) / kQuantRows;
    int64_t gy = (groups + streams_per_cta - 1) / streams_per_cta;
    if (gy < 1) gy = 1;  // rows == 0: one row of CTAs still writes s_dec_out
    int64_t cap = target / gx;
    if (cap < 1) cap = 1;
    if (gy > cap) gy = cap;
    if (gy > 65535) gy = 65535;
    if (gx > 2147483647) return cudaErrorInvalidValue;
    dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
    const uint16_t *xp = reinterpret_cast<const uint16_t *>(x);
    if (dynamic)
        quantize_kernel<true><<<grid, kQuantThreads, 0, stream>>>(xp, rows, cols, scale_in, q, sf,
                                                                 s_dec_out, am);
    else
        quantize_kernel<false><<<grid, kQuantThreads, 0, stream>>>(xp, rows, cols, scale_in, q,
                                                                  sf, s_dec_out, am);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------
// quantize_dynamic, resident form: for tensors whose 16-element blocks fit in
// the shared memory of one CTA per SM (up to ~28 MB of bf16 on 148 SMs; the
// qkv input of a 1024^2 DiT block is 28.3 MB).  CTA b owns one contiguous
// slice of whole blocks (a multiple of 4, so a row's four-scale groups never
// straddle two CTAs) and issues bulk copies of all of it into shared memory
// at once, in kResPieces pieces with one mbarrier each; the warps of piece p
// reduce its amax as soon as it lands.  After the grid barrier the slice is
// quantized from shared memory.  x is read from HBM exactly once, all of it
// in flight from the start, and phase 2 re-reads nothing from L2.

constexpr int kResThreads = 1024;
constexpr int kResPieces = 8;
constexpr int kResWarpsPerPiece = kResThreads / 32 / kResPieces;
// Shared memory of the slice: leaves room for the static arrays below within
// the 227 KB a CTA may use.
constexpr int64_t kResMaxBytes = 216 * 1024;

namespace {

// Bulk-copy and mbarrier helpers of this translation unit (the GEMM's live
// in ptx.cuh, which only gemm.cu includes).
__device__ __forceinline__ uint32_t res_smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void res_mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(res_smem_addr(bar)), "r"(count));
}

__device__ __forceinline__ void res_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(res_smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

// Contiguous global -> shared copy (16-byte aligned addresses, size a
// multiple of 16), completion counted on bar in bytes.
__device__ __forceinline__ void res_bulk_load(void *dst, const void *src, uint32_t bytes,
                                              uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            res_smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(res_smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ bool res_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(res_smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for phase 0 of bar: false once the deadline (%globaltimer
// ns) has passed.
__device__ __forceinline__ bool res_wait(uint64_t *bar, uint64_t deadline) {
    while (!res_try_wait(bar, 0)) {
        if (globaltimer_ns() > deadline) return false;
    }
    return true;
}

__device__ __forceinline__ BF16x16 lds_32B(const uint8_t *p) {
    BF16x16 v;
    const uint4 a = *reinterpret_cast<const uint4 *>(p);
    const uint4 b = *reinterpret_cast<const uint4 *>(p + 16);
    v.w[0] = a.x; v.w[1] = a.y; v.w[2] = a.z; v.w[3] = a.w;
    v.w[4] = b.x; v.w[5] = b.y; v.w[6] = b.z; v.w[7] = b.w;
    return v;
}

}  // namespace

__global__ void __launch_bounds__(kResThreads, 1) quantize_dynamic_resident_kernel(
    const uint8_t *__restrict__ x, int64_t rows, int64_t cols, uint32_t per_cta,
    uint8_t *__restrict__ q, uint8_t *__restrict__ sf, float *__restrict__ s_dec_out,
    float *__restrict__ amax_out, DynWorkspace *ws, int *err) {
    extern __shared__ __align__(128) uint8_t xs[];  // the slice, 32 bytes per block
    __shared__ uint64_t bars[kResPieces];
    __shared__ unsigned s_amax;
    __shared__ int s_fail, s_lost;
    __shared__ uint32_t red[kResThreads / 32];
    __shared__ float inv_tab[128];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const unsigned long long state0 = tid == 0 ? ld_relaxed_gpu_u64(&ws->state) : 0ull;

    // 32-bit indices: the launch checks that blocks and padded scale
    // offsets stay below 2^31.
    const uint32_t kb = static_cast<uint32_t>(cols >> 4);
    const uint32_t kb4 = kb >> 2;
    const uint32_t nvec = static_cast<uint32_t>(rows) * kb;  // a multiple of 4
    const uint32_t lo = min(blockIdx.x * per_cta, nvec);
    const uint32_t cnt = min(per_cta, nvec - lo);  // a multiple of 4
    // Piece p: blocks [piece(p), piece(p + 1)) of the slice, multiples of 4.
    auto piece = [&](int p) -> uint32_t {
        return p >= kResPieces ? cnt : (cnt / 4 * p / kResPieces) * 4;
    };

    if (tid == 0) {
        s_lost = 0;
        for (int p = 0; p < kResPieces; ++p) res_mbar_init(&bars[p], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (tid == 0) {
        for (int p = 0; p < kResPieces; ++p) {
            const uint32_t a = piece(p), bytes = (piece(p + 1) - a) * 32u;
            res_arrive_expect_tx(&bars[p], bytes);
            if (bytes != 0) res_bulk_load(xs + 32u * a, x + 32 * (int64_t(lo) + a), bytes, &bars[p]);
        }
    }

    // Phase 1: the warps of piece p wait for it, then reduce its amax.
    uint32_t m = 0;
    {
        const int p = warp / kResWarpsPerPiece;
        const uint32_t t = static_cast<uint32_t>(tid - p * kResWarpsPerPiece * 32);
        const uint64_t deadline = globaltimer_ns() + kBarrierTimeoutNs;
        if (res_wait(&bars[p], deadline)) {
            for (uint32_t i = piece(p) + t; i < piece(p + 1); i += kResWarpsPerPiece * 32)
                m = max(m, absmax_bf16x16(lds_32B(xs + 32u * i)));
        } else {
            s_lost = 1;  // benign race: every writer stores 1
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    if (warp == 0) {
        m = red[lane];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if (lane == 0) {
            if (s_lost && err != nullptr && atomicCAS(err, 0, 5) == 0) err[1] = 8;
            // A CTA whose copies never landed still joins the barrier, so the
            // others are not left waiting; the error word already says the
            // result is invalid.
            unsigned bits = 0;
            s_fail = grid_amax_barrier(ws, static_cast<unsigned>(state0 >> 32), m, err, &bits) ? 0 : 1;
            s_amax = bits;
        }
    }
    __syncthreads();
    if (s_fail || s_lost) {
        // Copies may still be in flight into this CTA's shared memory: wait
        // for them (bounded) before the CTA exits.
        if (tid == 0) {
            const uint64_t deadline = globaltimer_ns() + kBarrierTimeoutNs;
            for (int p = 0; p < kResPieces; ++p) res_wait(&bars[p], deadline);
        }
        return;
    }
    const float amax = __uint_as_float(s_amax);
    const float s_enc = tensor_encode_scale(amax);
    if (blockIdx.x == 0 && tid == 0) {
        if (s_dec_out != nullptr) *s_dec_out = __fdiv_rn(1.0f, s_enc);
        if (amax_out != nullptr) *amax_out = amax;
    }
    fill_inv_table(inv_tab, s_enc);
    __syncthreads();

    // Phase 2: quantize the slice from shared memory.  Validity is uniform
    // over each group of 4 lanes (cnt and kResThreads are multiples of 4),
    // so the scale gather's shuffles see consistent neighbours.
    for (uint32_t base = 0; base < cnt; base += kResThreads) {
        const uint32_t i = base + static_cast<uint32_t>(tid);
        const bool valid = i < cnt;
        BF16x16 v;
        if (valid) {
            v = lds_32B(xs + 32u * i);
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) v.w[k] = 0u;
        }
        const BlockScale bs = block_scale(__uint_as_float(absmax_bf16x16(v) << 16), s_enc, inv_tab);
        const uint32_t idx = lo + i;
        if (valid) {
            const uint4 a = make_uint4(v.w[0], v.w[1], v.w[2], v.w[3]);
            const uint4 b = make_uint4(v.w[4], v.w[5], v.w[6], v.w[7]);
            *reinterpret_cast<uint2 *>(q + 8 * static_cast<int64_t>(idx)) =
                make_uint2(quantize_bf16x8(a, bs.inv), quantize_bf16x8(b, bs.inv));
        }
        const uint32_t sfc = valid ? bs.sf : 0u;
        const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, sfc, 1);
        const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, sfc, 2);
        const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, sfc, 3);
        if (valid && (lane & 3) == 0) {
            const uint32_t r = idx / kb;
            const uint32_t c = idx - r * kb;
            *reinterpret_cast<uint32_t *>(sf + sf_offset(r, c, kb4)) =
                sfc | (s1 << 8) | (s2 << 16) | (s3 << 24);
        }
    }
    // Zero scales of the padding rows [rows, pad128(rows)).
    const uint32_t rows_i = static_cast<uint32_t>(rows);
    const uint32_t n_pad = (((rows_i + 127u) & ~127u) - rows_i) * kb4;
    const uint32_t S = gridDim.x * kResThreads;
    for (uint32_t i = blockIdx.x * kResThreads + tid; i < n_pad; i += S) {
        const uint32_t pr = i / kb4;
        *reinterpret_cast<uint32_t *>(sf + sf_offset(rows_i + pr, 4 * (i - pr * kb4), kb4)) = 0u;
    }
}

cudaError_t launch_quantize_dynamic(const void *x, int64_t rows, int64_t cols, uint8_t *q,
                                    uint8_t *sf, float *s_dec_out, float *amax_out,
                                    DynWorkspace *ws, int num_sms, cudaStream_t stream) {
    // Per device, from the occupancy queries (atomics: host threads may make
    // their first calls concurrently; they all store the same values).
    static std::atomic<int> resident_rows[64];
    static std::atomic<int> resident_flat[64];
    static std::atomic<int> res_ready[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    const bool flat = cols % 64 == 0;
    std::atomic<int> &resident_slot = flat ? resident_flat[dev] : resident_rows[dev];
    int resident = resident_slot.load(std::memory_order_relaxed);
    if (resident == 0) {
        int per_sm = 0;
        // Both index widths of the flat kernel have the same launch bounds.
        e = flat ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                       &per_sm, quantize_dynamic_flat_kernel<int64_t>, kFlatThreads, 0)
                 : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quantize_dynamic_kernel,
                                                                 kDynThreads, 0);
        if (e != cudaSuccess || per_sm < 1) return e != cudaSuccess ? e : cudaErrorInvalidValue;
        resident = per_sm;
        resident_slot.store(per_sm, std::memory_order_relaxed);
    }
    int grid = num_sms * resident;
    int *err = device_error_word();
    // The grid barrier needs every CTA resident at once: the grid is exactly
    // what the occupancy query says fits, and the launch is cooperative, so
    // the runtime guarantees it (or refuses the launch).
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(flat ? kFlatThreads : kDynThreads);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (flat) {
        const uint8_t *xb = reinterpret_cast<const uint8_t *>(x);
        const int64_t nvec_all = rows * (cols / 16);
        const int64_t sf_all = ((rows + 127) / 128 * 128) * (cols / 16);
        // Resident form when one slice per SM fits in shared memory.
        const int64_t per = ((nvec_all + num_sms - 1) / num_sms + 3) / 4 * 4;
        if (per * 32 <= kResMaxBytes && nvec_all < (int64_t(1) << 31) &&
            sf_all < (int64_t(1) << 31)) {
            int ready = res_ready[dev].load(std::memory_order_relaxed);
            if (ready == 0) {
                e = cudaFuncSetAttribute(quantize_dynamic_resident_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kResMaxBytes));
                if (e != cudaSuccess) return e;
                int per_sm = 0;
                e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                    &per_sm, quantize_dynamic_resident_kernel, kResThreads,
                    static_cast<size_t>(kResMaxBytes));
                if (e != cudaSuccess) return e;
                ready = per_sm >= 1 ? 1 : -1;
                res_ready[dev].store(ready, std::memory_order_relaxed);
            }
            if (ready == 1) {
                cfg.gridDim = dim3(num_sms);
                cfg.blockDim = dim3(kResThreads);
                cfg.dynamicSmemBytes = static_cast<size_t>(per * 32);
                return cudaLaunchKernelEx(&cfg, quantize_dynamic_resident_kernel, xb, rows, cols,
                                          static_cast<uint32_t>(per), q, sf, s_dec_out, amax_out,
                                          ws, err);
            }
        }
        cfg.gridDim = dim3(grid);
        // 32-bit indices when every index the kernel forms (blocks, padded
        // scale offsets, the last round's overshoot) stays below 2^31.
        const int64_t nvec = rows * (cols / 16);
        const int64_t span = int64_t(grid) * kFlatThreads * kFlatU;
        const int64_t sf_span = ((rows + 127) / 128 * 128) * (cols / 16);
        if (nvec + span < (int64_t(1) << 31) && sf_span < (int64_t(1) << 31))
            return cudaLaunchKernelEx(&cfg, quantize_dynamic_flat_kernel<uint32_t>, xb, rows, cols,
                                      q, sf, s_dec_out, amax_out, ws, err);
        return cudaLaunchKernelEx(&cfg, quantize_dynamic_flat_kernel<int64_t>, xb, rows, cols, q,
                                  sf, s_dec_out, amax_out, ws, err);
    }
    const int64_t kbp = ((cols / 16 + 3) / 4) * 4;
    int gx = static_cast<int>((kbp + kSliceBlocks - 1) / kSliceBlocks);
    // Phase 2 needs at least one CTA per column slice; very wide rows use
    // the two-kernel path instead.
    if (gx > grid) return cudaErrorNotSupported;
    grid = (grid / gx) * gx;
    cfg.gridDim = dim3(grid);
    return cudaLaunchKernelEx(&cfg, quantize_dynamic_kernel, reinterpret_cast<const uint16_t *>(x),
                              rows, cols, q, sf, s_dec_out, amax_out, ws, err, gx);
}

}  // namespace nvfp4
