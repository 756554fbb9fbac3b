// Block-scaled FP4 GEMM on 5th-generation tensor cores (tcgen05, sm_100a):
//   Y[m,n] = bf16( alpha * sum_k e2m1(A[m,k]) sfA[m,k/16] e2m1(B[n,k]) sfB[n,k/16] )
// with alpha = a_s_dec * b_s_dec, fp32 accumulation in tensor memory (TMEM),
// optionally followed by the next layer's NVFP4 quantization of Y in the
// epilogue.  This is the NVFP4 linear layer of the FLUX DiT pages ("英伟达
// B200狂飙10.2倍！AI绘图告别龟速！", section "NVFP4量化"; the GEMM kernels compared
// in "NVIDIA shows how TensorRT-LLM VisualGen speeds up FLUX 3 Image Klein on
// Blackwell", optimisation section), written here from scratch.
//
// Design (persistent, warp-specialised, one CTA per SM):
//   warp 0      TMA producer: per k-stage of 256 elements, one 2-D TMA load of
//               the A tile (128 rows x 128 B, 128B swizzle), one of the B tile
//               (BN rows), and contiguous bulk copies of the matching
//               scale-factor tiles (the 128x4 tiled layout makes a 128-row x
//               256-K slice one contiguous 2 KB run).  No multicast.
//   warp 1      MMA issuer (one thread): copies the stage's scale factors from
//               shared memory into TMEM (tcgen05.cp 32x128b.warpx4), then four
//               tcgen05.mma kind::mxf4nvf4 block_scale scale_vec::4X (K = 64
//               each) into the tile's TMEM accumulator; tcgen05.commit frees the
//               smem stage and, after the last k-stage, publishes the tile.
//               Also allocates / frees TMEM.
//   warps 2-5   epilogue: tcgen05.ld of their 32-lane quadrant, alpha scaling,
//               bf16 rounding, global stores, optional fused NVFP4 quantize.
// The accumulator is double-buffered when it fits (BN = 128), so the
// epilogue of tile i overlaps the mainloop of tile i+1.
// Every wait is bounded (see mbar_wait): on timeout the kernel records
// NVFP4_ERR_TIMEOUT, all roles stop, in-flight copies and MMAs are drained
// with bounded waits, and TMEM is freed before exit.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "gemm.h"
#include "nvfp4_math.cuh"
#include "ptx.cuh"

namespace nvfp4 {

cudaError_t read_and_clear_device_error(int *code, int *detail) {
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(code, g_error_code, sizeof(int));
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(detail, g_error_detail, sizeof(int));
    if (e != cudaSuccess) return e;
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_error_code, &zero, sizeof(int));
    if (e != cudaSuccess) return e;
    return cudaMemcpyToSymbol(g_error_detail, &zero, sizeof(int));
}

constexpr int kBM = 128;
constexpr int kBKBytes = 128;  // 256 FP4 elements per k-stage per row
constexpr int kBK = 256;
constexpr int kThreads = 192;

template <int BN_, int STAGES_, int ACC_STAGES_, int SF_SLOTS_>
struct GemmConfig {
    static constexpr int BN = BN_;
    static constexpr int STAGES = STAGES_;
    static constexpr int ACC_STAGES = ACC_STAGES_;
    static constexpr int SF_SLOTS = SF_SLOTS_;
    static constexpr int NB = BN / 128;  // 128-row blocks of B per tile
    static constexpr int A_BYTES = kBM * kBKBytes;
    static constexpr int B_BYTES = BN * kBKBytes;
    static constexpr int SFA_BYTES = 2048;
    static constexpr int SFB_BYTES = 2048 * NB;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_SFA = OFF_B + STAGES * B_BYTES;
    static constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
    static constexpr int OFF_BAR = OFF_SFB + STAGES * SFB_BYTES;
    static constexpr int NUM_BARS = 2 * STAGES + 2 * ACC_STAGES + 1;  // + drain
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack for 1024 alignment
    // TMEM columns: accumulators, then per-slot scale factors.
    static constexpr int SFA_COLS = 16;       // 4 MMAs x 4 columns (128 rows)
    static constexpr int SFB_COLS = 16 * NB;  // 4 MMAs x 4*NB columns
    static constexpr int SF_BASE = ACC_STAGES * BN;
    static constexpr int TMEM_USED = SF_BASE + SF_SLOTS * (SFA_COLS + SFB_COLS);
    static constexpr int TMEM_COLS = TMEM_USED <= 32    ? 32
                                     : TMEM_USED <= 64  ? 64
                                     : TMEM_USED <= 128 ? 128
                                     : TMEM_USED <= 256 ? 256
                                                        : 512;
    static_assert(TMEM_USED <= 512, "TMEM budget");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static constexpr uint32_t IDESC = make_idesc_mxf4nvf4(kBM, BN);
};

struct TileCoord {
    int m_blk, n_blk;
};

// Tile t -> (m, n) block, walking groups of kGroupM row-blocks with n fastest
// inside a group column-by-column, so concurrently running CTAs share A rows.
constexpr int kGroupM = 8;
__device__ __forceinline__ TileCoord tile_coord(int t, int tiles_m, int tiles_n) {
    const int per_group = kGroupM * tiles_n;
    const int g = t / per_group;
    const int first_m = g * kGroupM;
    const int gsz = min(tiles_m - first_m, kGroupM);
    const int r = t - g * per_group;
    TileCoord c;
    c.m_blk = first_m + r % gsz;
    c.n_blk = r / gsz;
    return c;
}

template <class Cfg>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    uint64_t *full = bars;
    uint64_t *empty = bars + Cfg::STAGES;
    uint64_t *acc_full = bars + 2 * Cfg::STAGES;
    uint64_t *acc_empty = acc_full + Cfg::ACC_STAGES;
    uint64_t *drain = acc_empty + Cfg::ACC_STAGES;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + Cfg::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Cfg::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int tiles_m = static_cast<int>((p.M + kBM - 1) / kBM);
    const int tiles_n = static_cast<int>((p.N + Cfg::BN - 1) / Cfg::BN);
    const int num_tiles = tiles_m * tiles_n;
    const int k_stages = static_cast<int>((p.K + kBK - 1) / kBK);
    const int64_t kb4_a = p.K / 64;  // scale tiles per 128-row block (K % 64 == 0)

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < Cfg::ACC_STAGES; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 4);  // one arrive per epilogue warp
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            const uint64_t pol_a = policy_evict_normal();
            const uint64_t pol_b = policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;  // stages whose copies may still be in flight
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                const TileCoord tc = tile_coord(t, tiles_m, tiles_n);
                for (int ks = 0; ks < k_stages; ++ks) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, 1)) {
                        ok = false;
                        break;
                    }
                    const int nsub = min(4, static_cast<int>((p.K - int64_t(ks) * kBK) / 64));
                    uint32_t sfb_bytes = 0;
                    for (int rb = 0; rb < Cfg::NB; ++rb)
                        if (int64_t(tc.n_blk) * Cfg::NB + rb < p.n_sf_blocks) sfb_bytes += nsub * 512;
                    mbar_arrive_expect_tx(&full[stage],
                                          Cfg::A_BYTES + Cfg::B_BYTES + nsub * 512 + sfb_bytes);
                    uint8_t *sa = smem + Cfg::OFF_A + stage * Cfg::A_BYTES;
                    uint8_t *sb = smem + Cfg::OFF_B + stage * Cfg::B_BYTES;
                    tma_load_2d(&tmap_a, &full[stage], sa, ks * kBKBytes, tc.m_blk * kBM, pol_a);
                    tma_load_2d(&tmap_b, &full[stage], sb, ks * kBKBytes, tc.n_blk * Cfg::BN, pol_b);
                    bulk_load(smem + Cfg::OFF_SFA + stage * Cfg::SFA_BYTES,
                              p.asf + (int64_t(tc.m_blk) * kb4_a + int64_t(ks) * 4) * 512,
                              nsub * 512, &full[stage], pol_a);
                    for (int rb = 0; rb < Cfg::NB; ++rb) {
                        const int64_t brow = int64_t(tc.n_blk) * Cfg::NB + rb;
                        if (brow < p.n_sf_blocks)
                            bulk_load(smem + Cfg::OFF_SFB + stage * Cfg::SFB_BYTES + rb * 2048,
                                      p.bsf + (brow * kb4_a + int64_t(ks) * 4) * 512, nsub * 512,
                                      &full[stage], pol_b);
                    }
                    if (issued < Cfg::STAGES) ++issued;
                    if (++stage == Cfg::STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            if (!ok) {
                // Drain: the last `issued` stages may still be receiving data.
                int s = stage;
                uint32_t ph = phase;
                for (int i = 0; i < issued; ++i) {
                    if (--s < 0) {
                        s = Cfg::STAGES - 1;
                        ph ^= 1;
                    }
                    mbar_wait_drain(&full[s], ph);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int local = 0;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++local) {
                const int acc = local % Cfg::ACC_STAGES;
                const uint32_t acc_phase = (local / Cfg::ACC_STAGES) & 1;
                if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1, abort_flag, 2)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * Cfg::BN;
                for (int ks = 0; ks < k_stages; ++ks) {
                    if (!mbar_wait(&full[stage], phase, abort_flag, 3)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nsub = min(4, static_cast<int>((p.K - int64_t(ks) * kBK) / 64));
                    const int slot = stage % Cfg::SF_SLOTS;
                    const uint32_t sfa_t =
                        tmem_base + Cfg::SF_BASE + slot * (Cfg::SFA_COLS + Cfg::SFB_COLS);
                    const uint32_t sfb_t = sfa_t + Cfg::SFA_COLS;
                    const uint32_t sa = smem_addr(smem + Cfg::OFF_A + stage * Cfg::A_BYTES);
                    const uint32_t sb = smem_addr(smem + Cfg::OFF_B + stage * Cfg::B_BYTES);
                    const uint32_t ssfa = smem_addr(smem + Cfg::OFF_SFA + stage * Cfg::SFA_BYTES);
                    const uint32_t ssfb = smem_addr(smem + Cfg::OFF_SFB + stage * Cfg::SFB_BYTES);
                    for (int j = 0; j < nsub; ++j) {
                        // 512-byte chunk j: 128 rows x 4 scales (K = 64) -> 4 columns.
                        tc_cp_32x128b_warpx4(sfa_t + 4 * j, make_smem_desc(ssfa + 512 * j, 0, 128, 0));
                        for (int rb = 0; rb < Cfg::NB; ++rb)
                            tc_cp_32x128b_warpx4(sfb_t + 4 * Cfg::NB * j + 4 * rb,
                                                 make_smem_desc(ssfb + 2048 * rb + 512 * j, 0, 128, 0));
                    }
                    for (int j = 0; j < nsub; ++j) {
                        const uint64_t adesc = make_smem_desc(sa + 32 * j, 16, 1024, 2);
                        const uint64_t bdesc = make_smem_desc(sb + 32 * j, 16, 1024, 2);
                        mma_mxf4nvf4(d_tmem, adesc, bdesc, Cfg::IDESC, sfa_t + 4 * j,
                                     sfb_t + 4 * Cfg::NB * j, (ks > 0 || j > 0) ? 1u : 0u);
                    }
                    tc_commit(&empty[stage]);
                    if (++stage == Cfg::STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                tc_commit(&acc_full[acc]);
            }
            // Arrives once every tcgen05 operation issued here has completed;
            // the teardown waits on it when the CTA aborted, before TMEM is freed.
            tc_commit(drain);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue
        const int quad = warp & 3;  // TMEM lanes [32*quad, 32*quad+32)
        const int row_in_tile = quad * 32 + lane;
        const float alpha = __fmul_rn(*p.a_s_dec, *p.b_s_dec);
        const bool fused = p.yq != nullptr;
        const float s_enc_y = fused ? *p.s_enc_y : 1.0f;
        const int64_t nb_y = p.N / 16;
        const int64_t nb4_y = (nb_y + 3) / 4;
        uint32_t amax_bits = 0;
        int local = 0;
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++local) {
            const TileCoord tc = tile_coord(t, tiles_m, tiles_n);
            const int acc = local % Cfg::ACC_STAGES;
            const uint32_t acc_phase = (local / Cfg::ACC_STAGES) & 1;
            if (!mbar_wait_warp(&acc_full[acc], acc_phase, abort_flag, 4)) break;
            tc_fence_after();
            const int64_t m = int64_t(tc.m_blk) * kBM + row_in_tile;
            const bool row_ok = m < p.M;
            uint32_t sf_word = 0;
#pragma unroll 1
            for (int ch = 0; ch < Cfg::BN / 32; ++ch) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem_base + acc * Cfg::BN + ch * 32 + ((quad * 32) << 16), r);
                tmem_ld_wait();
                if (ch == Cfg::BN / 32 - 1) {
                    // Accumulator fully read: hand it back to the MMA warp.
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&acc_empty[acc]);
                }
                const int64_t n0 = int64_t(tc.n_blk) * Cfg::BN + ch * 32;
                uint32_t packed[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float lo = __fmul_rn(__uint_as_float(r[2 * i]), alpha);
                    const float hi = __fmul_rn(__uint_as_float(r[2 * i + 1]), alpha);
                    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
                    packed[i] = *reinterpret_cast<const uint32_t *>(&h);
                }
                if (row_ok && p.y != nullptr) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        if (n0 + 8 * g < p.N)
                            *reinterpret_cast<uint4 *>(p.y + (m * p.N + n0 + 8 * g) * 2) =
                                make_uint4(packed[4 * g], packed[4 * g + 1], packed[4 * g + 2],
                                           packed[4 * g + 3]);
                    }
                }
                if (fused) {
#pragma unroll
                    for (int b = 0; b < 2; ++b) {
                        const int64_t nblk = (n0 >> 4) + b;
                        const bool ok_blk = row_ok && nblk < nb_y;
                        const uint4 v0 = make_uint4(packed[8 * b], packed[8 * b + 1],
                                                    packed[8 * b + 2], packed[8 * b + 3]);
                        const uint4 v1 = make_uint4(packed[8 * b + 4], packed[8 * b + 5],
                                                    packed[8 * b + 6], packed[8 * b + 7]);
                        const uint32_t mb = max(absmax_bf16x8(v0), absmax_bf16x8(v1));
                        const BlockScale bs = block_scale(__uint_as_float(mb << 16), s_enc_y);
                        if (ok_blk) {
                            amax_bits = max(amax_bits, mb);
                            const uint2 codes = make_uint2(quantize_bf16x8(v0, bs.inv),
                                                           quantize_bf16x8(v1, bs.inv));
                            *reinterpret_cast<uint2 *>(p.yq + m * (p.N / 2) + nblk * 8) = codes;
                        }
                        const uint32_t sfc = ok_blk ? bs.sf : 0u;
                        sf_word |= sfc << (8 * ((nblk & 3)));
                    }
                    // Four blocks (64 columns) complete a 4-byte scale group.
                    if (ch & 1) {
                        const int64_t nblk0 = ((n0 >> 4) + 1) & ~int64_t(3);
                        if (nblk0 < nb4_y * 4)
                            *reinterpret_cast<uint32_t *>(p.ysf + sf_offset(m, nblk0, nb4_y)) =
                                sf_word;
                        sf_word = 0;
                    }
                }
            }
        }
        if (fused && p.amax_y != nullptr) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                amax_bits = max(amax_bits, __shfl_xor_sync(0xFFFFFFFFu, amax_bits, o));
            if (lane == 0 && amax_bits != 0)
                atomicMax(reinterpret_cast<unsigned *>(p.amax_y), amax_bits << 16);
        }
    }

    // ------------------------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        if (*abort_flag) {
            // Bounded wait for the drain commit issued above.
            if (lane == 0) mbar_wait_drain(drain, 0);
            __syncwarp();
        }
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

template <class Cfg>
static cudaError_t launch_cfg(const CUtensorMap &ta, const CUtensorMap &tb, const GemmParams &p,
                              int num_sms, cudaStream_t stream) {
    static int configured_device = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_device != dev) {
        cudaError_t e = cudaFuncSetAttribute(gemm_kernel<Cfg>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             Cfg::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        configured_device = dev;
    }
    const int64_t tiles = ((p.M + kBM - 1) / kBM) * ((p.N + Cfg::BN - 1) / Cfg::BN);
    const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
    gemm_kernel<Cfg><<<grid, kThreads, Cfg::SMEM_BYTES, stream>>>(ta, tb, p);
    return cudaGetLastError();
}

using Cfg128 = GemmConfig<128, 6, 2, 6>;
using Cfg256 = GemmConfig<256, 4, 1, 4>;

int gemm_tile_n(int64_t M, int64_t N) {
    (void)M;
    (void)N;
    return 128;
}

cudaError_t launch_gemm(const CUtensorMap &ta, const CUtensorMap &tb, const GemmParams &p,
                        int tile_n, int num_sms, cudaStream_t stream) {
    if (tile_n == 256) return launch_cfg<Cfg256>(ta, tb, p, num_sms, stream);
    return launch_cfg<Cfg128>(ta, tb, p, num_sms, stream);
}

}  // namespace nvfp4
