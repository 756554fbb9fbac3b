// Block-scaled FP4 GEMM on 5th-generation tensor cores (tcgen05, sm_100a):
//   Y[m,n] = bf16( alpha * sum_k e2m1(A[m,k]) sfA[m,k/16] e2m1(B[n,k]) sfB[n,k/16] )
// with alpha = a_s_dec * b_s_dec, fp32 accumulation in tensor memory (TMEM),
// optionally followed by the next layer's NVFP4 quantization of Y in the
// epilogue.  This is the NVFP4 linear layer of the FLUX DiT pages ("英伟达
// B200狂飙10.2倍！AI绘图告别龟速！", section "NVFP4量化"; the NVFP4 GEMM kernels
// compared in "NVIDIA介绍用TensorRT LLM VisualGen加速Blackwell上的FLUX 3 Image
// Klein", paragraph on the tested optimisations), written here from scratch.
//
// Design (persistent, warp-specialised, one CTA per SM, 128 x BN tiles):
//   warp 0        TMA producer: per k-stage of 256 elements, a 2-D TMA load of
//                 the A tile (128 rows x 128 B, 128B swizzle), one of the B
//                 tile (BN rows), and one 3-D TMA box per operand of the
//                 matching scale factors (the 128x4-tiled layout makes a
//                 128-row x 256-K slice one contiguous 2 KB run: 8 lines of
//                 256 bytes per 128-row block).  No multicast.
//   warp 1        MMA issuer (one thread): four tcgen05.mma kind::mxf4nvf4
//                 block_scale scale_vec::4X (K = 64 each) per stage into the
//                 tile's TMEM accumulator; tcgen05.commit frees the stage and,
//                 after the last stage, publishes the tile.  Descriptors are
//                 precomputed, so the issue loop is a handful of adds: the MMA
//                 issue queue is shallow and any per-stage work here shows up
//                 as idle tensor cycles.  Also allocates / frees TMEM.
//   warps 2-5     scale-factor warps: each copies the stage's scale factors
//                 from shared memory into its 32-lane quadrant of TMEM with
//                 tcgen05.st (the MMA reads every quadrant's copy), keeping
//                 tcgen05.cp off the MMA issue stream, then arrives on the
//                 stage's `full` barrier: the MMA thread waits once per stage
//                 for operands (TMA bytes) and scales (these arrivals) alike.
//   warps 6..     epilogue, two warps per TMEM quadrant for BN = 256: drain
//                 the accumulator into registers (alpha scaling, bf16
//                 rounding), hand TMEM back to the MMA warp, then store Y and
//                 optionally quantize it (next-layer NVFP4 in blocks of 16).
// Every wait is bounded (mbar_wait): on timeout the kernel records
// NVFP4_ERR_TIMEOUT, all roles stop, in-flight copies and MMAs are drained
// with bounded waits, and TMEM is freed before exit.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "gemm.h"
#include "gemm_common.cuh"
#include "nvfp4_math.cuh"
#include "ptx.cuh"

namespace nvfp4 {

cudaError_t read_and_clear_device_error(int *code, int *detail) {
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return e;
    int v[2] = {0, 0};
    e = cudaMemcpyFromSymbol(v, g_error, sizeof(v));
    if (e != cudaSuccess) return e;
    *code = v[0];
    *detail = v[1];
    const int zero[2] = {0, 0};
    return cudaMemcpyToSymbol(g_error, zero, sizeof(zero));
}

int *device_error_word() {
    // Per device, taken once; atomic because host threads may make their
    // first calls at the same time (they all store the same address).
    static std::atomic<int *> addr[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    int *a = addr[dev].load(std::memory_order_acquire);
    if (a == nullptr) {
        void *v = nullptr;
        if (cudaGetSymbolAddress(&v, g_error) != cudaSuccess) return nullptr;
        a = static_cast<int *>(v);
        addr[dev].store(a, std::memory_order_release);
    }
    return a;
}

// Failure-detection self-test: one warp waits, through the kernels' own
// bounded mbar_wait, on a barrier that nothing will ever complete (its
// arrival count is 2 and one thread arrives once).  The wait gives up after
// timeout_ns, records NVFP4_ERR_TIMEOUT with `tag` in the device error word
// and the kernel returns normally, so the context stays usable.
__global__ void selftest_wait_timeout_kernel(uint64_t timeout_ns, int tag) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 2);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_arrive(&bar);   // one of the two arrivals; the phase stays open
    __syncwarp();
    if (threadIdx.x == 0) mbar_wait_for(&bar, 0, &abort_flag, tag, timeout_ns);
    __syncwarp();
}

cudaError_t launch_selftest_wait_timeout(uint64_t timeout_ns, int tag, cudaStream_t stream) {
    selftest_wait_timeout_kernel<<<1, 32, 0, stream>>>(timeout_ns, tag);
    return cudaGetLastError();
}

constexpr int kBM = 128;
constexpr int kBKBytes = 128;  // 256 FP4 elements per k-stage per row
constexpr int kBK = 256;

template <int BN_, int STAGES_, int ACC_STAGES_>
struct GemmConfig {
    static constexpr int BN = BN_;
    static constexpr int STAGES = STAGES_;
    static constexpr int ACC_STAGES = ACC_STAGES_;
    static constexpr int NB = BN / 128;  // 128-row blocks of B per tile
    static constexpr int SF_WARPS = 4;
    static constexpr int EPI_WARPS = 4 * NB;
    static constexpr int FIRST_SF_WARP = 2;
    static constexpr int FIRST_EPI_WARP = FIRST_SF_WARP + SF_WARPS;
    static constexpr int THREADS = 32 * (FIRST_EPI_WARP + EPI_WARPS);
    static constexpr int A_BYTES = kBM * kBKBytes;
    static constexpr int B_BYTES = BN * kBKBytes;
    static constexpr int SFA_BYTES = 2048;
    static constexpr int SFB_BYTES = 2048 * NB;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_SFA = OFF_B + STAGES * B_BYTES;
    static constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
    static constexpr int OFF_BAR = OFF_SFB + STAGES * SFB_BYTES;
    // full, sfload, empty per stage; acc_full, acc_empty per accumulator; drain
    static constexpr int NUM_BARS = 3 * STAGES + 2 * ACC_STAGES + 1;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int OFF_INV = OFF_MISC + 16;  // 128-entry block-multiplier table
    static constexpr int SMEM_BYTES = OFF_INV + 512 + 1024;  // + slack for 1024 alignment
    // TMEM columns: accumulators, then one scale-factor slot per stage.
    static constexpr int SFA_COLS = 16;       // 4 MMAs x 4 columns (128 rows)
    static constexpr int SFB_COLS = 16 * NB;  // 4 MMAs x 4*NB columns
    static constexpr int SLOT_COLS = SFA_COLS + SFB_COLS;
    static constexpr int SF_BASE = ACC_STAGES * BN;
    static constexpr int TMEM_USED = SF_BASE + STAGES * SLOT_COLS;
    static constexpr int TMEM_COLS = TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
    static_assert(TMEM_USED <= 512, "TMEM budget");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static constexpr uint32_t IDESC = make_idesc_mxf4nvf4(kBM, BN);
};

template <class Cfg, bool kGelu>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
    gemm_kernel(const __grid_constant__ GemmMaps maps, const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    uint64_t *full = bars;
    uint64_t *sfload = bars + Cfg::STAGES;
    uint64_t *empty = bars + 2 * Cfg::STAGES;
    uint64_t *acc_full = bars + 3 * Cfg::STAGES;
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

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::STAGES; ++s) {
            mbar_init(&full[s], 1 + Cfg::SF_WARPS);  // producer + scale-factor warps
            mbar_init(&sfload[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < Cfg::ACC_STAGES; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], Cfg::EPI_WARPS);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&maps.a);
        prefetch_tmap(&maps.b);
        prefetch_tmap(&maps.sfa);
        prefetch_tmap(&maps.sfb);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    float *inv_tab = reinterpret_cast<float *>(smem + Cfg::OFF_INV);
    if (p.yq != nullptr) fill_inv_table(inv_tab, *p.s_enc_y);
    if (p.s_dec_y != nullptr && blockIdx.x == 0 && threadIdx.x == 0)
        *p.s_dec_y = __fdiv_rn(1.0f, *p.s_enc_y);
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
                    mbar_arrive_expect_tx(&full[stage], Cfg::A_BYTES + Cfg::B_BYTES);
                    // Scales: one box of this k-stage's 8 lines (four 512-byte
                    // tiles) for the A row block and one for the tile's NB B row
                    // blocks, counted whole (lines past K, blocks past the
                    // tensor arrive as zeros).
                    mbar_arrive_expect_tx(&sfload[stage], Cfg::SFA_BYTES + Cfg::SFB_BYTES);
                    tma_load_2d(&maps.a, &full[stage], smem + Cfg::OFF_A + stage * Cfg::A_BYTES,
                                ks * kBKBytes, tc.m_blk * kBM, pol_a);
                    tma_load_2d(&maps.b, &full[stage], smem + Cfg::OFF_B + stage * Cfg::B_BYTES,
                                ks * kBKBytes, tc.n_blk * Cfg::BN, pol_b);
                    tma_load_3d(&maps.sfa, &sfload[stage], smem + Cfg::OFF_SFA + stage * Cfg::SFA_BYTES,
                                0, ks * 8, tc.m_blk, pol_a);
                    tma_load_3d(&maps.sfb, &sfload[stage], smem + Cfg::OFF_SFB + stage * Cfg::SFB_BYTES,
                                0, ks * 8, tc.n_blk * Cfg::NB, pol_b);
                    if (issued < Cfg::STAGES) ++issued;
                    if (++stage == Cfg::STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            if (!ok) {
                // Drain: the last `issued` stages may still be receiving data.
                // One bounded deadline for all of them (`full` may also miss
                // scale-warp arrivals that will never come).
                const uint64_t deadline = globaltimer() + kWaitTimeoutNs;
                int s = stage;
                uint32_t ph = phase;
                for (int i = 0; i < issued; ++i) {
                    if (--s < 0) {
                        s = Cfg::STAGES - 1;
                        ph ^= 1;
                    }
                    mbar_wait_until(&sfload[s], ph, deadline);
                    mbar_wait_until(&full[s], ph, deadline);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint64_t adesc0 = make_smem_desc(smem_addr(smem + Cfg::OFF_A), 16, 1024, 2);
            const uint64_t bdesc0 = make_smem_desc(smem_addr(smem + Cfg::OFF_B), 16, 1024, 2);
            const int k_full = static_cast<int>(p.K / kBK);          // stages of 4 MMAs
            const int k_tail = static_cast<int>((p.K % kBK) / 64);  // MMAs in a last short stage
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
                // Full 256-element stages: one wait, four MMAs, one commit.
                for (int ks = 0; ks < k_full; ++ks) {
                    if (!mbar_wait(&full[stage], phase, abort_flag, 3)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t adesc = adesc0 + static_cast<uint64_t>((stage * Cfg::A_BYTES) >> 4);
                    const uint64_t bdesc = bdesc0 + static_cast<uint64_t>((stage * Cfg::B_BYTES) >> 4);
                    const uint32_t sfa_t = tmem_base + Cfg::SF_BASE + stage * Cfg::SLOT_COLS;
                    const uint32_t sfb_t = sfa_t + Cfg::SFA_COLS;
                    mma_mxf4nvf4(d_tmem, adesc, bdesc, Cfg::IDESC, sfa_t, sfb_t, ks > 0 ? 1u : 0u);
#pragma unroll
                    for (int j = 1; j < 4; ++j)
                        mma_mxf4nvf4(d_tmem, adesc + 2 * j, bdesc + 2 * j, Cfg::IDESC,
                                     sfa_t + 4 * j, sfb_t + 4 * Cfg::NB * j, 1u);
                    tc_commit(&empty[stage]);
                    if (++stage == Cfg::STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (ok && k_tail > 0) {
                    // Last stage of a K that is not a multiple of 256.
                    if (!mbar_wait(&full[stage], phase, abort_flag, 5)) {
                        ok = false;
                    } else {
                        tc_fence_after();
                        const uint64_t adesc =
                            adesc0 + static_cast<uint64_t>((stage * Cfg::A_BYTES) >> 4);
                        const uint64_t bdesc =
                            bdesc0 + static_cast<uint64_t>((stage * Cfg::B_BYTES) >> 4);
                        const uint32_t sfa_t = tmem_base + Cfg::SF_BASE + stage * Cfg::SLOT_COLS;
                        const uint32_t sfb_t = sfa_t + Cfg::SFA_COLS;
                        for (int j = 0; j < k_tail; ++j)
                            mma_mxf4nvf4(d_tmem, adesc + 2 * j, bdesc + 2 * j, Cfg::IDESC,
                                         sfa_t + 4 * j, sfb_t + 4 * Cfg::NB * j,
                                         (k_full > 0 || j > 0) ? 1u : 0u);
                        tc_commit(&empty[stage]);
                        if (++stage == Cfg::STAGES) {
                            stage = 0;
                            phase ^= 1;
                        }
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
    } else if (warp < Cfg::FIRST_EPI_WARP) {
        // ---------------------------------------------------------------- scale factors
        // Warp w writes TMEM lanes 32*(w%4)..+31; lane i holds 16-byte line i
        // of every 512-byte scale chunk (rows i, i+32, i+64, i+96 x 4 scales),
        // the layout a 32x128b.warpx4 tensor-memory copy would produce.
        const uint32_t lane_base = tmem_base + ((static_cast<uint32_t>(warp & 3) * 32) << 16);
        const uint32_t ssfa0 = smem_addr(smem + Cfg::OFF_SFA) + lane * 16;
        const uint32_t ssfb0 = smem_addr(smem + Cfg::OFF_SFB) + lane * 16;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
            for (int ks = 0; ks < k_stages; ++ks) {
                if (!mbar_wait_warp(&sfload[stage], phase, abort_flag, 6)) {
                    ok = false;
                    break;
                }
                const uint32_t slot = lane_base + Cfg::SF_BASE + stage * Cfg::SLOT_COLS;
                uint32_t va[16];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 v = lds128(ssfa0 + stage * Cfg::SFA_BYTES + 512 * j);
                    va[4 * j] = v.x;
                    va[4 * j + 1] = v.y;
                    va[4 * j + 2] = v.z;
                    va[4 * j + 3] = v.w;
                }
                tmem_st_32x32b_x16(slot, va);
#pragma unroll
                for (int h = 0; h < Cfg::NB; ++h) {
                    // B scale column 8j + 4rb + c (NB = 2) or 4j + c (NB = 1):
                    // MMA step j, 128-row block rb, 32-bit word c of the line.
                    uint32_t vb[16];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int col = 16 * h + 4 * q;
                        const int j = col / (4 * Cfg::NB);
                        const int rb = (col / 4) % Cfg::NB;
                        const uint4 v =
                            lds128(ssfb0 + stage * Cfg::SFB_BYTES + rb * 2048 + 512 * j);
                        vb[4 * q] = v.x;
                        vb[4 * q + 1] = v.y;
                        vb[4 * q + 2] = v.z;
                        vb[4 * q + 3] = v.w;
                    }
                    tmem_st_32x32b_x16(slot + Cfg::SFA_COLS + 16 * h, vb);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_relaxed(&full[stage]);
                if (++stage == Cfg::STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        const int e = warp - Cfg::FIRST_EPI_WARP;
        const int quad = warp & 3;        // TMEM lanes [32*quad, 32*quad+32)
        const int col0 = (e >> 2) * 128;  // this warp's 128 columns of the tile
        const int row_in_tile = quad * 32 + lane;
        // alpha = S_dec,A * S_dec,B; with per-row scales of A, S_dec,A of this
        // thread's row of the tile.
        const float b_s_dec = *p.b_s_dec;
        const float alpha_tensor = p.a_row_scale ? 0.0f : __fmul_rn(*p.a_s_dec, b_s_dec);
        const float s_enc_y = p.yq != nullptr ? *p.s_enc_y : 1.0f;
        uint32_t amax_bits = 0;
        int local = 0;
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++local) {
            const TileCoord tc = tile_coord(t, tiles_m, tiles_n);
            const int64_t m_row = int64_t(tc.m_blk) * kBM + row_in_tile;
            const float alpha = p.a_row_scale
                                    ? __fmul_rn(p.a_s_dec[m_row < p.M ? m_row : p.M - 1], b_s_dec)
                                    : alpha_tensor;
            const int acc = local % Cfg::ACC_STAGES;
            const uint32_t acc_phase = (local / Cfg::ACC_STAGES) & 1;
            if (!mbar_wait_warp(&acc_full[acc], acc_phase, abort_flag, 4)) break;
            tc_fence_after();
            // Drain 128 accumulator columns into 64 packed bf16x2 registers.
            uint32_t pk[64];
            drain_cols<128, kGelu>(tmem_base + acc * Cfg::BN + col0 + ((static_cast<uint32_t>(quad) * 32) << 16),
                      alpha, pk);
            // Accumulator read: hand it back to the MMA warp.
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_relaxed(&acc_empty[acc]);
            store_row<128>(p, pk, int64_t(tc.m_blk) * kBM + row_in_tile,
                          int64_t(tc.n_blk) * Cfg::BN + col0, s_enc_y, inv_tab, amax_bits);
        }
        flush_amax_y(p, amax_bits, lane);
    }

    // ------------------------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        if (*abort_flag) {
            // Bounded wait for the drain commit issued by the MMA thread.
            if (lane == 0) mbar_wait_drain(drain, 0);
            __syncwarp();
        }
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

template <class Cfg, bool kGelu>
static cudaError_t launch_cfg(const GemmMaps &maps, const GemmParams &p, int num_sms,
                              cudaStream_t stream) {
    static std::atomic<int> configured[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev].load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(gemm_kernel<Cfg, kGelu>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             Cfg::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        configured[dev].store(1, std::memory_order_release);
    }
    const int64_t tiles = ((p.M + kBM - 1) / kBM) * ((p.N + Cfg::BN - 1) / Cfg::BN);
    const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
    gemm_kernel<Cfg, kGelu><<<grid, Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(maps, p);
    return cudaGetLastError();
}

using Cfg128 = GemmConfig<128, 6, 2>;
using Cfg256 = GemmConfig<256, 4, 1>;

GemmKind gemm_kind(int64_t M, int64_t N) {
    if (N < 256) return kGemm128;
    // CTA pairs need at least two 128-row blocks of A to be worth it.
    return M > 128 ? kGemmPair : kGemm256;
}

}  // namespace nvfp4

#include "gemm_pair.cuh"

namespace nvfp4 {

cudaError_t launch_gemm(const GemmMaps &maps, const GemmParams &p, GemmKind kind, int num_sms,
                        cudaStream_t stream) {
    // The activation is a template parameter, so the plain kernels keep their
    // register allocation and only the GELU variants carry erff.
    const bool gelu = p.act == 1;
    if (p.fp8) {  // the FP8 variant runs on CTA pairs only (the entry point checks the shape)
        if (kind != kGemmPair) return cudaErrorInvalidValue;
        return gelu ? launch_pair<true, true>(maps, p, num_sms, stream)
                    : launch_pair<false, true>(maps, p, num_sms, stream);
    }
    if (kind == kGemmPair)
        return gelu ? launch_pair<true, false>(maps, p, num_sms, stream)
                    : launch_pair<false, false>(maps, p, num_sms, stream);
    if (kind == kGemm256)
        return gelu ? launch_cfg<Cfg256, true>(maps, p, num_sms, stream)
                    : launch_cfg<Cfg256, false>(maps, p, num_sms, stream);
    return gelu ? launch_cfg<Cfg128, true>(maps, p, num_sms, stream)
                : launch_cfg<Cfg128, false>(maps, p, num_sms, stream);
}

}  // namespace nvfp4
