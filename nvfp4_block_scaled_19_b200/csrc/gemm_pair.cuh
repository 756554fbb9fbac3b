// Block-scaled FP4 GEMM on CTA pairs (tcgen05 cta_group::2), 256 x 256 tiles.
//
// Same computation as gemm_kernel (see gemm.cu), with each tile computed by
// a cluster of two CTAs on two SMs: CTA r holds rows 128r..128r+127 of the
// tile's A slice and rows 128r..128r+127 of its B slice in its own shared
// memory, and one 256x256x64 MMA issued by the pair leader (CTA 0) reads both
// CTAs' halves, leaving rows 128r..128r+127 of the accumulator in CTA r's
// tensor memory.  Per SM this loads A 16 KB + B 16 KB per 256-element
// k-stage for 128x256 outputs, a third less L2 -> SM traffic than the 1-CTA
// 128x256 tile (A 16 KB + B 32 KB), which measured bound at ~20 TB/s.
//
// Roles (both CTAs unless noted):
//   warp 0     producer: waits its own `empty` ring slot; the leader arms its
//              `full` barrier with both CTAs' A+B bytes; each CTA issues
//              `.cta_group::2` TMA loads (no multicast) of its A and B halves
//              into its own shared memory that complete on the leader's
//              `full` barrier, and loads its scale factors (its 128 A rows,
//              all 256 B rows: one 3-D TMA box each) against its own
//              `sfload` barrier.
//   warp 1     leader only: issues the MMAs (cta_group::2) and commits to the
//              `empty`, `acc_full` barriers of both CTAs (tcgen05.commit
//              multicast); both CTAs' warp 1 allocate / free the TMEM pair.
//   warps 2-5  scale factors into this CTA's TMEM (tcgen05.st), then arrive
//              on the leader's `full` barrier (remote for CTA 1), so that one
//              wait per stage covers operands and scales alike.
//   warps 6.. epilogue of this CTA's 128 rows, EPI_WARPS / 4 warps per TMEM
//              lane quadrant (8 warps, 128 accumulator columns each, measured
//              faster on B200 than 16 warps of 64 columns); arrive on the
//              leader's `acc_empty` barrier once the accumulator is read.
// The scale-factor TMEM layout per CTA is the 1-CTA N = 256 one: SFA for its
// own 128 rows, SFB for all 256 B rows, replicated in every lane quadrant.
//
// The MMA issue loop is the critical path.  Measured on B200, every cycle
// added to the issuing thread's k-stage adds at least a cycle to the kernel,
// and the ring's round trip (commit, producer, TMA, scale warps, barrier) is
// nearly as long as five stages: waiting less often, or through another
// warp, lengthened that round trip and was slower.  Hence one `full` barrier
// per stage for operands and scales alike, and stage loops unrolled over the
// ring so that no slot address is computed at run time.
#pragma once

#include <type_traits>

namespace nvfp4 {

// Runs body(std::integral_constant<int, S>{}) for the ring slots S = stage,
// stage + 1, ..., 4 in order while it returns true.  The stage loops of the
// producer, the scale warps and the MMA thread are unrolled over the 5-slot
// ring this way, so every slot address, descriptor and TMEM offset in a body
// is a constant; a body advances its own state and returns false to stop.
template <class F>
__device__ __forceinline__ void ring5_from(int stage, F &&body) {
    switch (stage) {
        case 0:
            if (!body(std::integral_constant<int, 0>{})) return;
            [[fallthrough]];
        case 1:
            if (!body(std::integral_constant<int, 1>{})) return;
            [[fallthrough]];
        case 2:
            if (!body(std::integral_constant<int, 2>{})) return;
            [[fallthrough]];
        case 3:
            if (!body(std::integral_constant<int, 3>{})) return;
            [[fallthrough]];
        default:
            body(std::integral_constant<int, 4>{});
    }
}

template <int STAGES_, int EPI_WARPS_>
struct PairConfig {
    static constexpr int STAGES = STAGES_;
    static constexpr int BN = 256;  // tile columns (B rows), split 128 per CTA
    static constexpr int BM = 256;  // tile rows, split 128 per CTA
    static constexpr int SF_WARPS = 4;
    static constexpr int EPI_WARPS = EPI_WARPS_;  // 8 or 16
    static constexpr int EPI_COLS = 256 / (EPI_WARPS / 4);  // accumulator columns per warp
    static constexpr int FIRST_SF_WARP = 2;
    static constexpr int FIRST_EPI_WARP = FIRST_SF_WARP + SF_WARPS;
    static constexpr int THREADS = 32 * (FIRST_EPI_WARP + EPI_WARPS);
    static constexpr int A_BYTES = 128 * kBKBytes;
    static constexpr int B_BYTES = 128 * kBKBytes;
    static constexpr int SFA_BYTES = 2048;
    static constexpr int SFB_BYTES = 4096;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_SFA = OFF_B + STAGES * B_BYTES;
    static constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
    static constexpr int OFF_BAR = OFF_SFB + STAGES * SFB_BYTES;
    // full, sfload, empty per stage; acc_full, acc_empty, drain
    static constexpr int NUM_BARS = 3 * STAGES + 3;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int OFF_INV = OFF_MISC + 16;  // 128-entry block-multiplier table
    // Y leaves through TMA stores of 32-row x 64-column boxes staged in shared
    // memory (whole 128-byte lines, instead of 32-byte pieces of 32 rows per
    // store instruction); 4 KB per epilogue warp.  The 16-warp (GELU)
    // configuration has no room for it and stores from registers.
    static constexpr bool TMA_Y = EPI_WARPS == 8;
    static constexpr int OFF_STG = (OFF_INV + 512 + 1023) / 1024 * 1024;
    static constexpr int STG_BYTES = TMA_Y ? EPI_WARPS * 4096 : 0;
    static constexpr int SMEM_BYTES = OFF_STG + STG_BYTES + 1024;
    static constexpr int SFA_COLS = 16;
    static constexpr int SFB_COLS = 32;
    static constexpr int SLOT_COLS = SFA_COLS + SFB_COLS;
    static constexpr int SF_BASE = BN;  // one 256-column accumulator
    static constexpr int TMEM_USED = SF_BASE + STAGES * SLOT_COLS;
    static_assert(STAGES == 5, "the stage loops are unrolled over a 5-slot ring (ring5_from)");
    static constexpr int TMEM_COLS = 512;
    static_assert(TMEM_USED <= 512, "TMEM budget");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static constexpr uint32_t IDESC = make_idesc_mxf4nvf4(256, 256);
};

// kFp8: the FP8 variant (E4M3 operands, per-tensor scales only): a 128-byte
// k-stage holds 128 elements, four tcgen05.mma kind::f8f6f4 (K = 32) cover
// it, and there are no block scales (no scale copies; the scale warps only
// forward their arrival so the barrier counts stay the same).
template <class Cfg, bool kGelu, bool kFp8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Cfg::THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ GemmMaps maps, const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    uint64_t *full = bars;
    uint64_t *sfload = bars + Cfg::STAGES;
    uint64_t *empty = bars + 2 * Cfg::STAGES;
    uint64_t *acc_full = bars + 3 * Cfg::STAGES;
    uint64_t *acc_empty = acc_full + 1;
    uint64_t *drain = acc_full + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + Cfg::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Cfg::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int tiles_m = static_cast<int>((p.M + Cfg::BM - 1) / Cfg::BM);
    const int tiles_n = static_cast<int>((p.N + Cfg::BN - 1) / Cfg::BN);
    const int num_tiles = tiles_m * tiles_n;
    const int pair = blockIdx.x >> 1;
    const int n_pairs = gridDim.x >> 1;
    // Operand bytes per row and k-stages of 128 bytes (256 FP4 / 128 FP8
    // elements); one MMA covers 32 bytes of K.
    const int64_t kbytes = kFp8 ? p.K : p.K / 2;
    const int k_stages = static_cast<int>((kbytes + kBKBytes - 1) / kBKBytes);

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::STAGES; ++s) {
            // The leader's producer arrival (with both CTAs' operand bytes)
            // plus every scale-factor warp of the pair.
            mbar_init(&full[s], 1 + 2 * Cfg::SF_WARPS);
            mbar_init(&sfload[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 2 * Cfg::EPI_WARPS);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&maps.a);
        prefetch_tmap(&maps.b);
        if (!kFp8) {
            prefetch_tmap(&maps.sfa);
            prefetch_tmap(&maps.sfb);
        }
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_holder, Cfg::TMEM_COLS);
        tmem_relinquish_pair();
    }
    float *inv_tab = reinterpret_cast<float *>(smem + Cfg::OFF_INV);
    if (p.yq != nullptr) fill_inv_table(inv_tab, *p.s_enc_y);
    if (p.s_dec_y != nullptr && blockIdx.x == 0 && threadIdx.x == 0)
        *p.s_dec_y = __fdiv_rn(1.0f, *p.s_enc_y);
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // barrier inits of both CTAs visible before any remote use
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            const uint64_t pol_a = policy_evict_normal();
            const uint64_t pol_b = policy_evict_last();
            const uint32_t full0 = mapa_shared(smem_addr(&full[0]), 0);  // leader's full[0]
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            bool ok = true;
            const uint32_t smem_s = smem_addr(smem);
            const uint32_t empty_a = smem_addr(empty);
            const uint32_t full_a = smem_addr(full);
            const uint32_t sfload_a = smem_addr(sfload);
            for (int t = pair; t < num_tiles && ok; t += n_pairs) {
                const TileCoord tc = tile_coord(t, tiles_m, tiles_n);
                const int a_row = tc.m_blk * Cfg::BM + static_cast<int>(rank) * 128;
                const int b_row = tc.n_blk * Cfg::BN + static_cast<int>(rank) * 128;
                const int sfa_blk = tc.m_blk * 2 + static_cast<int>(rank);
                int ks = 0;
                // One k-stage into ring slot S (unrolled: constant addresses).
                auto step = [&](auto slot) -> bool {
                    constexpr int S = decltype(slot)::value;
                    if (ks == k_stages) return false;
                    if (!mbar_wait_at(empty_a + 8 * S, phase ^ 1, abort_flag, 11)) {
                        ok = false;
                        return false;
                    }
                    if (leader)
                        mbar_arrive_expect_tx_at(full_a + 8 * S, 2 * (Cfg::A_BYTES + Cfg::B_BYTES));
                    // One box per operand's scales: 8 lines (this k-stage's four
                    // 512-byte tiles) of this CTA's A row block, and of both B row
                    // blocks of the tile.  Boxes are counted whole; lines past K
                    // or row blocks past the tensor arrive as zeros.
                    mbar_arrive_expect_tx_at(sfload_a + 8 * S,
                                             kFp8 ? 0u : uint32_t(Cfg::SFA_BYTES + Cfg::SFB_BYTES));
                    if (!kFp8) {
                        tma_load_3d_at(&maps.sfa, sfload_a + 8 * S,
                                       smem_s + Cfg::OFF_SFA + S * Cfg::SFA_BYTES, 0, ks * 8,
                                       sfa_blk, pol_a);
                        tma_load_3d_at(&maps.sfb, sfload_a + 8 * S,
                                       smem_s + Cfg::OFF_SFB + S * Cfg::SFB_BYTES, 0, ks * 8,
                                       tc.n_blk * 2, pol_b);
                    }
                    // Operands after the scales: the scales travel a longer way
                    // (scale warps, TMEM) before the stage is ready; issued
                    // first they land first (measured 1-4% faster on B200).
                    tma_load_2d_pair_at(&maps.a, full0 + 8 * S, smem_s + Cfg::OFF_A + S * Cfg::A_BYTES,
                                        ks * kBKBytes, a_row, pol_a);
                    tma_load_2d_pair_at(&maps.b, full0 + 8 * S, smem_s + Cfg::OFF_B + S * Cfg::B_BYTES,
                                        ks * kBKBytes, b_row, pol_b);
                    if (issued < Cfg::STAGES) ++issued;
                    ++ks;
                    if constexpr (S + 1 == Cfg::STAGES) {
                        stage = 0;
                        phase ^= 1;
                    } else {
                        stage = S + 1;
                    }
                    return true;
                };
                while (ok && ks < k_stages) ring5_from(stage, step);
            }
            if (!ok) {
                // Drain this CTA's in-flight scale copies (and, on the leader,
                // both CTAs' operand copies) under one bounded deadline; `full`
                // may also miss scale-warp arrivals that will never come.
                const uint64_t deadline = globaltimer() + kWaitTimeoutNs;
                int s = stage;
                uint32_t ph = phase;
                for (int i = 0; i < issued; ++i) {
                    if (--s < 0) {
                        s = Cfg::STAGES - 1;
                        ph ^= 1;
                    }
                    mbar_wait_until(&sfload[s], ph, deadline);
                    if (leader) mbar_wait_until(&full[s], ph, deadline);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (leader && lane == 0) {
            const uint64_t adesc0 = make_smem_desc(smem_addr(smem + Cfg::OFF_A), 16, 1024, 2);
            const uint64_t bdesc0 = make_smem_desc(smem_addr(smem + Cfg::OFF_B), 16, 1024, 2);
            const int k_full = static_cast<int>(kbytes / kBKBytes);         // stages of 4 MMAs
            const int k_tail = static_cast<int>((kbytes % kBKBytes) / 32);  // MMAs in a short stage
            constexpr uint32_t kIdesc = kFp8 ? make_idesc_f8_e4m3(256, 256) : Cfg::IDESC;
            // One MMA of the stage at smem descriptors (a, b), 32-byte K step j.
            auto mma = [&](uint64_t a, uint64_t b, uint32_t sfa_t, uint32_t sfb_t, int j,
                           uint32_t acc) {
                if constexpr (kFp8)
                    mma_f8f6f4_pair(tmem_base, a + 2 * j, b + 2 * j, kIdesc, acc);
                else
                    mma_mxf4nvf4_pair(tmem_base, a + 2 * j, b + 2 * j, kIdesc, sfa_t + 4 * j,
                                      sfb_t + 8 * j, acc);
            };
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int local = 0;
            const uint32_t full_a = smem_addr(full);
            const uint32_t empty_a = smem_addr(empty);
            const uint32_t sf_t0 = tmem_base + Cfg::SF_BASE;
            // One full 256-element stage in ring slot S: wait, four MMAs, one
            // commit.  S is a compile-time constant, so every address and
            // descriptor here is a constant offset from a register.
            auto full_stage = [&](auto slot, uint32_t acc0) -> bool {
                constexpr int S = decltype(slot)::value;
                if (!mbar_wait_at(full_a + 8 * S, phase, abort_flag, 13)) return false;
                tc_fence_after();
                const uint64_t adesc = adesc0 + ((uint64_t(S) * Cfg::A_BYTES) >> 4);
                const uint64_t bdesc = bdesc0 + ((uint64_t(S) * Cfg::B_BYTES) >> 4);
                const uint32_t sfa_t = sf_t0 + S * Cfg::SLOT_COLS;
                const uint32_t sfb_t = sfa_t + Cfg::SFA_COLS;
                mma(adesc, bdesc, sfa_t, sfb_t, 0, acc0);
#pragma unroll
                for (int j = 1; j < 4; ++j) mma(adesc, bdesc, sfa_t, sfb_t, j, 1u);
                tc_commit_pair_at(empty_a + 8 * S, 0x3);
                return true;
            };
            for (int t = pair; t < num_tiles && ok; t += n_pairs, ++local) {
                if (!mbar_wait(acc_empty, (local & 1) ^ 1, abort_flag, 12)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // Full 256-element stages, unrolled over the ring and entered
                // at the current slot.
                int ks = 0;
                auto step = [&](auto slot) -> bool {
                    constexpr int S = decltype(slot)::value;
                    if (ks == k_full) return false;
                    if (!full_stage(slot, ks > 0 ? 1u : 0u)) {
                        ok = false;
                        return false;
                    }
                    ++ks;
                    if constexpr (S + 1 == Cfg::STAGES) {
                        stage = 0;
                        phase ^= 1;
                    } else {
                        stage = S + 1;
                    }
                    return true;
                };
                while (ok && ks < k_full) ring5_from(stage, step);
                if (ok && k_tail > 0) {
                    // Last stage of a K that is not a multiple of 256.
                    if (!mbar_wait(&full[stage], phase, abort_flag, 14)) {
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
                            mma(adesc, bdesc, sfa_t, sfb_t, j, (k_full > 0 || j > 0) ? 1u : 0u);
                        tc_commit_pair(&empty[stage], 0x3);
                        if (++stage == Cfg::STAGES) {
                            stage = 0;
                            phase ^= 1;
                        }
                    }
                }
                if (!ok) break;
                tc_commit_pair(acc_full, 0x3);
            }
            tc_commit_pair(drain, 0x3);
        }
        __syncwarp();
    } else if (warp < Cfg::FIRST_EPI_WARP) {
        // ---------------------------------------------------------------- scale factors
        const uint32_t lane_base = tmem_base + ((static_cast<uint32_t>(warp & 3) * 32) << 16);
        const uint32_t ssfa0 = smem_addr(smem + Cfg::OFF_SFA) + lane * 16;
        const uint32_t ssfb0 = smem_addr(smem + Cfg::OFF_SFB) + lane * 16;
        const uint32_t full0 = mapa_shared(smem_addr(&full[0]), 0);  // leader's full[0]
        const uint32_t sfload_a = smem_addr(sfload);
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int t = pair; t < num_tiles && ok; t += n_pairs) {
            int ks = 0;
            // The scales of one k-stage in ring slot S (unrolled: constant
            // offsets).
            auto step = [&](auto slot) -> bool {
                constexpr int S = decltype(slot)::value;
                if (ks == k_stages) return false;
                if (!mbar_wait_warp_at(sfload_a + 8 * S, phase, abort_flag, 15)) {
                    ok = false;
                    return false;
                }
                if constexpr (!kFp8) {
                    const uint32_t slot_t = lane_base + Cfg::SF_BASE + S * Cfg::SLOT_COLS;
                    uint32_t va[16];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint4 v = lds128(ssfa0 + S * Cfg::SFA_BYTES + 512 * j);
                        va[4 * j] = v.x;
                        va[4 * j + 1] = v.y;
                        va[4 * j + 2] = v.z;
                        va[4 * j + 3] = v.w;
                    }
                    tmem_st_32x32b_x16(slot_t, va);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        // B scale column 8j + 4rb + c: MMA step j, 128-row block rb.
                        uint32_t vb[16];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int col = 16 * h + 4 * q;
                            const int j = col / 8;
                            const int rb = (col / 4) % 2;
                            const uint4 v =
                                lds128(ssfb0 + S * Cfg::SFB_BYTES + rb * 2048 + 512 * j);
                            vb[4 * q] = v.x;
                            vb[4 * q + 1] = v.y;
                            vb[4 * q + 2] = v.z;
                            vb[4 * q + 3] = v.w;
                        }
                        tmem_st_32x32b_x16(slot_t + Cfg::SFA_COLS + 16 * h, vb);
                    }
                    tmem_st_wait();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster_relaxed(full0 + 8 * S);
                ++ks;
                if constexpr (S + 1 == Cfg::STAGES) {
                    stage = 0;
                    phase ^= 1;
                } else {
                    stage = S + 1;
                }
                return true;
            };
            while (ok && ks < k_stages) ring5_from(stage, step);
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        const int e = warp - Cfg::FIRST_EPI_WARP;
        const int quad = warp & 3;
        const int col0 = (e >> 2) * Cfg::EPI_COLS;
        const int row_in_tile = static_cast<int>(rank) * 128 + quad * 32 + lane;
        // alpha = S_dec,A * S_dec,B; with per-row scales of A, S_dec,A of this
        // thread's row of the tile.
        const float b_s_dec = *p.b_s_dec;
        const float alpha_tensor = p.a_row_scale ? 0.0f : __fmul_rn(*p.a_s_dec, b_s_dec);
        const float s_enc_y = p.yq != nullptr ? *p.s_enc_y : 1.0f;
        const uint32_t acc_empty_l = mapa_shared(smem_addr(acc_empty), 0);
        uint32_t amax_bits = 0;
        int local = 0;
        for (int t = pair; t < num_tiles; t += n_pairs, ++local) {
            const TileCoord tc = tile_coord(t, tiles_m, tiles_n);
            const int64_t m_row = int64_t(tc.m_blk) * Cfg::BM + row_in_tile;
            const float alpha = p.a_row_scale
                                    ? __fmul_rn(p.a_s_dec[m_row < p.M ? m_row : p.M - 1], b_s_dec)
                                    : alpha_tensor;
            if (!mbar_wait_warp(acc_full, local & 1, abort_flag, 16)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + col0 + ((static_cast<uint32_t>(quad) * 32) << 16);
            uint32_t pk[Cfg::EPI_COLS / 2];
            if constexpr (kGelu && Cfg::EPI_COLS == 64) {
                // All 64 raw columns in registers, accumulator handed back,
                // then the GELU arithmetic overlaps the next tile's MMAs.
                uint32_t r0[32], r1[32];
                tmem_ld_32x32b_x32(taddr, r0);
                tmem_ld_32x32b_x32(taddr + 32, r1);
                tmem_ld_wait();
                tmem_regs_ready(r0);
                tmem_regs_ready(r1);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster_relaxed(acc_empty_l);
                store_blocks_64<true>(p, r0, r1, alpha, int64_t(tc.m_blk) * Cfg::BM + row_in_tile,
                                      int64_t(tc.n_blk) * Cfg::BN + col0, s_enc_y, inv_tab,
                                      amax_bits);
                continue;
            } else {
                drain_cols<Cfg::EPI_COLS, kGelu>(taddr, alpha, pk);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster_relaxed(acc_empty_l);
            }
            const int64_t n0 = int64_t(tc.n_blk) * Cfg::BN + col0;
            if constexpr (Cfg::TMA_Y) {
                if (p.y != nullptr) {
                    // Lane = row of the warp's 32 rows; 128-byte swizzle: 16-byte
                    // chunk j of row r sits at chunk j ^ (r % 8), which also keeps
                    // the shared-memory writes free of bank conflicts.
                    uint8_t *stg = smem + Cfg::OFF_STG + e * 4096;
                    const uint32_t srow = smem_addr(stg) + lane * 128;
                    const int64_t m0 = int64_t(tc.m_blk) * Cfg::BM + static_cast<int>(rank) * 128 +
                                       quad * 32;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (lane == 0) bulk_wait_group_read<0>();  // previous box read out
                        __syncwarp();
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            sts128(srow + ((j ^ (lane & 7)) << 4), pk[32 * h + 4 * j],
                                   pk[32 * h + 4 * j + 1], pk[32 * h + 4 * j + 2],
                                   pk[32 * h + 4 * j + 3]);
                        fence_proxy_async_smem();
                        __syncwarp();
                        // A box starting inside Y (partial boxes are clipped by
                        // the TMA); boxes that would start past M or N are skipped.
                        if (lane == 0 && m0 < p.M && n0 + 64 * h < p.N) {
                            tma_store_2d(&maps.y, stg, static_cast<int>(n0 + 64 * h),
                                         static_cast<int>(m0));
                            bulk_commit_group();
                        }
                    }
                }
            }
            store_row<Cfg::EPI_COLS>(p, pk, int64_t(tc.m_blk) * Cfg::BM + row_in_tile, n0, s_enc_y,
                                     inv_tab, amax_bits, !Cfg::TMA_Y);
        }
        flush_amax_y(p, amax_bits, lane);
        if constexpr (Cfg::TMA_Y) {
            if (lane == 0) bulk_wait_group<0>();  // Y boxes written before the CTA exits
            __syncwarp();
        }
    }

    // ------------------------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    if (leader && warp == 1 && *abort_flag) {
        if (lane == 0) mbar_wait_drain(drain, 0);
        __syncwarp();
    }
    // Neither CTA leaves while the pair's MMAs may still read its shared
    // memory or a remote arrive may still target it.
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
    }
}

// Plain epilogue: 8 warps of 128 columns.  GELU epilogue: 16 warps of 64
// columns, so a warp holds its raw columns while it hands the accumulator
// back and computes the activation afterwards.
template <bool kGelu>
using PairCfgFor = PairConfig<5, kGelu ? 16 : 8>;

template <bool kGelu, bool kFp8>
inline cudaError_t launch_pair(const GemmMaps &maps, const GemmParams &p, int num_sms,
                               cudaStream_t stream) {
    using Cfg = PairCfgFor<kGelu>;
    // Per device: clusters that fit at once, published by `configured`
    // (atomics: host threads may make their first calls concurrently).
    static std::atomic<int> configured[64];
    static std::atomic<int> max_clusters[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(gemm_pair_kernel<Cfg, kGelu, kFp8>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (num_sms / 2));
        cfg.blockDim = dim3(Cfg::THREADS);
        cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, gemm_pair_kernel<Cfg, kGelu, kFp8>, &cfg);
        if (e != cudaSuccess || n < 1) {
            cudaGetLastError();
            n = num_sms / 2;
        }
        max_clusters[dev].store(n, std::memory_order_relaxed);
        configured[dev].store(1, std::memory_order_release);
    }
    const int64_t tiles = ((p.M + 255) / 256) * ((p.N + 255) / 256);
    int64_t pairs = max_clusters[dev].load(std::memory_order_relaxed);
    if (pairs > tiles) pairs = tiles;
    gemm_pair_kernel<Cfg, kGelu, kFp8><<<static_cast<unsigned>(2 * pairs), Cfg::THREADS,
                                Cfg::SMEM_BYTES, stream>>>(maps, p);
    return cudaGetLastError();
}

}  // namespace nvfp4
