// tc_pair.cuh -- the base GEMMs (Y = X W, dX = dY W^T, each with the low-rank branch folded in)
// on pairs of SMs: tcgen05.mma.cta_group::2, M = 256 rows per tile across a cluster of two CTAs.
//
// Each CTA of the pair stages its own 128 rows of A and its own half (128 of 256 columns) of B, so
// a pair moves half the B bytes per output that two independent CTAs would, and a 32 KB stage fits
// a 6-deep ring.  The even CTA ("leader") issues the MMAs; both CTAs' TMA loads complete on the
// leader's full barrier; the leader's commits arrive on the barriers of both CTAs (multicast
// commit); both CTAs' epilogue warps release an accumulator on the leader's barrier.  Each CTA's
// TMEM holds its own 128 rows x 256 columns of the fp32 tile.  No load uses cluster multicast.
#pragma once
#include "tc.cuh"

namespace plora {

constexpr int kPairTileM = 2 * kTileM;           // 256 output rows per pair tile
constexpr int kPairStageBytes = kABytes + kABytes; // A: 128 x 64, B half: 128 x 64 (or 2 x 64 x 64)

template <Op OP>
__global__ void __launch_bounds__(kTcThreads, 1)
tc_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
               const __grid_constant__ CUtensorMap tmC, const TcParams p) {
    static_assert(OP == Op::BaseFwd || OP == Op::BaseDx, "pair kernel covers the base GEMMs");
    constexpr bool kBmn = (OP == Op::BaseDx);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOffset);
    uint64_t* full_bar = bars;
    uint64_t* empty_bar = bars + kMaxStages;
    uint64_t* accf_bar = bars + 2 * kMaxStages;
    uint64_t* acce_bar = bars + 2 * kMaxStages + 2;
    uint64_t* drain_bar = bars + 2 * kMaxStages + 4;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kMaxStages + 5);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const int nst = p.stages;
    const int stb = p.stage_bytes;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t crank = ptx::cluster_ctarank();
    const bool leader = crank == 0;
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; ++s) {
            ptx::mbar_init(&full_bar[s], 1);
            ptx::mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&accf_bar[b], 1);
            ptx::mbar_init(&acce_bar[b], 8);   // 4 epilogue warps in each CTA of the pair
        }
        ptx::mbar_init(drain_bar, 1);
        *abort_flag = 0;
        ptx::fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::tma_prefetch_desc(&tmA);
        ptx::tma_prefetch_desc(&tmB);
        ptx::tma_prefetch_desc(&tmC);
        if (p.fuse) {
            ptx::tma_prefetch_desc(&tmA2);
            ptx::tma_prefetch_desc(&tmB2);
        }
    }
    if (warp == 1) {
        ptx::tmem_alloc_pair<kTmemCols>(tmem_slot);
        ptx::tmem_relinquish_pair();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();   // both CTAs' barriers exist before any load or commit may reach them
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint64_t lim = p.timeout_ns;

    // Tile t of the pair schedule: grouped rasterisation over 256-row m-tiles and 256-column n-tiles.
    auto tile_mn = [&](int t, int& mb, int& nb) {
        const int per_group = p.group_m * p.tiles_n;
        const int g = t / per_group;
        const int first_m = g * p.group_m;
        const int gm = min(p.tiles_m - first_m, p.group_m);
        const int r = t - g * per_group;
        mb = first_m + r % gm;
        nb = r / gm;
    };
    auto rec_of = [&](int t) {
        MTileRec r;
        r.q0 = r.q1 = 0;
        if (p.fuse && t < p.num_tiles) {
            int mb, nb;
            tile_mn(t, mb, nb);
            r = p.mt_rec[mb];
        }
        return r;
    };
    const int kblocks = (p.K_total + kBlockK - 1) / kBlockK;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t armed = 0, armed_par = 0;
            bool ok = true;
            MTileRec lr_next = rec_of(pair);
            const uint32_t a_bytes = (uint32_t)kABytes;
            for (int t = pair; t < p.num_tiles && ok; t += npairs) {
                int mb, nb;
                tile_mn(t, mb, nb);
                const MTileRec lr = lr_next;
                lr_next = rec_of(t + npairs);
                const int a_row = mb * kPairTileM + (int)crank * kTileM;
                const int b_col = nb * kTileN + (int)crank * kTileM;   // this CTA's 128 of the 256 columns
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!ptx::mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, lim, p.err_flag)) { ok = false; break; }
                    uint8_t* sA = smem + stage * stb;
                    uint8_t* sB = sA + kABytes;
                    if (leader) {
                        ptx::mbar_arrive_expect_tx(&full_bar[stage], 2u * (a_bytes + (uint32_t)kABytes));
                        armed |= 1u << stage;
                        armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                    }
                    const uint32_t fb = ptx::pair_leader_addr(&full_bar[stage]);
                    ptx::tma_load_2d_pair(sA, &tmA, fb, kb * kBlockK, a_row);
                    if constexpr (kBmn) {
                        ptx::tma_load_2d_pair(sB, &tmB, fb, b_col, kb * kBlockK);
                        ptx::tma_load_2d_pair(sB + 8192, &tmB, fb, b_col + 64, kb * kBlockK);
                    } else {
                        ptx::tma_load_2d_pair(sB, &tmB, fb, kb * kBlockK, b_col);
                    }
                    if (++stage == nst) { stage = 0; phase ^= 1u; }
                }
                // Folded low-rank branch: A = this CTA's 128 rows of adapter j's zero-padded block,
                // B = this CTA's 128 columns of j's factor, with the base B's major-ness (Y: the
                // B pack, one K-major 128 x 64 box; dX: the A pack, 16-row MN-major boxes).
                for (int q = lr.q0; q < lr.q1 && ok; ++q) {
                    const LoraSeg sg = mtile_seg(p, lr, q);
                    for (int kb = 0; kb * kBlockK < sg.rp16; ++kb) {
                        const int R = min(kBlockK, sg.rp16 - kb * kBlockK);
                        if (!ptx::mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, lim, p.err_flag)) { ok = false; break; }
                        uint8_t* sA = smem + stage * stb;
                        uint8_t* sB = sA + kABytes;
                        if (leader) {
                            const uint32_t lb_bytes = kBmn ? 2u * (uint32_t)R * 128u : (uint32_t)kABytes;
                            ptx::mbar_arrive_expect_tx(&full_bar[stage], 2u * (a_bytes + lb_bytes));
                            armed |= 1u << stage;
                            armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                        }
                        const uint32_t fb = ptx::pair_leader_addr(&full_bar[stage]);
                        ptx::tma_load_2d_pair(sA, &tmA2, fb, kb * kBlockK, sg.h_y + (int)crank * kTileM);
                        if constexpr (kBmn) {
                            for (int h = 0; h < 2; ++h)
                                for (int r16 = 0; r16 < R; r16 += 16)
                                    ptx::tma_load_2d_pair(sB + h * R * 128 + r16 * 128, &tmB2, fb, b_col + 64 * h,
                                                          sg.adapter * p.RP + kb * kBlockK + r16);
                        } else {
                            ptx::tma_load_3d_pair(sB, &tmB2, fb, kb * kBlockK, b_col, sg.adapter);
                        }
                        if (++stage == nst) { stage = 0; phase ^= 1u; }
                    }
                }
            }
            // Drain: the leader's full barriers count both CTAs' bytes; every load of the pair has
            // landed once they complete.  (The final cluster barrier holds the odd CTA until then.)
            if (leader)
                for (int s = 0; s < nst; ++s)
                    if (armed & (1u << s)) {
                        int dummy = 0;
                        ptx::mbar_wait(&full_bar[s], (armed_par >> s) & 1u, &dummy, lim, p.err_flag);
                    }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (even CTA only)
        if (lane == 0 && leader) {
            int stage = 0;
            uint32_t phase = 0;
            int abuf = 0;
            uint32_t aphase = 0;
            bool ok = true;
            const uint32_t idesc = ptx::idesc_bf16_f32(kPairTileM, kTileN, false, kBmn);
            const uint32_t idesc_lr = ptx::idesc_bf16_f32(kPairTileM, kTileN, false, kBmn);
            MTileRec lr_next = rec_of(pair);
            for (int t = pair; t < p.num_tiles && ok; t += npairs) {
                const MTileRec lr = lr_next;
                lr_next = rec_of(t + npairs);
                if (!ptx::mbar_wait(&acce_bar[abuf], aphase ^ 1u, abort_flag, lim, p.err_flag)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(abuf * kTileN);
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!ptx::mbar_wait(&full_bar[stage], phase, abort_flag, lim, p.err_flag)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t sA = ptx::smem_u32(smem + stage * stb);
                    const uint32_t sB = sA + kABytes;
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint64_t adesc = ptx::smem_desc_sw128(sA + ks * 32, 16, 1024);
                        const uint64_t bdesc = kBmn ? ptx::smem_desc_sw128(sB + ks * 2048, 8192, 1024)
                                                    : ptx::smem_desc_sw128(sB + ks * 32, 16, 1024);
                        ptx::tc_mma_f16_pair(d_tmem, adesc, bdesc, idesc, (kb | ks) ? 1u : 0u);
                    }
                    ptx::tc_commit_pair_both(&empty_bar[stage]);
                    if (++stage == nst) { stage = 0; phase ^= 1u; }
                }
                for (int q = lr.q0; q < (ok ? lr.q1 : lr.q0); ++q) {
                    const LoraSeg sg = mtile_seg(p, lr, q);
                    for (int kb = 0; kb * kBlockK < sg.rp16; ++kb) {
                        const int R = min(kBlockK, sg.rp16 - kb * kBlockK);
                        if (!ptx::mbar_wait(&full_bar[stage], phase, abort_flag, lim, p.err_flag)) { ok = false; break; }
                        ptx::tc_fence_after();
                        const uint32_t sA = ptx::smem_u32(smem + stage * stb);
                        const uint32_t sB = sA + kABytes;
                        for (int ks = 0; ks < R / 16; ++ks) {
                            const uint64_t bdesc = kBmn ? ptx::smem_desc_sw128(sB + ks * 2048, (uint32_t)R * 128u, 1024)
                                                        : ptx::smem_desc_sw128(sB + ks * 32, 16, 1024);
                            ptx::tc_mma_f16_pair(d_tmem, ptx::smem_desc_sw128(sA + ks * 32, 16, 1024), bdesc,
                                                 idesc_lr, 1u);
                        }
                        ptx::tc_commit_pair_both(&empty_bar[stage]);
                        if (++stage == nst) { stage = 0; phase ^= 1u; }
                    }
                    if (!ok) break;
                }
                if (!ok) break;
                ptx::tc_commit_pair_both(&accf_bar[abuf]);
                if (++abuf == 2) { abuf = 0; aphase ^= 1u; }
            }
            ptx::tc_commit_pair_both(drain_bar);
            int dummy = 0;
            ptx::mbar_wait(drain_bar, 0, &dummy, lim, p.err_flag);
        }
    } else {
        // ------------------------------------------------------------ epilogue (warps 2..5, both CTAs)
        const int q = warp & 3;
        uint8_t* wbuf = smem + kEpiOffset + q * kEpiWarpBytes;
        int abuf = 0;
        uint32_t aphase = 0;
        uint32_t epi_seq = 0;    // this warp's output chunks so far (staging buffer = epi_seq & 1)
        for (int t = pair; t < p.num_tiles; t += npairs) {
            int mb, nb;
            tile_mn(t, mb, nb);
            if (!ptx::mbar_wait(&accf_bar[abuf], aphase, abort_flag, lim, p.err_flag)) break;
            ptx::tc_fence_after();
            const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(abuf * kTileN);
            const int out_row = mb * kPairTileM + (int)crank * kTileM;
            epilogue_store_tma(&tmC, t_row, wbuf, lane, out_row + q * 32, nb * kTileN, p.M_total, p.N_total, epi_seq);
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_cluster(&acce_bar[abuf], 0);
            if (++abuf == 2) { abuf = 0; aphase ^= 1u; }
        }
        if (lane == 0) ptx::bulk_wait<0>();   // every output store performed before the CTA exits
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();   // no CTA leaves while the other may still signal its barriers
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc_pair<kTmemCols>(tmem_base);
}

}  // namespace plora
