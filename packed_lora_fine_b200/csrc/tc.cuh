// tc.cuh -- the tensor-core (tcgen05 + TMEM + TMA) kernels of the bf16 path.
//
// One persistent, warp-specialised kernel template covers every product of
// the packed LoRA forward and backward (the "four cases" of PLoRA's packed
// operators -- forward, input gradient, and the two weight gradients that
// reduce over the sequence -- plus the shared frozen-base GEMMs; PLoRA
// summary, gist.science, arXiv 2508.02932, 技术摘要 › 方法论 › 2 › 算子设计):
//
//   op         computes                                 A operand (smem)        B operand (smem)
//   BaseFwd    Y  = X W            (all tokens)          X      K-major          W_store    K-major
//   BaseDx     dX = dY W^T         (all tokens)          dY     K-major          W_store    MN-major
//   ShrinkX    H_i = X_i A_i       (per 128-token tile)   X      K-major          A pack     K-major
//   ShrinkDy   G_i = s_i dY_i B_i^T                       dY     K-major          B^T pack   K-major
//   ExpandY    Y_i += s_i H_i B_i                         H      K-major          B^T pack   MN-major
//              (by default folded into BaseFwd instead: B row-padded pack, K-major)
//   ExpandDx   dX_i += G_i A_i^T                          G      K-major          A pack     MN-major
//   WgradB     dB_i = s_i dY_i^T H_i (sum over tokens)    dY     MN-major         H          MN-major
//   WgradA     dA_i = X_i^T G_i      (sum over tokens)    X      MN-major         G          MN-major
//
// Tiles run along the token (sequence) dimension for the shrink/expand
// products and along the hidden dimension for the weight gradients -- never
// along the small rank dimension; the rank is only the MMA's N (shrink) or K
// (expand) extent, padded to 16.  Every tile of every adapter is one work
// item of a static persistent schedule over all SMs, so adapters of unequal
// rank and token count share one launch (the load balancing of 算子设计).
//
// Warp roles (192 threads): warp 0 issues TMA loads into a 4-stage ring,
// warp 1 owns TMEM and issues tcgen05.mma into one of two 128x256 fp32
// accumulators, warps 2-5 drain an accumulator (tcgen05.ld) and run the
// op's epilogue while the next tile is being multiplied.
//
// A launch may carry a second, independent op (tc_kernel<OP, OP2>): its work
// items follow OP's in the same persistent grid (the backward runs dB's items
// after G's, filling the last wave of G's equal-cost token tiles).
//
// Output blocks: W may stack P projections that read the same X (q|k|v).  Each
// adapter then has one rank-r pair per block; H' and G hold block b in columns
// [b rblk, b rblk + r).  Y's folded product and dB read only their block's
// columns; G (through a block-diagonal B^T pack) and the folded dX product
// span all of them.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include "plan.cuh"
#include "ptx.cuh"

namespace plora {

enum class Op : int { BaseFwd = 0, BaseDx, ShrinkX, ShrinkDy, ExpandY, ExpandDx, WgradB, WgradA };

template <Op OP> struct OpTraits {
    static constexpr bool kAmn = (OP == Op::WgradB || OP == Op::WgradA);
    static constexpr bool kBmn = (OP == Op::BaseDx || OP == Op::ExpandY || OP == Op::ExpandDx ||
                                  OP == Op::WgradB || OP == Op::WgradA);
    static constexpr bool kBase = (OP == Op::BaseFwd || OP == Op::BaseDx);
    static constexpr bool kShrink = (OP == Op::ShrinkX || OP == Op::ShrinkDy);
    static constexpr bool kExpand = (OP == Op::ExpandY || OP == Op::ExpandDx);
    static constexpr bool kWgrad = (OP == Op::WgradB || OP == Op::WgradA);
};

constexpr int kStages = 4;                        // stages of the largest (48 KB) layout
constexpr int kMaxStages = 8;                     // ring slots when the op's stages are smaller
constexpr int kTileN = 256;                       // N of the base / expand tiles (TMEM columns)
constexpr int kABytes = kTileM * kBlockK * 2;     // 16 KB: 128 rows x 64 bf16
constexpr int kBBytesMax = kTileN * kBlockK * 2;  // 32 KB: 256 rows x 64 bf16
constexpr int kStageBytes = kABytes + kBBytesMax;
constexpr int kTmemCols = 512;                    // two 256-column fp32 accumulators
constexpr int kTcThreads = 192;
constexpr int kRingBytes = kStages * kStageBytes; // 192 KB of operand ring
constexpr int kEpiStageFloats = 32 * 33;          // per epilogue warp: a 32 x 32 fp32 chunk (padded rows)
constexpr int kTcSmemBytes = kRingBytes + 1024 /* align */ + 256 /* barriers */ + 4 * kEpiStageFloats * 4;

struct TcParams {
    int32_t M_total;        // Base: T; Wgrad: d (rows of dB_i or columns of dA_i)
    int32_t N_total;        // Base / Expand: output columns
    int32_t K_total;        // Base / Shrink: reduction length
    int32_t tiles_m, tiles_n, num_tiles;
    int32_t group_m;        // Base: rasterisation group (m tiles sharing an L2 window)
    int32_t RP;             // padded rank pitch of H / G / packs
    int32_t b_box_rows;     // K-major B: rows of the B box (Base: 256, Shrink: RP)
    int32_t red_dtiles;     // Wgrad: 128-row tiles along d
    const AdapterDev* adapters;
    const TokTile* tok;
    const RedEntry* red;
    void* out;              // bf16 output of Base / Shrink / Expand
    int64_t out_ld;         // its row pitch in elements
    float* partials;        // Wgrad split partials, [slot][dtile][128][RP]
    int32_t* counters;      // Wgrad split arrival counters
    int* err_flag;
    uint64_t timeout_ns;
    // Base ops with the low-rank branch folded in (fuse != 0): for global m-tile mb, the
    // adapters overlapping its 128 rows are mt_seg[mt_rec[mb].q0 .. mt_rec[mb].q1).
    const MTileRec* mt_rec;
    const LoraSeg* mt_seg;
    int32_t fuse;
    int32_t stages;         // operand ring depth (<= kMaxStages)
    int32_t stage_bytes;    // bytes per ring stage: A tile + this op's largest B tile
    // Output blocks (shared-input projections stacked along d_out): block b holds the output
    // columns [blk_end[b-1], blk_end[b]); nblk = 1 for a single projection.
    int32_t nblk;
    int32_t blk_end[kMaxOutBlocks];
};

// The output block holding output column `col`.
__device__ __forceinline__ int out_block(const TcParams& p, int col) {
    int b = 0;
    while (b + 1 < p.nblk && col >= p.blk_end[b]) ++b;
    return b;
}

struct TileInfo {
    int32_t a_x, a_y, b_x, b_y;
    int32_t kblocks, last_ksteps, mma_n, nb_boxes;
    int32_t adapter, out_row, rows_valid, n0, cols_valid, red_idx;
    int32_t mtile;
    float scale;
};

template <Op OP>
__device__ __forceinline__ TileInfo decode_tile(const TcParams& p, int t) {
    using Tr = OpTraits<OP>;
    TileInfo ti;
    ti.last_ksteps = 4;
    ti.nb_boxes = 1;
    ti.scale = 1.f;
    ti.adapter = -1;
    ti.red_idx = -1;
    if constexpr (Tr::kBase) {
        // Grouped rasterisation: group_m m-tiles walk all n-tiles together.
        const int per_group = p.group_m * p.tiles_n;
        const int g = t / per_group;
        const int first_m = g * p.group_m;
        const int gm = min(p.tiles_m - first_m, p.group_m);
        const int r = t - g * per_group;
        const int mb = first_m + r % gm;
        const int nb = r / gm;
        ti.mtile = mb;
        ti.a_x = 0;
        ti.a_y = mb * kTileM;
        if constexpr (OP == Op::BaseFwd) { ti.b_x = 0; ti.b_y = nb * kTileN; }
        else { ti.b_x = nb * kTileN; ti.b_y = 0; ti.nb_boxes = kTileN / 64; }
        ti.kblocks = (p.K_total + kBlockK - 1) / kBlockK;
        ti.mma_n = kTileN;
        ti.out_row = mb * kTileM;
        ti.rows_valid = min(kTileM, p.M_total - ti.out_row);
        ti.n0 = nb * kTileN;
        ti.cols_valid = min(kTileN, p.N_total - ti.n0);
    } else if constexpr (Tr::kShrink) {
        const TokTile tt = p.tok[t];
        const AdapterDev ad = p.adapters[tt.adapter];
        ti.adapter = tt.adapter;
        ti.a_x = 0;
        ti.a_y = tt.x_row;
        ti.b_x = 0;
        ti.b_y = tt.adapter * p.RP;
        ti.kblocks = (p.K_total + kBlockK - 1) / kBlockK;
        ti.mma_n = ad.rp16;
        ti.out_row = tt.h_row;
        ti.rows_valid = tt.rows;
        ti.n0 = 0;
        ti.cols_valid = p.RP;
        ti.scale = ad.scale;   // H' = s X A and G = s dY B^T carry the adapter's scale
    } else if constexpr (Tr::kExpand) {
        const int mt = t / p.tiles_n;
        const int nb = t - mt * p.tiles_n;
        const TokTile tt = p.tok[mt];
        const AdapterDev ad = p.adapters[tt.adapter];
        ti.adapter = tt.adapter;
        ti.a_x = 0;
        ti.a_y = tt.h_row;
        ti.b_x = nb * kTileN;
        ti.b_y = tt.adapter * p.RP;
        ti.nb_boxes = kTileN / 64;
        const int ksteps = ad.rp16 / 16;
        ti.kblocks = (ksteps + 3) / 4;
        ti.last_ksteps = ksteps - (ti.kblocks - 1) * 4;
        ti.mma_n = kTileN;
        ti.out_row = tt.x_row;
        ti.rows_valid = tt.rows;
        ti.n0 = nb * kTileN;
        ti.cols_valid = min(kTileN, p.N_total - ti.n0);
        ti.scale = 1.f;        // H' and G already carry the scale
    } else {
        const int e = t / p.red_dtiles;
        const int db = t - e * p.red_dtiles;
        const RedEntry re = p.red[e];
        const AdapterDev ad = p.adapters[re.adapter];
        ti.adapter = re.adapter;
        ti.red_idx = e;
        ti.a_x = db * kTileM;
        ti.a_y = re.x_row;
        ti.b_y = re.h_row;
        if constexpr (OP == Op::WgradB) {
            // dB rows of output block b pair with block b's columns of H' only
            ti.b_x = out_block(p, db * kTileM) * ad.rblk;
            ti.mma_n = (ad.rblk + 63) / 64 * 64;
        } else {
            ti.b_x = 0;
            ti.mma_n = ad.rp64;
        }
        ti.nb_boxes = ti.mma_n / 64;
        ti.kblocks = re.kblocks;
        ti.out_row = db * kTileM;
        ti.rows_valid = min(kTileM, p.M_total - ti.out_row);
        ti.n0 = db;  // the d-tile index (for partial slots)
        ti.cols_valid = ad.rank;
        ti.scale = 1.f;        // H' and G already carry the scale
    }
    return ti;
}

// The folded low-rank record of base tile t (empty when not folding or past the end).
template <Op OP>
__device__ __forceinline__ MTileRec load_mtile(const TcParams& p, int t) {
    MTileRec r;
    r.q0 = r.q1 = 0;
    if (OpTraits<OP>::kBase && p.fuse && t < p.num_tiles) {
        const TileInfo ti = decode_tile<OP>(p, t);
        r = p.mt_rec[ti.mtile / (kLoraTileM / kTileM)];
        // a 128-row tile reads its half of the 256-row record's rows
        const int shift = (ti.mtile % (kLoraTileM / kTileM)) * kTileM;
        r.s[0].h_y += shift;
        r.s[1].h_y += shift;
        r.pad_[0] = shift;
    }
    return r;
}
__device__ __forceinline__ LoraSeg mtile_seg(const TcParams& p, const MTileRec& r, int q) {
    if (q - r.q0 < 2) return r.s[q - r.q0];
    LoraSeg s = p.mt_seg[q];
    s.h_y += r.pad_[0];
    return s;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 unpack_bf16x2(uint32_t u) {
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
    return __bfloat1622float2(v);
}

// Operand-ring position of one role thread, carried across the work items of a launch.
struct RingPos {
    int stage;
    uint32_t phase;
    __device__ __forceinline__ void advance(int nst) {
        if (++stage == nst) { stage = 0; phase ^= 1u; }
    }
};

// Producer (one thread): TMA loads of every k-block of work item ti into the ring.  Returns
// false when a wait ran out of time (the error flag is then set).
template <Op OP>
__device__ __forceinline__ bool produce_item(const TcParams& p, const TileInfo& ti, const MTileRec& lr,
                                             const CUtensorMap* tmA, const CUtensorMap* tmB,
                                             const CUtensorMap* tmA2, const CUtensorMap* tmB2, uint8_t* smem,
                                             int stb, int nst, uint64_t* full_bar, uint64_t* empty_bar,
                                             RingPos& rp, uint32_t& armed, uint32_t& armed_par,
                                             volatile int* abort_flag, uint64_t lim) {
    using Tr = OpTraits<OP>;
    const uint32_t b_bytes = Tr::kBmn ? (uint32_t)ti.nb_boxes * 8192u : (uint32_t)p.b_box_rows * 128u;
    for (int kb = 0; kb < ti.kblocks; ++kb) {
        if (!ptx::mbar_wait(&empty_bar[rp.stage], rp.phase ^ 1u, abort_flag, lim, p.err_flag)) return false;
        uint8_t* sA = smem + rp.stage * stb;
        uint8_t* sB = sA + kABytes;
        ptx::mbar_arrive_expect_tx(&full_bar[rp.stage], (uint32_t)kABytes + b_bytes);
        armed |= 1u << rp.stage;
        armed_par = (armed_par & ~(1u << rp.stage)) | (rp.phase << rp.stage);
        if constexpr (Tr::kAmn) {
            ptx::tma_load_2d(sA, tmA, &full_bar[rp.stage], ti.a_x, ti.a_y + kb * kBlockK);
            ptx::tma_load_2d(sA + 8192, tmA, &full_bar[rp.stage], ti.a_x + 64, ti.a_y + kb * kBlockK);
        } else {
            ptx::tma_load_2d(sA, tmA, &full_bar[rp.stage], ti.a_x + kb * kBlockK, ti.a_y);
        }
        if constexpr (Tr::kBmn) {
            for (int h = 0; h < ti.nb_boxes; ++h)
                ptx::tma_load_2d(sB + h * 8192, tmB, &full_bar[rp.stage], ti.b_x + 64 * h, ti.b_y + kb * kBlockK);
        } else {
            ptx::tma_load_2d(sB, tmB, &full_bar[rp.stage], ti.b_x + kb * kBlockK, ti.b_y);
        }
        rp.advance(nst);
    }
    if constexpr (Tr::kBase) {
        // Low-rank branch folded into the same accumulator: for every adapter j whose
        // tokens overlap this m-tile, K-steps over its rank with A = its H' (or G) rows,
        // read at the tile's row offset inside j's zero-padded block (rows outside j's
        // segment load as zeros).  B has the base B's major-ness: for Y, rows n0.. of
        // j's row-padded B (K-major, one 256 x 64 box); for dX, j's packed A
        // (MN-major, 16-row boxes so that only the rank's rows are staged).  With output
        // blocks, Y's tile reads only its block's columns of H' (K = rblk from b rblk); dX's
        // sums over every block (K = P rblk).
        for (int q = lr.q0; q < lr.q1; ++q) {
            const LoraSeg sg = mtile_seg(p, lr, q);
            const int kext = Tr::kBmn ? sg.rp16 : sg.rblk;
            const int hx0 = Tr::kBmn ? 0 : out_block(p, ti.n0) * sg.rblk;
            for (int kb = 0; kb * kBlockK < kext; ++kb) {
                const int R = min(kBlockK, kext - kb * kBlockK);
                if (!ptx::mbar_wait(&empty_bar[rp.stage], rp.phase ^ 1u, abort_flag, lim, p.err_flag)) return false;
                uint8_t* sA = smem + rp.stage * stb;
                uint8_t* sB = sA + kABytes;
                const uint32_t lb_bytes = Tr::kBmn ? 4u * (uint32_t)R * 128u : (uint32_t)kTileN * 128u;
                ptx::mbar_arrive_expect_tx(&full_bar[rp.stage], (uint32_t)kABytes + lb_bytes);
                armed |= 1u << rp.stage;
                armed_par = (armed_par & ~(1u << rp.stage)) | (rp.phase << rp.stage);
                ptx::tma_load_2d(sA, tmA2, &full_bar[rp.stage], hx0 + kb * kBlockK, sg.h_y);
                if constexpr (Tr::kBmn) {
                    for (int h = 0; h < 4; ++h)
                        for (int r16 = 0; r16 < R; r16 += 16)
                            ptx::tma_load_2d(sB + h * R * 128 + r16 * 128, tmB2, &full_bar[rp.stage],
                                             ti.n0 + 64 * h, sg.adapter * p.RP + kb * kBlockK + r16);
                } else {
                    ptx::tma_load_2d(sB, tmB2, &full_bar[rp.stage], kb * kBlockK, sg.adapter * p.N_total + ti.n0);
                }
                rp.advance(nst);
            }
        }
    }
    return true;
}

// MMA issuer (one thread): the tcgen05.mma of every k-block of work item ti into the
// accumulator at d_tmem, releasing each ring stage as its MMAs complete.
template <Op OP>
__device__ __forceinline__ bool mma_item(const TcParams& p, const TileInfo& ti, const MTileRec& lr, uint8_t* smem,
                                         int stb, int nst, uint64_t* full_bar, uint64_t* empty_bar,
                                         uint32_t d_tmem, RingPos& rp, volatile int* abort_flag, uint64_t lim) {
    using Tr = OpTraits<OP>;
    const uint32_t idesc = ptx::idesc_bf16_f32(kTileM, ti.mma_n, Tr::kAmn, Tr::kBmn);
    for (int kb = 0; kb < ti.kblocks; ++kb) {
        if (!ptx::mbar_wait(&full_bar[rp.stage], rp.phase, abort_flag, lim, p.err_flag)) return false;
        ptx::tc_fence_after();
        const uint32_t sA = ptx::smem_u32(smem + rp.stage * stb);
        const uint32_t sB = sA + kABytes;
        const int steps = (kb == ti.kblocks - 1) ? ti.last_ksteps : 4;
        for (int ks = 0; ks < steps; ++ks) {
            const uint64_t adesc = Tr::kAmn ? ptx::smem_desc_sw128(sA + ks * 2048, 8192, 1024)
                                            : ptx::smem_desc_sw128(sA + ks * 32, 16, 1024);
            const uint64_t bdesc = Tr::kBmn ? ptx::smem_desc_sw128(sB + ks * 2048, 8192, 1024)
                                            : ptx::smem_desc_sw128(sB + ks * 32, 16, 1024);
            ptx::tc_mma_f16(d_tmem, adesc, bdesc, idesc, (kb | ks) ? 1u : 0u);
        }
        ptx::tc_commit(&empty_bar[rp.stage]);
        rp.advance(nst);
    }
    if constexpr (Tr::kBase) {
        const uint32_t idesc_lr = ptx::idesc_bf16_f32(kTileM, kTileN, false, Tr::kBmn);
        for (int q = lr.q0; q < lr.q1; ++q) {
            const LoraSeg sg = mtile_seg(p, lr, q);
            const int kext = Tr::kBmn ? sg.rp16 : sg.rblk;   // as the producer staged it
            for (int kb = 0; kb * kBlockK < kext; ++kb) {
                const int R = min(kBlockK, kext - kb * kBlockK);
                if (!ptx::mbar_wait(&full_bar[rp.stage], rp.phase, abort_flag, lim, p.err_flag)) return false;
                ptx::tc_fence_after();
                const uint32_t sA = ptx::smem_u32(smem + rp.stage * stb);
                const uint32_t sB = sA + kABytes;
                for (int ks = 0; ks < R / 16; ++ks) {
                    const uint64_t bdesc = Tr::kBmn ? ptx::smem_desc_sw128(sB + ks * 2048, (uint32_t)R * 128u, 1024)
                                                    : ptx::smem_desc_sw128(sB + ks * 32, 16, 1024);
                    ptx::tc_mma_f16(d_tmem, ptx::smem_desc_sw128(sA + ks * 32, 16, 1024), bdesc, idesc_lr, 1u);
                }
                ptx::tc_commit(&empty_bar[rp.stage]);
                rp.advance(nst);
            }
        }
    }
    return true;
}

// Epilogue (warps 2..5, one accumulator row per thread): drains work item ti's accumulator
// rows from TMEM at t_row and runs the op's output step.
template <Op OP>
__device__ __forceinline__ void epilogue_item(const TcParams& p, const TileInfo& ti, uint32_t t_row, int q, int lane,
                                              float* epi_stage, int* red_flag) {
    using Tr = OpTraits<OP>;
    const int row = q * 32 + lane;          // accumulator row handled by this thread
    const bool row_ok = row < ti.rows_valid;
    if constexpr (Tr::kBase) {
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + (int64_t)(ti.out_row + row) * p.out_ld + ti.n0;
        for (int c = 0; c < kTileN; c += 16) {
            uint32_t r[16];
            ptx::tmem_ld16(t_row + c, r);
            ptx::tmem_ld_wait();
            if (row_ok) {
                uint4 v0, v1;
                v0.x = pack_bf16x2(__uint_as_float(r[0]), __uint_as_float(r[1]));
                v0.y = pack_bf16x2(__uint_as_float(r[2]), __uint_as_float(r[3]));
                v0.z = pack_bf16x2(__uint_as_float(r[4]), __uint_as_float(r[5]));
                v0.w = pack_bf16x2(__uint_as_float(r[6]), __uint_as_float(r[7]));
                v1.x = pack_bf16x2(__uint_as_float(r[8]), __uint_as_float(r[9]));
                v1.y = pack_bf16x2(__uint_as_float(r[10]), __uint_as_float(r[11]));
                v1.z = pack_bf16x2(__uint_as_float(r[12]), __uint_as_float(r[13]));
                v1.w = pack_bf16x2(__uint_as_float(r[14]), __uint_as_float(r[15]));
                if (c + 8 <= ti.cols_valid) *reinterpret_cast<uint4*>(out + c) = v0;
                if (c + 16 <= ti.cols_valid) *reinterpret_cast<uint4*>(out + c + 8) = v1;
            }
        }
    } else if constexpr (Tr::kShrink) {
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + (int64_t)(ti.out_row + row) * p.out_ld;
        for (int c = 0; c < ti.cols_valid; c += 16) {
            uint4 v0 = make_uint4(0, 0, 0, 0), v1 = make_uint4(0, 0, 0, 0);
            if (c < ti.mma_n) {
                uint32_t r[16];
                ptx::tmem_ld16(t_row + c, r);
                ptx::tmem_ld_wait();
                if (row_ok) {
                    const float s = ti.scale;
                    v0.x = pack_bf16x2(s * __uint_as_float(r[0]), s * __uint_as_float(r[1]));
                    v0.y = pack_bf16x2(s * __uint_as_float(r[2]), s * __uint_as_float(r[3]));
                    v0.z = pack_bf16x2(s * __uint_as_float(r[4]), s * __uint_as_float(r[5]));
                    v0.w = pack_bf16x2(s * __uint_as_float(r[6]), s * __uint_as_float(r[7]));
                    v1.x = pack_bf16x2(s * __uint_as_float(r[8]), s * __uint_as_float(r[9]));
                    v1.y = pack_bf16x2(s * __uint_as_float(r[10]), s * __uint_as_float(r[11]));
                    v1.z = pack_bf16x2(s * __uint_as_float(r[12]), s * __uint_as_float(r[13]));
                    v1.w = pack_bf16x2(s * __uint_as_float(r[14]), s * __uint_as_float(r[15]));
                }
            }
            *reinterpret_cast<uint4*>(out + c) = v0;
            *reinterpret_cast<uint4*>(out + c + 8) = v1;
        }
        // The adapter's block has kLoraPad zero rows before and after its (128-rounded) rows, so that
        // a base tile straddling the segment can read it at any row offset; the first and the last
        // tile of the adapter write them.
        const AdapterDev ad = p.adapters[ti.adapter];
        const bool first = ti.out_row == ad.h_row;
        const bool last = ti.out_row + kTileM >= ad.h_row + ad.n;
        if (first || last) {
            const uint4 z = make_uint4(0, 0, 0, 0);
            __nv_bfloat16* base = static_cast<__nv_bfloat16*>(p.out);
            const int tail = ad.h_row + ((ad.n + kTileM - 1) / kTileM) * kTileM;
            for (int pr = row; pr < kLoraPad; pr += kTileM) {
                if (first) {
                    uint4* dst = reinterpret_cast<uint4*>(base + (int64_t)(ad.h_row - kLoraPad + pr) * p.out_ld);
                    for (int c = 0; c < p.RP / 8; ++c) dst[c] = z;
                }
                if (last) {
                    uint4* dst = reinterpret_cast<uint4*>(base + (int64_t)(tail + pr) * p.out_ld);
                    for (int c = 0; c < p.RP / 8; ++c) dst[c] = z;
                }
            }
        }
    } else if constexpr (Tr::kExpand) {
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + (int64_t)(ti.out_row + row) * p.out_ld + ti.n0;
        const float s = ti.scale;
        for (int h = 0; h < kTileN; h += 128) {
            uint4 y[16];
            if (row_ok) {
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    if (h + 8 * u + 8 <= ti.cols_valid) y[u] = *reinterpret_cast<const uint4*>(out + h + 8 * u);
            }
#pragma unroll
            for (int u = 0; u < 16; u += 2) {
                uint32_t r[16];
                ptx::tmem_ld16(t_row + h + 8 * u, r);
                ptx::tmem_ld_wait();
                if (row_ok) {
#pragma unroll
                    for (int w = 0; w < 2; ++w) {
                        if (h + 8 * (u + w) + 8 > ti.cols_valid) continue;
                        uint4 o = y[u + w];
                        uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            float2 f = unpack_bf16x2(ow[e]);
                            f.x += s * __uint_as_float(r[8 * w + 2 * e]);
                            f.y += s * __uint_as_float(r[8 * w + 2 * e + 1]);
                            ow[e] = pack_bf16x2(f.x, f.y);
                        }
                        *reinterpret_cast<uint4*>(out + h + 8 * (u + w)) = o;
                    }
                }
            }
        }
    } else {
        // Weight gradients: row = hidden index (d_out for dB, d_in for dA), column = rank index.
        const RedEntry re = p.red[ti.red_idx];
        const AdapterDev ad = p.adapters[ti.adapter];
        const int rank = ad.rank;
        const int hid = ti.out_row + row;
        const float s = ti.scale;
        if (re.nsplit == 1 && OP == Op::WgradB) {
            // dB_i's 128-row tile is one contiguous block ([row][rank]); stage 32 x 32 chunks of
            // this warp's rows in shared memory and store them with consecutive lanes on
            // consecutive addresses.
            float* stg = epi_stage + q * kEpiStageFloats;
            const int row0 = ti.out_row + q * 32;                 // first hidden row of this warp
            const int nrows = min(32, p.M_total - row0);
            float* blk = ad.dB + (int64_t)row0 * rank;
            for (int c0 = 0; c0 < ti.mma_n && c0 < rank; c0 += 32) {
                uint32_t r[16];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    ptx::tmem_ld16(t_row + c0 + 16 * hh, r);
                    ptx::tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 16; ++e) stg[lane * 33 + 16 * hh + e] = s * __uint_as_float(r[e]);
                }
                __syncwarp();
                const int ncols = min(32, rank - c0);
                if (rank <= 32) {
                    // the whole [nrows][rank] block is contiguous: linear stores
                    for (int idx = lane; idx < nrows * rank; idx += 32) {
                        const int rr = idx / rank, cc = idx - rr * rank;
                        blk[idx] = stg[rr * 33 + cc];
                    }
                } else {
                    for (int rr = 0; rr < nrows; ++rr)
                        if (lane < ncols) blk[(int64_t)rr * rank + c0 + lane] = stg[rr * 33 + lane];
                }
                __syncwarp();
            }
        } else if (re.nsplit == 1) {
            for (int c = 0; c < ti.mma_n; c += 16) {
                uint32_t r[16];
                ptx::tmem_ld16(t_row + c, r);
                ptx::tmem_ld_wait();
                if (row_ok) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        // column k of X^T G is block pb's rank row kk (rows pb rank + kk of dA)
                        const int k = c + e;
                        const int pb = k / ad.rblk, kk = k - pb * ad.rblk;
                        if (pb < p.nblk && kk < rank)
                            ad.dA[(int64_t)(pb * rank + kk) * p.M_total + hid] = s * __uint_as_float(r[e]);
                    }
                }
            }
        } else {
            // Split along the tokens: write this split's partial, the last split of the
            // tile to arrive sums all partials in split order (deterministic) and stores.
            const int64_t slot_elems = (int64_t)kTileM * p.RP;
            // accumulator columns that reach an output: dB's rank, or every block's columns of dA
            const int ncols = (OP == Op::WgradB || p.nblk == 1) ? rank : ad.rp16;
            // partial layout [slot][d-tile][rank column][128 rows]: a warp's lanes touch
            // consecutive rows, so both the writes here and the reduction below coalesce.
            float* mine = p.partials + ((int64_t)(re.slot + re.split) * p.red_dtiles + ti.n0) * slot_elems + row;
            for (int c = 0; c < ti.mma_n; c += 16) {
                uint32_t r[16];
                ptx::tmem_ld16(t_row + c, r);
                ptx::tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    if (c + e < ncols) mine[(int64_t)(c + e) * kTileM] = __uint_as_float(r[e]);
            }
            __threadfence();
            ptx::named_bar_sync(1, 128);
            if (threadIdx.x == 64) {
                const int old = atomicAdd(&p.counters[re.counter + ti.n0], 1);
                *red_flag = (old == re.nsplit - 1) ? 1 : 0;
            }
            ptx::named_bar_sync(1, 128);
            if (*red_flag) {
                __threadfence();
                if (row_ok) {
                    const float* first = p.partials + ((int64_t)re.slot * p.red_dtiles + ti.n0) * slot_elems + row;
                    const int64_t split_stride = (int64_t)p.red_dtiles * slot_elems;
                    for (int k0 = 0; k0 < ncols; k0 += 8) {
                        // 8 ranks at a time: all of a split's loads are in flight together,
                        // the sum still runs over the splits in order.
                        float acc[8];
#pragma unroll
                        for (int u = 0; u < 8; ++u) acc[u] = 0.f;
                        for (int sp = 0; sp < re.nsplit; ++sp) {
                            float v[8];
#pragma unroll
                            for (int u = 0; u < 8; ++u)
                                v[u] = (k0 + u < ncols) ? __ldcg(first + sp * split_stride + (int64_t)(k0 + u) * kTileM) : 0.f;
#pragma unroll
                            for (int u = 0; u < 8; ++u) acc[u] += v[u];
                        }
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const int k = k0 + u;
                            if constexpr (OP == Op::WgradB) {
                                if (k < rank) ad.dB[(int64_t)hid * rank + k] = s * acc[u];
                            } else {
                                const int pb = k / ad.rblk, kk = k - pb * ad.rblk;
                                if (pb < p.nblk && kk < rank)
                                    ad.dA[(int64_t)(pb * rank + kk) * p.M_total + hid] = s * acc[u];
                            }
                        }
                    }
                }
                if (threadIdx.x == 64) p.counters[re.counter + ti.n0] = 0;
            }
            ptx::named_bar_sync(1, 128);
        }
    }
}

// One persistent launch runs the work items of OP (p.num_tiles of them) followed, when OP2
// differs from OP, by those of OP2 (p2.num_tiles, with operands from tmA2 / tmB2).  Both ops
// use the ring layout of p (stages, stage_bytes).  Items are dealt round-robin over the CTAs,
// so the second op's items fill the last, partial wave of the first op's.
template <Op OP, Op OP2 = OP>
__global__ void __launch_bounds__(kTcThreads, 1)
tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
          const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2, const TcParams p,
          const TcParams p2) {
    using Tr = OpTraits<OP>;
    constexpr bool kDual = OP2 != OP;
    static_assert(!kDual || (!Tr::kBase && !OpTraits<OP2>::kBase),
                  "a base GEMM reads its low-rank branch through tmA2 / tmB2");
    const int total = p.num_tiles + (kDual ? p2.num_tiles : 0);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kRingBytes);
    uint64_t* full_bar = bars;                       // [kMaxStages]
    uint64_t* empty_bar = bars + kMaxStages;         // [kMaxStages]
    uint64_t* accf_bar = bars + 2 * kMaxStages;      // [2]
    uint64_t* acce_bar = bars + 2 * kMaxStages + 2;  // [2]
    uint64_t* drain_bar = bars + 2 * kMaxStages + 4;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kMaxStages + 5);
    const int nst = p.stages;                        // ring depth of this launch
    const int stb = p.stage_bytes;                   // bytes per stage (multiple of 1024)
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* red_flag = reinterpret_cast<int*>(tmem_slot + 2);
    float* epi_stage = reinterpret_cast<float*>(smem + kRingBytes + 256);   // [4 warps][32][33]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; ++s) {
            ptx::mbar_init(&full_bar[s], 1);
            ptx::mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&accf_bar[b], 1);
            ptx::mbar_init(&acce_bar[b], 4);
        }
        ptx::mbar_init(drain_bar, 1);
        *abort_flag = 0;
        ptx::fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::tma_prefetch_desc(&tmA);
        ptx::tma_prefetch_desc(&tmB);
        if ((Tr::kBase && p.fuse) || kDual) {
            ptx::tma_prefetch_desc(&tmA2);
            ptx::tma_prefetch_desc(&tmB2);
        }
    }
    if (warp == 1) {
        ptx::tmem_alloc<kTmemCols>(tmem_slot);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint64_t lim = p.timeout_ns;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            RingPos rp{0, 0u};
            uint32_t armed = 0, armed_par = 0;
            bool ok = true;
            // The folded low-rank record of a base tile is fetched one tile ahead.
            MTileRec lr_next = load_mtile<OP>(p, blockIdx.x);
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const MTileRec lr = lr_next;
                lr_next = load_mtile<OP>(p, t + gridDim.x);
                if (kDual && t >= p.num_tiles)
                    ok = produce_item<OP2>(p2, decode_tile<OP2>(p2, t - p.num_tiles), lr, &tmA2, &tmB2, &tmA2, &tmB2,
                                           smem, stb, nst, full_bar, empty_bar, rp, armed, armed_par, abort_flag, lim);
                else
                    ok = produce_item<OP>(p, decode_tile<OP>(p, t), lr, &tmA, &tmB, &tmA2, &tmB2, smem, stb, nst,
                                          full_bar, empty_bar, rp, armed, armed_par, abort_flag, lim);
            }
            // Drain: every load this thread issued must have landed before the CTA exits.
            for (int s = 0; s < nst; ++s)
                if (armed & (1u << s)) {
                    int dummy = 0;
                    ptx::mbar_wait(&full_bar[s], (armed_par >> s) & 1u, &dummy, lim, p.err_flag);
                }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            RingPos rp{0, 0u};
            int abuf = 0;
            uint32_t aphase = 0;
            MTileRec lr_next = load_mtile<OP>(p, blockIdx.x);
            for (int t = blockIdx.x; t < total; t += gridDim.x) {
                const MTileRec lr = lr_next;
                lr_next = load_mtile<OP>(p, t + gridDim.x);
                if (!ptx::mbar_wait(&acce_bar[abuf], aphase ^ 1u, abort_flag, lim, p.err_flag)) break;
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(abuf * kTileN);
                const bool ok = (kDual && t >= p.num_tiles)
                    ? mma_item<OP2>(p2, decode_tile<OP2>(p2, t - p.num_tiles), lr, smem, stb, nst, full_bar,
                                    empty_bar, d_tmem, rp, abort_flag, lim)
                    : mma_item<OP>(p, decode_tile<OP>(p, t), lr, smem, stb, nst, full_bar, empty_bar, d_tmem, rp,
                                   abort_flag, lim);
                if (!ok) break;
                ptx::tc_commit(&accf_bar[abuf]);
                if (++abuf == 2) { abuf = 0; aphase ^= 1u; }
            }
            // Drain: all issued MMAs complete before TMEM is released.
            ptx::tc_commit(drain_bar);
            int dummy = 0;
            ptx::mbar_wait(drain_bar, 0, &dummy, lim, p.err_flag);
        }
    } else {
        // ------------------------------------------------------------ epilogue (warps 2..5)
        const int q = warp & 3;                 // TMEM lane quarter this warp may access
        int abuf = 0;
        uint32_t aphase = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x) {
            if (!ptx::mbar_wait(&accf_bar[abuf], aphase, abort_flag, lim, p.err_flag)) break;
            ptx::tc_fence_after();
            const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(abuf * kTileN);
            if (kDual && t >= p.num_tiles)
                epilogue_item<OP2>(p2, decode_tile<OP2>(p2, t - p.num_tiles), t_row, q, lane, epi_stage, red_flag);
            else
                epilogue_item<OP>(p, decode_tile<OP>(p, t), t_row, q, lane, epi_stage, red_flag);
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&acce_bar[abuf]);
            if (++abuf == 2) { abuf = 0; aphase ^= 1u; }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc<kTmemCols>(tmem_base);
}

// ---------------------------------------------------------------------------
// Packing of the small per-adapter factors into the MMA-ready padded layouts.
//   packA [n*RP][d_in]:  row i*RP + b*rblk_i + k = A_i[b*r_i + k][:] (k < r_i), zero up to rblk_i
//   packBT[n*RP][d_out]: row i*RP + b*rblk_i + k = B_i[:][k] on block b's columns (k < r_i), else zero
// (b = output block, rblk_i = r_i rounded up to 16; one block: b = 0 and rblk_i = rp16_i).
// Rows rp16_i <= k < RP are never read by an MMA and are left unwritten.
// ---------------------------------------------------------------------------
__global__ void pack_a_kernel(const AdapterDev* __restrict__ ad, int n, int RP, int64_t d_in,
                              __nv_bfloat16* __restrict__ packA) {
    const int64_t vec_per_row = d_in / 8;
    const int64_t total = (int64_t)n * RP * vec_per_row;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t rowi = e / vec_per_row;
        const int64_t v = e - rowi * vec_per_row;
        const int i = (int)(rowi / RP);
        const int j = (int)(rowi - (int64_t)i * RP);
        if (j >= ad[i].rp16) continue;   // rows past the MMA extent are never read
        // row j is output block pb's rank row k (A_store row pb rank + k)
        const int pb = j / ad[i].rblk, k = j - pb * ad[i].rblk;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (k < ad[i].rank)
            val = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(ad[i].A) +
                                                 (int64_t)(pb * ad[i].rank + k) * d_in)[v];
        reinterpret_cast<uint4*>(packA + rowi * d_in)[v] = val;
    }
}

// Row-padded copy of every B for the fused forward (the expand's B operand, K-major like W):
// packB[(i d_out + c) RP + k] = B_i[c][k] for k < r_i, 0 for r_i <= k < rblk_i (r_i rounded up to
// 16); columns at or past rblk_i are never multiplied and stay unwritten.  grid.y = adapter; one thread per 16-byte
// chunk of the rp16_i columns, so consecutive threads read consecutive bytes of B_i.
__global__ void __launch_bounds__(256) pack_b_kernel(const AdapterDev* __restrict__ ad, int RP, int d_out,
                                                     __nv_bfloat16* __restrict__ packB) {
    const int i = blockIdx.y;
    const int r = ad[i].rank;
    const unsigned vc = (unsigned)ad[i].rblk / 8u;          // chunks per row
    const unsigned total = (unsigned)d_out * vc;
    const __nv_bfloat16* B = static_cast<const __nv_bfloat16*>(ad[i].B);
    __nv_bfloat16* dst = packB + (int64_t)i * d_out * RP;
    for (unsigned e = blockIdx.x * blockDim.x + threadIdx.x; e < total; e += gridDim.x * blockDim.x) {
        const unsigned c = e / vc;
        const int ch = (int)(e - c * vc);
        const __nv_bfloat16* src = B + (int64_t)c * r;
        uint4 val;
        if ((r & 7) == 0 && ch * 8 < r) {
            val = reinterpret_cast<const uint4*>(src)[ch];
        } else {
            __nv_bfloat16 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int k = ch * 8 + u;
                v[u] = k < r ? src[k] : __float2bfloat16_rn(0.f);
            }
            val = *reinterpret_cast<const uint4*>(v);
        }
        *reinterpret_cast<uint4*>(dst + (int64_t)c * RP + ch * 8) = val;
    }
}

// grid: (ceil(d_out/128), n); block 256.  Stages B_i[c0..c0+127][0..r) in shared memory (dynamic,
// 128 x (r + 2) bf16), then writes rows k < rp16 of packBT, 128 columns each.
__global__ void __launch_bounds__(256) pack_bt_kernel(const AdapterDev* __restrict__ ad, int RP, int64_t d_out,
                                                      OutBlocks blocks, __nv_bfloat16* __restrict__ packBT) {
    extern __shared__ __nv_bfloat16 tile[];
    const int i = blockIdx.y;
    const int64_t c0 = (int64_t)blockIdx.x * 128;
    const int r = ad[i].rank;
    const int ld = r + 2;
    const __nv_bfloat16* B = static_cast<const __nv_bfloat16*>(ad[i].B);
    const int cols = (int)(d_out - c0 < 128 ? d_out - c0 : 128);
    if ((r & 7) == 0) {
        // rows of B are 16-byte multiples: 16-byte loads, 8 ranks each
        const int vr = r >> 3;
        const uint4* src = reinterpret_cast<const uint4*>(B + c0 * r);
        for (int e = threadIdx.x; e < cols * vr; e += blockDim.x) {
            const int cc = e / vr, v = e - cc * vr;
            const uint4 q = src[e];
            const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&q);
#pragma unroll
            for (int u = 0; u < 8; ++u) tile[cc * ld + v * 8 + u] = h[u];
        }
    } else {
        for (int e = threadIdx.x; e < cols * r; e += blockDim.x) {
            const int cc = e / r, k = e - cc * r;
            tile[cc * ld + k] = B[(c0 + cc) * r + k];
        }
    }
    __syncthreads();
    // With output blocks the pack is block-diagonal: row pb rblk + k holds B's column k on block
    // pb's output columns and zeros elsewhere, so block pb of G sums over block pb's columns only.
    // A 128-column tile lies in one block (block ends are multiples of 256).
    int cb = 0;
    while (cb + 1 < blocks.n && c0 >= blocks.end[cb]) ++cb;
    const int rblk = ad[i].rblk;
    const int rows = ad[i].rp16;   // rows past the MMA extent are never read
    for (int e = threadIdx.x; e < rows * 64; e += blockDim.x) {
        const int j = e >> 6, cc = (e & 63) * 2;
        const int pb = j / rblk, k = j - pb * rblk;
        const bool live = pb == cb && k < r;
        if (cc < cols) {
            __nv_bfloat162 v;
            v.x = live ? tile[cc * ld + k] : __float2bfloat16_rn(0.f);
            v.y = live ? tile[(cc + 1) * ld + k] : __float2bfloat16_rn(0.f);
            *reinterpret_cast<__nv_bfloat162*>(packBT + ((int64_t)i * RP + j) * d_out + c0 + cc) = v;
        }
    }
}

}  // namespace plora
