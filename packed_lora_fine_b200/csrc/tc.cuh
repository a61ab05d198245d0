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
//   ShrinkDy   G_i = s_i dY_i B_i^T                       dY     K-major          B pack     MN-major
//   ExpandY    Y_i += s_i H_i B_i                         H      K-major          B pack     K-major
//              (by default folded into BaseFwd instead, with the same B pack)
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
// Warp roles (192 threads): warp 0 issues TMA loads into the operand ring,
// warp 1 owns TMEM and issues tcgen05.mma into one of two 128x256 fp32
// accumulators, warps 2-5 drain an accumulator (tcgen05.ld) and run the
// op's epilogue while the next tile is being multiplied.  A base-GEMM tile
// is 256 x 256: its two 128-row halves use both accumulators and share each
// k-block's B tile (see mma_wide for how the halves overlap the epilogue).
//
// A launch may carry a second, independent op (tc_kernel<OP, OP2>): its work
// items follow OP's in the same persistent grid, with operands from their own
// tensor maps (the backward runs dB's items after G's, filling the last wave of
// G's equal-cost token tiles, and dA's after the dX GEMM's tiles, filling its
// last, partial wave).
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

constexpr int kStages = 4;                        // stages of the 48 KB layout (128-row A, 256-row B)
constexpr int kMaxStages = 8;                     // ring slots when the op's stages are smaller
constexpr int kTileN = 256;                       // N of the base / expand tiles (TMEM columns)
constexpr int kABytes = kTileM * kBlockK * 2;     // 16 KB: 128 rows x 64 bf16
constexpr int kBBytesMax = kTileN * kBlockK * 2;  // 32 KB: 256 rows x 64 bf16
constexpr int kStageBytes = kABytes + kBBytesMax;
constexpr int kTmemCols = 512;                    // two 256-column fp32 accumulators
constexpr int kTcThreads = 192;
constexpr int kRingBytes = kStages * kStageBytes; // 192 KB of operand ring

// Rows of a base-GEMM tile.  256: two M = 128 accumulators share every k-block's 256 x 64 B tile, so a
// k-block stages 64 KB of operands for 8.4 MFLOP (64 bytes per clock at the full tensor rate, within
// what L2 delivers to an SM); the ring then holds three 64 KB stages.  128: one accumulator per tile,
// 48 KB for 4.2 MFLOP (96 bytes per clock).
#ifndef PLORA_BASE_TILE_ROWS
#define PLORA_BASE_TILE_ROWS 256
#endif
constexpr int kBaseRows = PLORA_BASE_TILE_ROWS;
static_assert(kBaseRows == 128 || kBaseRows == 256, "base tile rows");
constexpr int kWideStageBytes = 2 * kABytes + kBBytesMax;   // 64 KB
constexpr int kWideStages = kRingBytes / kWideStageBytes;   // 3

template <Op OP> struct OpTraits {
    static constexpr bool kAmn = (OP == Op::WgradB || OP == Op::WgradA);
    static constexpr bool kBmn = (OP == Op::BaseDx || OP == Op::ShrinkDy || OP == Op::ExpandDx ||
                                  OP == Op::WgradB || OP == Op::WgradA);
    static constexpr bool kBase = (OP == Op::BaseFwd || OP == Op::BaseDx);
    static constexpr bool kShrink = (OP == Op::ShrinkX || OP == Op::ShrinkDy);
    static constexpr bool kExpand = (OP == Op::ExpandY || OP == Op::ExpandDx);
    static constexpr bool kWgrad = (OP == Op::WgradB || OP == Op::WgradA);
    static constexpr bool kWide = kBase && kBaseRows == 256;   // 256-row tile, two accumulators
    static constexpr int kARows = kWide ? 256 : kTileM;        // rows of A per tile
    static constexpr uint32_t kAStage = (uint32_t)kARows * kBlockK * 2;   // A bytes per stage
};
// Epilogue staging, per epilogue warp: two 4 KB buffers, each one 128-byte-swizzled TMA box of 32 rows x
// 64 bf16 (the base GEMMs' output stores); the dB epilogue uses the same space for a 32 x 33 fp32 chunk.
constexpr int kEpiBufBytes = 32 * 64 * 2;
constexpr int kEpiWarpBytes = 2 * kEpiBufBytes;
constexpr int kEpiStageFloats = 32 * 33;
static_assert(kEpiStageFloats * 4 <= kEpiWarpBytes, "dB staging fits a warp's epilogue space");
// Layout: [operand ring][4 warps' epilogue staging][barriers], from a 1024-byte-aligned base.
constexpr int kEpiOffset = kRingBytes;
constexpr int kBarOffset = kRingBytes + 4 * kEpiWarpBytes;
constexpr int kTcSmemBytes = kBarOffset + 512 /* barriers, flags, item queue */ + 1024 /* align */;
static_assert(kTcSmemBytes <= 232448, "shared memory per CTA");

struct TcParams {
    int32_t M_total;        // Base: T; Wgrad: d (rows of dB_i or columns of dA_i)
    int32_t N_total;        // Base / Expand: output columns
    int32_t K_total;        // Base / Shrink: reduction length
    int32_t tiles_m, tiles_n, num_tiles;
    int32_t group_m;        // Base: rasterisation group (m tiles sharing an L2 window)
    int32_t RP;             // padded rank pitch of H / G / packs
    int32_t b_box_rows;     // BaseFwd: rows of the K-major B box (256)
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
    // Extents of what the kernel addresses through plain pointers (checked by the PLORA_DEBUG build).
    int64_t out_elems;      // elements of the output buffer `out`
    int64_t part_elems;     // floats of the split partials
    int32_t n_counters;     // ints of the arrival counters
    int32_t n_adapters;     // entries of the adapter table
    int32_t n_items;        // entries of tok (shrink, expand) or red (weight gradients)
    int32_t n_mtrec, n_mtseg;   // entries of mt_rec, mt_seg
};

// The output block holding output column `col`.
__device__ __forceinline__ int out_block(const TcParams& p, int col) {
    int b = 0;
    while (b + 1 < p.nblk && col >= p.blk_end[b]) ++b;
    return b;
}

struct TileInfo {
    int32_t a_x, a_y, b_x, b_y, b_z;
    int32_t kblocks, last_ksteps, mma_n, nb_boxes;
    int32_t adapter, out_row, rows_valid, n0, cols_valid, cols_live, red_idx;
    int32_t mtile;
    float scale;
};

template <Op OP>
__device__ __forceinline__ TileInfo decode_tile(const TcParams& p, int t) {  // t: work item (a copy)
    using Tr = OpTraits<OP>;
    TileInfo ti;
    ti.last_ksteps = 4;
    ti.nb_boxes = 1;
    ti.b_z = 0;
    ti.scale = 1.f;
    ti.adapter = -1;
    ti.red_idx = -1;
    if constexpr (Tr::kBase) {
        constexpr int kRows = Tr::kARows;
        // Grouped rasterisation: group_m m-tiles walk all n-tiles together.
        const int per_group = p.group_m * p.tiles_n;
        const int g = t / per_group;
        const int first_m = g * p.group_m;
        const int gm = min(p.tiles_m - first_m, p.group_m);
        const int r = t - g * per_group;
        const int mb = first_m + r % gm;          // m-tiles fastest within the window
        const int nb = r / gm;
        ti.mtile = mb;
        ti.a_x = 0;
        ti.a_y = mb * kRows;
        if constexpr (OP == Op::BaseFwd) { ti.b_x = 0; ti.b_y = nb * kTileN; }
        else { ti.b_x = nb * kTileN; ti.b_y = 0; ti.nb_boxes = kTileN / 64; }
        ti.kblocks = (p.K_total + kBlockK - 1) / kBlockK;
        ti.mma_n = kTileN;
        ti.out_row = mb * kRows;
        ti.rows_valid = min(kRows, p.M_total - ti.out_row);
        ti.n0 = nb * kTileN;
        ti.cols_valid = min(kTileN, p.N_total - ti.n0);
    } else if constexpr (Tr::kShrink) {
        if (!dcheck(p.err_flag, t >= 0 && t < p.n_items)) t = 0;
        TokTile tt = p.tok[t];
        if (!dcheck(p.err_flag, tt.adapter >= 0 && tt.adapter < p.n_adapters && tt.rows >= 1 && tt.rows <= kTileM))
            tt = p.tok[0];
        const AdapterDev ad = p.adapters[tt.adapter];
        ti.adapter = tt.adapter;
        ti.a_x = 0;
        ti.a_y = tt.x_row;
        ti.b_x = 0;
        if constexpr (OP == Op::ShrinkX) {
            // B = the adapter's rp16 rows of the A pack, K-major, in 16-row boxes
            ti.b_y = tt.adapter * p.RP;
            ti.mma_n = ad.rp16;
            ti.nb_boxes = ad.rp16 / 16;
        } else {
            // B = the adapter's B pack [d_out][RP] read MN-major (64 rank columns x 64 rows per box)
            // over rp64 columns; the columns past rp16 are not the adapter's and are stored as zeros
            ti.b_y = 0;
            ti.b_z = tt.adapter;
            ti.mma_n = ad.rp64;
            ti.nb_boxes = ad.rp64 / 64;
        }
        ti.kblocks = (p.K_total + kBlockK - 1) / kBlockK;
        ti.out_row = tt.h_row;
        ti.rows_valid = tt.rows;
        ti.n0 = 0;
        ti.cols_valid = p.RP;
        ti.cols_live = ad.rp16;
        ti.scale = ad.scale;   // H' = s X A and G = s dY B^T carry the adapter's scale
    } else if constexpr (Tr::kExpand) {
        int mt = t / p.tiles_n;
        const int nb = t - mt * p.tiles_n;
        if (!dcheck(p.err_flag, mt >= 0 && mt < p.n_items)) mt = 0;
        TokTile tt = p.tok[mt];
        if (!dcheck(p.err_flag, tt.adapter >= 0 && tt.adapter < p.n_adapters)) tt = p.tok[0];
        const AdapterDev ad = p.adapters[tt.adapter];
        ti.adapter = tt.adapter;
        ti.a_x = 0;
        ti.a_y = tt.h_row;
        if constexpr (OP == Op::ExpandY) {
            // B = rows nb*256.. of the adapter's B pack, K-major (3-D map: rank column, row, adapter)
            ti.b_x = 0;
            ti.b_y = nb * kTileN;
            ti.b_z = tt.adapter;
        } else {
            ti.b_x = nb * kTileN;
            ti.b_y = tt.adapter * p.RP;
            ti.nb_boxes = kTileN / 64;
        }
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
        int e = t / p.red_dtiles;
        const int db = t - e * p.red_dtiles;
        if (!dcheck(p.err_flag, e >= 0 && e < p.n_items)) e = 0;
        RedEntry re = p.red[e];
        if (!dcheck(p.err_flag, re.adapter >= 0 && re.adapter < p.n_adapters)) re = p.red[e = 0];
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
        constexpr int kPer = kLoraTileM / OpTraits<OP>::kARows;   // tiles per 256-row record
        const int rec = ti.mtile / kPer;
        if (!dcheck(p.err_flag, rec >= 0 && rec < p.n_mtrec)) return r;
        r = p.mt_rec[rec];
        if (!dcheck(p.err_flag, r.q0 >= 0 && r.q0 <= r.q1 && r.q1 <= p.n_mtseg)) r.q1 = r.q0;
        // a 128-row tile reads its half of the 256-row record's rows
        const int shift = (ti.mtile % kPer) * kTileM;
        r.s[0].h_y += shift;
        r.s[1].h_y += shift;
        r.pad_[0] = shift;
    }
    return r;
}
__device__ __forceinline__ LoraSeg mtile_seg(const TcParams& p, const MTileRec& r, int q) {
    if (q == r.q0) return r.s[0];       // constant indices keep the record in registers
    if (q == r.q0 + 1) return r.s[1];
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
// false when a wait ran out of time (the error flag is then set).  m: the segment's five tensor maps
// (A, B, a base GEMM's fold A2 and B2, and the output C; for the shrink of H, B, A2, B2 and C are the A
// pack in boxes of 16, 32, 64 and 128 rows).
template <Op OP>
__device__ __forceinline__ bool produce_item(const TcParams& p, const TileInfo& ti, const MTileRec& lr,
                                             const CUtensorMap* m, uint8_t* smem,
                                             int stb, int nst, uint64_t* full_bar, uint64_t* empty_bar,
                                             RingPos& rp, uint32_t& armed, uint32_t& armed_par,
                                             volatile int* abort_flag, uint64_t lim) {
    using Tr = OpTraits<OP>;
    const CUtensorMap* tmA = &m[0];
    const CUtensorMap* tmB = &m[1];
    const CUtensorMap* tmA2 = &m[2];
    const CUtensorMap* tmB2 = &m[3];
    uint32_t b_bytes;
    if constexpr (OP == Op::ShrinkX) b_bytes = (uint32_t)ti.mma_n * 128u;        // rp16 rows of 64
    else if constexpr (OP == Op::ExpandY) b_bytes = (uint32_t)kTileN * 128u;     // 256 rows of 64
    else if constexpr (Tr::kBmn) b_bytes = (uint32_t)ti.nb_boxes * 8192u;        // 64 x 64 boxes
    else b_bytes = (uint32_t)p.b_box_rows * 128u;
    for (int kb = 0; kb < ti.kblocks; ++kb) {
        if (!ptx::mbar_wait(&empty_bar[rp.stage], rp.phase ^ 1u, abort_flag, lim, p.err_flag)) return false;
        uint8_t* sA = smem + rp.stage * stb;
        uint8_t* sB = sA + Tr::kAStage;
        ptx::mbar_arrive_expect_tx(&full_bar[rp.stage], Tr::kAStage + b_bytes);
        armed |= 1u << rp.stage;
        armed_par = (armed_par & ~(1u << rp.stage)) | (rp.phase << rp.stage);
        if constexpr (Tr::kAmn) {
            ptx::tma_load_2d(sA, tmA, &full_bar[rp.stage], ti.a_x, ti.a_y + kb * kBlockK);
            ptx::tma_load_2d(sA + 8192, tmA, &full_bar[rp.stage], ti.a_x + 64, ti.a_y + kb * kBlockK);
        } else {
            ptx::tma_load_2d(sA, tmA, &full_bar[rp.stage], ti.a_x + kb * kBlockK, ti.a_y);
        }
        if constexpr (OP == Op::ShrinkX) {
            // the adapter's rp16 rows as boxes of 128, 64, 32 and 16 rows (m[4], m[3], m[2], m[1]):
            // at most four copies of exactly its rows (16-row boxes alone took up to eight, and the
            // copies, more than their bytes, set this launch's rate)
            int r0 = 0;
            for (int lg = 3; lg >= 0; --lg) {
                const int box = 16 << lg;
                while (ti.mma_n - r0 >= box) {
                    ptx::tma_load_2d(sB + r0 * 128, &m[1 + lg], &full_bar[rp.stage], kb * kBlockK, ti.b_y + r0);
                    r0 += box;
                }
            }
        } else if constexpr (OP == Op::ShrinkDy) {
            for (int h = 0; h < ti.nb_boxes; ++h)
                ptx::tma_load_3d(sB + h * 8192, tmB, &full_bar[rp.stage], 64 * h, kb * kBlockK, ti.b_z);
        } else if constexpr (OP == Op::ExpandY) {
            ptx::tma_load_3d(sB, tmB, &full_bar[rp.stage], kb * kBlockK, ti.b_y, ti.b_z);
        } else if constexpr (Tr::kBmn) {
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
        // segment load as zeros; a 256-row tile stages both halves' rows in one box).  B has the base B's major-ness: for Y, rows n0.. of
        // j's B pack (K-major, one 256 x 64 box); for dX, j's packed A (MN-major, 16-row
        // boxes so that only the rank's rows are staged).  With output blocks, Y's tile reads
        // only its block's columns of H' and of the block-diagonal B pack (K = rblk from
        // b rblk); dX's sums over every block (K = P rblk).
        for (int q = lr.q0; q < lr.q1; ++q) {
            const LoraSeg sg = mtile_seg(p, lr, q);
            const int kext = Tr::kBmn ? sg.rp16 : sg.rblk;
            const int hx0 = Tr::kBmn ? 0 : out_block(p, ti.n0) * sg.rblk;
            for (int kb = 0; kb * kBlockK < kext; ++kb) {
                const int R = min(kBlockK, kext - kb * kBlockK);
                if (!ptx::mbar_wait(&empty_bar[rp.stage], rp.phase ^ 1u, abort_flag, lim, p.err_flag)) return false;
                uint8_t* sA = smem + rp.stage * stb;
                uint8_t* sB = sA + Tr::kAStage;
                const uint32_t lb_bytes = Tr::kBmn ? 4u * (uint32_t)R * 128u : (uint32_t)kTileN * 128u;
                ptx::mbar_arrive_expect_tx(&full_bar[rp.stage], Tr::kAStage + lb_bytes);
                armed |= 1u << rp.stage;
                armed_par = (armed_par & ~(1u << rp.stage)) | (rp.phase << rp.stage);
                ptx::tma_load_2d(sA, tmA2, &full_bar[rp.stage], hx0 + kb * kBlockK, sg.h_y);
                if constexpr (Tr::kBmn) {
                    for (int h = 0; h < 4; ++h)
                        for (int r16 = 0; r16 < R; r16 += 16)
                            ptx::tma_load_2d(sB + h * R * 128 + r16 * 128, tmB2, &full_bar[rp.stage],
                                             ti.n0 + 64 * h, sg.adapter * p.RP + kb * kBlockK + r16);
                } else {
                    // the block-diagonal B pack holds block b's B in the same columns as H'
                    ptx::tma_load_3d(sB, tmB2, &full_bar[rp.stage], hx0 + kb * kBlockK, ti.n0, sg.adapter);
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
    // Descriptors of stage 0; a stage and a k-step only move the start address (bits 0-13, in 16-byte
    // units; shared addresses stay below 2^18 bytes, so the sum never carries out of the field).
    const uint32_t s0 = ptx::smem_u32(smem);
    const uint64_t adesc0 = Tr::kAmn ? ptx::smem_desc_sw128(s0, 8192, 1024) : ptx::smem_desc_sw128(s0, 16, 1024);
    const uint64_t bdesc0 = Tr::kBmn ? ptx::smem_desc_sw128(s0 + Tr::kAStage, 8192, 1024)
                                     : ptx::smem_desc_sw128(s0 + Tr::kAStage, 16, 1024);
    constexpr uint32_t kAstep = Tr::kAmn ? 2048 / 16 : 32 / 16;
    constexpr uint32_t kBstep = Tr::kBmn ? 2048 / 16 : 32 / 16;
    for (int kb = 0; kb < ti.kblocks; ++kb) {
        if (!ptx::mbar_wait(&full_bar[rp.stage], rp.phase, abort_flag, lim, p.err_flag)) return false;
        ptx::tc_fence_after();
        const uint64_t so = (uint64_t)((uint32_t)(rp.stage * stb) >> 4);
        const int steps = (kb == ti.kblocks - 1) ? ti.last_ksteps : 4;
        for (int ks = 0; ks < steps; ++ks)
            ptx::tc_mma_f16(d_tmem, adesc0 + so + ks * kAstep, bdesc0 + so + ks * kBstep, idesc, (kb | ks) ? 1u : 0u);
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
                const uint32_t sB = sA + Tr::kAStage;
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

// MMA issuer of a 256-row base tile.  Rows 0-127 (half 0) accumulate into TMEM columns b0 * 256..,
// rows 128-255 (half 1) into b1 * 256.., and both halves multiply each stage's B tile; a stage is
// released once both have read it.  The fold's k-blocks follow the base ones, as the producer staged
// them (both halves fold every adapter of the 256-row record: rows outside an adapter's tokens read
// the zero padding of its H' / G block).  Each half's products run in the order of the 128-row tile,
// so its sums are bit-identical to it.
//
// The halves go k-block by k-block, except over the first and the last `nst` k-blocks (what the ring
// holds at once), where the half-0 products of all of them go first.  At the end of a tile half 0 then
// completes early and its accumulator drains while half 1's last k-blocks run; at the start of the next
// tile half 0 has work queued while half 1 of the previous tile is still draining.  With both
// accumulators in one tile, this is what keeps the epilogue off the tensor pipe's critical path.
// aph: the parity of each accumulator's uses so far (bit b for accumulator b).
template <Op OP>
__device__ __forceinline__ bool mma_wide(const TcParams& p, const TileInfo& ti, const MTileRec& lr, uint8_t* smem,
                                         int stb, int nst, uint64_t* full_bar, uint64_t* empty_bar,
                                         uint64_t* accf_bar, uint64_t* acce_bar, int b0, uint32_t aph,
                                         uint32_t tmem_base, RingPos& rp, volatile int* abort_flag, uint64_t lim) {
    using Tr = OpTraits<OP>;
    static_assert(Tr::kWide, "256-row base tiles only");
    const uint32_t idesc = ptx::idesc_bf16_f32(kTileM, kTileN, false, Tr::kBmn);
    const uint32_t s0 = ptx::smem_u32(smem);
    const uint64_t adesc0 = ptx::smem_desc_sw128(s0, 16, 1024);
    const uint64_t bdesc0 = Tr::kBmn ? ptx::smem_desc_sw128(s0 + Tr::kAStage, 8192, 1024)
                                     : ptx::smem_desc_sw128(s0 + Tr::kAStage, 16, 1024);
    constexpr uint32_t kBstep = Tr::kBmn ? 2048 / 16 : 32 / 16;
    const int b1 = b0 ^ 1;
    const uint32_t d_acc[2] = {tmem_base + (uint32_t)(b0 * kTileN), tmem_base + (uint32_t)(b1 * kTileN)};

    // k-block cursor: base k-block kb < kblocks, then k-block f of fold segment q
    struct Cur { int kb, q, f; };
    auto kext_of = [&](int q) {
        const LoraSeg sg = mtile_seg(p, lr, q);
        return Tr::kBmn ? sg.rp16 : sg.rblk;
    };
    int nk = ti.kblocks;
    for (int q = lr.q0; q < lr.q1; ++q) nk += (kext_of(q) + kBlockK - 1) / kBlockK;
    auto next = [&](Cur& c) {
        if (c.kb < ti.kblocks) {
            if (++c.kb == ti.kblocks) { c.q = lr.q0; c.f = 0; }
        } else if (++c.f * kBlockK >= kext_of(c.q)) {
            ++c.q;
            c.f = 0;
        }
    };
    // the MMAs of half h over the k-block at cursor c, staged in ring stage `stage`
    auto issue = [&](const Cur& c, int h, int stage) {
        const uint32_t sA = s0 + (uint32_t)(stage * stb);
        if (c.kb < ti.kblocks) {
            const uint64_t so = (uint64_t)(((uint32_t)(stage * stb)) >> 4);
            const uint64_t ah = (uint64_t)((uint32_t)(h * kABytes) >> 4);
            const int steps = (c.kb == ti.kblocks - 1) ? ti.last_ksteps : 4;
            for (int ks = 0; ks < steps; ++ks)
                ptx::tc_mma_f16(d_acc[h], adesc0 + so + ah + (uint64_t)(ks * 2), bdesc0 + so + ks * kBstep, idesc,
                                (c.kb | ks) ? 1u : 0u);
        } else {
            const int R = min(kBlockK, kext_of(c.q) - c.f * kBlockK);
            const uint32_t sB = sA + Tr::kAStage;
            for (int ks = 0; ks < R / 16; ++ks) {
                const uint64_t bdesc = Tr::kBmn ? ptx::smem_desc_sw128(sB + ks * 2048, (uint32_t)R * 128u, 1024)
                                                : ptx::smem_desc_sw128(sB + ks * 32, 16, 1024);
                ptx::tc_mma_f16(d_acc[h], ptx::smem_desc_sw128(sA + h * kABytes + ks * 32, 16, 1024), bdesc, idesc,
                                1u);
            }
        }
    };
    auto wait_full = [&]() {
        if (!ptx::mbar_wait(&full_bar[rp.stage], rp.phase, abort_flag, lim, p.err_flag)) return false;
        ptx::tc_fence_after();
        return true;
    };
    auto wait_drained = [&](int b) {   // accumulator b drained by the epilogue (its previous use)
        if (!ptx::mbar_wait(&acce_bar[b], ((aph >> b) & 1u) ^ 1u, abort_flag, lim, p.err_flag)) return false;
        ptx::tc_fence_after();
        return true;
    };
    const int head = min(nst, nk);
    const int tail = min(nst, nk - head);
    Cur c{0, lr.q0, 0};
    // head: half 0 of the first `head` k-blocks, then half 1 of them
    if (!wait_drained(b0)) return false;
    RingPos r0 = rp;
    Cur c0 = c;
    for (int i = 0; i < head; ++i) {
        if (!wait_full()) return false;
        issue(c, 0, rp.stage);
        next(c);
        rp.advance(nst);
    }
    if (tail == 0) ptx::tc_commit(&accf_bar[b0]);
    if (!wait_drained(b1)) return false;
    rp = r0;
    c = c0;
    for (int i = 0; i < head; ++i) {
        issue(c, 1, rp.stage);
        ptx::tc_commit(&empty_bar[rp.stage]);
        next(c);
        rp.advance(nst);
    }
    if (tail == 0) {
        ptx::tc_commit(&accf_bar[b1]);
        return true;
    }
    // middle: both halves per k-block
    for (int i = head; i < nk - tail; ++i) {
        if (!wait_full()) return false;
        issue(c, 0, rp.stage);
        issue(c, 1, rp.stage);
        ptx::tc_commit(&empty_bar[rp.stage]);
        next(c);
        rp.advance(nst);
    }
    // tail: half 0 of the last `tail` k-blocks (then half 0 is complete), then half 1 of them
    r0 = rp;
    c0 = c;
    for (int i = 0; i < tail; ++i) {
        if (!wait_full()) return false;
        issue(c, 0, rp.stage);
        next(c);
        rp.advance(nst);
    }
    ptx::tc_commit(&accf_bar[b0]);
    rp = r0;
    c = c0;
    for (int i = 0; i < tail; ++i) {
        issue(c, 1, rp.stage);
        ptx::tc_commit(&empty_bar[rp.stage]);
        next(c);
        rp.advance(nst);
    }
    ptx::tc_commit(&accf_bar[b1]);
    return true;
}

// Base-GEMM epilogue of one epilogue warp: its 32 accumulator rows (TMEM lanes from t_row) x 256
// columns, rounded to bf16 (nearest even) and written to rows row0.. and columns n0.. of the output
// through its two staging buffers: per 64 columns, the lanes write their rows into a 128-byte-swizzled
// 32 x 64 box (16-byte stores, conflict-free) and one lane issues a TMA tensor store, so whole lines
// reach L2 and the conversion of a chunk overlaps the store of the one before.  The store clips rows
// and columns outside the output tensor.  seq counts the warp's chunks over the whole launch and picks
// the buffer, so the alternation carries across calls: a call may store an odd number of chunks (a
// narrow last n-tile), and the next call's first chunk must not take the buffer whose store may still
// be reading it.
__device__ __forceinline__ void epilogue_store_tma(const CUtensorMap* tmC, uint32_t t_row, uint8_t* wbuf, int lane,
                                                   int row0, int n0, int M_total, int N_total, uint32_t& seq) {
    if (row0 >= M_total) return;
    const uint32_t sw = (uint32_t)(lane & 7);
    for (int ch = 0; ch < kTileN / 64; ++ch) {
        const int col0 = n0 + ch * 64;
        if (col0 >= N_total) break;
        uint32_t ra[32], rb[32];
        ptx::tmem_ld32(t_row + ch * 64, ra);
        ptx::tmem_ld32(t_row + ch * 64 + 32, rb);
        ptx::tmem_ld_wait();
        uint8_t* buf = wbuf + (seq++ & 1u) * kEpiBufBytes;
        if (lane == 0) ptx::bulk_wait_read<1>();   // the store that last read this buffer is done
        __syncwarp();
        const uint32_t rowaddr = ptx::smem_u32(buf) + (uint32_t)lane * 128u;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t* v = j < 4 ? ra + 8 * j : rb + 8 * (j - 4);
            uint4 o;
            o.x = pack_bf16x2(__uint_as_float(v[0]), __uint_as_float(v[1]));
            o.y = pack_bf16x2(__uint_as_float(v[2]), __uint_as_float(v[3]));
            o.z = pack_bf16x2(__uint_as_float(v[4]), __uint_as_float(v[5]));
            o.w = pack_bf16x2(__uint_as_float(v[6]), __uint_as_float(v[7]));
            ptx::st_shared_v4(rowaddr + ((((uint32_t)j) ^ sw) << 4), o);
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            ptx::tma_store_2d(tmC, buf, col0, row0);
            ptx::bulk_commit();
        }
    }
}

// Epilogue (warps 2..5, one accumulator row per thread): drains work item ti's accumulator
// rows from TMEM at t_row and runs the op's output step.
template <Op OP>
__device__ __forceinline__ void epilogue_item(const TcParams& p, const TileInfo& ti, uint32_t t_row, int q, int lane,
                                              uint8_t* wbuf, const CUtensorMap* tmC, int* red_flag, uint32_t& epi_seq) {
    using Tr = OpTraits<OP>;
    const int row = q * 32 + lane;          // accumulator row handled by this thread
    const bool row_ok = row < ti.rows_valid;
    float* epi_stage = reinterpret_cast<float*>(wbuf);
    if constexpr (Tr::kBase) {
        epilogue_store_tma(tmC, t_row, wbuf, lane, ti.out_row + q * 32, ti.n0, p.M_total, p.N_total, epi_seq);
    } else if constexpr (Tr::kShrink) {
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + (int64_t)(ti.out_row + row) * p.out_ld;
        // (the TMEM loads below are warp-collective: a failed check skips this thread's stores only)
        const bool out_ok = dcheck(p.err_flag, ti.out_row + row >= 0 && ti.cols_valid <= p.out_ld &&
                                                   (int64_t)(ti.out_row + row + 1) * p.out_ld <= p.out_elems);
        for (int c = 0; c < ti.cols_valid; c += 16) {
            uint4 v0 = make_uint4(0, 0, 0, 0), v1 = make_uint4(0, 0, 0, 0);
            if (c < ti.cols_live) {
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
            if (out_ok) {
                *reinterpret_cast<uint4*>(out + c) = v0;
                *reinterpret_cast<uint4*>(out + c + 8) = v1;
            }
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
            const bool pads_ok = dcheck(p.err_flag, ad.h_row - kLoraPad >= 0 && p.RP <= p.out_ld &&
                                                        (int64_t)(tail + kLoraPad) * p.out_ld <= p.out_elems);
            for (int pr = row; pr < kLoraPad && pads_ok; pr += kTileM) {
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
        // (the TMEM loads below are warp-collective: a failed check skips this thread's accesses only)
        const bool rw = row_ok && dcheck(p.err_flag, ti.n0 + ti.cols_valid <= p.out_ld &&
                                                         (int64_t)(ti.out_row + row + 1) * p.out_ld <= p.out_elems);
        for (int h = 0; h < kTileN; h += 128) {
            uint4 y[16];
            if (rw) {
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    if (h + 8 * u + 8 <= ti.cols_valid) y[u] = *reinterpret_cast<const uint4*>(out + h + 8 * u);
            }
#pragma unroll
            for (int u = 0; u < 16; u += 2) {
                uint32_t r[16];
                ptx::tmem_ld16(t_row + h + 8 * u, r);
                ptx::tmem_ld_wait();
                if (rw) {
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
            float* stg = epi_stage;
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
            const bool split_ok = dcheck(p.err_flag, re.slot >= 0 && re.counter >= 0 && re.split < re.nsplit &&
                                                         ((int64_t)(re.slot + re.nsplit - 1) * p.red_dtiles + ti.n0 + 1) *
                                                                 slot_elems <= p.part_elems &&
                                                         re.counter + ti.n0 < p.n_counters);
            if (!split_ok) return;   // every thread of the tile takes the same branch
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

// One persistent launch runs the work items of up to kMaxSeg independent products ("segments"):
// segments [0, n_op1) run OP and the others OP2 (the backward runs dB's items after G's, filling the
// last wave of G's equal-cost token tiles, and dA's after the dX GEMM's tiles, filling its last,
// partial wave; the layer calls run one product kind of several projections together).  Segment j
// owns items [begin[j], begin[j+1]) and has its own parameters and tensor maps: m[j][0..1] the
// operands, m[j][2..3] a base GEMM's folded low-rank branch, m[j][4] a base GEMM's output.  Every
// segment uses the ring layout of segment 0 (stages, stage_bytes), which must hold all their tiles.
// Items are dealt round-robin over the CTAs.
constexpr int kMaxSeg = 16;

struct GroupParams {
    int32_t n_seg, n_op1;
    int32_t begin[kMaxSeg + 1];
    // With a second op, a counter that starts at zero (the call's schedule copy clears it): its items
    // are then claimed one at a time (nullptr: every item dealt round-robin).
    int32_t* dyn;
    TcParams p[kMaxSeg];
};
constexpr int kItemQ = 4;   // item queue slots (producer -> MMA and epilogue roles) for claimed items
struct GroupMaps {
    CUtensorMap m[kMaxSeg][5];
};

template <Op OP, Op OP2 = OP>
__global__ void __launch_bounds__(kTcThreads, 1)
tc_kernel(const __grid_constant__ GroupMaps maps, const __grid_constant__ GroupParams g) {
    using Tr = OpTraits<OP>;
    static_assert(OP2 == OP || !OpTraits<OP2>::kBase, "the second op of a launch is not a base GEMM");
    const TcParams& p0 = g.p[0];
    const int total = g.begin[g.n_seg];
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOffset);
    uint64_t* full_bar = bars;                       // [kMaxStages]
    uint64_t* empty_bar = bars + kMaxStages;         // [kMaxStages]
    uint64_t* accf_bar = bars + 2 * kMaxStages;      // [2]
    uint64_t* acce_bar = bars + 2 * kMaxStages + 2;  // [2]
    uint64_t* drain_bar = bars + 2 * kMaxStages + 4;
    uint64_t* itemf_bar = bars + 2 * kMaxStages + 5;             // [kItemQ] a claimed item is published
    uint64_t* iteme_bar = bars + 2 * kMaxStages + 5 + kItemQ;    // [kItemQ] its slot has been read
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kMaxStages + 5 + 2 * kItemQ);
    const int nst = p0.stages;                       // ring depth of this launch
    const int stb = p0.stage_bytes;                  // bytes per stage (multiple of 1024)
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* red_flag = reinterpret_cast<int*>(tmem_slot + 2);
    volatile int32_t* item_q = reinterpret_cast<volatile int32_t*>(tmem_slot + 4);   // [kItemQ]
    // Items [0, n_static) are dealt round-robin over the CTAs.  With g.dyn, the second op's items
    // [n_static, total) are claimed one at a time once a CTA's share of the first op is done, so the
    // CTAs that hold no item of the first op's last, partial wave take more of them.  The producer
    // claims and publishes each item; the MMA and epilogue roles read the same sequence.  Which CTA
    // runs an item changes no result: every item is computed on its own.
    const bool dyn = OP2 != OP && g.dyn != nullptr && g.n_seg > g.n_op1;
    const int n_static = dyn ? g.begin[g.n_op1] : total;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // The segment of item t (a short scan: at most kMaxSeg segments).
    auto seg_of = [&](int t) {
        int j = 0;
        while (j + 1 < g.n_seg && t >= g.begin[j + 1]) ++j;
        return j;
    };
    // The folded low-rank record of item t of a base GEMM (empty otherwise, and past the end).
    auto rec_of = [&](int t) {
        MTileRec r;
        r.q0 = r.q1 = 0;
        if (!Tr::kBase || t >= total) return r;
        const int j = seg_of(t);
        return j < g.n_op1 ? load_mtile<OP>(g.p[j], t - g.begin[j]) : r;
    };

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
        for (int s = 0; s < kItemQ; ++s) {
            ptx::mbar_init(&itemf_bar[s], 1);
            ptx::mbar_init(&iteme_bar[s], 5);   // the MMA lane and the four epilogue warps
        }
        *abort_flag = 0;
        ptx::fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        // every map slot of every segment holds a valid map (the host fills unused slots with copies)
        for (int j = 0; j < g.n_seg; ++j)
            for (int k = 0; k < 5; ++k) ptx::tma_prefetch_desc(&maps.m[j][k]);
    }
    if (warp == 1) {
        ptx::tmem_alloc<kTmemCols>(tmem_slot);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint64_t lim = p0.timeout_ns;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            RingPos rp{0, 0u};
            uint32_t armed = 0, armed_par = 0;
            bool ok = true;
            // The folded low-rank record of a base tile is fetched one tile ahead.
            MTileRec lr_next = rec_of(blockIdx.x);
            for (int t = blockIdx.x; t < n_static && ok; t += gridDim.x) {
                const MTileRec lr = lr_next;
                lr_next = rec_of(t + gridDim.x);
                const int j = seg_of(t);
                const CUtensorMap* m = maps.m[j];
                const TcParams& pj = g.p[j];
                if (j >= g.n_op1)
                    ok = produce_item<OP2>(pj, decode_tile<OP2>(pj, t - g.begin[j]), lr, m, smem, stb, nst, full_bar,
                                           empty_bar, rp, armed, armed_par, abort_flag, lim);
                else
                    ok = produce_item<OP>(pj, decode_tile<OP>(pj, t - g.begin[j]), lr, m, smem, stb, nst, full_bar,
                                          empty_bar, rp, armed, armed_par, abort_flag, lim);
            }
            if (dyn && ok) {
                int qs = 0;
                uint32_t qph = 0;
                for (;;) {
                    const int idx = atomicAdd(g.dyn, 1);
                    const int t = idx < total - n_static ? n_static + idx : -1;   // -1: no items left
                    if (!ptx::mbar_wait(&iteme_bar[qs], qph ^ 1u, abort_flag, lim, p0.err_flag)) break;
                    item_q[qs] = t;
                    ptx::mbar_arrive(&itemf_bar[qs]);
                    if (++qs == kItemQ) { qs = 0; qph ^= 1u; }
                    if (t < 0) break;
                    const int j = seg_of(t);
                    if (!produce_item<OP2>(g.p[j], decode_tile<OP2>(g.p[j], t - g.begin[j]), MTileRec{}, maps.m[j],
                                           smem, stb, nst, full_bar, empty_bar, rp, armed, armed_par, abort_flag,
                                           lim))
                        break;
                }
            }
            // Drain: every load this thread issued must have landed before the CTA exits.
            for (int s = 0; s < nst; ++s)
                if (armed & (1u << s)) {
                    int dummy = 0;
                    ptx::mbar_wait(&full_bar[s], (armed_par >> s) & 1u, &dummy, lim, p0.err_flag);
                }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            RingPos rp{0, 0u};
            int abuf = 0;
            uint32_t aph = 0;    // bit b: parity of accumulator b's uses so far
            bool ok = true;
            MTileRec lr_next = rec_of(blockIdx.x);
            for (int t = blockIdx.x; t < n_static; t += gridDim.x) {
                const MTileRec lr = lr_next;
                lr_next = rec_of(t + gridDim.x);
                const int j = seg_of(t);
                const TcParams& pj = g.p[j];
                if constexpr (Tr::kWide) {
                    if (j < g.n_op1) {   // a 256-row base tile: both accumulators, in the order abuf, abuf ^ 1
                        if (!mma_wide<OP>(pj, decode_tile<OP>(pj, t - g.begin[j]), lr, smem, stb, nst, full_bar,
                                          empty_bar, accf_bar, acce_bar, abuf, aph, tmem_base, rp, abort_flag, lim)) {
                            ok = false;
                            break;
                        }
                        aph ^= 3u;
                        continue;
                    }
                }
                if (!ptx::mbar_wait(&acce_bar[abuf], ((aph >> abuf) & 1u) ^ 1u, abort_flag, lim, p0.err_flag)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(abuf * kTileN);
                ok = (j >= g.n_op1)
                    ? mma_item<OP2>(pj, decode_tile<OP2>(pj, t - g.begin[j]), lr, smem, stb, nst, full_bar,
                                    empty_bar, d_tmem, rp, abort_flag, lim)
                    : mma_item<OP>(pj, decode_tile<OP>(pj, t - g.begin[j]), lr, smem, stb, nst, full_bar, empty_bar,
                                   d_tmem, rp, abort_flag, lim);
                if (!ok) break;
                ptx::tc_commit(&accf_bar[abuf]);
                aph ^= 1u << abuf;
                abuf ^= 1;
            }
            if (dyn && ok) {
                int qs = 0;
                uint32_t qph = 0;
                for (;;) {
                    if (!ptx::mbar_wait(&itemf_bar[qs], qph, abort_flag, lim, p0.err_flag)) break;
                    const int t = item_q[qs];
                    ptx::mbar_arrive(&iteme_bar[qs]);
                    if (++qs == kItemQ) { qs = 0; qph ^= 1u; }
                    if (t < 0) break;
                    if (!ptx::mbar_wait(&acce_bar[abuf], ((aph >> abuf) & 1u) ^ 1u, abort_flag, lim, p0.err_flag)) break;
                    ptx::tc_fence_after();
                    const int j = seg_of(t);
                    if (!mma_item<OP2>(g.p[j], decode_tile<OP2>(g.p[j], t - g.begin[j]), MTileRec{}, smem, stb, nst,
                                       full_bar, empty_bar, tmem_base + (uint32_t)(abuf * kTileN), rp, abort_flag, lim))
                        break;
                    ptx::tc_commit(&accf_bar[abuf]);
                    aph ^= 1u << abuf;
                    abuf ^= 1;
                }
            }
            // Drain: all issued MMAs complete before TMEM is released.
            ptx::tc_commit(drain_bar);
            int dummy = 0;
            ptx::mbar_wait(drain_bar, 0, &dummy, lim, p0.err_flag);
        }
    } else {
        // ------------------------------------------------------------ epilogue (warps 2..5)
        const int q = warp & 3;                 // TMEM lane quarter this warp may access
        uint8_t* wbuf = smem + kEpiOffset + q * kEpiWarpBytes;
        int abuf = 0;
        uint32_t aph = 0;        // bit b: parity of accumulator b's uses so far
        uint32_t epi_seq = 0;    // this warp's output chunks so far (staging buffer = epi_seq & 1)
        bool ok = true;
        for (int t = blockIdx.x; t < n_static && ok; t += gridDim.x) {
            const int j = seg_of(t);
            const TcParams& pj = g.p[j];
            if constexpr (Tr::kWide) {
                if (j < g.n_op1) {   // a 256-row base tile: half 0 from accumulator abuf, half 1 from abuf ^ 1
                    const TileInfo ti = decode_tile<OP>(pj, t - g.begin[j]);
                    for (int h = 0; h < 2 && ok; ++h) {
                        const int b = abuf ^ h;
                        if (!ptx::mbar_wait(&accf_bar[b], (aph >> b) & 1u, abort_flag, lim, p0.err_flag)) {
                            ok = false;
                            break;
                        }
                        ptx::tc_fence_after();
                        const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * kTileN);
                        epilogue_store_tma(&maps.m[j][4], t_row, wbuf, lane, ti.out_row + h * kTileM + q * 32, ti.n0,
                                           pj.M_total, pj.N_total, epi_seq);
                        ptx::tc_fence_before();
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive(&acce_bar[b]);
                    }
                    aph ^= 3u;
                    continue;
                }
            }
            if (!ptx::mbar_wait(&accf_bar[abuf], (aph >> abuf) & 1u, abort_flag, lim, p0.err_flag)) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(abuf * kTileN);
            if (j >= g.n_op1)
                epilogue_item<OP2>(pj, decode_tile<OP2>(pj, t - g.begin[j]), t_row, q, lane, wbuf, &maps.m[j][4],
                                   red_flag, epi_seq);
            else
                epilogue_item<OP>(pj, decode_tile<OP>(pj, t - g.begin[j]), t_row, q, lane, wbuf, &maps.m[j][4],
                                  red_flag, epi_seq);
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&acce_bar[abuf]);
            aph ^= 1u << abuf;
            abuf ^= 1;
        }
        if (dyn && ok) {
            int qs = 0;
            uint32_t qph = 0;
            for (;;) {
                if (!ptx::mbar_wait(&itemf_bar[qs], qph, abort_flag, lim, p0.err_flag)) break;
                const int t = item_q[qs];
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&iteme_bar[qs]);
                if (++qs == kItemQ) { qs = 0; qph ^= 1u; }
                if (t < 0) break;
                if (!ptx::mbar_wait(&accf_bar[abuf], (aph >> abuf) & 1u, abort_flag, lim, p0.err_flag)) break;
                ptx::tc_fence_after();
                const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(abuf * kTileN);
                const int j = seg_of(t);
                epilogue_item<OP2>(g.p[j], decode_tile<OP2>(g.p[j], t - g.begin[j]), t_row, q, lane, wbuf, &maps.m[j][4],
                                   red_flag, epi_seq);
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&acce_bar[abuf]);
                aph ^= 1u << abuf;
                abuf ^= 1;
            }
        }
        // Every output store has been performed before the CTA (and its staging) goes away.
        if (Tr::kBase && lane == 0) ptx::bulk_wait<0>();
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc<kTmemCols>(tmem_base);
}

// ---------------------------------------------------------------------------
// Packing of the small per-adapter factors into the MMA-ready padded layouts, once per forward, into
// the `saved` buffer that the backward reads as well (b = output block, rblk_i = r_i rounded up to 16,
// rp16_i = P rblk_i; one block: b = 0 and rblk_i = rp16_i):
//   packA [n RP][d_in]:    row i RP + b rblk_i + k = A_i[b r_i + k][:] for k < r_i, zero up to rblk_i
//   packB [n][d_out][RP]:  packB[i][c][b rblk_i + k] = B_i[c][k] if column c lies in block b and k < r_i,
//                          else zero (block-diagonal over the output blocks)
// packA rows at or past rp16_i and packB columns at or past rp16_i are never multiplied (the shrink of
// G reads them and discards the accumulator columns) and stay unwritten.
//
// packA feeds the shrink of H (K-major) and the fold of G A^T into dX (MN-major); packB feeds the fold
// of H' B into Y (K-major, block b's columns) and the shrink of G = s dY B^T (MN-major: column
// b rblk + k of G sums over block b's output columns only, as output blocks need).
// ---------------------------------------------------------------------------
// One projection's pack: its adapter table, the pitch RP, the sizes, the output blocks and where the
// two packs go (with their extents, for the PLORA_DEBUG checks).
struct PackJob {
    const AdapterDev* ad;
    __nv_bfloat16* packA;
    __nv_bfloat16* packB;
    int64_t d_in, d_out, packA_elems, packB_elems;
    int32_t n, RP;
    OutBlocks blocks;
    int* err_flag;
};
constexpr int kMaxPackJobs = 16;
struct PackJobs {
    int32_t n;
    PackJob j[kMaxPackJobs];
};

// grid (gx, adapters, jobs), block 256: per adapter of a job, a grid-stride loop over its 16-byte
// chunks, first the rp16 x d_in/8 chunks of packA, then the d_out x rp16/8 chunks of packB (consecutive
// threads on consecutive bytes of both sources and destinations).
__global__ void __launch_bounds__(256) pack_ab_kernel(const __grid_constant__ PackJobs jobs) {
    if ((int)blockIdx.z >= jobs.n) return;
    const PackJob& J = jobs.j[blockIdx.z];
    const int i = blockIdx.y;
    if (i >= J.n) return;
    const AdapterDev a = J.ad[i];
    const int RP = J.RP;
    const int64_t d_in = J.d_in, d_out = J.d_out;
    __nv_bfloat16* __restrict__ packA = J.packA;
    __nv_bfloat16* __restrict__ packB = J.packB;
    const int r = a.rank, rblk = a.rblk;
    const int64_t va = d_in / 8;
    const int64_t ua = (int64_t)a.rp16 * va;
    const int vb = a.rp16 / 8;
    const int64_t ub = d_out * vb;
    const __nv_bfloat16* A = static_cast<const __nv_bfloat16*>(a.A);
    const __nv_bfloat16* B = static_cast<const __nv_bfloat16*>(a.B);
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < ua + ub; e += (int64_t)gridDim.x * blockDim.x) {
        uint4 val = make_uint4(0, 0, 0, 0);
        if (e < ua) {
            const int j = (int)(e / va);
            const int64_t v = e - (int64_t)j * va;
            const int pb = j / rblk, k = j - pb * rblk;      // output block pb's rank row k
            if (!dcheck(J.err_flag, pb < J.blocks.n && j < RP &&
                                        ((int64_t)i * RP + j) * d_in + (v + 1) * 8 <= J.packA_elems))
                continue;
            if (k < r) val = reinterpret_cast<const uint4*>(A + (int64_t)(pb * r + k) * d_in)[v];
            reinterpret_cast<uint4*>(packA + ((int64_t)i * RP + j) * d_in)[v] = val;
        } else {
            const int64_t f = e - ua;
            const int64_t c = f / vb;
            const int col = (int)(f - c * vb) * 8;
            const int pb = col / rblk, k0 = col - pb * rblk;  // 8 columns of one block (rblk % 16 == 0)
            int cb = 0;
            while (cb + 1 < J.blocks.n && c >= J.blocks.end[cb]) ++cb;
            if (cb == pb && k0 < r) {
                const __nv_bfloat16* src = B + c * r + k0;
                if ((r & 7) == 0) {
                    val = *reinterpret_cast<const uint4*>(src);
                } else {
                    __nv_bfloat16 v[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) v[u] = k0 + u < r ? src[u] : __float2bfloat16_rn(0.f);
                    val = *reinterpret_cast<const uint4*>(v);
                }
            }
            if (!dcheck(J.err_flag, col + 8 <= RP && ((int64_t)i * d_out + c) * RP + col + 8 <= J.packB_elems)) continue;
            *reinterpret_cast<uint4*>(packB + ((int64_t)i * d_out + c) * RP + col) = val;
        }
    }
}

}  // namespace plora
