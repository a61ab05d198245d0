// plan.cuh -- per-call schedule structures shared by the host code and the kernels.
//
// A call's schedule is built on the host from the segment offsets and the
// adapter table, copied once to the device (by a small kernel, from mapped
// pinned staging), and read by every kernel of the call.
#pragma once
#include <cstdint>

namespace plora {

constexpr int kTileM = 128;     // token rows (or hidden rows) per tensor-core tile
constexpr int kBlockK = 64;     // K elements per pipeline stage (128 bytes of bf16)
constexpr int kRankAlign = 64;  // the padded rank width RP of the saved/G buffers is a multiple of this
constexpr int kSplitTokens = 16384; // weight-gradient split size along the tokens (fixed: deterministic)
constexpr int kLoraPad = 256;       // zero rows before and after each adapter's H' / G block
constexpr int kLoraTileM = 256;     // base-GEMM rows per overlap record (one 256-row tile, 1-SM or SM pair)

constexpr int kMaxOutBlocks = 8;    // output blocks (shared-input projections stacked along d_out)

// Device-side bounds checks (the PLORA_DEBUG build).  A kernel compares each index it forms from the
// schedule with the extent of the buffer it addresses, as the host allocated it; a failed check records
// kErrBounds (PLORA_ERR_BOUNDS) in the handle's error flag and the access is skipped (or the schedule
// entry replaced by entry 0), so a wrong schedule shows up as an error status, never as a fault.  In
// release builds the checks compile to nothing.
#ifdef PLORA_DEBUG
constexpr bool kDeviceChecks = true;
#else
constexpr bool kDeviceChecks = false;
#endif
constexpr int kErrBounds = 6;

__device__ __forceinline__ bool dcheck(int* err_flag, bool ok) {
    if constexpr (kDeviceChecks) {
        if (!ok) {
            if (err_flag) atomicCAS(err_flag, 0, kErrBounds);
            return false;
        }
    }
    return true;
}

// The output blocks of a handle: block b holds output columns [end[b-1], end[b]).
struct OutBlocks {
    int32_t n;
    int32_t end[kMaxOutBlocks];
};

// One adapter, as the kernels see it.  With P output blocks an adapter has one rank-r pair
// per block; H' and G hold block p in columns [p rblk, p rblk + r) (zeros up to (p+1) rblk).
struct AdapterDev {
    const void* A;     // A_store [P rank][d_in] (block p = rows p rank ..)
    const void* B;     // B_store [d_out][rank]
    float* dA;         // [P rank][d_in]
    float* dB;         // [d_out][rank]
    int32_t x_row;     // first token row in X / Y / dY / dX (= off[i])
    int32_t n;         // tokens of this adapter
    int32_t h_row;     // first row of this adapter's block in the saved H / workspace G buffers
    int32_t rank;
    float scale;
    int32_t rp16;      // width of its H' / G columns, P rblk (the shrink's N, the dX fold's K)
    int32_t rp64;      // rp16 rounded up to 64 (the MN-major tile width of dA)
    int32_t rblk;      // rank rounded up to 16 (one block's pitch: the Y fold's and dB's extent)
};
static_assert(sizeof(AdapterDev) == 64, "AdapterDev layout");

// A 128-row tile of one adapter's tokens (shrink / expand kernels).
struct TokTile {
    int32_t adapter;
    int32_t rows;      // valid rows in this tile, 1..128
    int32_t x_row;     // first token row
    int32_t h_row;     // first row in H / G
};
static_assert(sizeof(TokTile) == 16, "TokTile layout");

// One split of one adapter's tokens for the weight gradients (dB, dA).
struct RedEntry {
    int32_t adapter;
    int32_t x_row;     // first token row of the split
    int32_t h_row;     // first H / G row of the split
    int32_t kblocks;   // 64-token blocks in the split
    int32_t split;     // index of the split within the adapter
    int32_t nsplit;    // number of splits of the adapter
    int32_t slot;      // first partial slot of the adapter (nsplit > 1), else -1
    int32_t counter;   // first arrival counter of the adapter (nsplit > 1), else -1
};
static_assert(sizeof(RedEntry) == 32, "RedEntry layout");

// One adapter overlapping one 256-row record (kLoraTileM rows) of a base GEMM (low-rank branch folded in).
struct LoraSeg {
    int32_t adapter;
    int32_t h_y;       // H' / G row holding the record's first token, inside the adapter's zero-padded block
    int32_t rp16;      // K extent of the folded dX product (the adapter's P rblk)
    int32_t rblk;      // K extent of the folded Y product (one output block's rank, rounded up to 16)
};
static_assert(sizeof(LoraSeg) == 16, "LoraSeg layout");

// Per 256-row record of a base GEMM's rows: the range of its LoraSeg entries, with the first two
// inlined so that one 48-byte load gives everything in the common case.
struct MTileRec {
    int32_t q0, q1;    // entries mt_seg[q0 .. q1)
    int32_t pad_[2];
    LoraSeg s[2];      // mt_seg[q0], mt_seg[q0 + 1] (when present)
};
static_assert(sizeof(MTileRec) == 48, "MTileRec layout");

// A generic strided product for the SIMT path:
//   C(m, n) = alpha * sum_k A(m, k) B(k, n)  (+ C(m, n) if accumulate)
// with A(m,k) = A[m*a_sm + k*a_sk], B(k,n) = B[k*b_sk + n*b_sn], C(m,n) = C[m*c_sm + n*c_sn].
struct SimtOp {
    const void* A;
    const void* B;
    void* C;
    int64_t a_sm, a_sk, b_sk, b_sn, c_sm, c_sn;
    int32_t M, N, K;
    float alpha;
    int32_t accumulate;
    int32_t c_fp32;      // 1: C is fp32; 0: C has the input element type
    int32_t tile_begin;  // first block index of this op in the launch
    int32_t tiles_n;     // 64-wide tiles along N
};
static_assert(sizeof(SimtOp) == 104, "SimtOp layout");

}  // namespace plora
