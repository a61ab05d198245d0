// plora.cu -- host side of the packed LoRA library: argument checking, the
// per-call schedule (segment tiles, weight-gradient splits, LPT order), the
// tensor maps, the workspace, and the launches of the sm_100a kernels.
//
// The C ABI is declared and documented in include/plora.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <memory>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include "../../include/plora.h"
#include "plan.cuh"
#include "simt.cuh"
#include "tc.cuh"
#include "tc_pair.cuh"
#include "adamw.cuh"

using namespace plora;

namespace {

constexpr int kSlots = 4;                   // host staging / device schedule ring depth
// Rasterisation windows of the base GEMMs (rows of A whose tiles walk every n-tile together): 2048
// rows, eight 256-row m-tiles, so that a wave of 148 tiles spans about 18 n-tiles and A's window (16 MB
// of X for d_in = 4096) stays in L2 while W streams past it.  Measured on whole benchmark steps against
// 1024, 4096 and 8192 rows (and mixed forward / dX windows): 2048 was the fastest.
#ifndef PLORA_WINDOW_ROWS
#define PLORA_WINDOW_ROWS 2048
#endif
#ifndef PLORA_DX_WINDOW_ROWS
#define PLORA_DX_WINDOW_ROWS 2048
#endif
constexpr int kWindowRows = PLORA_WINDOW_ROWS;
constexpr int kDxWindowRows = PLORA_DX_WINDOW_ROWS;
constexpr uint64_t kTimeoutNs = 4000000000ull;

struct Region {
    size_t off = 0, bytes = 0;
};

}  // namespace

// The segments of one tc_kernel launch (see GroupParams): segment parameters and their five tensor
// maps (operands A, B; a base GEMM's folded branch A2, B2 and output C; unused slots hold copies of A).
// The launch copies them when it is enqueued, so one host copy serves every launch.
struct Segments {
    GroupParams g{};
    GroupMaps m{};
    int n_op2 = 0;
    TcParams p2[kMaxSeg];
    CUtensorMap m2[kMaxSeg][5];
};

struct plora_ctx {
    plora_config cfg{};
    int device = 0;
    int num_sms = 0;
    size_t esize = 2;
    int RPmax = 64;
    int64_t max_h_rows = 0;
    int64_t max_slots = 0, max_counters = 0;
    size_t blob_bytes = 0;
    bool tc = false;           // tensor-core path (bf16 without PLORA_FLAG_SIMT)
    int nblk = 1;              // output blocks (shared-input projections stacked along d_out)
    int32_t blk_end[kMaxOutBlocks] = {};   // cumulative output-column ends of the blocks
    int pairs_fwd = 0, pairs_dx = 0;   // co-resident SM pairs for the pair-tile base GEMMs

    uint8_t* ws = nullptr;     // one device allocation, carved into regions
    size_t ws_bytes = 0;
    Region r_G, r_part, r_cnt, r_err, r_blob[kSlots];

    uint8_t* h_blob[kSlots] = {};       // mapped pinned staging of each slot (host view)
    uint8_t* h_blob_dev[kSlots] = {};   // the same buffers as the device addresses them
    // Schedule slots for calls made while their stream is being captured into a CUDA graph: each
    // captured call keeps its slot (staging and device copy) until plora_capture_release, so every
    // replay of the graph re-runs its staging copy from buffers no later call overwrites.
    struct CaptureSlot {
        uint8_t* host = nullptr;
        uint8_t* host_dev = nullptr;
        uint8_t* dev = nullptr;
    };
    std::vector<CaptureSlot> cap;
    size_t cap_next = 0;
    bool in_capture = false;   // the current call's stream is capturing (no profiling events then)
    cudaEvent_t ev[kSlots] = {};
    int next_slot = 0;

    std::string last_error;

    // Launch accounting and optional per-kernel timing (CUDA events on the launching stream).
    bool profiling = false;
    int64_t launches[16] = {};
    double total_ms[16] = {};
    struct Rec { int kind; cudaEvent_t a, b; };
    std::vector<Rec> pending;
    std::vector<cudaEvent_t> pool;

    // host scratch for building one launch's segment table (kernel parameters, ~14 KB)
    std::unique_ptr<Segments> segs;

    template <typename T> T* at(const Region& r) const { return reinterpret_cast<T*>(ws + r.off); }
};

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

plora_status fail(plora_ctx* h, plora_status s, const char* fmt, ...) {
    if (h) {
        char buf[512];
        va_list ap;
        va_start(ap, fmt);
        vsnprintf(buf, sizeof buf, fmt, ap);
        va_end(ap);
        h->last_error = buf;
    }
    return s;
}

plora_status cuda_fail(plora_ctx* h, cudaError_t e, const char* what) {
    return fail(h, PLORA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }
int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

bool get_encode() {
    if (g_encode) return true;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
        return false;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return true;
}

// [p, p + bytes) must lie inside one device allocation: every tensor pointer is checked against the
// driver's record of the allocation that contains it, so that no kernel is ever launched on a host
// pointer, an unallocated address or a buffer that is too small.
PFN_cuMemGetAddressRange_v3020 g_range = nullptr;

bool get_range_fn() {
    if (g_range) return true;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
        return false;
    g_range = reinterpret_cast<PFN_cuMemGetAddressRange_v3020>(fn);
    return true;
}

bool in_device_allocation(const void* p, size_t bytes) {
    if (bytes == 0) return true;
    if (!p || !g_range) return false;
    CUdeviceptr base = 0;
    size_t size = 0;
    if (g_range(&base, &size, reinterpret_cast<CUdeviceptr>(p)) != CUDA_SUCCESS) return false;
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    if (a < base || a - base > size) return false;
    return bytes <= size - (a - base);
}

// A wait that is never satisfied: exercises the bounded-wait timeout path and the error flag.
__global__ void timeout_probe_kernel(int* err_flag, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar, 1);
        abort_flag = 0;
        ptx::fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) ptx::mbar_wait(&bar, 0, &abort_flag, limit_ns, err_flag);
    __syncthreads();
}

// Kernel kinds for launch accounting / profiling.
enum Kind { kPack = 0, kBaseFwd, kShrinkX, kExpandY, kBaseDx, kShrinkDy, kExpandDx, kWgradB, kWgradA,
            kSimt, kAdamw, kShrinkDyWgradB, kStage, kBaseDxWgradA, kKinds };
const char* const kKindNames[kKinds] = {"pack_ab", "base_fwd", "shrink_x", "expand_y", "base_dx",
                                        "shrink_dy", "expand_dx", "wgrad_b", "wgrad_a", "simt_gemm", "adamw",
                                        "shrink_dy+wgrad_b", "stage_copy", "base_dx+wgrad_a"};

cudaEvent_t take_event(plora_ctx* h) {
    if (!h->pool.empty()) {
        cudaEvent_t e = h->pool.back();
        h->pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

// Bracket one launch: record a start event (when profiling), run `launch`, record the end event.
template <typename F>
void tracked(plora_ctx* h, int kind, cudaStream_t st, F&& launch) {
    h->launches[kind] += 1;
    if (!h->profiling || h->in_capture) {
        launch();
        return;
    }
    plora_ctx::Rec r{kind, take_event(h), take_event(h)};
    cudaEventRecord(r.a, st);
    launch();
    cudaEventRecord(r.b, st);
    h->pending.push_back(r);
}

// 2-D bf16 tensor map, 128-byte swizzle, out-of-bounds elements read as zero.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_elems,
              uint32_t box_inner, uint32_t box_outer) {
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_elems * 2};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------
// Per-call schedule
// ---------------------------------------------------------------------------
struct HostPlan {
    int32_t n = 0, RP = kRankAlign;
    int64_t T = 0, h_rows = 0;
    std::vector<AdapterDev> ad;
    std::vector<TokTile> tok;
    std::vector<RedEntry> red;
    std::vector<int32_t> empty;    // adapters with no tokens
    std::vector<int32_t> mt_off;   // per global 128-row tile: first entry in mt_seg (+ end)
    std::vector<MTileRec> mt_rec;  // per global 128-row tile: the range, first two entries inlined
    std::vector<LoraSeg> mt_seg;   // adapters overlapping each global tile
    int32_t slots = 0, counters = 0;
};

plora_status check_table(plora_ctx* h, int32_t n, const int64_t* off, const plora_adapter* tab, bool grads) {
    if (n < 0 || n > h->cfg.max_adapters)
        return fail(h, PLORA_ERR_INVALID_ARG, "n_adapters=%d outside [0, max_adapters=%d]", n, h->cfg.max_adapters);
    if (!off) return fail(h, PLORA_ERR_INVALID_ARG, "off is NULL");
    if (n > 0 && !tab) return fail(h, PLORA_ERR_INVALID_ARG, "adapter table is NULL");
    if (off[0] != 0) return fail(h, PLORA_ERR_INVALID_ARG, "off[0]=%lld, must be 0", (long long)off[0]);
    for (int32_t i = 0; i < n; ++i) {
        if (off[i + 1] < off[i])
            return fail(h, PLORA_ERR_INVALID_ARG, "offsets decrease at adapter %d (%lld > %lld)", i,
                        (long long)off[i], (long long)off[i + 1]);
    }
    if (off[n] > h->cfg.max_tokens)
        return fail(h, PLORA_ERR_INVALID_ARG, "off[n]=%lld exceeds max_tokens=%lld", (long long)off[n],
                    (long long)h->cfg.max_tokens);
    for (int32_t i = 0; i < n; ++i) {
        const plora_adapter& a = tab[i];
        if (a.rank < 1 || a.rank > h->cfg.max_rank)
            return fail(h, PLORA_ERR_INVALID_ARG, "adapter %d: rank %d outside [1, max_rank=%d]", i, a.rank,
                        h->cfg.max_rank);
        if (!std::isfinite(a.scale)) return fail(h, PLORA_ERR_INVALID_ARG, "adapter %d: scale is not finite", i);
        if (!a.A || !a.B) return fail(h, PLORA_ERR_INVALID_ARG, "adapter %d: A or B is NULL", i);
        if (!aligned16(a.A) || !aligned16(a.B))
            return fail(h, PLORA_ERR_INVALID_ARG, "adapter %d: A or B not 16-byte aligned", i);
        if (grads) {
            if (!a.dA || !a.dB) return fail(h, PLORA_ERR_INVALID_ARG, "adapter %d: dA or dB is NULL", i);
            if (!aligned16(a.dA) || !aligned16(a.dB))
                return fail(h, PLORA_ERR_INVALID_ARG, "adapter %d: dA or dB not 16-byte aligned", i);
        }
    }
    return PLORA_OK;
}

void build_plan(const plora_ctx* h, int32_t n, const int64_t* off, const plora_adapter* tab, HostPlan& P) {
    P.n = n;
    P.T = off[n];
    int maxr = 1;
    for (int32_t i = 0; i < n; ++i) maxr = std::max(maxr, tab[i].rank);
    P.RP = (int32_t)round_up(h->nblk * round_up(maxr, 16), kRankAlign);   // the widest adapter's P rblk
    P.ad.resize(n);
    int64_t hrow = 0;
    const int64_t dtiles = std::max(ceil_div(h->cfg.d_in, kTileM), ceil_div(h->cfg.d_out, kTileM));
    for (int32_t i = 0; i < n; ++i) {
        AdapterDev& a = P.ad[i];
        a.A = tab[i].A;
        a.B = tab[i].B;
        a.dA = tab[i].dA;
        a.dB = tab[i].dB;
        a.x_row = (int32_t)off[i];
        a.n = (int32_t)(off[i + 1] - off[i]);
        a.h_row = (int32_t)hrow;
        a.rank = tab[i].rank;
        a.scale = tab[i].scale;
        a.rblk = (int32_t)round_up(a.rank, 16);
        a.rp16 = h->nblk * a.rblk;
        a.rp64 = (int32_t)round_up(a.rp16, 64);
        if (a.n == 0) {
            P.empty.push_back(i);
            continue;
        }
        // H' / G block: 128 zero rows, the adapter's rows rounded up to 128, 128 zero rows.
        a.h_row = (int32_t)(hrow + kLoraPad);
        hrow += round_up(a.n, kTileM) + 2 * kLoraPad;
        for (int32_t t = 0; t < a.n; t += kTileM)
            P.tok.push_back(TokTile{i, std::min(kTileM, a.n - t), a.x_row + t, a.h_row + t});
        // Weight-gradient splits: a function of this adapter's token count alone, so an
        // adapter's dA/dB do not depend on what else is packed with it.
        const int32_t nsplit = (int32_t)ceil_div(a.n, kSplitTokens);
        const int32_t slot = nsplit > 1 ? P.slots : -1;
        const int32_t cnt = nsplit > 1 ? P.counters : -1;
        if (nsplit > 1) {
            P.slots += nsplit;
            P.counters += (int32_t)dtiles;
        }
        for (int32_t s = 0; s < nsplit; ++s) {
            const int32_t t0 = s * kSplitTokens;
            const int32_t len = std::min(kSplitTokens, a.n - t0);
            P.red.push_back(RedEntry{i, a.x_row + t0, a.h_row + t0, (int32_t)ceil_div(len, kBlockK), s, nsplit,
                                     slot, cnt});
        }
    }
    P.h_rows = hrow;
    // Adapters overlapping each global 128-row tile (for the base GEMMs with the low-rank branch folded in).
    const int64_t tiles_m = ceil_div(P.T, kLoraTileM);
    P.mt_off.assign(tiles_m + 1, 0);
    int32_t first = 0;
    for (int64_t mb = 0; mb < tiles_m; ++mb) {
        const int64_t m0 = mb * kLoraTileM, m1 = std::min<int64_t>(P.T, m0 + kLoraTileM);
        P.mt_off[mb] = (int32_t)P.mt_seg.size();
        while (first < n && off[first + 1] <= m0) ++first;
        for (int32_t j = first; j < n && off[j] < m1; ++j)
            if (off[j + 1] > off[j])
                P.mt_seg.push_back(LoraSeg{j, (int32_t)(P.ad[j].h_row + (m0 - off[j])), P.ad[j].rp16, P.ad[j].rblk});
    }
    P.mt_off[tiles_m] = (int32_t)P.mt_seg.size();
    P.mt_rec.assign(tiles_m, MTileRec{});
    for (int64_t mb = 0; mb < tiles_m; ++mb) {
        MTileRec& r = P.mt_rec[mb];
        r.q0 = P.mt_off[mb];
        r.q1 = P.mt_off[mb + 1];
        for (int k = 0; k < 2 && r.q0 + k < r.q1; ++k) r.s[k] = P.mt_seg[r.q0 + k];
    }
    // Longest-first order of the weight-gradient work (the static persistent schedule
    // then deals items round-robin over the SMs).
    std::stable_sort(P.red.begin(), P.red.end(),
                     [](const RedEntry& a, const RedEntry& b) { return a.kblocks > b.kblocks; });
}

// The `saved` buffer a forward fills and the backward reads: the zero-padded blocks of H' = s X A
// ([h_rows][RP], at offset 0), then on the tensor-core path the packed factors of the call (packA
// [n RP][d_in] and packB [n][d_out][RP], see pack_ab_kernel), each from a 256-byte boundary.
struct SavedLayout {
    size_t o_packA = 0, o_packB = 0, bytes = 0;
};

SavedLayout saved_layout(const plora_ctx* h, const HostPlan& P) {
    SavedLayout L;
    const size_t hb = (size_t)P.h_rows * (size_t)P.RP * h->esize;
    if (!h->tc) {
        L.bytes = hb;
        return L;
    }
    L.o_packA = (size_t)round_up((int64_t)hb, 256);
    L.o_packB = L.o_packA + (size_t)round_up((int64_t)P.n * P.RP * h->cfg.d_in * 2, 256);
    L.bytes = L.o_packB + (size_t)P.n * (size_t)h->cfg.d_out * (size_t)P.RP * 2;
    return L;
}

size_t saved_bytes_of(const plora_ctx* h, const HostPlan& P) { return saved_layout(h, P).bytes; }

// Extents of every tensor a call reads or writes (see include/plora.h for the layouts).
struct TensorArgs {
    const void* X = nullptr;
    const void* W = nullptr;
    const void* Y = nullptr;
    const void* dY = nullptr;
    const void* dX = nullptr;
    const void* saved = nullptr;
    bool adapters_AB = true;   // check each A_i, B_i
    bool adapters_dA = false;  // check each dA_i
    bool adapters_dB = false;  // check each dB_i
};

plora_status check_extents(plora_ctx* h, const HostPlan& P, const plora_adapter* tab, const TensorArgs& a) {
    if (!get_range_fn()) return fail(h, PLORA_ERR_CUDA, "cuMemGetAddressRange is not available");
    const size_t es = h->esize;
    const size_t T = (size_t)P.T, di = (size_t)h->cfg.d_in, dout = (size_t)h->cfg.d_out;
    struct Item { const void* p; size_t bytes; const char* name; };
    const Item items[] = {{a.X, T * di * es, "X"}, {a.W, dout * di * es, "W"}, {a.Y, T * dout * es, "Y"},
                          {a.dY, T * dout * es, "dY"}, {a.dX, T * di * es, "dX"},
                          {a.saved, T ? saved_bytes_of(h, P) : 0, "saved"}};
    for (const Item& it : items)
        if (it.p && !in_device_allocation(it.p, it.bytes))
            return fail(h, PLORA_ERR_INVALID_ARG, "%s is not a device buffer of %zu bytes", it.name, it.bytes);
    for (int32_t i = 0; i < P.n; ++i) {
        const size_t r = (size_t)tab[i].rank;
        const size_t ra = r * (size_t)h->nblk;   // rows of A and dA: one rank-r block per output block
        if (a.adapters_AB && (!in_device_allocation(tab[i].A, ra * di * es) ||
                              !in_device_allocation(tab[i].B, dout * r * es)))
            return fail(h, PLORA_ERR_INVALID_ARG, "adapter %d: A or B is not a device buffer of its size", i);
        if (a.adapters_dA && !in_device_allocation(tab[i].dA, ra * di * sizeof(float)))
            return fail(h, PLORA_ERR_INVALID_ARG, "adapter %d: dA is not a device buffer of its size", i);
        if (a.adapters_dB && !in_device_allocation(tab[i].dB, dout * r * sizeof(float)))
            return fail(h, PLORA_ERR_INVALID_ARG, "adapter %d: dB is not a device buffer of its size", i);
    }
    return PLORA_OK;
}

// Copy the plan blob to the device through the staging ring. Returns device pointers.
// Item counters of the launches that claim their second op's items (GroupParams::dyn): the
// backward's shrink of G with dB, and its dX GEMM with dA.
constexpr int kDynCounters = 4;
constexpr int kDynShrinkDyWgradB = 0;
constexpr int kDynBaseDxWgradA = 1;

struct DevPlan {
    AdapterDev* ad = nullptr;
    TokTile* tok = nullptr;
    RedEntry* red = nullptr;
    SimtOp* ops = nullptr;
    MTileRec* mt_rec = nullptr;
    LoraSeg* mt_seg = nullptr;
    int32_t* dyn = nullptr;   // kDynCounters item counters, zero when the call's launches start
    int slot = 0;
};

// Copies calls' schedules from their slots' mapped pinned staging buffers into device memory, one
// copy per blockIdx.y.  A kernel rather than cudaMemcpyAsync: its reads of host memory do not wait in
// the copy-engine queue behind bulk host-to-device copies that the caller may have in flight (the next
// step's inputs, say).
struct StageCopies {
    int32_t n;
    int32_t pad_;
    const uint4* src[kMaxSeg];
    uint4* dst[kMaxSeg];
    int64_t n16[kMaxSeg];
    int64_t cap16[kMaxSeg];        // 16-byte words of each destination region
    int* err_flag;
};

__global__ void stage_copy_kernel(const __grid_constant__ StageCopies cs) {
    const int k = blockIdx.y;
    if (k >= cs.n || !dcheck(cs.err_flag, cs.n16[k] <= cs.cap16[k])) return;
    const uint4* __restrict__ src = cs.src[k];
    uint4* __restrict__ dst = cs.dst[k];
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < cs.n16[k]; i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = src[i];
}

// One launch copying every schedule queued in `cs` (device views of the staging in src).
cudaError_t stage_copy_run(plora_ctx* h, const StageCopies& cs, cudaStream_t st) {
    if (cs.n == 0) return cudaSuccess;
    int64_t most = 0;
    for (int k = 0; k < cs.n; ++k) most = std::max(most, cs.n16[k]);
    const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>(ceil_div(most, 256), 64));
    tracked(h, kStage, st, [&] { stage_copy_kernel<<<dim3((unsigned)blocks, (unsigned)cs.n), 256, 0, st>>>(cs); });
    return cudaGetLastError();
}

// Queues `bytes` of staging (device view `src`) for the device region at d (rounded up to 16 bytes;
// the staging and the device region are both whole multiples of 256 bytes).
void stage_copy_add(plora_ctx* h, StageCopies& cs, const uint8_t* src, uint8_t* d, size_t bytes) {
    if (cs.n == 0) cs.err_flag = h->at<int>(h->r_err);
    cs.cap16[cs.n] = (int64_t)(h->blob_bytes / 16);
    cs.src[cs.n] = reinterpret_cast<const uint4*>(src);
    cs.dst[cs.n] = reinterpret_cast<uint4*>(d);
    cs.n16[cs.n] = (int64_t)((bytes + 15) / 16);
    ++cs.n;
}

cudaError_t stage_copy(plora_ctx* h, const uint8_t* src, uint8_t* d, size_t bytes, cudaStream_t st) {
    StageCopies cs{};
    stage_copy_add(h, cs, src, d, bytes);
    return stage_copy_run(h, cs, st);
}

bool stream_capturing(cudaStream_t st) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    return cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive;
}

// The schedule slot of the current call: the next ring slot once its previous use has finished, or,
// while the stream is being captured, the next reserved capture slot (slot index -1 - k).
struct Slot {
    int index = 0;
    uint8_t* host = nullptr;
    const uint8_t* host_dev = nullptr;
    uint8_t* dev = nullptr;
};

plora_status take_slot(plora_ctx* h, cudaStream_t st, Slot& sl) {
    h->in_capture = stream_capturing(st);
    if (h->in_capture) {
        if (h->cap_next >= h->cap.size())
            return fail(h, PLORA_ERR_INVALID_ARG, "the stream is being captured and no reserved schedule slot is "
                        "left (plora_capture_reserve before the capture)");
        const plora_ctx::CaptureSlot& c = h->cap[h->cap_next];
        sl.index = -1 - (int)h->cap_next;
        ++h->cap_next;
        sl.host = c.host;
        sl.host_dev = c.host_dev;
        sl.dev = c.dev;
        return PLORA_OK;
    }
    const int slot = h->next_slot;
    h->next_slot = (h->next_slot + 1) % kSlots;
    cudaError_t e = cudaEventSynchronize(h->ev[slot]);
    if (e != cudaSuccess) return cuda_fail(h, e, "cudaEventSynchronize(staging slot)");
    sl.index = slot;
    sl.host = h->h_blob[slot];
    sl.host_dev = h->h_blob_dev[slot];
    sl.dev = h->at<uint8_t>(h->r_blob[slot]);
    return PLORA_OK;
}

// With `defer`, the copy is queued there instead of launched (a layer call stages every projection's
// schedule with one launch).
plora_status upload(plora_ctx* h, const HostPlan& P, const std::vector<SimtOp>& ops, cudaStream_t st,
                    DevPlan& D, StageCopies* defer = nullptr) {
    Slot sl;
    plora_status ps = take_slot(h, st, sl);
    if (ps != PLORA_OK) return ps;
    size_t o = 0;
    auto put = [&](const void* src, size_t bytes) {
        const size_t at = o;
        if (bytes) memcpy(sl.host + at, src, bytes);
        o = round_up((int64_t)(o + bytes), 256);
        return at;
    };
    const size_t o_ad = put(P.ad.data(), P.ad.size() * sizeof(AdapterDev));
    const size_t o_tok = put(P.tok.data(), P.tok.size() * sizeof(TokTile));
    const size_t o_red = put(P.red.data(), P.red.size() * sizeof(RedEntry));
    const size_t o_ops = put(ops.data(), ops.size() * sizeof(SimtOp));
    const size_t o_mto = put(P.mt_rec.data(), P.mt_rec.size() * sizeof(MTileRec));
    const size_t o_mtl = put(P.mt_seg.data(), P.mt_seg.size() * sizeof(LoraSeg));
    const int32_t zeros[kDynCounters] = {};
    const size_t o_dyn = put(zeros, sizeof(zeros));   // the schedule copy clears the item counters
    if (o > h->blob_bytes) return fail(h, PLORA_ERR_INVALID_ARG, "schedule exceeds the handle's staging size");
    uint8_t* d = sl.dev;
    if (defer) {
        stage_copy_add(h, *defer, sl.host_dev, d, o);
    } else {
        cudaError_t e = stage_copy(h, sl.host_dev, d, o, st);
        if (e != cudaSuccess) return cuda_fail(h, e, "copying the schedule to the device");
    }
    D.ad = reinterpret_cast<AdapterDev*>(d + o_ad);
    D.tok = reinterpret_cast<TokTile*>(d + o_tok);
    D.red = reinterpret_cast<RedEntry*>(d + o_red);
    D.ops = reinterpret_cast<SimtOp*>(d + o_ops);
    D.mt_rec = reinterpret_cast<MTileRec*>(d + o_mto);
    D.mt_seg = reinterpret_cast<LoraSeg*>(d + o_mtl);
    D.dyn = reinterpret_cast<int32_t*>(d + o_dyn);
    D.slot = sl.index;
    return PLORA_OK;
}

// Copy two host arrays to the device through the staging ring (same slot discipline as upload()).
plora_status upload_parts(plora_ctx* h, const void* a, size_t na, const void* b, size_t nb, cudaStream_t st,
                          uint8_t** da, uint8_t** db, int* slot_out) {
    const size_t ob = (size_t)round_up((int64_t)na, 256);
    const size_t total = ob + nb;
    if (total > h->blob_bytes) return fail(h, PLORA_ERR_INVALID_ARG, "optimizer tables exceed the staging size");
    Slot sl;
    plora_status ps = take_slot(h, st, sl);
    if (ps != PLORA_OK) return ps;
    if (na) memcpy(sl.host, a, na);
    if (nb) memcpy(sl.host + ob, b, nb);
    uint8_t* d = sl.dev;
    cudaError_t e = stage_copy(h, sl.host_dev, d, total, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "copying the optimizer tables to the device");
    *da = d;
    *db = d + ob;
    *slot_out = sl.index;
    return PLORA_OK;
}

plora_status finish(plora_ctx* h, const DevPlan& D, cudaStream_t st) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(h, e, "kernel launch");
    if (D.slot >= 0) {   // a ring slot: its event guards reuse (a capture slot is never reused)
        e = cudaEventRecord(h->ev[D.slot], st);
        if (e != cudaSuccess) return cuda_fail(h, e, "cudaEventRecord");
    }
    return PLORA_OK;
}

// ---------------------------------------------------------------------------
// SIMT ops
// ---------------------------------------------------------------------------
void add_op(std::vector<SimtOp>& ops, int32_t& tiles, const void* A, int64_t a_sm, int64_t a_sk, const void* B,
            int64_t b_sk, int64_t b_sn, void* C, int64_t c_sm, int64_t c_sn, int64_t M, int64_t N, int64_t K,
            float alpha, bool acc, bool c_fp32) {
    if (M <= 0 || N <= 0) return;
    SimtOp o{};
    o.A = A; o.B = B; o.C = C;
    o.a_sm = a_sm; o.a_sk = a_sk; o.b_sk = b_sk; o.b_sn = b_sn; o.c_sm = c_sm; o.c_sn = c_sn;
    o.M = (int32_t)M; o.N = (int32_t)N; o.K = (int32_t)K;
    o.alpha = alpha;
    o.accumulate = acc ? 1 : 0;
    o.c_fp32 = c_fp32 ? 1 : 0;
    o.tile_begin = tiles;
    o.tiles_n = (int32_t)ceil_div(N, 64);
    tiles += (int32_t)(ceil_div(M, 64) * o.tiles_n);
    ops.push_back(o);
}

template <typename T>
void launch_simt(plora_ctx* h, const SimtOp* d_ops, int n_ops, int tiles, cudaStream_t st) {
    if (tiles > 0)
        tracked(h, kSimt, st, [&] { simt_gemm_kernel<T><<<tiles, 256, 0, st>>>(d_ops, n_ops); });
}

// ---------------------------------------------------------------------------
// Tensor-core launches
// ---------------------------------------------------------------------------
struct SegMaps {
    const CUtensorMap *a, *b, *a2, *b2, *c;
};

// Appends a segment of the first op (op2 = false) or of the second (op2 = true).
void seg_add(Segments& S, const TcParams& p, const SegMaps& mp, bool op2) {
    const CUtensorMap* src[5] = {mp.a, mp.b, mp.a2 ? mp.a2 : mp.a, mp.b2 ? mp.b2 : mp.a, mp.c ? mp.c : mp.a};
    if (op2) {
        for (int k = 0; k < 5; ++k) S.m2[S.n_op2][k] = *src[k];
        S.p2[S.n_op2++] = p;
    } else {
        for (int k = 0; k < 5; ++k) S.m.m[S.g.n_op1][k] = *src[k];
        S.g.p[S.g.n_op1++] = p;
    }
}

// Orders the segments (first op's, then second op's), sets the item ranges; returns the item count.
int seg_finish(Segments& S) {
    S.g.n_seg = S.g.n_op1 + S.n_op2;
    for (int j = 0; j < S.n_op2; ++j) {
        S.g.p[S.g.n_op1 + j] = S.p2[j];
        for (int k = 0; k < 5; ++k) S.m.m[S.g.n_op1 + j][k] = S.m2[j][k];
    }
    S.g.begin[0] = 0;
    for (int j = 0; j < S.g.n_seg; ++j) S.g.begin[j + 1] = S.g.begin[j] + std::max(0, S.g.p[j].num_tiles);
    return S.g.begin[S.g.n_seg];
}

template <Op OP, Op OP2 = OP>
cudaError_t launch_segments(Segments& S, int num_sms, cudaStream_t st) {
    const int total = seg_finish(S);
    if (total <= 0) return cudaSuccess;
    tc_kernel<OP, OP2><<<std::min(total, num_sms), kTcThreads, kTcSmemBytes, st>>>(S.m, S.g);
    return cudaGetLastError();
}

// c: the output tensor map of a base GEMM (TMA-stored epilogue); other ops ignore it.
template <Op OP>
void launch_tc(plora_ctx* h, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& a2, const CUtensorMap& b2,
               const CUtensorMap& c, const TcParams& p, cudaStream_t st) {
    if (p.num_tiles <= 0) return;
    constexpr int kind = OP == Op::BaseFwd ? kBaseFwd : OP == Op::BaseDx ? kBaseDx : OP == Op::ShrinkX ? kShrinkX
                       : OP == Op::ShrinkDy ? kShrinkDy : OP == Op::ExpandY ? kExpandY : OP == Op::ExpandDx ? kExpandDx
                       : OP == Op::WgradB ? kWgradB : kWgradA;
    Segments& S = *h->segs;
    S = Segments{};
    seg_add(S, p, SegMaps{&a, &b, &a2, &b2, &c}, false);
    tracked(h, kind, st, [&] { launch_segments<OP>(S, h->num_sms, st); });
}

// Two independent ops in one persistent launch: OP's items (operands a, b; a base GEMM's fold a2, b2
// and output c) then OP2's (a3, b3).
template <Op OP, Op OP2>
void launch_tc2(plora_ctx* h, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& a2,
                const CUtensorMap& b2, const CUtensorMap& c, const CUtensorMap& a3, const CUtensorMap& b3,
                const TcParams& p, const TcParams& p2, int kind, cudaStream_t st) {
    if (p.num_tiles + p2.num_tiles <= 0) return;
    Segments& S = *h->segs;
    S = Segments{};
    seg_add(S, p, SegMaps{&a, &b, &a2, &b2, &c}, false);
    seg_add(S, p2, SegMaps{&a3, &b3, nullptr, nullptr, nullptr}, true);
    tracked(h, kind, st, [&] { launch_segments<OP, OP2>(S, h->num_sms, st); });
}

// Base GEMMs on SM pairs: a cluster of two CTAs per 256x256 tile, persistent over the pairs that
// can be resident at once (a GPC with an odd number of free SMs leaves one unpaired).
template <Op OP>
cudaLaunchConfig_t pair_config(int pairs, cudaStream_t st, cudaLaunchAttribute* attr) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(2 * pairs));
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = kTcSmemBytes;
    cfg.stream = st;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

template <Op OP>
void launch_pair(plora_ctx* h, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& a2,
                 const CUtensorMap& b2, const CUtensorMap& c, const TcParams& p, cudaStream_t st) {
    if (p.num_tiles <= 0) return;
    const int resident = OP == Op::BaseFwd ? h->pairs_fwd : h->pairs_dx;
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = pair_config<OP>(std::min(p.num_tiles, resident), st, attr);
    constexpr int kind = OP == Op::BaseFwd ? kBaseFwd : kBaseDx;
    tracked(h, kind, st, [&] { cudaLaunchKernelEx(&cfg, tc_pair_kernel<OP>, a, b, a2, b2, c, p); });
}

template <Op OP>
cudaError_t pair_setup(int& pairs) {
    cudaError_t e = cudaFuncSetAttribute(tc_pair_kernel<OP>, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tc_pair_kernel<OP>, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = pair_config<OP>(1, nullptr, attr);
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, tc_pair_kernel<OP>, &cfg);
    if (e != cudaSuccess) return e;
    pairs = clusters;
    return pairs > 0 ? cudaSuccess : cudaErrorInvalidConfiguration;
}

// Pair-tile parameters of a base GEMM over T rows: 256-row m-tiles, 32 KB stages, a 6-deep ring.
void pair_params(TcParams& p, int64_t T, int64_t N, int window_rows) {
    p.tiles_m = (int32_t)ceil_div(T, 2 * kTileM);
    p.tiles_n = (int32_t)ceil_div(N, kTileN);
    p.num_tiles = p.tiles_m * p.tiles_n;
    p.group_m = std::max(1, window_rows / (2 * kTileM));   // the row window in 256-row pair tiles
    p.stage_bytes = kPairStageBytes;
    p.stages = std::min(kMaxStages, kRingBytes / kPairStageBytes);
}

// A deeper operand ring for ops whose B tile is narrower than 256 rows: A tile + RP rows of B.
void narrow_ring(TcParams& p, int RP) {
    p.stage_bytes = kABytes + RP * kBlockK * 2;
    p.stages = std::min(kMaxStages, kRingBytes / p.stage_bytes);
}

// Tile geometry of a single-SM base GEMM over T rows and N output columns: kBaseRows-row m-tiles, the
// rasterisation window in those tiles, and the ring layout of that tile (three 64 KB stages for
// 256-row tiles).
void base_tiles(TcParams& p, int64_t T, int64_t N, int window_rows) {
    p.tiles_m = (int32_t)ceil_div(T, kBaseRows);
    p.tiles_n = (int32_t)ceil_div(N, kTileN);
    p.num_tiles = p.tiles_m * p.tiles_n;
    p.group_m = std::max(1, window_rows / kBaseRows);
    if (kBaseRows == 256) {
        p.stages = kWideStages;
        p.stage_bytes = kWideStageBytes;
    }
}

template <Op OP, Op OP2 = OP>
cudaError_t set_tc_attr() {
    return cudaFuncSetAttribute(tc_kernel<OP, OP2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmemBytes);
}

TcParams base_params(const plora_ctx* h, const HostPlan& P, const DevPlan& D) {
    TcParams p{};
    p.RP = P.RP;
    p.adapters = D.ad;
    p.tok = D.tok;
    p.red = D.red;
    p.err_flag = h->at<int>(h->r_err);
    p.timeout_ns = kTimeoutNs;
    p.partials = h->at<float>(h->r_part);
    p.counters = h->at<int32_t>(h->r_cnt);
    p.mt_rec = D.mt_rec;
    p.mt_seg = D.mt_seg;
    p.fuse = 0;
    p.stages = kStages;
    p.stage_bytes = kStageBytes;
    p.nblk = h->nblk;
    for (int b = 0; b < kMaxOutBlocks; ++b) p.blk_end[b] = h->blk_end[b];
    p.part_elems = (int64_t)(h->r_part.bytes / sizeof(float));
    p.n_counters = (int32_t)(h->r_cnt.bytes / sizeof(int32_t));
    p.n_adapters = P.n;
    p.n_mtrec = (int32_t)P.mt_rec.size();
    p.n_mtseg = (int32_t)P.mt_seg.size();
    return p;
}

// Packs every adapter's A and B into the saved buffer in the layouts the tensor-core operands want
// (pack_ab_kernel), once per forward; the backward reads the same packs.  pack_job describes one
// call's pack; pack_run launches one grid over every queued job.
PackJob pack_job(plora_ctx* h, const HostPlan& P, const DevPlan& D, void* saved) {
    const SavedLayout L = saved_layout(h, P);
    uint8_t* sv = static_cast<uint8_t*>(saved);
    PackJob J{};
    J.ad = D.ad;
    J.packA = reinterpret_cast<__nv_bfloat16*>(sv + L.o_packA);
    J.packB = reinterpret_cast<__nv_bfloat16*>(sv + L.o_packB);
    J.d_in = h->cfg.d_in;
    J.d_out = h->cfg.d_out;
    J.packA_elems = (int64_t)((L.o_packB - L.o_packA) / 2);
    J.packB_elems = (int64_t)((L.bytes - L.o_packB) / 2);
    J.n = P.n;
    J.RP = P.RP;
    J.blocks.n = h->nblk;
    for (int b = 0; b < kMaxOutBlocks; ++b) J.blocks.end[b] = h->blk_end[b];
    J.err_flag = h->at<int>(h->r_err);
    return J;
}

// Chunks of the largest adapter of a job (sizes the grid's x extent).
int64_t pack_chunks(const plora_ctx* h, const HostPlan& P) {
    int64_t most = 1;
    for (const AdapterDev& a : P.ad)
        most = std::max<int64_t>(most, (int64_t)a.rp16 * (h->cfg.d_in / 8) + h->cfg.d_out * (a.rp16 / 8));
    return most;
}

void pack_run(plora_ctx* h, const PackJobs& jobs, int64_t most_chunks, int most_adapters, cudaStream_t st) {
    if (jobs.n == 0 || most_adapters == 0) return;
    const int gx = (int)std::min<int64_t>(ceil_div(most_chunks, 256), 1024);
    tracked(h, kPack, st, [&] {
        pack_ab_kernel<<<dim3((unsigned)gx, (unsigned)most_adapters, (unsigned)jobs.n), 256, 0, st>>>(jobs);
    });
}


// 3-D bf16 tensor map of the B pack [n][d_out][RP] (rank column innermost), 128-byte swizzle, a box of
// 64 columns x box_rows rows of one adapter; rows past d_out read as zero.
bool make_packb_map(CUtensorMap* m, const void* base, uint64_t RP, uint64_t d_out, uint64_t n, uint32_t box_rows) {
    cuuint64_t dims[3] = {RP, d_out, n};
    cuuint64_t strides[2] = {RP * 2, d_out * RP * 2};
    cuuint32_t box[3] = {64, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The argument checks of a forward (everything before the first enqueue); builds the call's plan.
plora_status fwd_args(plora_ctx* h, const void* X, const void* W, const void* Y, int32_t n, const int64_t* off,
                      const plora_adapter* tab, const void* saved, HostPlan& P) {
    plora_status s = check_table(h, n, off, tab, false);
    if (s != PLORA_OK) return s;
    const bool any_tokens = off[n] > 0;   // with no tokens, X, Y and saved are never touched
    if (!W || (any_tokens && (!X || !Y || !saved)))
        return fail(h, PLORA_ERR_INVALID_ARG, "X, W, Y or saved is NULL");
    if (!aligned16(X) || !aligned16(W) || !aligned16(Y))
        return fail(h, PLORA_ERR_INVALID_ARG, "X, W or Y not 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(saved) & 255u) != 0)
        return fail(h, PLORA_ERR_INVALID_ARG, "saved not 256-byte aligned");
    cudaError_t ce = cudaSetDevice(h->device);
    if (ce != cudaSuccess) return cuda_fail(h, ce, "cudaSetDevice");
    build_plan(h, n, off, tab, P);
    if (P.T == 0) return PLORA_OK;
    TensorArgs ta;
    ta.X = X; ta.W = W; ta.Y = Y; ta.saved = saved;
    return check_extents(h, P, tab, ta);
}

// The argument checks of a backward; builds the call's plan.
plora_status bwd_args(plora_ctx* h, const void* X, const void* W, const void* dY, const void* dX, int32_t n,
                      const int64_t* off, const plora_adapter* tab, const void* saved, HostPlan& P) {
    plora_status s = check_table(h, n, off, tab, true);
    if (s != PLORA_OK) return s;
    const bool any_tokens = off[n] > 0;   // with no tokens, only dA and dB are written (zeros)
    if (!W || (any_tokens && (!X || !dY || !saved)))
        return fail(h, PLORA_ERR_INVALID_ARG, "X, W, dY or saved is NULL");
    if (!aligned16(X) || !aligned16(W) || !aligned16(dY) || (dX && !aligned16(dX)))
        return fail(h, PLORA_ERR_INVALID_ARG, "X, W, dY or dX not 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(saved) & 255u) != 0)
        return fail(h, PLORA_ERR_INVALID_ARG, "saved not 256-byte aligned");
    cudaError_t ce = cudaSetDevice(h->device);
    if (ce != cudaSuccess) return cuda_fail(h, ce, "cudaSetDevice");
    build_plan(h, n, off, tab, P);
    TensorArgs ta;
    if (P.T > 0) { ta.X = X; ta.W = W; ta.dY = dY; ta.dX = dX; ta.saved = saved; }
    ta.adapters_AB = P.T > 0;
    ta.adapters_dA = ta.adapters_dB = true;
    return check_extents(h, P, tab, ta);
}

// Adapters without tokens get zero weight gradients (enqueued once every check has passed).
plora_status zero_empty_grads(plora_ctx* h, const HostPlan& P, const plora_adapter* tab, cudaStream_t st) {
    for (int32_t i : P.empty) {
        cudaError_t ce = cudaMemsetAsync(tab[i].dA, 0, (size_t)tab[i].rank * h->nblk * h->cfg.d_in * sizeof(float), st);
        if (ce == cudaSuccess) ce = cudaMemsetAsync(tab[i].dB, 0, (size_t)tab[i].rank * h->cfg.d_out * sizeof(float), st);
        if (ce != cudaSuccess) return cuda_fail(h, ce, "cudaMemsetAsync(dA/dB of an empty adapter)");
    }
    return PLORA_OK;
}

// ---------------------------------------------------------------------------
// Tensor-core calls, prepared one by one and launched together: a single call, or the projections of
// a layer call, whose products of one kind run as one persistent launch over all of them (each
// projection a segment of the launch, with its own parameters and tensor maps).
// ---------------------------------------------------------------------------
struct FwdCall {
    plora_ctx* h = nullptr;
    const void* X = nullptr;
    const void* W = nullptr;
    void* Y = nullptr;
    void* saved = nullptr;
    HostPlan P;
    DevPlan D;
    CUtensorMap mX, mXb, mW, mW128, mPA16, mPA32, mPA64, mPA128, mHk, mHkb, mPBk, mPBk128, mY;
    TcParams q{}, p{};
};

// After the argument checks: stages the call's schedule (queued into cs), encodes its tensor maps and
// fills the parameters of its shrink (q) and base GEMM (p).
plora_status fwd_prepare(FwdCall& c, cudaStream_t st, StageCopies& cs) {
    plora_ctx* h = c.h;
    const HostPlan& P = c.P;
    plora_status s = upload(h, P, {}, st, c.D, &cs);
    if (s != PLORA_OK) return s;
    const int64_t d_in = h->cfg.d_in, d_out = h->cfg.d_out;
    // mPA16 .. mPA128: the A pack in boxes of 16 to 128 rows (the shrink's K-major B, an adapter's rows
    // in at most four copies per k-block); mPBk / mPBk128: the B pack, K-major,
    // 256 rows for the 1-SM tile and the expand, 128 per CTA of an SM pair; mXb / mHkb: X and H' in
    // boxes of a 1-SM base tile's rows.
    const SavedLayout L = saved_layout(h, P);
    const uint8_t* sv = static_cast<const uint8_t*>(c.saved);
    bool ok = make_map(&c.mX, c.X, d_in, P.T, d_in, 64, kTileM) &&
              make_map(&c.mY, c.Y, d_out, P.T, d_out, 64, 32) &&
              make_map(&c.mW, c.W, d_in, d_out, d_in, 64, kTileN) &&
              make_map(&c.mW128, c.W, d_in, d_out, d_in, 64, kTileM) &&
              make_map(&c.mPA16, sv + L.o_packA, d_in, (uint64_t)P.n * P.RP, d_in, 64, 16) &&
              make_map(&c.mPA32, sv + L.o_packA, d_in, (uint64_t)P.n * P.RP, d_in, 64, 32) &&
              make_map(&c.mPA64, sv + L.o_packA, d_in, (uint64_t)P.n * P.RP, d_in, 64, 64) &&
              make_map(&c.mPA128, sv + L.o_packA, d_in, (uint64_t)P.n * P.RP, d_in, 64, 128) &&
              make_map(&c.mHk, c.saved, P.RP, P.h_rows, P.RP, 64, kTileM) &&
              make_map(&c.mXb, c.X, d_in, P.T, d_in, 64, kBaseRows) &&
              make_map(&c.mHkb, c.saved, P.RP, P.h_rows, P.RP, 64, kBaseRows) &&
              make_packb_map(&c.mPBk, sv + L.o_packB, P.RP, d_out, P.n, kTileN) &&
              make_packb_map(&c.mPBk128, sv + L.o_packB, P.RP, d_out, P.n, kTileM);
    if (!ok) return fail(h, PLORA_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    // K2: H'_i = s_i X_i A_i per 128-token tile (into the zero-padded blocks of `saved`).
    TcParams& q = c.q;
    q = base_params(h, P, c.D);
    q.K_total = (int32_t)d_in;
    q.num_tiles = (int32_t)P.tok.size();
    q.out = c.saved; q.out_ld = P.RP;
    q.out_elems = P.h_rows * P.RP;
    q.n_items = (int32_t)P.tok.size();
    // K1 (+K3): Y = X W over all packed tokens; fused, each tile also accumulates H'_j B_j of every
    // adapter j overlapping it, so Y is written once.
    TcParams& p = c.p;
    p = base_params(h, P, c.D);
    p.M_total = (int32_t)P.T; p.N_total = (int32_t)d_out; p.K_total = (int32_t)d_in;
    base_tiles(p, P.T, d_out, kWindowRows);
    p.b_box_rows = kTileN;
    p.out = c.Y; p.out_ld = d_out;
    p.fuse = (h->cfg.flags & PLORA_FLAG_UNFUSED) ? 0 : 1;
    return PLORA_OK;
}

// The calls in decreasing order of their K (the cost of one work item of a given kind): items are dealt
// round-robin in segment order, so the longest come first and the last wave holds the shortest.  The
// order changes no result: every item is computed on its own.
template <typename C, typename F>
std::vector<int> by_k(const C* calls, int nc, F k_of) {
    std::vector<int> o(nc);
    for (int k = 0; k < nc; ++k) o[k] = k;
    std::stable_sort(o.begin(), o.end(), [&](int a, int b) { return k_of(calls[a]) > k_of(calls[b]); });
    return o;
}

// The forward of every prepared call: one schedule copy, one pack, one shrink launch, one base-GEMM
// launch per call (the SM-pair and unfused variants, single calls only, keep their own launches).
plora_status fwd_launch(FwdCall* calls, int nc, cudaStream_t st, StageCopies& cs) {
    plora_ctx* h0 = calls[0].h;
    cudaError_t e = stage_copy_run(h0, cs, st);
    if (e != cudaSuccess) return cuda_fail(h0, e, "copying the schedule to the device");
    PackJobs jobs{};
    int64_t most = 1;
    int most_n = 0, RPmax = kRankAlign;
    for (int k = 0; k < nc; ++k) {
        FwdCall& c = calls[k];
        jobs.j[jobs.n++] = pack_job(c.h, c.P, c.D, c.saved);
        most = std::max(most, pack_chunks(c.h, c.P));
        most_n = std::max(most_n, c.P.n);
        RPmax = std::max(RPmax, c.P.RP);
    }
    pack_run(h0, jobs, most, most_n, st);
    Segments& S = *h0->segs;
    S = Segments{};
    const std::vector<int> order = by_k(calls, nc, [](const FwdCall& c) { return c.p.K_total; });
    for (int k : order) {   // one narrow ring that holds every call's widest B tile
        FwdCall& c = calls[k];
        narrow_ring(c.q, RPmax);
        seg_add(S, c.q, SegMaps{&c.mX, &c.mPA16, &c.mPA32, &c.mPA64, &c.mPA128}, false);
    }
    tracked(h0, kShrinkX, st, [&] { launch_segments<Op::ShrinkX>(S, h0->num_sms, st); });
    const uint32_t flags = h0->cfg.flags;
    if (nc == 1 && (flags & (PLORA_FLAG_BASE_PAIR | PLORA_FLAG_UNFUSED))) {
        FwdCall& c = calls[0];
        plora_ctx* h = c.h;
        const bool fused = c.p.fuse != 0;
        if (flags & PLORA_FLAG_BASE_PAIR) {
            pair_params(c.p, c.P.T, h->cfg.d_out, kWindowRows);
            launch_pair<Op::BaseFwd>(h, c.mX, c.mW128, c.mHk, fused ? c.mPBk128 : c.mW128, c.mY, c.p, st);
        } else {
            launch_tc<Op::BaseFwd>(h, c.mXb, c.mW, c.mHkb, c.mW, c.mY, c.p, st);
        }
        if (!fused) {
            // K3 as its own pass: Y_i += H'_i B_i (read-modify-write of Y).
            TcParams r = base_params(h, c.P, c.D);
            r.N_total = (int32_t)h->cfg.d_out;
            r.tiles_n = (int32_t)ceil_div(h->cfg.d_out, kTileN);
            r.num_tiles = (int32_t)c.P.tok.size() * r.tiles_n;
            r.out = c.Y; r.out_ld = h->cfg.d_out;
            r.out_elems = c.P.T * h->cfg.d_out;
            r.n_items = (int32_t)c.P.tok.size();
            launch_tc<Op::ExpandY>(h, c.mHk, c.mPBk, c.mHk, c.mPBk, c.mHk, r, st);
        }
    } else {
        // One base-GEMM launch per call.  A persistent launch over several projections deals every
        // SM the same number of tiles of each, except that some get one more of the first: with tiles
        // of different lengths (K = 14336 and 4096 in a LLaMA layer), those that got one fewer start
        // the next projection a tile early and stay ahead through it, so the tiles in flight spread
        // over several waves and W's slices leave L2 before the window's m-tiles have all read them.
        for (int k : order) {
            FwdCall& c = calls[k];
            S = Segments{};
            seg_add(S, c.p, SegMaps{&c.mXb, &c.mW, &c.mHkb, &c.mPBk, &c.mY}, false);
            tracked(h0, kBaseFwd, st, [&] { launch_segments<Op::BaseFwd>(S, h0->num_sms, st); });
        }
    }
    for (int k = 0; k < nc; ++k) {
        const plora_status s = finish(calls[k].h, calls[k].D, st);
        if (s != PLORA_OK) return s;
    }
    return PLORA_OK;
}

struct BwdCall {
    plora_ctx* h = nullptr;
    const void* X = nullptr;
    const void* W = nullptr;
    const void* dY = nullptr;
    void* dX = nullptr;
    const void* saved = nullptr;
    HostPlan P;
    DevPlan D;
    CUtensorMap mdY_k, mdY_kb, mdY_mn, mW_mn, mPB_mn, mG_k, mG_kb, mG_mn, mPA_mn, mPA16, mH_mn, mX_mn, mdX;
    TcParams q{}, wb{}, p{}, wa{};
};

// After the argument checks (and the zero gradients of empty adapters): stages the call's schedule
// (queued into cs), encodes its tensor maps and fills the parameters of the shrink of G (q), dB (wb),
// the dX GEMM (p) and dA (wa).
plora_status bwd_prepare(BwdCall& c, cudaStream_t st, StageCopies& cs) {
    plora_ctx* h = c.h;
    const HostPlan& P = c.P;
    plora_status s = upload(h, P, {}, st, c.D, &cs);
    if (s != PLORA_OK) return s;
    const int64_t d_in = h->cfg.d_in, d_out = h->cfg.d_out;
    void* G = h->at<void>(h->r_G);
    // The factors were packed into `saved` by the forward; the backward packs nothing.
    const SavedLayout L = saved_layout(h, P);
    const uint8_t* sv = static_cast<const uint8_t*>(c.saved);
    // the output map of the dX GEMM (dX may be NULL: the GEMM is skipped then)
    bool ok = (!c.dX || make_map(&c.mdX, c.dX, d_in, P.T, d_in, 64, 32)) &&
              make_map(&c.mdY_k, c.dY, d_out, P.T, d_out, 64, kTileM) &&
              make_map(&c.mdY_mn, c.dY, d_out, P.T, d_out, 64, 64) &&
              make_map(&c.mW_mn, c.W, d_in, d_out, d_in, 64, 64) &&
              make_packb_map(&c.mPB_mn, sv + L.o_packB, P.RP, d_out, P.n, 64) &&
              make_map(&c.mG_k, G, P.RP, P.h_rows, P.RP, 64, kTileM) &&
              make_map(&c.mdY_kb, c.dY, d_out, P.T, d_out, 64, kBaseRows) &&   // boxes of a 1-SM base tile
              make_map(&c.mG_kb, G, P.RP, P.h_rows, P.RP, 64, kBaseRows) &&
              make_map(&c.mG_mn, G, P.RP, P.h_rows, P.RP, 64, 64) &&
              make_map(&c.mPA_mn, sv + L.o_packA, d_in, (uint64_t)P.n * P.RP, d_in, 64, 64) &&
              make_map(&c.mPA16, sv + L.o_packA, d_in, (uint64_t)P.n * P.RP, d_in, 64, 16) &&
              make_map(&c.mH_mn, c.saved, P.RP, P.h_rows, P.RP, 64, 64) &&
              make_map(&c.mX_mn, c.X, d_in, P.T, d_in, 64, 64);
    if (!ok) return fail(h, PLORA_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    if (!c.dX) c.mdX = c.mdY_k;   // an unused slot still holds a valid map
    // K5: G_i = s_i dY_i B_i^T per 128-token tile (into the zero-padded workspace blocks).
    TcParams& q = c.q;
    q = base_params(h, P, c.D);
    q.K_total = (int32_t)d_out;
    q.num_tiles = (int32_t)P.tok.size();
    q.out = G; q.out_ld = P.RP;
    q.out_elems = (int64_t)(h->r_G.bytes / h->esize);
    q.n_items = (int32_t)P.tok.size();
    // K7: dB_i = H'_i^T dY_i (a sum over each adapter's tokens) needs neither G nor dX, so its items
    // share K5's launch and fill the last wave of K5's equal-cost token tiles.
    TcParams& wb = c.wb;
    wb = base_params(h, P, c.D);
    wb.M_total = (int32_t)d_out;
    wb.red_dtiles = (int32_t)ceil_div(d_out, kTileM);
    wb.num_tiles = (int32_t)P.red.size() * wb.red_dtiles;
    wb.n_items = (int32_t)P.red.size();
    // K4 (+K6): dX = dY W^T; fused, each tile also accumulates G_j A_j^T of every adapter j
    // overlapping it, so dX is written once.
    TcParams& p = c.p;
    p = base_params(h, P, c.D);
    p.M_total = (int32_t)P.T; p.N_total = (int32_t)d_in; p.K_total = (int32_t)d_out;
    base_tiles(p, P.T, d_in, kDxWindowRows);
    if (!c.dX) p.num_tiles = 0;
    p.out = c.dX; p.out_ld = d_in;
    p.fuse = (h->cfg.flags & PLORA_FLAG_UNFUSED) ? 0 : 1;
    // K8: dA_i = X_i^T G_i (a sum over each adapter's tokens).
    TcParams& wa = c.wa;
    wa = base_params(h, P, c.D);
    wa.M_total = (int32_t)d_in;
    wa.red_dtiles = (int32_t)ceil_div(d_in, kTileM);
    wa.num_tiles = (int32_t)P.red.size() * wa.red_dtiles;
    wa.n_items = (int32_t)P.red.size();
    return PLORA_OK;
}

// The backward of every prepared call: one schedule copy, one launch of the shrink of G with dB's
// items, and per call one launch of the dX GEMM with its dA items filling its last wave (the SM-pair
// variant, single calls only, keeps dA in a launch of its own; the unfused one adds its expand pass).
plora_status bwd_launch(BwdCall* calls, int nc, cudaStream_t st, StageCopies& cs) {
    plora_ctx* h0 = calls[0].h;
    cudaError_t e = stage_copy_run(h0, cs, st);
    if (e != cudaSuccess) return cuda_fail(h0, e, "copying the schedule to the device");
    int RPmax = kRankAlign;
    for (int k = 0; k < nc; ++k) RPmax = std::max(RPmax, calls[k].P.RP);
    Segments& S = *h0->segs;
    S = Segments{};
    // G's shrink reduces over d_out, the dX GEMM too: the calls with the widest d_out first
    const std::vector<int> order = by_k(calls, nc, [](const BwdCall& c) { return c.p.K_total; });
    for (int k : order) {   // one narrow ring that holds every call's widest tiles
        BwdCall& c = calls[k];
        narrow_ring(c.q, RPmax);
        narrow_ring(c.wb, RPmax);
        seg_add(S, c.q, SegMaps{&c.mdY_k, &c.mPB_mn, nullptr, nullptr, nullptr}, false);
        seg_add(S, c.wb, SegMaps{&c.mdY_mn, &c.mH_mn, nullptr, nullptr, nullptr}, true);
    }
    S.g.dyn = calls[0].D.dyn + kDynShrinkDyWgradB;   // dB's items are claimed: they fill G's last wave
    tracked(h0, kShrinkDyWgradB, st, [&] { launch_segments<Op::ShrinkDy, Op::WgradB>(S, h0->num_sms, st); });
    const uint32_t flags = h0->cfg.flags;
    if (nc == 1 && (flags & PLORA_FLAG_BASE_PAIR)) {
        BwdCall& c = calls[0];
        plora_ctx* h = c.h;
        if (c.dX) {
            pair_params(c.p, c.P.T, h->cfg.d_in, kDxWindowRows);
            launch_pair<Op::BaseDx>(h, c.mdY_k, c.mW_mn, c.mG_k, c.mPA16, c.mdX, c.p, st);
        }
        narrow_ring(c.wa, c.P.RP);
        launch_tc<Op::WgradA>(h, c.mX_mn, c.mG_mn, c.mX_mn, c.mG_mn, c.mX_mn, c.wa, st);
    } else {
        // K8 needs neither dX nor K6, so a call's dA items follow its dX tiles in the same persistent
        // launch and fill its last, partial wave (on the dX GEMM's ring, whose stages hold them): one
        // launch per call with dX, for the reason the forward gives.  The calls without dX run their
        // dA items together, on a narrow ring.
        for (int k : order) {
            BwdCall& c = calls[k];
            if (!c.dX) continue;
            S = Segments{};
            seg_add(S, c.p, SegMaps{&c.mdY_kb, &c.mW_mn, &c.mG_kb, &c.mPA16, &c.mdX}, false);
            c.wa.stages = c.p.stages;
            c.wa.stage_bytes = c.p.stage_bytes;
            seg_add(S, c.wa, SegMaps{&c.mX_mn, &c.mG_mn, nullptr, nullptr, nullptr}, true);
            S.g.dyn = c.D.dyn + kDynBaseDxWgradA;   // dA's items are claimed: they fill the GEMM's last wave
            tracked(h0, kBaseDxWgradA, st, [&] { launch_segments<Op::BaseDx, Op::WgradA>(S, h0->num_sms, st); });
        }
        S = Segments{};
        for (int k : order) {
            BwdCall& c = calls[k];
            if (c.dX) continue;
            narrow_ring(c.wa, RPmax);
            seg_add(S, c.wa, SegMaps{&c.mX_mn, &c.mG_mn, nullptr, nullptr, nullptr}, false);
        }
        if (S.g.n_op1 > 0)
            tracked(h0, kWgradA, st, [&] { launch_segments<Op::WgradA>(S, h0->num_sms, st); });
        if (nc == 1 && (flags & PLORA_FLAG_UNFUSED) && calls[0].dX) {
            // K6 as its own pass: dX_i += G_i A_i^T (read-modify-write of dX).
            BwdCall& c = calls[0];
            plora_ctx* h = c.h;
            TcParams r = base_params(h, c.P, c.D);
            r.N_total = (int32_t)h->cfg.d_in;
            r.tiles_n = (int32_t)ceil_div(h->cfg.d_in, kTileN);
            r.num_tiles = (int32_t)c.P.tok.size() * r.tiles_n;
            r.out = c.dX; r.out_ld = h->cfg.d_in;
            r.out_elems = c.P.T * h->cfg.d_in;
            r.n_items = (int32_t)c.P.tok.size();
            launch_tc<Op::ExpandDx>(h, c.mG_k, c.mPA_mn, c.mG_k, c.mPA_mn, c.mG_k, r, st);
        }
    }
    for (int k = 0; k < nc; ++k) {
        const plora_status s = finish(calls[k].h, calls[k].D, st);
        if (s != PLORA_OK) return s;
    }
    return PLORA_OK;
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

const char* plora_status_string(plora_status s) {
    switch (s) {
        case PLORA_OK: return "PLORA_OK";
        case PLORA_ERR_INVALID_ARG: return "PLORA_ERR_INVALID_ARG";
        case PLORA_ERR_UNSUPPORTED: return "PLORA_ERR_UNSUPPORTED";
        case PLORA_ERR_OOM: return "PLORA_ERR_OOM";
        case PLORA_ERR_CUDA: return "PLORA_ERR_CUDA";
        case PLORA_ERR_TIMEOUT: return "PLORA_ERR_TIMEOUT";
        case PLORA_ERR_BOUNDS: return "PLORA_ERR_BOUNDS";
    }
    return "PLORA_ERR_UNKNOWN";
}

const char* plora_last_error(plora_handle h) { return h ? h->last_error.c_str() : ""; }

int32_t plora_version(void) { return 102; }

int32_t plora_debug_build(void) { return kDeviceChecks ? 1 : 0; }

// Output blocks of a config: 1 (one projection) or n_out_blocks, with the checks the header lists.
plora_status check_out_blocks(const plora_config* cfg, int* nblk) {
    *nblk = 1;
    if (cfg->n_out_blocks < 0 || cfg->n_out_blocks > PLORA_MAX_OUT_BLOCKS || cfg->reserved != 0)
        return PLORA_ERR_INVALID_ARG;
    if (cfg->n_out_blocks <= 1) return PLORA_OK;
    if (cfg->dtype != PLORA_BF16 || (cfg->flags & (PLORA_FLAG_SIMT | PLORA_FLAG_UNFUSED | PLORA_FLAG_BASE_PAIR)))
        return PLORA_ERR_UNSUPPORTED;
    int64_t prev = 0;
    for (int b = 0; b < cfg->n_out_blocks; ++b) {
        const int64_t e = cfg->out_block_end[b];
        if (e <= prev || e % 256) return PLORA_ERR_INVALID_ARG;
        prev = e;
    }
    if (prev != cfg->d_out) return PLORA_ERR_INVALID_ARG;
    if (cfg->n_out_blocks * round_up(cfg->max_rank, 16) > PLORA_MAX_RANK) return PLORA_ERR_INVALID_ARG;
    *nblk = cfg->n_out_blocks;
    return PLORA_OK;
}

plora_status plora_create(plora_handle* out, const plora_config* cfg) {
    if (!out) return PLORA_ERR_INVALID_ARG;
    *out = nullptr;
    if (!cfg) return PLORA_ERR_INVALID_ARG;
    if (cfg->dtype != PLORA_BF16 && cfg->dtype != PLORA_FP32) return PLORA_ERR_UNSUPPORTED;
    if (cfg->d_in < 8 || cfg->d_out < 8 || cfg->d_in > 65536 || cfg->d_out > 65536) return PLORA_ERR_UNSUPPORTED;
    if (cfg->d_in % 8 || cfg->d_out % 8) return PLORA_ERR_UNSUPPORTED;
    if (cfg->max_adapters < 1 || cfg->max_adapters > PLORA_MAX_ADAPTERS) return PLORA_ERR_INVALID_ARG;
    if (cfg->max_rank < 1 || cfg->max_rank > PLORA_MAX_RANK) return PLORA_ERR_INVALID_ARG;
    if (cfg->max_tokens < 1 || cfg->max_tokens > ((int64_t)1 << 30)) return PLORA_ERR_INVALID_ARG;
    if (cfg->flags & ~(uint32_t)(PLORA_FLAG_SIMT | PLORA_FLAG_UNFUSED | PLORA_FLAG_BASE_PAIR)) return PLORA_ERR_INVALID_ARG;
    int nblk = 1;
    const plora_status sb = check_out_blocks(cfg, &nblk);
    if (sb != PLORA_OK) return sb;

    plora_ctx* h = new (std::nothrow) plora_ctx();
    if (!h) return PLORA_ERR_OOM;
    h->segs.reset(new (std::nothrow) Segments());
    if (!h->segs) { delete h; return PLORA_ERR_OOM; }
    h->cfg = *cfg;
    h->nblk = nblk;
    for (int b = 0; b < nblk; ++b) h->blk_end[b] = (int32_t)(nblk > 1 ? cfg->out_block_end[b] : cfg->d_out);
    h->esize = cfg->dtype == PLORA_BF16 ? 2 : 4;
    h->tc = cfg->dtype == PLORA_BF16 && !(cfg->flags & PLORA_FLAG_SIMT);

    cudaError_t e = cudaGetDevice(&h->device);
    cudaDeviceProp prop{};
    if (e == cudaSuccess) e = cudaGetDeviceProperties(&prop, h->device);
    if (e != cudaSuccess) { delete h; return PLORA_ERR_CUDA; }
    if (prop.major != 10) { delete h; return PLORA_ERR_UNSUPPORTED; }
    h->num_sms = prop.multiProcessorCount;
    if (h->tc && !get_encode()) { delete h; return PLORA_ERR_CUDA; }

    // Workspace sizing (all bounds follow from the config).
    const int64_t na = cfg->max_adapters;
    h->RPmax = (int)round_up(nblk * round_up(cfg->max_rank, 16), kRankAlign);
    h->max_h_rows = cfg->max_tokens + (int64_t)(kTileM - 1 + 2 * kLoraPad) * na;
    const int64_t dtiles = std::max(ceil_div(cfg->d_in, kTileM), ceil_div(cfg->d_out, kTileM));
    h->max_slots = 2 * (cfg->max_tokens / kSplitTokens) + 1;
    h->max_counters = (cfg->max_tokens / (kSplitTokens + 1) + 1) * dtiles;
    const int64_t tok_max = cfg->max_tokens / kTileM + na + 1;
    const int64_t red_max = h->max_slots + na + 1;
    const int64_t ops_max = 4 * na + 4;
    h->blob_bytes = (size_t)round_up(na * (int64_t)sizeof(AdapterDev), 256) +
                    (size_t)round_up(tok_max * (int64_t)sizeof(TokTile), 256) +
                    (size_t)round_up(red_max * (int64_t)sizeof(RedEntry), 256) +
                    (size_t)round_up(ops_max * (int64_t)sizeof(SimtOp), 256) +
                    (size_t)round_up((tok_max + 1) * (int64_t)sizeof(MTileRec), 256) +
                    (size_t)round_up((tok_max + na) * (int64_t)sizeof(LoraSeg), 256) +
                    (size_t)round_up(kDynCounters * (int64_t)sizeof(int32_t), 256) + 1024;
    // The AdamW step's tables (segments and chunks) travel through the same staging ring.
    const int64_t adamw_chunks =
        2 * na + na * (int64_t)cfg->max_rank * (nblk * cfg->d_in + cfg->d_out) / kAdamwChunk;
    h->blob_bytes = std::max(h->blob_bytes, (size_t)round_up(2 * na * (int64_t)sizeof(AdamwSeg), 256) +
                                                (size_t)round_up(adamw_chunks * (int64_t)sizeof(AdamwChunk), 256) +
                                                1024);

    size_t o = 0;
    auto carve = [&](Region& r, size_t bytes) {
        r.off = o;
        r.bytes = bytes;
        o = (size_t)round_up((int64_t)(o + bytes), 1024);
    };
    carve(h->r_err, 256);
    carve(h->r_G, (size_t)h->max_h_rows * h->RPmax * h->esize);
    if (h->tc) {
        carve(h->r_part, (size_t)h->max_slots * dtiles * kTileM * h->RPmax * sizeof(float));
        carve(h->r_cnt, (size_t)h->max_counters * sizeof(int32_t));
    }
    for (int s = 0; s < kSlots; ++s) carve(h->r_blob[s], h->blob_bytes);
    h->ws_bytes = o;
    e = cudaMalloc(&h->ws, h->ws_bytes);
    if (e != cudaSuccess) { cudaGetLastError(); delete h; return PLORA_ERR_OOM; }
    e = cudaMemset(h->ws, 0, h->ws_bytes);
    for (int s = 0; s < kSlots && e == cudaSuccess; ++s) {
        e = cudaHostAlloc(&h->h_blob[s], h->blob_bytes, cudaHostAllocMapped | cudaHostAllocPortable);
        if (e == cudaSuccess) e = cudaHostGetDevicePointer(reinterpret_cast<void**>(&h->h_blob_dev[s]), h->h_blob[s], 0);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev[s], cudaEventDisableTiming);
    }
    if (e == cudaSuccess && h->tc) {
        e = set_tc_attr<Op::BaseFwd>();
        if (e == cudaSuccess) e = set_tc_attr<Op::BaseDx>();
        if (e == cudaSuccess) e = set_tc_attr<Op::ShrinkX>();
        if (e == cudaSuccess) e = set_tc_attr<Op::ShrinkDy>();
        if (e == cudaSuccess) e = set_tc_attr<Op::ExpandY>();
        if (e == cudaSuccess) e = set_tc_attr<Op::ExpandDx>();
        if (e == cudaSuccess) e = set_tc_attr<Op::WgradB>();
        if (e == cudaSuccess) e = set_tc_attr<Op::WgradA>();
        if (e == cudaSuccess) e = (set_tc_attr<Op::ShrinkDy, Op::WgradB>());
        if (e == cudaSuccess) e = (set_tc_attr<Op::BaseDx, Op::WgradA>());
        if (e == cudaSuccess) e = pair_setup<Op::BaseFwd>(h->pairs_fwd);
        if (e == cudaSuccess) e = pair_setup<Op::BaseDx>(h->pairs_dx);
    }
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        cudaGetLastError();
        plora_destroy(h);
        return e == cudaErrorMemoryAllocation ? PLORA_ERR_OOM : PLORA_ERR_CUDA;
    }
    *out = h;
    return PLORA_OK;
}

plora_status plora_destroy(plora_handle h) {
    if (!h) return PLORA_OK;
    cudaDeviceSynchronize();
    for (int s = 0; s < kSlots; ++s) {
        if (h->ev[s]) cudaEventDestroy(h->ev[s]);
        if (h->h_blob[s]) cudaFreeHost(h->h_blob[s]);
    }
    for (const plora_ctx::Rec& r : h->pending) {
        cudaEventDestroy(r.a);
        cudaEventDestroy(r.b);
    }
    for (cudaEvent_t e : h->pool) cudaEventDestroy(e);
    for (const plora_ctx::CaptureSlot& c : h->cap) {
        if (c.host) cudaFreeHost(c.host);
        if (c.dev) cudaFree(c.dev);
    }
    if (h->ws) cudaFree(h->ws);
    delete h;
    return PLORA_OK;
}

plora_status plora_capture_reserve(plora_handle h, int32_t n) {
    if (!h) return PLORA_ERR_INVALID_ARG;
    h->last_error.clear();
    if (n < 0 || n > 4096) return fail(h, PLORA_ERR_INVALID_ARG, "n=%d outside [0, 4096]", n);
    cudaError_t e = cudaSetDevice(h->device);
    for (int32_t k = 0; k < n && e == cudaSuccess; ++k) {
        plora_ctx::CaptureSlot c;
        e = cudaHostAlloc(&c.host, h->blob_bytes, cudaHostAllocMapped | cudaHostAllocPortable);
        if (e == cudaSuccess) e = cudaHostGetDevicePointer(reinterpret_cast<void**>(&c.host_dev), c.host, 0);
        if (e == cudaSuccess) e = cudaMalloc(&c.dev, h->blob_bytes);
        if (e != cudaSuccess) {
            if (c.host) cudaFreeHost(c.host);
            if (c.dev) cudaFree(c.dev);
            cudaGetLastError();
            break;
        }
        h->cap.push_back(c);
    }
    if (e != cudaSuccess)
        return e == cudaErrorMemoryAllocation ? fail(h, PLORA_ERR_OOM, "capture slots: out of memory")
                                              : cuda_fail(h, e, "reserving capture slots");
    return PLORA_OK;
}

plora_status plora_capture_release(plora_handle h) {
    if (!h) return PLORA_ERR_INVALID_ARG;
    h->last_error.clear();
    cudaError_t e = cudaSetDevice(h->device);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(h, e, "synchronising before releasing capture slots");
    for (const plora_ctx::CaptureSlot& c : h->cap) {
        if (c.host) cudaFreeHost(c.host);
        if (c.dev) cudaFree(c.dev);
    }
    h->cap.clear();
    h->cap_next = 0;
    return PLORA_OK;
}

plora_status plora_saved_bytes(plora_handle h, int32_t n, const int64_t* off, const plora_adapter* tab,
                               size_t* bytes) {
    if (!h) return PLORA_ERR_INVALID_ARG;
    h->last_error.clear();
    if (!bytes) return fail(h, PLORA_ERR_INVALID_ARG, "bytes is NULL");
    *bytes = 0;
    plora_status s = check_table(h, n, off, tab, false);
    if (s != PLORA_OK) return s;
    HostPlan P;
    build_plan(h, n, off, tab, P);
    *bytes = saved_bytes_of(h, P);
    return PLORA_OK;
}

plora_status plora_forward(plora_handle h, const void* X, const void* W, void* Y, int32_t n, const int64_t* off,
                           const plora_adapter* tab, void* saved, void* stream) {
    if (!h) return PLORA_ERR_INVALID_ARG;
    h->last_error.clear();
    HostPlan P;
    plora_status s = fwd_args(h, X, W, Y, n, off, tab, saved, P);
    if (s != PLORA_OK || P.T == 0) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t d_in = h->cfg.d_in, d_out = h->cfg.d_out;

    if (!h->tc) {
        std::vector<SimtOp> ops;
        int32_t t1 = 0, t2 = 0;
        const bool f32 = h->cfg.dtype == PLORA_FP32;
        const size_t es = h->esize;
        // K1: Y = X W.  K2: H'_i = s_i X_i A_i.
        add_op(ops, t1, X, d_in, 1, W, 1, d_in, Y, d_out, 1, P.T, d_out, d_in, 1.f, false, f32);
        for (const AdapterDev& a : P.ad) {
            if (a.n == 0) continue;
            add_op(ops, t1, (const uint8_t*)X + (size_t)a.x_row * d_in * es, d_in, 1, a.A, 1, d_in,
                   (uint8_t*)saved + (size_t)a.h_row * P.RP * es, P.RP, 1, a.n, a.rank, d_in, a.scale, false, f32);
        }
        const int n1 = (int)ops.size();
        // K3: Y_i += H'_i B_i.
        for (const AdapterDev& a : P.ad) {
            if (a.n == 0) continue;
            add_op(ops, t2, (const uint8_t*)saved + (size_t)a.h_row * P.RP * es, P.RP, 1, a.B, 1, a.rank,
                   (uint8_t*)Y + (size_t)a.x_row * d_out * es, d_out, 1, a.n, d_out, a.rank, 1.f, true, f32);
        }
        DevPlan D;
        s = upload(h, P, ops, st, D);
        if (s != PLORA_OK) return s;
        if (f32) {
            launch_simt<float>(h, D.ops, n1, t1, st);
            launch_simt<float>(h, D.ops + n1, (int)ops.size() - n1, t2, st);
        } else {
            launch_simt<__nv_bfloat16>(h, D.ops, n1, t1, st);
            launch_simt<__nv_bfloat16>(h, D.ops + n1, (int)ops.size() - n1, t2, st);
        }
        return finish(h, D, st);
    }

    // Tensor-core path.
    FwdCall c;
    c.h = h; c.X = X; c.W = W; c.Y = Y; c.saved = saved;
    c.P = std::move(P);
    StageCopies cs{};
    s = fwd_prepare(c, st, cs);
    if (s != PLORA_OK) return s;
    return fwd_launch(&c, 1, st, cs);
}

plora_status plora_backward(plora_handle h, const void* X, const void* W, const void* dY, void* dX, int32_t n,
                            const int64_t* off, const plora_adapter* tab, const void* saved, void* stream) {
    if (!h) return PLORA_ERR_INVALID_ARG;
    h->last_error.clear();
    HostPlan P;
    plora_status s = bwd_args(h, X, W, dY, dX, n, off, tab, saved, P);
    if (s != PLORA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t d_in = h->cfg.d_in, d_out = h->cfg.d_out;
    s = zero_empty_grads(h, P, tab, st);
    if (s != PLORA_OK || P.T == 0) return s;
    void* G = h->at<void>(h->r_G);

    if (!h->tc) {
        std::vector<SimtOp> ops;
        int32_t t1 = 0, t2 = 0;
        const bool f32 = h->cfg.dtype == PLORA_FP32;
        const size_t es = h->esize;
        // Phase 1 -- K4: dX = dY W^T; K5: G_i = s_i dY_i B_i^T; K7: dB_i = dY_i^T H'_i.
        if (dX) add_op(ops, t1, dY, d_out, 1, W, d_in, 1, dX, d_in, 1, P.T, d_in, d_out, 1.f, false, f32);
        for (const AdapterDev& a : P.ad) {
            if (a.n == 0) continue;
            add_op(ops, t1, (const uint8_t*)dY + (size_t)a.x_row * d_out * es, d_out, 1, a.B, a.rank, 1,
                   (uint8_t*)G + (size_t)a.h_row * P.RP * es, P.RP, 1, a.n, a.rank, d_out, a.scale, false, f32);
            add_op(ops, t1, (const uint8_t*)dY + (size_t)a.x_row * d_out * es, 1, d_out,
                   (const uint8_t*)saved + (size_t)a.h_row * P.RP * es, P.RP, 1, a.dB, a.rank, 1, d_out, a.rank,
                   a.n, 1.f, false, true);
        }
        const int n1 = (int)ops.size();
        // Phase 2 -- K6: dX_i += G_i A_i^T; K8: dA_i = X_i^T G_i.
        for (const AdapterDev& a : P.ad) {
            if (a.n == 0) continue;
            if (dX)
                add_op(ops, t2, (const uint8_t*)G + (size_t)a.h_row * P.RP * es, P.RP, 1, a.A, d_in, 1,
                       (uint8_t*)dX + (size_t)a.x_row * d_in * es, d_in, 1, a.n, d_in, a.rank, 1.f, true, f32);
            add_op(ops, t2, (const uint8_t*)X + (size_t)a.x_row * d_in * es, 1, d_in,
                   (const uint8_t*)G + (size_t)a.h_row * P.RP * es, P.RP, 1, a.dA, 1, d_in, d_in, a.rank, a.n,
                   1.f, false, true);
        }
        DevPlan D;
        s = upload(h, P, ops, st, D);
        if (s != PLORA_OK) return s;
        if (f32) {
            launch_simt<float>(h, D.ops, n1, t1, st);
            launch_simt<float>(h, D.ops + n1, (int)ops.size() - n1, t2, st);
        } else {
            launch_simt<__nv_bfloat16>(h, D.ops, n1, t1, st);
            launch_simt<__nv_bfloat16>(h, D.ops + n1, (int)ops.size() - n1, t2, st);
        }
        return finish(h, D, st);
    }

    BwdCall c;
    c.h = h; c.X = X; c.W = W; c.dY = dY; c.dX = dX; c.saved = saved;
    c.P = std::move(P);
    StageCopies cs{};
    s = bwd_prepare(c, st, cs);
    if (s != PLORA_OK) return s;
    return bwd_launch(&c, 1, st, cs);
}

plora_status plora_device_info(plora_handle h, int32_t* out, int32_t capacity, int32_t* count) {
    if (!h || !count || capacity < 0 || (capacity > 0 && !out)) return PLORA_ERR_INVALID_ARG;
    const int32_t v[6] = {h->num_sms, h->pairs_fwd, h->pairs_dx, kBaseRows, kWindowRows, kDxWindowRows};
    for (int32_t i = 0; i < 6 && i < capacity; ++i) out[i] = v[i];
    *count = 6;
    return PLORA_OK;
}

plora_status plora_check(plora_handle h, void* stream) {
    if (!h) return PLORA_ERR_INVALID_ARG;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(h, e, "cudaStreamSynchronize");
    int flag = 0;
    e = cudaMemcpy(&flag, h->at<int>(h->r_err), sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(h, e, "reading the device error flag");
    if (flag != 0) {
        int zero = 0;
        cudaMemcpy(h->at<int>(h->r_err), &zero, sizeof(int), cudaMemcpyHostToDevice);
        if (flag == kErrBounds)
            return fail(h, PLORA_ERR_BOUNDS, "a device-side bounds check failed; the access was skipped");
        return fail(h, PLORA_ERR_TIMEOUT, "a device-side wait ran out of time (flag %d)", flag);
    }
    return PLORA_OK;
}

plora_status plora_debug_unpack_saved(plora_handle h, int32_t n, const int64_t* off, const plora_adapter* tab,
                                      const void* saved, int32_t i, float* H_out, void* stream) {
    if (!h) return PLORA_ERR_INVALID_ARG;
    h->last_error.clear();
    plora_status s = check_table(h, n, off, tab, false);
    if (s != PLORA_OK) return s;
    if (i < 0 || i >= n) return fail(h, PLORA_ERR_INVALID_ARG, "adapter index %d outside [0, %d)", i, n);
    if (!saved || !H_out || !aligned16(H_out)) return fail(h, PLORA_ERR_INVALID_ARG, "saved or H_out bad");
    HostPlan P;
    build_plan(h, n, off, tab, P);
    const AdapterDev& a = P.ad[i];
    if (a.n == 0) return PLORA_OK;
    {
        TensorArgs ta;
        ta.saved = saved;
        ta.adapters_AB = false;
        s = check_extents(h, P, tab, ta);
        const size_t out_bytes = (size_t)a.n * a.rank * h->nblk * sizeof(float);
        if (s == PLORA_OK && !in_device_allocation(H_out, out_bytes))
            s = fail(h, PLORA_ERR_INVALID_ARG, "H_out is not a device buffer of %zu bytes", out_bytes);
        if (s != PLORA_OK) return s;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int grid = (int)std::min<int64_t>(ceil_div((int64_t)a.n * a.rank * h->nblk, 256), 1024);
    if (h->cfg.dtype == PLORA_FP32)
        unpack_saved_kernel<float><<<grid, 256, 0, st>>>((const float*)saved, a.h_row, P.RP, a.n, a.rank, h->nblk,
                                                         a.rblk, H_out);
    else
        unpack_saved_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)saved, a.h_row, P.RP, a.n,
                                                                 a.rank, h->nblk, a.rblk, H_out);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? PLORA_OK : cuda_fail(h, e, "unpack launch");
}

plora_status plora_adamw_step(plora_handle h, int32_t n, const plora_adapter* tab, const plora_adamw_state* st,
                              void* stream) {
    if (!h) return PLORA_ERR_INVALID_ARG;
    h->last_error.clear();
    if (n < 0 || n > h->cfg.max_adapters)
        return fail(h, PLORA_ERR_INVALID_ARG, "n_adapters=%d outside [0, max_adapters=%d]", n, h->cfg.max_adapters);
    if (n == 0) return PLORA_OK;
    if (!tab || !st) return fail(h, PLORA_ERR_INVALID_ARG, "adapter table or optimizer state is NULL");
    if (!get_range_fn()) return fail(h, PLORA_ERR_CUDA, "cuMemGetAddressRange is not available");
    const bool bf16 = h->cfg.dtype == PLORA_BF16;
    const size_t di = (size_t)h->cfg.d_in, dout = (size_t)h->cfg.d_out;
    std::vector<AdamwSeg> segs;
    std::vector<AdamwChunk> chunks;
    for (int32_t i = 0; i < n; ++i) {
        const plora_adapter& a = tab[i];
        const plora_adamw_state& o = st[i];
        if (a.rank < 1 || a.rank > h->cfg.max_rank)
            return fail(h, PLORA_ERR_INVALID_ARG, "adapter %d: rank %d outside [1, max_rank=%d]", i, a.rank,
                        h->cfg.max_rank);
        if (!(o.beta1 >= 0.f && o.beta1 < 1.f) || !(o.beta2 >= 0.f && o.beta2 < 1.f) || !(o.eps > 0.f) ||
            !std::isfinite(o.eps) || !std::isfinite(o.lr) || !std::isfinite(o.weight_decay) || o.step < 1)
            return fail(h, PLORA_ERR_INVALID_ARG, "adapter %d: invalid AdamW hyper-parameters", i);
        if (bf16 && (!o.A_master || !o.B_master))
            return fail(h, PLORA_ERR_INVALID_ARG, "adapter %d: a bf16 handle needs fp32 master copies", i);
        if (!bf16 && (o.A_master || o.B_master))
            return fail(h, PLORA_ERR_INVALID_ARG, "adapter %d: an fp32 handle updates A and B in place", i);
        const size_t r = (size_t)a.rank;
        const size_t ra = r * (size_t)h->nblk;   // rows of A: one rank-r block per output block
        const size_t es = h->esize;
        float* pA = bf16 ? o.A_master : const_cast<float*>(static_cast<const float*>(a.A));
        float* pB = bf16 ? o.B_master : const_cast<float*>(static_cast<const float*>(a.B));
        const void* ptrs[] = {a.A, a.B, a.dA, a.dB, pA, pB, o.mA, o.vA, o.mB, o.vB};
        const size_t bytes[] = {ra * di * es, dout * r * es, ra * di * 4, dout * r * 4, ra * di * 4, dout * r * 4,
                                ra * di * 4, ra * di * 4, dout * r * 4, dout * r * 4};
        for (int k = 0; k < 10; ++k) {
            if (!ptrs[k] || !aligned16(ptrs[k]))
                return fail(h, PLORA_ERR_INVALID_ARG, "adapter %d: a parameter, gradient or state pointer is NULL "
                            "or not 16-byte aligned", i);
            if (!in_device_allocation(ptrs[k], bytes[k]))
                return fail(h, PLORA_ERR_INVALID_ARG, "adapter %d: a parameter, gradient or state buffer is not a "
                            "device buffer of its size", i);
        }
        const double b1 = o.beta1, b2 = o.beta2;
        const double bc1 = 1.0 - std::pow(b1, (double)o.step);
        const double bc2 = 1.0 - std::pow(b2, (double)o.step);
        AdamwSeg sg{};
        sg.decay = (float)(1.0 - (double)o.lr * (double)o.weight_decay);
        sg.step_size = (float)((double)o.lr / bc1);
        sg.beta1 = o.beta1;
        sg.beta2 = o.beta2;
        sg.inv_sqrt_bc2 = (float)(1.0 / std::sqrt(bc2));
        sg.eps = o.eps;
        AdamwSeg sa = sg, sb = sg;
        sa.p = pA; sa.m = o.mA; sa.v = o.vA; sa.g = a.dA; sa.out = bf16 ? const_cast<void*>(a.A) : nullptr;
        sa.n = (int64_t)(ra * di);
        sb.p = pB; sb.m = o.mB; sb.v = o.vB; sb.g = a.dB; sb.out = bf16 ? const_cast<void*>(a.B) : nullptr;
        sb.n = (int64_t)(dout * r);
        for (const AdamwSeg& x : {sa, sb}) {
            const int32_t id = (int32_t)segs.size();
            segs.push_back(x);
            for (int64_t e = 0; e < x.n; e += kAdamwChunk) chunks.push_back(AdamwChunk{id, 0, e});
        }
    }
    cudaError_t ce = cudaSetDevice(h->device);
    if (ce != cudaSuccess) return cuda_fail(h, ce, "cudaSetDevice");
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    uint8_t *dsegs = nullptr, *dchunks = nullptr;
    int slot = 0;
    plora_status s = upload_parts(h, segs.data(), segs.size() * sizeof(AdamwSeg), chunks.data(),
                                  chunks.size() * sizeof(AdamwChunk), cs, &dsegs, &dchunks, &slot);
    if (s != PLORA_OK) return s;
    const unsigned grid = (unsigned)chunks.size();
    tracked(h, kAdamw, cs, [&] {
        adamw_kernel<<<grid, 256, 0, cs>>>(reinterpret_cast<const AdamwSeg*>(dsegs),
                                           reinterpret_cast<const AdamwChunk*>(dchunks));
    });
    DevPlan D;
    D.slot = slot;
    return finish(h, D, cs);
}

plora_status plora_debug_timeout_probe(plora_handle h, int64_t timeout_ns, void* stream) {
    if (!h) return PLORA_ERR_INVALID_ARG;
    h->last_error.clear();
    if (timeout_ns < 1000000 || timeout_ns > 10000000000LL)
        return fail(h, PLORA_ERR_INVALID_ARG, "timeout_ns=%lld outside [1 ms, 10 s]", (long long)timeout_ns);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    timeout_probe_kernel<<<1, 32, 0, st>>>(h->at<int>(h->r_err), (uint64_t)timeout_ns);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? PLORA_OK : cuda_fail(h, e, "timeout probe launch");
}

plora_status plora_profile_enable(plora_handle h, int32_t enable) {
    if (!h) return PLORA_ERR_INVALID_ARG;
    h->profiling = enable != 0;
    return PLORA_OK;
}

plora_status plora_profile_read(plora_handle h, int32_t capacity, int32_t* n_kinds, const char** names,
                                int64_t* launches, double* total_ms) {
    if (!h || !n_kinds) return PLORA_ERR_INVALID_ARG;
    h->last_error.clear();
    for (const plora_ctx::Rec& r : h->pending) {
        cudaError_t e = cudaEventSynchronize(r.b);
        float ms = 0.f;
        if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, r.a, r.b);
        if (e != cudaSuccess) return cuda_fail(h, e, "reading profile events");
        h->total_ms[r.kind] += ms;
        h->pool.push_back(r.a);
        h->pool.push_back(r.b);
    }
    h->pending.clear();
    *n_kinds = kKinds;
    for (int k = 0; k < kKinds && k < capacity; ++k) {
        if (names) names[k] = kKindNames[k];
        if (launches) launches[k] = h->launches[k];
        if (total_ms) total_ms[k] = h->total_ms[k];
        h->launches[k] = 0;
        h->total_ms[k] = 0.0;
    }
    return PLORA_OK;
}

plora_status plora_debug_schedule(const plora_config* cfg, int32_t n, const int64_t* off, const plora_adapter* tab,
                                  int32_t grads, int32_t which, int32_t* out, int64_t capacity, int64_t* count) {
    if (!cfg || !count) return PLORA_ERR_INVALID_ARG;
    *count = 0;
    plora_ctx tmp;
    tmp.cfg = *cfg;
    tmp.esize = cfg->dtype == PLORA_FP32 ? 4 : 2;
    plora_status s = check_out_blocks(cfg, &tmp.nblk);
    if (s != PLORA_OK) return s;
    s = check_table(&tmp, n, off, tab, grads != 0);
    if (s != PLORA_OK) return s;
    HostPlan P;
    build_plan(&tmp, n, off, tab, P);
    std::vector<int32_t> v;
    if (which == 0) {
        for (const TokTile& t : P.tok) v.insert(v.end(), {t.adapter, t.rows, t.x_row, t.h_row});
    } else if (which == 1) {
        for (const RedEntry& r : P.red)
            v.insert(v.end(), {r.adapter, r.x_row, r.h_row, r.kblocks, r.split, r.nsplit, r.slot, r.counter});
    } else if (which == 2) {
        for (const AdapterDev& a : P.ad) v.insert(v.end(), {a.x_row, a.n, a.h_row, a.rp16, a.rp64});
    } else if (which == 3) {
        v = {P.RP, (int32_t)P.h_rows};
    } else if (which == 4) {
        v = P.mt_off;
    } else if (which == 5) {
        for (const LoraSeg& g : P.mt_seg) v.push_back(g.adapter);
    } else {
        return PLORA_ERR_INVALID_ARG;
    }
    *count = (int64_t)v.size();
    if (out) memcpy(out, v.data(), sizeof(int32_t) * (size_t)std::min<int64_t>(capacity, (int64_t)v.size()));
    return PLORA_OK;
}

plora_status plora_partition(int32_t n, const int64_t* counts, const int32_t* ranks, int64_t d_in, int64_t d_out,
                             double flops_per_s, double bytes_per_s, int32_t n_parts, int32_t* owner,
                             double* part_cost) {
    if (n < 0 || n > PLORA_MAX_ADAPTERS || n_parts < 1 || n_parts > PLORA_MAX_ADAPTERS) return PLORA_ERR_INVALID_ARG;
    if (d_in < 1 || d_out < 1 || !(flops_per_s > 0.0) || !(bytes_per_s > 0.0) || !std::isfinite(flops_per_s) ||
        !std::isfinite(bytes_per_s))
        return PLORA_ERR_INVALID_ARG;
    if (n > 0 && (!counts || !ranks || !owner)) return PLORA_ERR_INVALID_ARG;
    for (int32_t i = 0; i < n; ++i)
        if (counts[i] < 0 || ranks[i] < 1 || ranks[i] > PLORA_MAX_RANK) return PLORA_ERR_INVALID_ARG;
    // An adapter's cost is the ideal time of its share of one packed step at the given peaks: its tokens'
    // share of the two base GEMMs and its low-rank products (4 d_in d_out + 6 r (d_in + d_out) flop per
    // token) plus the low-rank kernels' memory traffic (8 (d_in + d_out) + 12 r bytes per token).
    const double di = (double)d_in, dout = (double)d_out;
    std::vector<double> cost(n);
    for (int32_t i = 0; i < n; ++i) {
        const double r = (double)ranks[i];
        const double per_token = (4.0 * di * dout + 6.0 * r * (di + dout)) / flops_per_s +
                                 (8.0 * (di + dout) + 12.0 * r) / bytes_per_s;
        cost[i] = (double)counts[i] * per_token;
    }
    // Longest processing time first: adapters by decreasing cost (ties: lower index first), each to the
    // part with the least cost so far (ties: lower part index).  Deterministic.
    std::vector<int32_t> order(n);
    for (int32_t i = 0; i < n; ++i) order[i] = i;
    std::stable_sort(order.begin(), order.end(), [&](int32_t a, int32_t b) { return cost[a] > cost[b]; });
    std::vector<double> load(n_parts, 0.0);
    for (int32_t i : order) {
        int32_t best = 0;
        for (int32_t q = 1; q < n_parts; ++q)
            if (load[q] < load[best]) best = q;
        owner[i] = best;
        load[best] += cost[i];
    }
    if (part_cost)
        for (int32_t q = 0; q < n_parts; ++q) part_cost[q] = load[q];
    return PLORA_OK;
}

// ---------------------------------------------------------------------------
// Layer calls: several projections over one segment map as one launch set.
// ---------------------------------------------------------------------------
}  // extern "C"

struct plora_layer_ctx {
    int n = 0;
    plora_ctx* h[PLORA_MAX_LAYER_PROJ] = {};
    std::string last_error;
};

namespace {

// A projection's failure, reported on the layer with the projection's index.
plora_status layer_fail(plora_layer_ctx* L, int p, plora_status s) {
    L->last_error = "projection " + std::to_string(p) + ": " + L->h[p]->last_error;
    return s;
}

}  // namespace

extern "C" {

plora_status plora_layer_create(plora_layer* out, int32_t n_proj, const plora_config* cfgs) {
    if (!out) return PLORA_ERR_INVALID_ARG;
    *out = nullptr;
    if (n_proj < 1 || n_proj > PLORA_MAX_LAYER_PROJ || !cfgs) return PLORA_ERR_INVALID_ARG;
    for (int32_t p = 0; p < n_proj; ++p)
        if (cfgs[p].dtype != PLORA_BF16 || (cfgs[p].flags & (PLORA_FLAG_SIMT | PLORA_FLAG_UNFUSED | PLORA_FLAG_BASE_PAIR)))
            return PLORA_ERR_UNSUPPORTED;
    plora_layer_ctx* L = new (std::nothrow) plora_layer_ctx();
    if (!L) return PLORA_ERR_OOM;
    for (int32_t p = 0; p < n_proj; ++p) {
        const plora_status s = plora_create(&L->h[p], &cfgs[p]);
        if (s != PLORA_OK) {
            plora_layer_destroy(L);
            return s;
        }
        L->n = p + 1;
        if (L->h[p]->device != L->h[0]->device) {
            plora_layer_destroy(L);
            return PLORA_ERR_INVALID_ARG;
        }
    }
    *out = L;
    return PLORA_OK;
}

plora_status plora_layer_destroy(plora_layer L) {
    if (!L) return PLORA_OK;
    for (int p = 0; p < L->n; ++p) plora_destroy(L->h[p]);
    delete L;
    return PLORA_OK;
}

plora_status plora_layer_handle(plora_layer L, int32_t p, plora_handle* h) {
    if (!L || !h || p < 0 || p >= L->n) return PLORA_ERR_INVALID_ARG;
    *h = L->h[p];
    return PLORA_OK;
}

const char* plora_layer_last_error(plora_layer L) { return L ? L->last_error.c_str() : ""; }

plora_status plora_layer_saved_bytes(plora_layer L, int32_t n, const int64_t* off, const plora_proj* projs,
                                     size_t* bytes) {
    if (!L) return PLORA_ERR_INVALID_ARG;
    L->last_error.clear();
    if (!projs || !bytes) {
        L->last_error = "projs or bytes is NULL";
        return PLORA_ERR_INVALID_ARG;
    }
    for (int p = 0; p < L->n; ++p) {
        const plora_status s = plora_saved_bytes(L->h[p], n, off, projs[p].tab, &bytes[p]);
        if (s != PLORA_OK) return layer_fail(L, p, s);
    }
    return PLORA_OK;
}

plora_status plora_layer_forward(plora_layer L, int32_t n, const int64_t* off, const plora_proj* projs, void* stream) {
    if (!L) return PLORA_ERR_INVALID_ARG;
    L->last_error.clear();
    if (!projs) {
        L->last_error = "projs is NULL";
        return PLORA_ERR_INVALID_ARG;
    }
    std::vector<FwdCall> calls(L->n);
    for (int p = 0; p < L->n; ++p) {   // every check of every projection before anything is enqueued
        plora_ctx* h = L->h[p];
        h->last_error.clear();
        const plora_proj& io = projs[p];
        const plora_status s = fwd_args(h, io.X, io.W, io.Y, n, off, io.tab, io.saved, calls[p].P);
        if (s != PLORA_OK) return layer_fail(L, p, s);
        calls[p].h = h;
        calls[p].X = io.X; calls[p].W = io.W; calls[p].Y = io.Y; calls[p].saved = io.saved;
    }
    if (calls[0].P.T == 0) return PLORA_OK;   // the segment map is shared: no tokens anywhere
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    StageCopies cs{};
    for (int p = 0; p < L->n; ++p) {
        const plora_status s = fwd_prepare(calls[p], st, cs);
        if (s != PLORA_OK) return layer_fail(L, p, s);
    }
    const plora_status s = fwd_launch(calls.data(), L->n, st, cs);
    return s == PLORA_OK ? s : layer_fail(L, 0, s);
}

plora_status plora_layer_backward(plora_layer L, int32_t n, const int64_t* off, const plora_proj* projs, void* stream) {
    if (!L) return PLORA_ERR_INVALID_ARG;
    L->last_error.clear();
    if (!projs) {
        L->last_error = "projs is NULL";
        return PLORA_ERR_INVALID_ARG;
    }
    std::vector<BwdCall> calls(L->n);
    for (int p = 0; p < L->n; ++p) {
        plora_ctx* h = L->h[p];
        h->last_error.clear();
        const plora_proj& io = projs[p];
        const plora_status s = bwd_args(h, io.X, io.W, io.dY, io.dX, n, off, io.tab, io.saved, calls[p].P);
        if (s != PLORA_OK) return layer_fail(L, p, s);
        calls[p].h = h;
        calls[p].X = io.X; calls[p].W = io.W; calls[p].dY = io.dY; calls[p].dX = io.dX; calls[p].saved = io.saved;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    for (int p = 0; p < L->n; ++p) {
        const plora_status s = zero_empty_grads(L->h[p], calls[p].P, projs[p].tab, st);
        if (s != PLORA_OK) return layer_fail(L, p, s);
    }
    if (calls[0].P.T == 0) return PLORA_OK;
    StageCopies cs{};
    for (int p = 0; p < L->n; ++p) {
        const plora_status s = bwd_prepare(calls[p], st, cs);
        if (s != PLORA_OK) return layer_fail(L, p, s);
    }
    const plora_status s = bwd_launch(calls.data(), L->n, st, cs);
    return s == PLORA_OK ? s : layer_fail(L, 0, s);
}

plora_status plora_layer_check(plora_layer L, void* stream) {
    if (!L) return PLORA_ERR_INVALID_ARG;
    L->last_error.clear();
    plora_status first = PLORA_OK;
    for (int p = 0; p < L->n; ++p) {   // every projection's flag is read (and cleared)
        const plora_status s = plora_check(L->h[p], stream);
        if (s != PLORA_OK && first == PLORA_OK) {
            first = s;
            layer_fail(L, p, s);
        }
    }
    return first;
}

}  // extern "C"

// ===========================================================================
// Allocation-free variant of the dB weight-gradient product.
//
// Its scratch -- the adapter table and token splits the kernel reads, the split
// partials, their arrival counters and the device error flag -- lives in one
// file-scope device array instead of a handle's cudaMalloc'd workspace.  The
// array is created with the module on every GPU that loads this library and
// stays until the process exits.  Host code cannot use the array's name as a
// device address (on the host it only stands for the symbol), so the first
// call on each device looks the address up with cudaGetSymbolAddress and
// passes that pointer to the kernel.
//
// The schedule reaches the array through kernel parameters: the launch copies
// them when it is enqueued, so the call needs neither pinned staging (which it
// would have to allocate) nor a copy from pageable host memory (which may wait
// for the stream's earlier work).
// ===========================================================================
namespace {

constexpr size_t kStaticScratchBytes = PLORA_STATIC_SCRATCH_BYTES;
constexpr size_t kStaticSchedBytes = (size_t)1 << 20;      // error flag + adapter table + splits
constexpr int kStaticMaxDevices = 64;
constexpr int kStaticParam16 = 1536;                       // 24 KB of schedule per staging launch

// One staging launch: `n16` 16-byte words of schedule for [dst, dst + 16 n16) of the array and,
// on the first launch of a call, the error flag ([0, 256)) and `zero16` words at `zero` (the arrival
// counters) cleared, since the previous call may have left them set.
struct StaticStage {
    uint32_t dst;      // byte offset of the schedule words in the array
    uint32_t n16;
    uint32_t zero;     // byte offset of the counters to clear
    uint32_t zero16;
    uint32_t clear_flag;
    uint32_t pad_[3];
    uint4 words[kStaticParam16];
};
static_assert(sizeof(StaticStage) + sizeof(void*) < 32000, "kernel parameters of the staging launch");

}  // namespace

static __device__ __align__(256) uint8_t g_plora_static_scratch[kStaticScratchBytes];

namespace {

__global__ void static_stage_kernel(const __grid_constant__ StaticStage s, uint8_t* scratch) {
    const uint32_t tid = blockIdx.x * blockDim.x + threadIdx.x, nth = gridDim.x * blockDim.x;
    uint4* dst = reinterpret_cast<uint4*>(scratch + s.dst);
    for (uint32_t i = tid; i < s.n16; i += nth) dst[i] = s.words[i];
    uint4* z = reinterpret_cast<uint4*>(scratch + s.zero);
    for (uint32_t i = tid; i < s.zero16; i += nth) z[i] = make_uint4(0, 0, 0, 0);
    if (s.clear_flag && tid < 256 / 16) reinterpret_cast<uint4*>(scratch)[tid] = make_uint4(0, 0, 0, 0);
}

struct StaticDevice {
    uint8_t* scratch = nullptr;   // device address of g_plora_static_scratch on this device
    int num_sms = 0;
};
std::mutex g_static_mu;
StaticDevice g_static_dev[kStaticMaxDevices];

// Once per device, with that device current: resolve the array's device address, the
// tensor-map encoder and the kernel's shared-memory limit.  None of these allocate.
plora_status static_setup(int dev, StaticDevice& out) {
    std::lock_guard<std::mutex> lock(g_static_mu);
    StaticDevice& d = g_static_dev[dev];
    if (!d.scratch) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_plora_static_scratch);
        if (e != cudaSuccess || p == nullptr) return PLORA_ERR_CUDA;
        int sms = 0;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return PLORA_ERR_CUDA;
        if (!get_encode()) return PLORA_ERR_CUDA;
        e = cudaFuncSetAttribute(tc_kernel<Op::WgradB>, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmemBytes);
        if (e != cudaSuccess) return PLORA_ERR_CUDA;
        d.num_sms = sms;
        d.scratch = static_cast<uint8_t*>(p);
    }
    out = d;
    return PLORA_OK;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Byte layout of one call's scratch inside the static array.
struct StaticLayout {
    size_t o_ad, o_red, sched_end;   // [0, 256) error flag | adapter table | splits   (< kStaticSchedBytes)
    size_t o_cnt, cnt_bytes;         // arrival counters: the plan's count, one int each
    size_t o_part, part_end;         // split partials [slot][d_out tile][rank column][128 rows] fp32
};

StaticLayout static_layout(const HostPlan& P, int32_t dtiles_out) {
    StaticLayout L;
    L.o_ad = 256;
    L.o_red = align256(L.o_ad + P.ad.size() * sizeof(AdapterDev));
    L.sched_end = align256(L.o_red + P.red.size() * sizeof(RedEntry));
    L.o_cnt = kStaticSchedBytes;
    // build_plan spaces each split adapter's counters by max(d_in, d_out tiles): size the area from
    // its total, not from the d_out tiles the dB product reads.
    L.cnt_bytes = align256((size_t)P.counters * sizeof(int32_t));
    L.o_part = L.o_cnt + L.cnt_bytes;
    L.part_end = L.o_part + (size_t)P.slots * dtiles_out * kTileM * (size_t)P.RP * sizeof(float);
    return L;
}

}  // namespace

extern "C" plora_status plora_grad_B_static(const plora_config* cfg, const void* dY, int32_t n, const int64_t* off,
                                            const plora_adapter* tab, const void* saved, void* stream) {
    if (!cfg) return PLORA_ERR_INVALID_ARG;
    if (cfg->dtype != PLORA_BF16 || (cfg->flags & PLORA_FLAG_SIMT) || cfg->n_out_blocks > 1)
        return PLORA_ERR_UNSUPPORTED;
    if (cfg->d_in < 8 || cfg->d_out < 8 || cfg->d_in > 65536 || cfg->d_out > 65536 || cfg->d_in % 8 ||
        cfg->d_out % 8)
        return PLORA_ERR_UNSUPPORTED;
    if (cfg->max_adapters < 1 || cfg->max_adapters > PLORA_MAX_ADAPTERS || cfg->max_rank < 1 ||
        cfg->max_rank > PLORA_MAX_RANK || cfg->max_tokens < 1 || cfg->max_tokens > ((int64_t)1 << 30))
        return PLORA_ERR_INVALID_ARG;
    plora_ctx tmp;
    tmp.cfg = *cfg;
    tmp.esize = 2;
    plora_status s = check_table(&tmp, n, off, tab, false);
    if (s != PLORA_OK) return s;
    for (int32_t i = 0; i < n; ++i)
        if (!tab[i].dB || !aligned16(tab[i].dB)) return PLORA_ERR_INVALID_ARG;
    const bool any_tokens = off[n] > 0;
    if (any_tokens && (!dY || !saved)) return PLORA_ERR_INVALID_ARG;
    if (!aligned16(dY) || (reinterpret_cast<uintptr_t>(saved) & 255u) != 0) return PLORA_ERR_INVALID_ARG;

    HostPlan P;
    build_plan(&tmp, n, off, tab, P);
    const int64_t d_out = cfg->d_out;
    const int32_t dtiles = (int32_t)ceil_div(d_out, kTileM);
    const StaticLayout L = static_layout(P, dtiles);
    if (L.sched_end > kStaticSchedBytes || L.part_end > kStaticScratchBytes) return PLORA_ERR_UNSUPPORTED;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kStaticMaxDevices) return PLORA_ERR_CUDA;
    StaticDevice sd;
    s = static_setup(dev, sd);
    if (s != PLORA_OK) return s;
    {
        TensorArgs ta;
        if (P.T > 0) { ta.dY = dY; ta.saved = saved; }
        ta.adapters_AB = false;
        ta.adapters_dB = true;
        s = check_extents(&tmp, P, tab, ta);
        if (s != PLORA_OK) return s;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    // Adapters without tokens get dB = 0.
    for (int32_t i : P.empty)
        if (cudaMemsetAsync(tab[i].dB, 0, (size_t)tab[i].rank * d_out * sizeof(float), st) != cudaSuccess)
            return PLORA_ERR_CUDA;
    if (P.T == 0) return cudaGetLastError() == cudaSuccess ? PLORA_OK : PLORA_ERR_CUDA;

    // The array keeps the previous call's contents.  The schedule words ([256, sched_end): adapter
    // table, then splits) travel in the parameters of one or more staging launches; the first also
    // clears the error flag and this call's arrival counters.
    std::vector<uint8_t> blob(L.sched_end - L.o_ad, 0);
    memcpy(blob.data(), P.ad.data(), P.ad.size() * sizeof(AdapterDev));
    if (!P.red.empty()) memcpy(blob.data() + (L.o_red - L.o_ad), P.red.data(), P.red.size() * sizeof(RedEntry));
    uint8_t* base = sd.scratch;
    StaticStage stg{};
    const size_t chunk = sizeof(stg.words);
    size_t at = 0;
    do {   // blob.size() is a positive multiple of 256 (every call here has an adapter with tokens)
        const size_t bytes = std::min(chunk, blob.size() - at);
        const bool first = at == 0;
        stg.dst = (uint32_t)(L.o_ad + at);
        stg.n16 = (uint32_t)(bytes / 16);
        memcpy(stg.words, blob.data() + at, bytes);
        stg.zero = first ? (uint32_t)L.o_cnt : 0u;
        stg.zero16 = first ? (uint32_t)(L.cnt_bytes / 16) : 0u;
        stg.clear_flag = first ? 1u : 0u;
        static_stage_kernel<<<8, 256, 0, st>>>(stg, base);
        at += chunk;
    } while (at < blob.size());

    CUtensorMap mdY, mH;
    if (!make_map(&mdY, dY, d_out, P.T, d_out, 64, 64) || !make_map(&mH, saved, P.RP, P.h_rows, P.RP, 64, 64))
        return PLORA_ERR_CUDA;
    TcParams p{};
    p.RP = P.RP;
    p.nblk = 1;
    p.adapters = reinterpret_cast<const AdapterDev*>(base + L.o_ad);
    p.red = reinterpret_cast<const RedEntry*>(base + L.o_red);
    p.err_flag = reinterpret_cast<int*>(base);
    p.timeout_ns = kTimeoutNs;
    p.partials = reinterpret_cast<float*>(base + L.o_part);
    p.counters = reinterpret_cast<int32_t*>(base + L.o_cnt);
    p.group_m = 16;
    p.M_total = (int32_t)d_out;
    p.red_dtiles = dtiles;
    p.num_tiles = (int32_t)P.red.size() * dtiles;
    p.n_adapters = P.n;
    p.n_items = (int32_t)P.red.size();
    p.part_elems = (int64_t)((kStaticScratchBytes - L.o_part) / sizeof(float));
    p.n_counters = (int32_t)(L.cnt_bytes / sizeof(int32_t));
    narrow_ring(p, P.RP);
    std::unique_ptr<Segments> S(new (std::nothrow) Segments());   // host memory, not device
    if (!S) return PLORA_ERR_OOM;
    seg_add(*S, p, SegMaps{&mdY, &mH, nullptr, nullptr, nullptr}, false);
    if (launch_segments<Op::WgradB>(*S, sd.num_sms, st) != cudaSuccess) return PLORA_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? PLORA_OK : PLORA_ERR_CUDA;
}
