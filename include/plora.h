/*
 * plora.h -- C ABI of the packed LoRA fine-tuning library for NVIDIA B200 (sm_100a).
 *
 * One call computes, for N LoRA adapters that share one frozen base projection
 * W and own contiguous segments of one packed token buffer, the forward and
 * the backward of the layer
 *
 *     Y_i  = X_i W + s_i (X_i A_i) B_i
 *     dX_i = dY_i W^T + s_i (dY_i B_i^T) A_i^T
 *     dB_i = s_i (X_i A_i)^T dY_i          (a sum over the tokens of adapter i)
 *     dA_i = X_i^T (s_i dY_i B_i^T)        (a sum over the tokens of adapter i)
 *
 * where X_i are the rows off[i] .. off[i+1]-1 of X and s_i = alpha_i / r_i.
 * The layer is LoRA's: a frozen W plus a trainable low-rank branch A then B
 * whose output is scaled by alpha/r and added ("LLM+LoRA微调加速技术原理解析",
 * m.youleyou.com, 深入理解LoRA：基本原理与PEFT实现); only A and B get gradients
 * ("LoRA加速集成方案", cloud.baidu.com, 四、工作原理 › 3. 反向传播阶段).  Packing
 * many adapters over one shared frozen base and batching their operators over
 * the concatenated LoRA tensors, tiled along the sequence or hidden dimension
 * rather than the rank, with load balancing across adapters of unequal rank
 * and token count, is PLoRA's execution engine (PLoRA summary, gist.science,
 * arXiv 2508.02932, 技术摘要 › 方法论 › 2. LoRA 执行引擎 › 打包 LoRA 算子,
 * 算子设计).
 *
 * Layouts.  Every tensor is dense and row-major, in the PyTorch / PEFT module
 * layouts, so that module parameters can be passed without copies:
 *     X       [T][d_in]       packed tokens               (dtype)
 *     W       [d_out][d_in]   nn.Linear.weight = W^T      (dtype)
 *     A_i     [r_i][d_in]     lora_A.weight    = A_i^T    (dtype)
 *     B_i     [d_out][r_i]    lora_B.weight    = B_i^T    (dtype)
 *     Y, dY   [T][d_out]                                  (dtype)
 *     dX      [T][d_in]                                   (dtype)
 *     dA_i    [r_i][d_in],  dB_i [d_out][r_i]             (fp32)
 * T = off[N].  dtype is bf16 (products accumulated in fp32, outputs rounded
 * to nearest even) or fp32 (fp32 FMA throughout, no TF32).
 *
 * Ownership.  The caller owns every tensor.  A handle owns only its private
 * workspace (device scratch, pinned host staging, a device error flag).
 * `off` and the adapter table are HOST arrays, read during the call; every
 * pointer inside them, and every tensor pointer, is a DEVICE pointer that
 * must stay valid until the work enqueued on `stream` has run.
 *
 * Semantics.  Y, dX, dA_i and dB_i are overwritten, never accumulated into.
 * An adapter with no tokens (off[i] == off[i+1]) gets dA_i = dB_i = 0.
 * All work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 * stream); calls return once it is enqueued.  A handle stages each call's
 * schedule in one of four slots, so a call first waits until the work of the
 * call four before it on the same handle has run (calls captured into a CUDA
 * graph use reserved slots instead; see plora_capture_reserve).
 *
 * Errors.  Every argument is checked before anything is enqueued; on an
 * error nothing is written and the call returns a non-zero status, with a
 * message available from plora_last_error().  This includes the memory:
 * every tensor pointer must lie inside one device allocation that holds the
 * tensor's whole extent (checked against the driver's allocation record,
 * so at the granularity of cudaMalloc: a sub-allocator's slice is checked
 * against its whole segment), else the call returns PLORA_ERR_INVALID_ARG
 * and launches nothing.  No C++ exception crosses this
 * ABI.  An asynchronous device failure surfaces as PLORA_ERR_CUDA from the
 * call that observes it or from plora_check(); a device-side wait that ran
 * out of time surfaces as PLORA_ERR_TIMEOUT from plora_check().
 *
 * Threading.  A handle runs one call at a time (its workspace is reused by
 * the next call on the same stream); distinct handles are independent.
 */
#ifndef PLORA_H
#define PLORA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PLORA_API __attribute__((visibility("default")))
#else
#define PLORA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PLORA_OK = 0,
    PLORA_ERR_INVALID_ARG = 1,  /* a null/misaligned pointer, bad offsets, rank or count out of range */
    PLORA_ERR_UNSUPPORTED = 2,  /* a shape or dtype the library does not handle */
    PLORA_ERR_OOM = 3,          /* workspace allocation failed in plora_create */
    PLORA_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed */
    PLORA_ERR_TIMEOUT = 5,      /* a bounded device-side wait ran out (see plora_check) */
    PLORA_ERR_BOUNDS = 6        /* PLORA_DEBUG builds: a device-side bounds check failed (see plora_check) */
} plora_status;

typedef enum {
    PLORA_BF16 = 0,
    PLORA_FP32 = 1
} plora_dtype;

/* plora_config.flags */
enum {
    PLORA_FLAG_SIMT = 1u,     /* bf16 only: run the plain SIMT kernels instead of the tensor-core ones */
    PLORA_FLAG_UNFUSED = 2u,  /* tensor-core path: run the expand products (Y += s H B, dX += G A^T) as
                                 separate read-modify-write passes instead of inside the base GEMMs */
    PLORA_FLAG_BASE_PAIR = 4u /* tensor-core path: base GEMMs on SM pairs (256-row tiles, tcgen05
                                 cta_group::2, half the B staging per SM) instead of single SMs */
};

/* Limits. */
#define PLORA_MAX_RANK 256
#define PLORA_MAX_ADAPTERS 4096
#define PLORA_MAX_OUT_BLOCKS 8

/*
 * Handle configuration.  d_in, d_out: projection sizes, multiples of 8 in
 * [8, 65536].  dtype: a plora_dtype.  max_adapters in [1, PLORA_MAX_ADAPTERS],
 * max_rank in [1, PLORA_MAX_RANK], max_tokens >= 1: upper bounds of every
 * later call, used to size the workspace.
 *
 * Output blocks (shared-input projections in one base GEMM).  LoRA is usually
 * applied to the attention's query, key and value projections, which read the
 * same input ("LoRA加速集成方案", cloud.baidu.com, 七 › 2. 层的选择), and PEFT
 * configures them as one fused query_key_value module ("LLM+LoRA微调加速技术原理解析",
 * m.youleyou.com, 深入理解LoRA：基本原理与PEFT实现).  With n_out_blocks = P in
 * [2, PLORA_MAX_OUT_BLOCKS], W is P such projections stacked along d_out: block p
 * holds output columns [out_block_end[p-1], out_block_end[p]) (out_block_end[-1] = 0),
 * each end a multiple of 256, out_block_end[P-1] = d_out.  Every adapter then has its
 * own low-rank pair per block, all of rank r: Y[:, block p] = X W_p^T + s X A_p^T B_p^T.
 * The layouts stack the blocks (see plora_adapter).  P * roundup(max_rank, 16) must not
 * exceed 256.  Output blocks need the default tensor-core path (bf16, no
 * PLORA_FLAG_SIMT / UNFUSED / BASE_PAIR); other combinations return
 * PLORA_ERR_UNSUPPORTED.  n_out_blocks = 0 or 1 means one projection (the ends are
 * then ignored).
 */
typedef struct {
    int64_t d_in;
    int64_t d_out;
    int32_t dtype;
    int32_t max_adapters;
    int32_t max_rank;
    uint32_t flags;
    int64_t max_tokens;
    int32_t n_out_blocks;
    int32_t reserved;                               /* 0 */
    int64_t out_block_end[PLORA_MAX_OUT_BLOCKS];
} plora_config;

/*
 * One adapter.  rank r in [1, max_rank]; scale = alpha / r as the caller
 * computed it (finite); A: [r][d_in], B: [d_out][r] in the handle's dtype;
 * dA: [r][d_in], dB: [d_out][r] in fp32 (written by plora_backward, ignored
 * by plora_forward).  Every pointer 16-byte aligned.  With P output blocks,
 * A and dA are [P r][d_in] (rows p r .. p r + r - 1 are block p's A_p) and B, dB
 * stay [d_out][r] (the rows of block p's columns are its B_p).
 */
typedef struct {
    int32_t rank;
    float scale;
    const void* A;
    const void* B;
    float* dA;
    float* dB;
} plora_adapter;

typedef struct plora_ctx* plora_handle;

/*
 * Create a handle on the current CUDA device and allocate its workspace.
 * Returns PLORA_ERR_INVALID_ARG / PLORA_ERR_UNSUPPORTED for a bad config,
 * PLORA_ERR_OOM if the workspace cannot be allocated, PLORA_ERR_CUDA if no
 * usable sm_100 device is current.  *out is NULL on failure.
 */
PLORA_API plora_status plora_create(plora_handle* out, const plora_config* cfg);

/* Free the handle and its workspace (synchronises the device first). NULL is accepted. */
PLORA_API plora_status plora_destroy(plora_handle h);

/*
 * Size in bytes of the `saved` buffer that plora_forward fills and
 * plora_backward reads for this segment map and adapter table.  Its layout
 * is the library's: per-adapter zero-padded blocks of s_i X_i A_i rows and, on
 * the tensor-core path, every adapter's A and B packed as the tensor cores read
 * them (the forward packs them once; the backward reuses them, so A and B must
 * not change between the two calls).  Read it only through plora_debug_unpack_saved.
 */
PLORA_API plora_status plora_saved_bytes(plora_handle h, int32_t n_adapters, const int64_t* off,
                               const plora_adapter* tab, size_t* bytes);

/*
 * Forward.  X: [T][d_in], W: [d_out][d_in], Y (out): [T][d_out], all device.
 * n_adapters in [0, max_adapters]; off: host int64[n_adapters+1] with
 * off[0] = 0, non-decreasing, off[n] <= max_tokens; tab: host
 * plora_adapter[n_adapters].  saved (out): device buffer of
 * plora_saved_bytes() bytes, 256-byte aligned, kept for plora_backward.
 * When off[n] == 0 (no tokens), X, Y and saved may be NULL and nothing is written.
 */
PLORA_API plora_status plora_forward(plora_handle h, const void* X, const void* W, void* Y,
                           int32_t n_adapters, const int64_t* off, const plora_adapter* tab,
                           void* saved, void* stream);

/*
 * Backward.  Same X, W, off, tab and saved as the forward; dY: [T][d_out];
 * dX (out, may be NULL to skip the input gradient): [T][d_in]; writes every
 * adapter's dA and dB (which must be non-NULL).  When off[n] == 0, X, dY, dX
 * and saved may be NULL and only the (zero) weight gradients are written.
 */
PLORA_API plora_status plora_backward(plora_handle h, const void* X, const void* W, const void* dY,
                            void* dX, int32_t n_adapters, const int64_t* off,
                            const plora_adapter* tab, const void* saved, void* stream);

/*
 * Synchronise `stream` and report the handle's device error flag: PLORA_OK,
 * PLORA_ERR_TIMEOUT (a bounded device wait ran out), PLORA_ERR_BOUNDS (a
 * PLORA_DEBUG build's bounds check failed) or PLORA_ERR_CUDA.  A reported
 * flag is cleared.
 */
PLORA_API plora_status plora_check(plora_handle h, void* stream);

/* Static text for a status code. */
PLORA_API const char* plora_status_string(plora_status s);

/* Detail text of the handle's last failure ("" if none; valid until the next call on h). */
PLORA_API const char* plora_last_error(plora_handle h);

/*
 * Debug: copy adapter i's saved activation H'_i = s_i X_i A_i (the scaled
 * shrink, which both the expand and dB consume) out of `saved` as fp32
 * [n_i][r_i] into the device buffer H_out (16-byte aligned); with P output blocks,
 * [n_i][P r_i], block p in columns p r_i .. p r_i + r_i - 1.
 */
PLORA_API plora_status plora_debug_unpack_saved(plora_handle h, int32_t n_adapters, const int64_t* off,
                                      const plora_adapter* tab, const void* saved, int32_t i,
                                      float* H_out, void* stream);

/*
 * Debug / testing: the schedule one call would run for this configuration,
 * segment map and adapter table -- host logic only, no handle, no device.
 * Checks the arguments like plora_forward (or plora_backward if grads != 0)
 * and writes int32 records to out[0 .. capacity):
 *   which = 0: token tiles, 4 per tile: adapter, rows (1..128), first token
 *              row, first row in the saved H / workspace G buffers;
 *   which = 1: weight-gradient splits, 8 per split: adapter, first token row,
 *              first H/G row, 64-token blocks, split index, split count,
 *              first partial slot (-1 if unsplit), first counter (-1);
 *   which = 2: adapters, 5 per adapter: first token row, tokens, first H/G
 *              row (each adapter with tokens owns a block of 256 zero rows,
 *              its rows rounded up to 128, then 256 zero rows), the width of
 *              its H/G columns (P output blocks x the rank rounded up to 16;
 *              P = 1 without output blocks), that width rounded up to 64;
 *   which = 3: two values: the padded rank pitch RP and the H/G row count;
 *   which = 4: per global 256-row tile of the base GEMMs, the first index
 *              into the list of which = 5 (plus the end): ceil(T/256) + 1 values;
 *   which = 5: the adapters (with tokens) overlapping each such tile.
 * *count receives the number of int32 values the full answer needs.
 */
PLORA_API plora_status plora_debug_schedule(const plora_config* cfg, int32_t n_adapters, const int64_t* off,
                                            const plora_adapter* tab, int32_t grads, int32_t which,
                                            int32_t* out, int64_t capacity, int64_t* count);

/*
 * Optimizer state of one adapter for plora_adamw_step.  All arrays are fp32 device
 * buffers shaped like the adapter's factors (A: [r][d_in], B: [d_out][r]), 16-byte
 * aligned, updated in place.  A_master / B_master hold the fp32 parameters; with an
 * fp32 handle they may be NULL, and then the table's A / B are the fp32 parameters.
 */
typedef struct {
    float lr;            /* this step's learning rate for this adapter (after any schedule) */
    float beta1, beta2;  /* in [0, 1) */
    float eps;           /* > 0 */
    float weight_decay;  /* decoupled: p <- p (1 - lr weight_decay) */
    int32_t step;        /* 1-based count of this adapter's updates, for bias correction */
    float* A_master;
    float* B_master;
    float* mA;
    float* vA;
    float* mB;
    float* vB;
} plora_adamw_state;

/*
 * One AdamW step for every adapter in one launch (the optimizer update that follows the
 * backward in LoRA fine-tuning; "LLM+LoRA微调加速技术原理解析", m.youleyou.com, the PEFT
 * training loop with torch.optim.AdamW).  Per element of A_i and B_i, with g = dA_i / dB_i
 * from the table (fp32), in fp32:
 *     p <- p (1 - lr wd);   m <- b1 m + (1 - b1) g;   v <- b2 v + (1 - b2) g^2;
 *     p <- p - (lr / (1 - b1^t)) m / (sqrt(v) / sqrt(1 - b2^t) + eps)
 * then the table's A_i / B_i (the layer's parameters in the handle's dtype) receive p,
 * rounded to nearest even for bf16.  Adapters are independent: each has its own state.
 * tab: host plora_adapter[n] (rank, A, B written, dA, dB read); st: host
 * plora_adamw_state[n].  Errors as for plora_backward (every pointer is checked against
 * its device allocation before anything is launched).
 */
PLORA_API plora_status plora_adamw_step(plora_handle h, int32_t n_adapters, const plora_adapter* tab,
                                        const plora_adamw_state* st, void* stream);

/*
 * CUDA graph capture (a runtime facility; the pages describe no API).  A plora_forward,
 * plora_backward or plora_adamw_step called while its stream is being captured
 * (cudaStreamBeginCapture, torch.cuda.graph) takes one schedule slot reserved here instead
 * of the handle's ring, and keeps it: every replay of the graph re-copies that call's
 * schedule from the slot, which no later call overwrites.  Reserve before the capture begins
 * (these calls allocate: n pinned host buffers and n device buffers, each as large as one
 * call's schedule staging); a call captured with no reserved slot left returns
 * PLORA_ERR_INVALID_ARG and enqueues nothing.  Captured calls record no profiling events.
 * Replays and eager calls share the handle's workspace, so as for eager calls only one runs at
 * a time per handle.  plora_capture_release synchronises the device and frees every capture
 * slot: call it only once no graph that holds captured calls of this handle will replay again.
 * plora_destroy frees them too.
 */
PLORA_API plora_status plora_capture_reserve(plora_handle h, int32_t n);
PLORA_API plora_status plora_capture_release(plora_handle h);

/*
 * Launch geometry of the handle's device and of this build (a diagnostic; the method itself
 * has no such call): out[0] = SMs, out[1] / out[2] = the 2-SM clusters that can be resident at
 * once for the SM-pair Y / dX base GEMMs (PLORA_FLAG_BASE_PAIR), each <= SMs / 2; out[3] = rows
 * of a single-SM base-GEMM tile (256 or 128), out[4] / out[5] = the rasterisation windows of the
 * Y / dX base GEMMs in rows.  At most `capacity` values are written; *count receives 6.
 */
PLORA_API plora_status plora_device_info(plora_handle h, int32_t* out, int32_t capacity, int32_t* count);

/*
 * Profiling.  The handle always counts its kernel launches per kernel kind.
 * With profiling enabled, it also brackets every launch with CUDA events on
 * the launching stream and sums each kernel's device time.
 */
PLORA_API plora_status plora_profile_enable(plora_handle h, int32_t enable);

/*
 * Synchronise on the recorded events, then report, per kernel kind, the
 * launches and the summed device milliseconds since the last read (and reset
 * both).  *n_kinds receives the number of kinds; at most `capacity` entries
 * of names (static strings), launches and total_ms (each may be NULL) are
 * written.
 */
PLORA_API plora_status plora_profile_read(plora_handle h, int32_t capacity, int32_t* n_kinds,
                                          const char** names, int64_t* launches, double* total_ms);

/*
 * Allocation-free dB: dB_i = s_i H_i^T dY_i for every adapter -- the same
 * product, schedule and results as the dB part of plora_backward -- without a
 * handle and without allocating anything.  The paper has no counterpart; this
 * entry point exists for callers that cannot allocate device memory: code
 * running under a memory planner or a caching allocator that owns the whole
 * device and forbids any other cudaMalloc, code that must not synchronise the
 * device (cudaMalloc and cudaFree can), and hosts that hand a library only
 * the tensors it works on.
 *
 * Its scratch (schedule, token-split partials, arrival counters, error flag)
 * is one static device array of PLORA_STATIC_SCRATCH_BYTES that every GPU
 * loading this library holds until the process exits.  The call allocates
 * nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 *
 * cfg: as for plora_create (bf16, no PLORA_FLAG_SIMT, one output block; the max_*
 * fields bound the call).  dY: [T][d_out] bf16 device; saved: the buffer a plora_forward
 * with the same off and adapter ranks filled; off, tab: host arrays as for
 * plora_backward (only rank, scale and dB are read; dB must be non-NULL and
 * 16-byte aligned, A and B must still be valid pointers).  Writes every dB_i.
 *
 * Returns PLORA_ERR_UNSUPPORTED when the call does not fit the array, whose
 * first MiB holds the schedule and whose rest holds the split state:
 *   - the schedule, 256 + 64 x n_adapters + 32 x (token splits) bytes (each
 *     part rounded up to 256), must fit in 1 MiB; an adapter has
 *     ceil(n_i / 16384) token splits;
 *   - the split state of the adapters longer than 16384 tokens must fit in
 *     PLORA_STATIC_SCRATCH_BYTES - 1 MiB: their arrival counters,
 *     S x max(ceil(d_in/128), ceil(d_out/128)) x 4 bytes rounded up to 256
 *     (S = the number of such adapters), then their partials,
 *     (their token splits) x ceil(d_out/128) x 128 x RP x 4 bytes, with RP the
 *     largest rank rounded up to 64.
 * Other errors as for plora_backward; a device wait that runs out of time is
 * not reported (there is no handle to report it through).
 *
 * The schedule reaches the array through the parameters of small staging
 * kernels, which the launch copies when it is enqueued: the call copies
 * nothing from host memory and does not wait for the stream's earlier work.
 * The first call on each device resolves the array's device address and sets
 * the kernel up; make that first call before any stream capture begins.
 * Every call shares the one array and clears what must start at zero (the
 * error flag and the arrival counters); calls whose work overlaps on the GPU
 * (different streams, or different host threads) race on it and must be
 * serialised by the caller.
 */
#define PLORA_STATIC_SCRATCH_BYTES (16u << 20)
PLORA_API plora_status plora_grad_B_static(const plora_config* cfg, const void* dY, int32_t n_adapters,
                                           const int64_t* off, const plora_adapter* tab, const void* saved,
                                           void* stream);

/*
 * Layer calls: several projections that share one segment map (the same adapters over the same
 * packed token rows) and read and write independent tensors run as ONE launch set, one persistent
 * launch per product kind over all of them, instead of one set per projection.  A LoRA fine-tuning
 * job adapts several linear modules of each layer (query, key, value, output, and the MLP's gate, up
 * and down projections; "LoRA加速集成方案", cloud.baidu.com, 七 › 2. 层的选择), and PLoRA packs each
 * adapter's tokens through all of them.  Projections that read one input (q|k|v, gate|up) go in as
 * one projection with output blocks.  Each projection is a segment of the memory-bound launches, with its
 * own parameters and tensor maps: a forward launches one schedule copy, one pack and one shrink for
 * all projections, and one base GEMM per projection; a backward one schedule copy and one launch of
 * G's shrink with dB for all projections, and per projection one dX GEMM with its dA filling the last
 * wave (projections whose dX is skipped run their dA together).  The base GEMMs get a launch each
 * because their tiles differ in length between projections, and one persistent launch over them would
 * let the SMs drift apart in the tile order, at a cost in L2 reuse.  Results are bit for bit those of
 * separate plora_forward / plora_backward calls on the projections' handles.
 *
 * The projections must not depend on each other within a call (the launch set runs them
 * concurrently): in a model, a layer call groups projections whose inputs are all ready, for example
 * the independent targets of a benchmark, or the weight and input gradients of projections whose
 * output gradients are all known.
 */
#define PLORA_MAX_LAYER_PROJ 8
typedef struct plora_layer_ctx* plora_layer;

/* One projection of a layer call.  Shapes and layouts as for plora_forward / plora_backward with this
 * projection's d_in, d_out: X [T][d_in], W [d_out][d_in], Y and dY [T][d_out], dX [T][d_in] (device);
 * tab: host plora_adapter[n_adapters], this projection's factors (and gradients, for the backward);
 * saved: device, 256-byte aligned, plora_layer_saved_bytes() bytes, filled by the forward.  The
 * forward reads X, W, tab, saved and writes Y; the backward reads X, W, dY, tab, saved and writes dX
 * (may be NULL to skip it) and every dA, dB. */
typedef struct {
    const void* X;
    const void* W;
    void* Y;
    const void* dY;
    void* dX;
    const plora_adapter* tab;
    void* saved;
} plora_proj;

/*
 * Create a layer of n_proj in [1, PLORA_MAX_LAYER_PROJ] projections on the current device, one
 * handle per configuration (as plora_create; the tensor-core path only: bf16 without PLORA_FLAG_SIMT,
 * PLORA_FLAG_UNFUSED or PLORA_FLAG_BASE_PAIR, else PLORA_ERR_UNSUPPORTED).  *out is NULL on failure.
 */
PLORA_API plora_status plora_layer_create(plora_layer* out, int32_t n_proj, const plora_config* cfgs);
/* Free the layer and its handles (synchronises the device first).  NULL is accepted. */
PLORA_API plora_status plora_layer_destroy(plora_layer L);
/* The handle of projection p (owned by the layer): for plora_check, plora_adamw_step, the profile
 * calls (a layer call's launches are counted and timed on projection 0's handle) and the debug calls. */
PLORA_API plora_status plora_layer_handle(plora_layer L, int32_t p, plora_handle* h);
/* bytes (out): host size_t[n_proj], each projection's saved-buffer size for this call. */
PLORA_API plora_status plora_layer_saved_bytes(plora_layer L, int32_t n_adapters, const int64_t* off,
                                               const plora_proj* projs, size_t* bytes);
/* Forward of every projection (projs: host plora_proj[n_proj]; off as for plora_forward, shared). */
PLORA_API plora_status plora_layer_forward(plora_layer L, int32_t n_adapters, const int64_t* off,
                                           const plora_proj* projs, void* stream);
/* Backward of every projection, reading the saved buffers their layer forward filled. */
PLORA_API plora_status plora_layer_backward(plora_layer L, int32_t n_adapters, const int64_t* off,
                                            const plora_proj* projs, void* stream);
/* Errors: every argument of every projection is checked before anything is enqueued (nothing is
 * written on an error; plora_layer_last_error names the projection).  Device errors as for
 * plora_check, through plora_layer_check (synchronises `stream`, reports the first projection's
 * error, clears the flags). */
PLORA_API plora_status plora_layer_check(plora_layer L, void* stream);
PLORA_API const char* plora_layer_last_error(plora_layer L);

/*
 * Multi-GPU sharding of one adapter set: assign each adapter to one of n_parts GPUs (one process
 * per GPU, each running its own handle over its share), balancing the parts' costs.  PLoRA runs
 * each packed job on a chosen number of GPUs (PLoRA summary, gist.science, arXiv 2508.02932,
 * 技术摘要 › 方法论 › 1. LoRA 打包规划器 (parallelism degree per job)); adapters are independent, so a
 * part needs no data from another and no collective follows.  Host logic only: no device, no handle.
 *
 * counts: host int64[n] tokens per adapter (>= 0); ranks: host int32[n] in [1, PLORA_MAX_RANK];
 * d_in, d_out: the projection; flops_per_s, bytes_per_s (> 0): the tensor and memory peaks the cost
 * model divides by.  Adapter i costs
 *     n_i ( (4 d_in d_out + 6 r_i (d_in + d_out)) / flops_per_s + (8 (d_in + d_out) + 12 r_i) / bytes_per_s )
 * (its tokens' share of the two base GEMMs and the low-rank products, and the low-rank kernels' bytes).
 * Longest processing time first: adapters by decreasing cost (ties: lower index first) each go to the
 * part with the least cost so far (ties: lower part index), so the result is deterministic and the
 * largest part's cost is at most (4/3 - 1/(3 n_parts)) times the best possible.
 * owner (out): host int32[n], the part of each adapter; part_cost (out, may be NULL): host
 * double[n_parts], each part's summed cost.  n in [0, PLORA_MAX_ADAPTERS], n_parts in
 * [1, PLORA_MAX_ADAPTERS]; anything else returns PLORA_ERR_INVALID_ARG and writes nothing.
 */
PLORA_API plora_status plora_partition(int32_t n_adapters, const int64_t* counts, const int32_t* ranks,
                                       int64_t d_in, int64_t d_out, double flops_per_s, double bytes_per_s,
                                       int32_t n_parts, int32_t* owner, double* part_cost);

/*
 * Debug / failure detection: launch one CTA whose bounded wait is on a barrier that
 * nothing ever arrives at, through the same bounded-wait code the kernels use, with a
 * limit of timeout_ns (1 ms .. 10 s).  The wait runs out, the kernel records
 * PLORA_ERR_TIMEOUT in the handle's device error flag and returns; the next
 * plora_check(h, stream) reports PLORA_ERR_TIMEOUT (and clears the flag).  No trap, no
 * fault, no hang: the context stays usable.
 */
PLORA_API plora_status plora_debug_timeout_probe(plora_handle h, int64_t timeout_ns, void* stream);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
PLORA_API int32_t plora_version(void);

/*
 * 1 for the PLORA_DEBUG build of this library (libplora_debug.so), 0 otherwise (a diagnostic; the
 * method has no such call).  In the debug build every kernel compares each index it forms from a
 * call's schedule with the extent of the buffer it addresses, as the host allocated it (the output
 * and the saved activations, the packed factors, the split partials and arrival counters, the
 * schedule tables); a failed check sets the handle's error flag to PLORA_ERR_BOUNDS and the access
 * is skipped (an out-of-range schedule entry is replaced by entry 0), so plora_check reports the error
 * and nothing traps.  The checks cost time; results on valid inputs are those of the release build.
 */
PLORA_API int32_t plora_debug_build(void);

#ifdef __cplusplus
}
#endif

#endif /* PLORA_H */
