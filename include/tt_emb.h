/*
 * tt_emb.h -- C ABI of the B200 Tensor-Train embedding gather library (libttemb.so).
 *
 * The operation (FlowTT: Exploiting Computation Flow Reuse in Irregular
 * Tensor-Train Embedding -- Abstract, section 2.4 "Problem Definition",
 * section 3.2 "Flow-Aware Fused TT Embedding Execution", section 3.3
 * "Flow-Aligned Prefix-Based Index Grouping"):
 *
 *   A virtual table of N rows and D = d_1*...*d_k columns is held as k TT
 *   cores G_j, each a row-major float32 array of shape [r_{j-1}][n_j][d_j][r_j]
 *   with r_0 = r_k = 1 and N <= n_1*...*n_k.  Row i is split into mixed-radix
 *   digits (i_1..i_k) over (n_1..n_k), i_1 the most significant; the row is
 *   the chained product G_1[:, i_1] . G_2[:, i_2] ... G_k[:, i_k], column
 *   (a_1..a_k) flattened row-major.  Lookups are sum-pooled into bags.  Rows
 *   that share their first k-1 digits (the prefix) share the intermediate
 *   product of the first k-1 slices; the library groups a batch by prefix
 *   (sort, unique, run-length encoding) and computes each shared intermediate
 *   once.  Training adds dL/dG_j for L = sum_b <grad_out_b, out_b> and a plain
 *   SGD step.
 *
 * Conventions shared by every entry point
 *   - One handle holds T tables that share k, d and r; each table has its own
 *     (n_1..n_k) and its own valid row count N_t.  Limits: 1 <= T <=
 *     TT_EMB_MAX_TABLES, 1 <= k <= TT_EMB_MAX_CORES, N_t < 2^31 * ... see
 *     tt_emb_create.
 *   - "device" pointers are CUDA global-memory pointers of the current device;
 *     "host" pointers are ordinary CPU memory.  The library never frees memory
 *     it did not allocate; it only allocates the handle (host) and, in
 *     tt_emb_create, one small device status block (freed by tt_emb_destroy).
 *   - Bags are table-major: bag (t, b) holds indices[offsets[t*B+b] ..
 *     offsets[t*B+b+1]), and its pooled row goes to out[b][t*D .. (t+1)*D).
 *   - Calls that take a stream only enqueue work on it and never synchronise
 *     the host.  Errors found on the host (bad arguments, shapes, state) are
 *     returned at once.  Errors found on the device (an index outside
 *     [0, N_t), offsets that are not a valid partition of [0, L), a bounded
 *     wait that ran out) are recorded in the handle's device status block;
 *     every later kernel of the handle then does nothing, the outputs of the
 *     failed call are unspecified, and the code surfaces at the next
 *     tt_emb_sync().  No error ever crosses the ABI as an exception.
 *   - Calls on one handle must be ordered (same stream, or ordered streams);
 *     two handles are independent.
 */
#ifndef TT_EMB_H
#define TT_EMB_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TT_EMB_MAX_TABLES 64
#define TT_EMB_MAX_CORES 4
#define TT_EMB_ABI_VERSION 1

typedef struct tt_emb_handle* tt_emb_t;
/* A cudaStream_t passed as an opaque pointer (NULL = the legacy default stream). */
typedef void* tt_stream_t;

typedef enum {
    TT_OK = 0,
    TT_ERR_ARG = 1,          /* a null pointer, a negative size or an unknown option */
    TT_ERR_SHAPE = 2,        /* table / core shapes outside the supported set */
    TT_ERR_INDEX_RANGE = 3,  /* (device) an index outside [0, N_t) */
    TT_ERR_OFFSETS = 4,      /* (device) offsets not monotone, offsets[0] != 0 or offsets[T*B] != L */
    TT_ERR_WORKSPACE = 5,    /* no workspace, or one smaller than tt_emb_workspace_size() asked for */
    TT_ERR_STATE = 6,        /* cores not set, backward without a forward, grads not registered */
    TT_ERR_CUDA = 7,         /* a CUDA runtime call failed (launch, memset, copy) */
    TT_ERR_TIMEOUT = 8,      /* (device) a bounded wait ran out of iterations */
    TT_ERR_UNSUPPORTED = 9   /* a valid request this build does not implement */
} tt_status;

/* Scheduling of the fused kernels (FlowTT section 3.4 and the ablation in section 4). */
typedef enum {
    TT_SCHED_STATIC = 0,     /* each block takes a fixed, precomputed share of the prefix groups */
    TT_SCHED_STEAL = 1,      /* persistent blocks: own share first, then steal chunks of unfinished groups */
    TT_SCHED_STEAL_L2 = 2    /* as STEAL, and shared intermediates of split groups are checkpointed in L2 */
} tt_sched_mode;

/* Grouping depth (FlowTT section 4, "Prefix-Based Reuse over Exact Deduplication"). */
typedef enum {
    TT_GROUP_PREFIX = 0,     /* deduplicate rows and share each prefix intermediate */
    TT_GROUP_UNIQUE_ONLY = 1 /* deduplicate rows only: every distinct row is contracted on its own */
} tt_group_mode;

/*
 * Arithmetic of the prefix-level products (FlowTT section 3.3 computes the prefix
 * contraction C_p = G_1[0, i_1] . G_2[:, i_2] once per prefix group; the pages compute in
 * fp32).  TT_PREC_BF16_TC rounds the operands to bf16 (round to nearest even) and runs
 * the products on the fifth-generation tensor cores, accumulating in fp32 in tensor
 * memory: in the forward the prefix contraction; in the backward, for r_1 = r_2 = 64,
 * also the recomputed C_p and the two gradient products dG_1 += dC_p . G_2[:, i_2]^T and
 * dG_2[:, i_2] += G_1[0, i_1]^T . dC_p (dC_p itself is rounded to bf16 for them).  The
 * suffix contraction, the pooling and the per-row backward (dG_3, dC_p) stay fp32.
 * Results agree with the exact (fp64) definition to within 2e-2, measured normwise per
 * pooled row and per digit slice of a core gradient.  It needs three cores with
 * d = (4, 4, 8) and r_1 = r_2 in {32, 64}; tt_emb_create returns TT_ERR_SHAPE otherwise.
 */
typedef enum {
    TT_PREC_FP32 = 0,        /* fp32 operands and accumulation on the FP32 pipes (default) */
    TT_PREC_BF16_TC = 1,     /* bf16 operands, fp32 accumulation, tcgen05 tensor cores (bound 2e-2) */
    TT_PREC_FP32_SPLIT_TC = 2 /* fp32-accurate on the tensor cores: every operand value x is held as
                                 two bf16 terms hi = bf16(x), lo = bf16(x - hi) (|x - hi - lo| <=
                                 2^-18 |x|) and each product is hi.hi + hi.lo + lo.hi with fp32
                                 accumulation; same coverage as TT_PREC_BF16_TC, bound 1e-4 */
} tt_precision;

typedef struct {
    int32_t sched;           /* tt_sched_mode, default TT_SCHED_STEAL_L2 */
    int32_t grouping;        /* tt_group_mode, default TT_GROUP_PREFIX */
    int32_t chunk;           /* distinct rows per stealable subtask of the fused forward, 1..256;
                                0 = 256 (longer chunks of prefix groups are split) */
    int32_t grid;            /* persistent blocks; 0 = one wave on the current device (the fused forward
                                never runs more than one resident wave) */
    int32_t force_generic;   /* 1: run the shape-generic kernels even where a specialised path exists */
    int32_t precision;       /* tt_precision, default TT_PREC_FP32 */
    int32_t reserved[10];    /* must be zero */
} tt_emb_options;

/* Fills *opt with the defaults (scheduler STEAL_L2, prefix grouping, fp32 pipes).  The
 * options select among the pages' design points: FlowTT section 3.4 (scheduling), section 4
 * "Prefix-Based Reuse over Exact Deduplication" (grouping). */
void tt_emb_default_options(tt_emb_options* opt);

/*
 * Creates a handle for T tables sharing k, d and r (host call, no device work
 * besides allocating the 256-byte device status block).  The table is the TT
 * format of FlowTT section 2.4 "Problem Definition" (cores [r_{j-1}][n_j][d_j][r_j],
 * r_0 = r_k = 1) and of the TT-Rec abstract (TT-EmbeddingBag).
 *   num_tables   T, 1..TT_EMB_MAX_TABLES
 *   num_cores    k, 1..TT_EMB_MAX_CORES
 *   n_factors    host int64 [T][k]: n_j of each table, each >= 1; the product of
 *                a table's factors must be < 2^40
 *   n_rows       host int64 [T]: valid rows N_t, 1 <= N_t <= prod_j n_j and N_t < 2^32
 *   d_factors    host int32 [k]: d_j >= 1, D = prod d_j <= 1024
 *   ranks        host int32 [k+1]: r_0 = r_k = 1, 1 <= r_j <= 128
 *   opt          host, may be NULL (defaults)
 *   out          host: receives the handle
 * Returns TT_OK, TT_ERR_ARG, TT_ERR_SHAPE or TT_ERR_CUDA.
 */
int tt_emb_create(int32_t num_tables, int32_t num_cores, const int64_t* n_factors,
                  const int64_t* n_rows, const int32_t* d_factors, const int32_t* ranks,
                  const tt_emb_options* opt, tt_emb_t* out);

/*
 * Registers the cores (and optionally the gradient buffers) by borrowing
 * device pointers (FlowTT section 2.4: the TT cores G_j that replace the table).  Host arrays of T*k device pointers, table-major
 * (entry t*k + j is core j of table t, float32 [r_{j-1}][n_j][d_j][r_j],
 * 16-byte aligned).  core_grads may be NULL for inference; when given, each
 * buffer has the shape of its core and is overwritten by tt_emb_backward.
 * The caller keeps ownership and must keep the memory alive while the handle
 * uses it.  Returns TT_OK or TT_ERR_ARG.
 */
int tt_emb_set_cores(tt_emb_t h, float* const* cores, float* const* core_grads);

/*
 * Device workspace needed for batches of at most max_lookups lookups and
 * batch bags per table (host call).  *bytes receives the size.  It holds the
 * grouping of FlowTT section 3.3 (sort buffers, distinct rows, prefix groups) and
 * the plan of section 3.4, plus the row checkpoint of the fused kernels; FlowTT
 * section 5 reports peak memory, which this figure bounds for the library's part.
 * Returns TT_OK or TT_ERR_ARG (null handle or pointer, negative sizes,
 * max_lookups >= 2^31 - 1).
 */
int tt_emb_workspace_size(tt_emb_t h, int64_t max_lookups, int64_t batch, size_t* bytes);

/*
 * Registers caller-owned device workspace (256-byte aligned) of `bytes` bytes,
 * sized for (max_lookups, batch) by tt_emb_workspace_size.  The workspace
 * holds the segmentation between a forward and its backward (FlowTT section 3.2:
 * the backward reverses the forward's flow); it must not be shared by two
 * handles that run at the same time.  Returns TT_OK, TT_ERR_ARG (null or
 * misaligned pointer, bad sizes) or TT_ERR_WORKSPACE (bytes below the size asked).
 */
int tt_emb_set_workspace(tt_emb_t h, void* workspace, size_t bytes, int64_t max_lookups,
                         int64_t batch);

/*
 * Forward pass (FlowTT section 3.3 grouping, section 3.2 fused execution "C = A.B,
 * then E = C.D, followed by pooling", section 3.4 persistent scheduling):
 * out[b][t*D + c] = sum over bag (t, b) of row_t(i)[c] (float32,
 * fp32 accumulation).  Enqueues on `stream`: index validation, digit/key
 * extraction, radix sort, unique + prefix run-length grouping, and the fused
 * gather + pooling kernel.
 *   indices   device int64 [num_lookups], each in [0, N_t) of its table
 *   offsets   device int64 [T*batch + 1], non-decreasing, offsets[0] = 0,
 *             offsets[T*batch] = num_lookups
 *   out       device float32 [batch][T*D], overwritten (empty bags give 0)
 * num_lookups and batch must not exceed the workspace's sizes.  The
 * segmentation is kept in the workspace for tt_emb_backward.  Host errors:
 * TT_ERR_ARG, TT_ERR_STATE (no cores), TT_ERR_WORKSPACE, TT_ERR_CUDA (a launch
 * failed); device errors (TT_ERR_INDEX_RANGE, TT_ERR_OFFSETS, TT_ERR_TIMEOUT)
 * surface at tt_emb_sync.
 */
int tt_emb_forward(tt_emb_t h, const int64_t* indices, const int64_t* offsets,
                   int64_t num_lookups, int64_t batch, float* out, tt_stream_t stream);

/*
 * Backward pass of the last forward on this handle (FlowTT section 3.2: "the
 * backward path reverses this structure"): overwrites the registered
 * core_grads with dL/dG_j for L = sum <grad_out, out> (zero for slices no
 * lookup touched).  grad_out: device float32 [batch][T*D] of the last forward's
 * batch.  Reuses the forward's segmentation (no re-sort).  Returns
 * TT_ERR_STATE without a preceding forward or without registered core_grads.
 */
int tt_emb_backward(tt_emb_t h, const float* grad_out, tt_stream_t stream);

/* SGD step on every registered core: G <- G - lr * dG (float32, elementwise).  The
 * training step the pages time (FlowTT section 4, training latency) ends with an
 * optimiser step; the pages name none, so this is plain SGD without momentum.
 * Returns TT_OK, TT_ERR_ARG, TT_ERR_STATE (cores or gradients missing) or TT_ERR_CUDA. */
int tt_emb_sgd_update(tt_emb_t h, float lr, tt_stream_t stream);

/*
 * Backward pass and SGD step fused, with a sparse update of the middle core (the
 * "sparse fused optimizer" follow-on to FlowTT section 3.2's backward).  The result for the
 * cores is that of tt_emb_backward followed by tt_emb_sgd_update(lr).  On three-core
 * tables served by the shape-specialised kernels, the block that reduces a column group's
 * dG_2[:, i_2] on chip applies G_2[:, i_2] -= lr * dG_2[:, i_2] itself, so dG_2 is neither
 * zero-filled, written nor read back; G_2 slices no lookup touched are not visited.  In that
 * case the registered core_grads of the middle cores are left unchanged (not gradients);
 * those of the other cores hold their gradients.  Other tables take the unfused
 * path (every registered gradient is written).  Same arguments and errors as
 * tt_emb_backward; registered core_grads are required (the first and last cores' gradients
 * are reduced there).
 */
int tt_emb_backward_sgd(tt_emb_t h, const float* grad_out, float lr, tt_stream_t stream);

/*
 * Test and inspection hook: device views of the last forward's segmentation
 * (FlowTT section 3.3: sorted indices, unique extraction, prefix run-length
 * groups), valid until the next forward on the handle.  Synchronises the stream
 * of the last call to read the counts.  TT_ERR_STATE without a forward.
 */
typedef struct {
    int64_t num_lookups;        /* L */
    int64_t num_unique;         /* U: distinct (table, row) pairs */
    int64_t num_groups;         /* G: distinct (table, prefix) pairs */
    int32_t key_bits;           /* bits of the row field in a sort key */
    int32_t key_bytes;          /* 4 or 8 */
    const void* sorted_keys;    /* device [L]: (table << key_bits) | row, ascending */
    const int32_t* perm;        /* device [L]: input position of each sorted lookup (stable) */
    const void* uniq_keys;      /* device [U]: the distinct keys */
    const int32_t* uniq_start;  /* device [U+1]: first sorted lookup of each distinct key */
    const int32_t* grp_start;   /* device [G+1]: first distinct key of each prefix group */
    const int32_t* bag_sorted;  /* device [L]: bag t*B + b of each sorted lookup */
} tt_seg_view;

int tt_emb_get_segmentation(tt_emb_t h, tt_seg_view* view);

/*
 * Copies the last forward's segmentation arrays (see tt_seg_view for shapes)
 * into caller buffers, host or device (any pointer may be NULL to skip it).
 * Synchronous.  Test and inspection hook.
 */
int tt_emb_copy_segmentation(tt_emb_t h, void* sorted_keys, int32_t* perm, void* uniq_keys,
                             int32_t* uniq_start, int32_t* grp_start, int32_t* bag_sorted);

/*
 * Waits for the handle's work on the stream of its last call and returns the
 * first device-side error recorded since the last tt_emb_sync (then clears it),
 * or TT_ERR_CUDA if the stream itself failed.  The device errors are the input
 * checks of the grouping step (FlowTT section 3.3) and the bounded waits of the
 * persistent scheduler (section 3.4).
 */
int tt_emb_sync(tt_emb_t h);

/*
 * The most recent failure on this handle, then cleared: the code of the last
 * call on it that returned an error (host-detected), or of a device error that
 * tt_emb_sync reported, whichever came last; TT_OK when nothing failed since the
 * handle was created or since the previous tt_emb_last_error.  Host call; it
 * never waits for the device (use tt_emb_sync for that).  A null handle gives
 * TT_ERR_ARG.
 */
int tt_emb_last_error(tt_emb_t h);

/* Message for a status code (static storage, never null). */
const char* tt_emb_error_string(int code);

/* Destroys the handle (host + its status block).  NULL is ignored. */
void tt_emb_destroy(tt_emb_t h);

/*
 * Per-phase device timing, for benchmarks.  While enabled, every call records
 * CUDA events on its stream around each phase below; tt_emb_sync() folds the
 * finished intervals into per-phase totals.  tt_emb_phase_times copies the
 * totals (milliseconds, host double [TT_EMB_NUM_PHASES]) and the number of
 * kernels the handle has launched since timing was last enabled (host int64,
 * may be NULL).  Enabling resets both.  The launch count is kept whether or
 * not timing is on.
 */
typedef enum {
    TT_PHASE_FWD_KEYS = 0,   /* offsets/index validation and key extraction */
    TT_PHASE_FWD_SORT = 1,   /* radix sort of the keys */
    TT_PHASE_FWD_SEGMENT = 2,/* unique + prefix run-length segmentation */
    TT_PHASE_FWD_FUSED = 3,  /* fused gather + pooling (includes zeroing out) */
    TT_PHASE_BWD_FUSED = 4,  /* fused backward kernel (prefix/suffix partial products, dG per digit) */
    TT_PHASE_BWD_REDUCE = 5, /* gradient zero fill and the merged-core split of four-core tables */
    TT_PHASE_SGD = 6,        /* SGD update */
    TT_PHASE_BWD_ROWSUM = 7, /* upstream gradient summed per distinct row (reverse of pooling) */
    TT_EMB_NUM_PHASES = 8
} tt_phase;

int tt_emb_enable_timing(tt_emb_t h, int enable);
int tt_emb_phase_times(tt_emb_t h, double* ms, int64_t* launches);

/*
 * tt_emb_forward_noalloc -- the forward pass (same arguments and output contract
 * as tt_emb_forward) for callers that cannot allocate device memory.  The paper
 * has no counterpart; this is a deployment variant of this library.
 *
 * Arithmetic: it always runs the shape-generic FP32 kernels, whatever the
 * handle's precision option, so its output matches tt_emb_forward within the
 * parity tolerance (1e-4 normwise per pooled row), not bit for bit; on a handle
 * in TT_PREC_BF16_TC mode it is the more exact of the two.
 *
 * Who needs it: hosts that give an embedded library neither an allocator nor
 * a workspace (plugin interfaces with fixed buffers), processes that forbid
 * device allocation once they are serving so that memory use and latency stay
 * fixed, and C callers that do not link PyTorch or any other allocator.  None
 * of them can provide the workspace that tt_emb_set_workspace expects.
 *
 * Instead, the sort buffers, histograms and segmentation arrays live in one
 * fixed device array of TT_EMB_NOALLOC_SCRATCH_BYTES (16 MiB) that is part of
 * the library: every GPU on which the library is used holds it until the
 * process exits.  The call itself allocates nothing (no cudaMalloc, cudaFree or
 * allocating library routine); the caller still passes inputs and outputs, and
 * the handle (created beforehand) supplies cores and its status block.
 *   - num_lookups above TT_EMB_NOALLOC_MAX_LOOKUPS (262144) is rejected with
 *     TT_ERR_WORKSPACE before any work is enqueued.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and keeps it.  With
 *     CUDA's lazy module loading (the default since CUDA 12.2) that lookup is
 *     also what loads the library's module holding the array, which reserves its
 *     16 MiB on that device at that moment and can fail if the device is full.
 *     So make the first call at start-up, before serving and before any stream
 *     capture; a call with num_lookups = 0 does the set-up (it only zero-fills
 *     `out`).
 *   - The handle's device (the one current at tt_emb_create) must be current;
 *     otherwise the call returns TT_ERR_STATE before enqueuing anything.
 *   - Every call, on every handle and stream, shares the one array, which keeps
 *     the previous call's contents (the call clears what must start at zero).
 *     Calls that overlap on the GPU race: order them (one stream, or events).
 *   - The segmentation of this call is not kept for tt_emb_backward; a backward
 *     after it returns TT_ERR_STATE until the next tt_emb_forward.
 */
#define TT_EMB_NOALLOC_MAX_LOOKUPS 262144
#define TT_EMB_NOALLOC_SCRATCH_BYTES (16u << 20)

int tt_emb_forward_noalloc(tt_emb_t h, const int64_t* indices, const int64_t* offsets,
                           int64_t num_lookups, int64_t batch, float* out, tt_stream_t stream);

/*
 * Balance probe of the persistent scheduler (FlowTT section 2.4: skewed prefix frequencies
 * create load imbalance; section 3.4 balances it).  While `records` is set, every block of
 * the fused forward kernel (slot 0) and of the fused backward kernel (slot 1) writes one
 * record of 4 uint64 at records[(slot * max_blocks + block) * 4]: SM id (bits 0-15) | the
 * number of C tiles the block read from an L2 checkpoint slot (bits 16-31) | tasks << 32, the
 * block's start and end on the GPU's global timer (ns), and the nanoseconds it spent in
 * bounded waits (pooling tasks waiting for their table).  Blocks >= max_blocks write nothing;
 * each launch overwrites its slot.  records: device memory of 2 * max_blocks * 4 uint64,
 * 8-byte aligned, owned by the caller; NULL turns the probe off.  Returns TT_OK or TT_ERR_ARG.
 */
int tt_emb_set_probe(tt_emb_t h, uint64_t* records, int32_t max_blocks);

/*
 * Test hook for failure detection (no GPU fault is involved).  Arms one
 * injected failure of a bounded device wait; it is consumed by the next call
 * that runs the wait:
 *   TT_INJECT_POOL_WAIT      next tt_emb_forward on the shape-specialised path:
 *                            every pooling task waits for one more finished
 *                            chunk of its table than there is, polling at most
 *                            `spin_limit` times (0 = the library's default)
 *                            before it records TT_ERR_TIMEOUT and returns.
 *   TT_INJECT_MMA_WAIT_FWD   next tt_emb_forward in a tensor-core precision: the
 *   TT_INJECT_MMA_WAIT_BWD   (or next backward's) first tensor-core completion
 *                            wait reports that it ran out once the products have
 *                            completed, so the kernel takes its timeout exit
 *                            (copies drained, tensor memory freed) and records
 *                            TT_ERR_TIMEOUT.
 *   TT_INJECT_NONE           disarms.
 * The error surfaces at tt_emb_sync like any device error; the handle is then
 * usable again.  Returns TT_OK, TT_ERR_ARG or TT_ERR_UNSUPPORTED (the handle has
 * no such wait: generic kernels, or no tensor-core precision).
 */
typedef enum {
    TT_INJECT_NONE = 0,
    TT_INJECT_POOL_WAIT = 1,
    TT_INJECT_MMA_WAIT_FWD = 2,
    TT_INJECT_MMA_WAIT_BWD = 3
} tt_inject;

int tt_emb_debug_inject(tt_emb_t h, int32_t what, int32_t spin_limit);

/* ABI version of the loaded library (TT_EMB_ABI_VERSION). */
int tt_emb_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* TT_EMB_H */
