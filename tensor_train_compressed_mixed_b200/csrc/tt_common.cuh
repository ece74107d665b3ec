// Internal declarations shared by the kernels and the C ABI of libttemb.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "tt_emb.h"

namespace tt {

constexpr int kMaxT = TT_EMB_MAX_TABLES;
constexpr int kMaxK = TT_EMB_MAX_CORES;
constexpr unsigned kFull = 0xffffffffu;

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

// ---------------------------------------------------------------------------
// Device status block (one per handle, 256 bytes): word 0 holds the first
// error code raised by any kernel, word 1 a detail (e.g. the bad position).
// Every kernel returns at once when word 0 is set, so one bad input stops the
// rest of the call without touching memory it was not given.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void raise_error(int32_t* st, int code, int info)
{
    if (atomicCAS(st, 0, code) == 0) st[1] = info;
}

__device__ __forceinline__ bool has_error(const int32_t* st)
{
    return *reinterpret_cast<const volatile int32_t*>(st) != 0;
}

// Counters that the grouping kernels leave in the workspace header.
struct WsCounters {
    int64_t num_unique;  // U: distinct (table, row) keys
    int64_t num_groups;  // G: prefix groups
    int64_t pad[30];
};

// Parameters of the key / grouping kernels.
struct KeyParams {
    int32_t T;
    int32_t ibits;        // bits of the row field of a key
    int64_t B;            // bags per table
    int64_t L;            // lookups
    int32_t unique_only;  // 1: every distinct row is its own group
    int32_t pad;
    uint32_t nrows[kMaxT];  // valid rows per table
    uint32_t nlast[kMaxT];  // n_k per table (prefix = row / n_k)
};

// Shapes and cores of the fused kernels.
struct CoreParams {
    int32_t T, k, D;
    int32_t P;            // rows of the prefix intermediate, D / d_k
    int32_t d[kMaxK];
    int32_t r[kMaxK + 1];
    int32_t ibits;
    int32_t unique_only;
    int64_t B;
    uint32_t n[kMaxT][kMaxK];
    const float* cores[kMaxT][kMaxK];
    // specialised path: the last core re-laid out as [n_k][r_{k-1}][d_k], so that one
    // row's last slice is a contiguous block (built by k3_transpose_last each forward)
    const float* last_t[kMaxT];
    // tensor-core prefix step: G_1 as [n_1][d_1][terms][r_1] and G_2 as [n_2][terms] operand
    // tiles (n = (a_2, rho_2) rows x K = rho_1, 8 x 8 core matrices) in bf16, built by k3_to_bf16
    const uint16_t* bf1[kMaxT];
    const uint16_t* bf2[kMaxT];
    // failure injection (tt_emb_debug_inject; zero in normal calls): inj_pool = 1 makes every
    // pooling wait want one finished chunk more than its table has; inj_mma = 1 makes the
    // first tensor-core completion wait report a timeout after the products completed;
    // inj_spin > 0 replaces the pooling wait's iteration limit
    int32_t inj_pool, inj_mma, inj_spin, inj_pad;
    // balance probe (tt_emb_set_probe; null in normal calls): each block of a fused kernel
    // writes one record of kProbeWords words at probe[(probe_slot * probe_cap + block) * 4]
    unsigned long long* probe;
    int32_t probe_slot, probe_cap;
};

// Balance probe record of one block of a fused kernel: SM id | C tiles read from a checkpoint
// slot << 16 | tasks << 32, start and end (global timer, ns), nanoseconds spent waiting (pooling
// waits for unfinished tables).
constexpr int kProbeWords = 4;
__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ unsigned sm_id()
{
    unsigned id;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(id));
    return id;
}
__device__ __forceinline__ void probe_write(const CoreParams& cp, unsigned long long t0, int tasks,
                                            unsigned long long wait_ns, int ckpt_loads = 0)
{
    if (cp.probe == nullptr || (int)blockIdx.x >= cp.probe_cap || threadIdx.x != 0) return;
    unsigned long long* r = cp.probe + ((size_t)cp.probe_slot * cp.probe_cap + blockIdx.x) * kProbeWords;
    r[0] = (unsigned long long)(sm_id() & 0xffffu) | ((unsigned long long)(min(ckpt_loads, 0xffff)) << 16) |
           ((unsigned long long)(unsigned)tasks << 32);
    r[1] = t0;
    r[2] = global_ns();
    r[3] = wait_ns;
}

struct GradPtrs {
    // gradient buffers in the core layouts; the three-core specialised backward takes the last
    // core's gradient in the transposed layout [n3][R][D3] instead
    float* g[kMaxT][kMaxK];
    // fused SGD (tt_emb_backward_sgd): the middle core is updated in place by the block that
    // reduces its column group, G_2[:, i_2] -= lr * dB, instead of writing dG_2
    float* upd1[kMaxT];
    float lr;
    int32_t fused;
};

// Up to T*k float buffers handled by one elementwise launch (zero fill, SGD).
struct BufferList {
    int32_t count;
    int32_t pad;
    int64_t chunk_start[kMaxT * kMaxK + 1];  // prefix sums of per-buffer chunk counts
    int64_t size[kMaxT * kMaxK];             // floats per buffer
    float* a[kMaxT * kMaxK];                 // updated buffers (16-byte aligned)
    const float* b[kMaxT * kMaxK];           // second operand (gradients), may be null
};
constexpr int kElemChunk = 8192;             // floats per block of an elementwise launch

struct SortBuffers {
    void* keys[2];        // ping-pong key arrays (uint32 or uint64)
    int32_t* vals[2];     // ping-pong positions
    uint32_t* hist;       // [256 * tiles]
    uint32_t* digit_total;// [256]
};

// Parameters of the column-group planner and of the specialised kernels.
struct PlanParams {
    int32_t T, k, ibits, col_digit;  // col_digit: prefix digit that names a column (1 = i_2)
    int64_t B;
    int32_t MP;                      // prefix groups per forward chunk
    int32_t NB;                      // bags per pooling task
    int32_t ncols;                   // sum over tables of n_{col_digit}
    int32_t sched;                   // tt_sched_mode
    int32_t grid;                    // persistent blocks of the fused forward (owner ranges)
    int32_t slot_cap;                // checkpoint slots for split chunks (TT_SCHED_STEAL_L2)
    int32_t split_rows;              // distinct rows per forward subtask at most (1 .. kSplitRows)
    uint32_t n[kMaxT][kMaxK];
    int32_t col_base[kMaxT + 1];     // first column of each table
};

// Distinct rows per forward subtask at most (the default; tt_emb_options.chunk may lower it):
// chunks with more rows are split into row ranges of at most this many (FlowTT section 3.4's
// chunks of long prefix groups, the stealing granule).  It may not exceed the row table.
constexpr int kSplitRows = 256;
constexpr int kMaxGrid = 4096;       // persistent blocks the scheduler arrays hold
constexpr int kDequeBias = 1 << 30;  // offset of both halves of a block's (head, tail) word
constexpr int kCkptFloats = 16384;   // one forward C tile (MF x N = 16384 floats for every shape)
constexpr int64_t kCkptSlots = 2048; // checkpoint slots at most (128 MB, about the size of L2)
// subtasks of a chunk of `rows` distinct rows; first subtask owned by block b of G (of S)
__host__ __device__ __forceinline__ int subtasks_of(int rows, int split)
{
    return rows > split ? (rows + split - 1) / split : 1;
}
__host__ __device__ __forceinline__ int owner_start(int S, int b, int G) { return (int)((int64_t)S * b / G); }

// Device-side plan header (workspace).  Queue cursors and per-table
// completion counters are reset by the planner on every forward.
struct PlanHeader {
    int32_t nsub, nchunks, nP, nslots;   // forward subtasks, chunks, pooling tasks per table, used slots
    int32_t pool_head, col_head, ncols_busy, pad2;   // ncols_busy: columns with work (backward queue)
    int32_t nC[kMaxT];             // forward subtasks per table (pooling of t waits for all of them)
    int32_t done[kMaxT];           // finished forward subtasks per table
};

struct PlanBuffers {
    SortBuffers sort;              // uint32 column keys / group ids, ping-pong
    int32_t* sorted_groups;        // set by launch_plan: group ids in column order
    int32_t* col_count;            // [ncols]
    int32_t* col_rows;             // [ncols] distinct rows of each column
    int32_t* col_order;            // [ncols] backward column queue: non-empty columns, costliest first
    int32_t* col_start;            // [ncols + 1]
    int32_t* chunk_base;           // [ncols + 1]
    PlanHeader* hdr;
    int4* chunks;                  // (first sorted position, groups, table, column digit)
    int4* grec;                    // [G] per sorted group position: (first distinct row, rows,
                                   //     first digit i_1, 0), so chunk metadata is one load
    // forward subtask scheduler (FlowTT section 3.4): chunks split into row ranges, each
    // block owning a contiguous range of subtasks, claims, and the C checkpoint slots
    int32_t* crow;                 // [chunks] distinct rows of each chunk
    int32_t* sub_base;             // [chunks + 1] first subtask of each chunk
    int32_t* slot_of;              // [chunks] checkpoint slot of a split chunk, or -1
    int4* subs;                    // [subtasks] (chunk, first row, end row, slot)
    unsigned long long* deque;     // [kMaxGrid] (head + bias) << 32 | (tail + bias) of each owner range
    int32_t* exhausted;            // [kMaxGrid] hint: the block's range is fully claimed
    int32_t* slot_flag;            // [slot_cap] 0 empty, 1 being written, 2 ready
    float* ckpt;                   // [slot_cap][16384] the forward C tile of a split chunk
};

// ---------------------------------------------------------------------------
// Block-wide exclusive scan for 256-thread blocks (8 warps).  All threads
// must call it; `total` receives the block sum.  s_tmp: 8 elements of smem.
// ---------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ T block256_exclusive_scan(T v, T* total, T* s_tmp)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    T x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        T y = __shfl_up_sync(kFull, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_tmp[wid] = x;
    __syncthreads();
    if (wid == 0) {
        T w = lane < 8 ? s_tmp[lane] : T(0);
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) {
            T y = __shfl_up_sync(kFull, w, o);
            if (lane >= o) w += y;
        }
        if (lane < 8) s_tmp[lane] = w;
    }
    __syncthreads();
    const T before = wid ? s_tmp[wid - 1] : T(0);
    *total = s_tmp[7];
    __syncthreads();
    return before + x - v;
}

// ---------------------------------------------------------------------------
// Host-side launchers (stream-ordered, no host synchronisation).
// ---------------------------------------------------------------------------

constexpr int kSortItems = 12;
constexpr int kSortTile = 256 * kSortItems;
constexpr int kScanTile = 256 * 16;

__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

cudaError_t launch_make_keys(const KeyParams& kp, bool key64, const int64_t* indices,
                             const int64_t* offsets, void* keys, int32_t* vals,
                             int32_t* bag_of_pos, int32_t* status, cudaStream_t s, int* nl);

// Sorts (keys, vals) by the low `bits` bits of the key; returns in *which the
// buffer index (0 or 1) that holds the result.
// `dev_n` (may be null): a device count that caps n, for counts known only on the device.
cudaError_t radix_sort_pairs(bool key64, int64_t n, int bits, SortBuffers& sb, int* which,
                             int32_t* status, cudaStream_t s, int* nl,
                             const int64_t* dev_n = nullptr);

cudaError_t launch_segment(const KeyParams& kp, bool key64, const void* sorted_keys,
                           const int32_t* perm, const int32_t* bag_of_pos, void* uniq_keys,
                           int32_t* uniq_start, int32_t* grp_start, int32_t* bag_sorted,
                           uint64_t* partials, WsCounters* counters, int32_t* uid_at_pos,
                           int32_t* uid_sorted, int32_t* status, cudaStream_t s, int* nl);

cudaError_t launch_forward_generic(const CoreParams& cp, bool key64, const void* uniq_keys,
                                   const int32_t* uniq_start, const int32_t* grp_start,
                                   const int32_t* bag_sorted, const WsCounters* counters,
                                   int64_t max_groups, float* out, int32_t* status,
                                   cudaStream_t s, int grid, int* nl);

cudaError_t launch_backward_generic(const CoreParams& cp, const GradPtrs& gp, bool key64,
                                    const void* uniq_keys, const int32_t* uniq_start,
                                    const int32_t* grp_start, const int32_t* bag_sorted,
                                    const WsCounters* counters, int64_t max_groups,
                                    const float* grad_out, int32_t* status, cudaStream_t s,
                                    int grid, int* nl);

cudaError_t launch_plan(const PlanParams& pp, bool key64, const void* uniq_keys,
                        const int32_t* grp_start, const WsCounters* counters, int64_t max_groups,
                        PlanBuffers& pb, int32_t* status, cudaStream_t s, int* nl);

// Shape-specialised three-core kernels (fused_k3.cu).
struct K3Args {
    const CoreParams* cp;
    const PlanParams* pp;
    bool key64;
    const void* uniq_keys;
    const int32_t* uniq_start;
    const int32_t* grp_start;
    const int32_t* bag_sorted;
    const int32_t* uid_at_pos;
    const int32_t* uid_sorted;
    const WsCounters* counters;
    const PlanBuffers* pb;
    const int4* grec;              // plan's per-group records in sorted (column) order
    const int64_t* offsets;
    float* rowbuf;                 // [U][D]: pooled-row checkpoint (forward), upstream sums (backward)
    int64_t L;
    int grid;
    int tc;                        // prefix-level products on the tensor cores: 0 = no (FP32 pipes),
                                   // 1 = bf16 operands, 3 = two bf16 terms per operand (three products)
    int32_t* status;
};
// Four-core tables run the three-core kernels on the merged first core
// G_12 = G_1 . G_2 (merge.cu).
struct MergeParams {
    int32_t T, d1, d2, r1, r2, pad;
    int32_t blk_base[kMaxT + 1];   // first block of each table (prefix sums of n_2)
    uint32_t n1[kMaxT], n2[kMaxT];
    const float* g1[kMaxT];
    const float* g2[kMaxT];
    float* g12[kMaxT];
    const float* dg12[kMaxT];
    float* dg1[kMaxT];
    float* dg2[kMaxT];
};
bool merge_fits(const MergeParams& mp);
cudaError_t launch_merge(const MergeParams& mp, int32_t* status, cudaStream_t s, int* nl);
cudaError_t launch_unmerge(const MergeParams& mp, int32_t* status, cudaStream_t s, int* nl);

constexpr int kPoolBags = 64;     // bags per pooling task of the specialised forward
bool k3_supported(const CoreParams& cp);
int k3_plan_mp(const CoreParams& cp);
int k3_blocks_per_sm(const CoreParams& cp, bool backward, bool tc = false);
// shapes with a tensor-core (bf16) variant of the forward prefix GEMM
bool k3_tc_supported(const CoreParams& cp);
// shapes whose backward also runs its prefix-level products on the tensor cores (rank 64)
bool k3_tc_bwd_supported(const CoreParams& cp);
// bf16 operand copies of G_1 and G_2 for the tensor-core forward (cp.cores -> dst1/dst2)
// terms = 2 stores every value as hi = bf16(x) and lo = bf16(x - hi)
cudaError_t k3_to_bf16(const CoreParams& cp, int terms, uint16_t* const* dst1, uint16_t* const* dst2,
                      cudaStream_t s, int* nl);
cudaError_t k3_forward(const K3Args& a, float* out, cudaStream_t s, int* nl);
// last core [r][n_k][d_k] -> [n_k][r][d_k] into cp.last_t (before k3_forward / k3_backward)
cudaError_t k3_transpose_last(const CoreParams& cp, float* const* dst, cudaStream_t s, int* nl);
// [n3][R][D3] per table -> dst in the core layout [R][n3][D3] (gradients of the last cores)
cudaError_t k3_transpose_last_back(const CoreParams& cp, const float* const* src, float* const* dst, cudaStream_t s,
                                   int* nl);
// upstream sums per distinct row (must run before k3_backward)
cudaError_t k3_rowsum(const K3Args& a, const float* grad_out, cudaStream_t s, int* nl);
cudaError_t k3_backward(const K3Args& a, const GradPtrs& gp, const float* grad_out, cudaStream_t s,
                        int* nl);

cudaError_t launch_fill_zero(const BufferList& bl, int32_t* status, cudaStream_t s, int* nl);
cudaError_t launch_sgd(const BufferList& bl, float lr, int32_t* status, cudaStream_t s, int* nl);

// Shared-memory floats the generic fused kernels need for these shapes.
int64_t generic_forward_smem_floats(const CoreParams& cp);
int64_t generic_backward_smem_floats(const CoreParams& cp);

}  // namespace tt
