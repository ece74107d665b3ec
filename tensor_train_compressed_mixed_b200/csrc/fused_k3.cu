// Shape-specialised fused TT gather for three cores with d_2 = 4 and equal
// inner ranks R in {16, 32, 64} (the benchmark shapes d = (4,4,4) / (4,4,8)).
//
// FlowTT section 3.2 ("Flow-Aware Fused TT Embedding Execution") and 3.4:
//   * A work unit is a chunk of prefix groups that share their middle digit
//     i_2 (a column group).  The middle slice B = G_2[:, i_2] (R x 4R floats)
//     is staged in shared memory once and reused by every prefix of the
//     chunk; the chunk's prefix intermediates C_p = A_p . B (A_p = G_1[0, i_1])
//     form one register-tiled FP32 GEMM whose result stays on chip.
//   * Each distinct row of the chunk applies its last slice, E = C_p . D,
//     from shared memory, and E goes to an L2-resident row checkpoint.
//   * Pooling runs in the same persistent kernel: pooling tasks of table t
//     wait (bounded) until every chunk of t has finished, then gather each
//     bag's rows in bag order and write the pooled row once.  Tables are
//     interleaved so a table's rows are pooled while the next table computes
//     and the rows are still in L2 (the inter-block reuse FlowTT obtains with
//     L2 checkpointing).
//   * The backward pass takes whole column groups: per distinct row the
//     upstream sum H (precomputed by a balanced segmented pass) gives the
//     last-slice gradient C_p^T H and dC_p += H D^T; per prefix dA = dC B^T
//     and dB += A^T dC.  dB is reduced on chip over the whole column group and
//     written once; dA and the last-slice gradients are reduced into the
//     small, L2-resident gradient arrays with 16-byte vector reductions.
//   * With the tensor-core precisions (d = (4,4,8), R in {32, 64}) the
//     prefix-level products run as tcgen05 MMAs with fp32 accumulators in
//     tensor memory: C = A . B in the forward; in the backward (R = 64) the
//     transposed C^T = B^T A^T, which each warp reads straight from tensor
//     memory, then dA = dC . B^T and dB += A^T . dC.
#include <cuda_bf16.h>
#include <string.h>

#include "tt_common.cuh"

#define TT_K3_CASES_INNER(X) \
    X(4, 4, 8, 64)           \
    X(4, 4, 8, 32)           \
    X(4, 4, 8, 16)           \
    X(4, 4, 4, 32)           \
    X(4, 4, 4, 16)           \
    X(8, 4, 4, 32)

// Optional phase timing (build with -DTT_PROFILE_PHASES): thread 0 of every
// block adds the clock64 cycles it spent in each phase to a device array that
// tt_emb_debug_phase_cycles() reads and clears.  Off in normal builds.
#ifdef TT_PROFILE_PHASES
__device__ unsigned long long g_tt_phase_cycles[32];
#define TT_PH_START() long long tt_ph_t0 = clock64()
#define TT_PH(i)                                                             \
    do {                                                                     \
        if (threadIdx.x == 0) {                                              \
            const long long tt_ph_t = clock64();                             \
            atomicAdd(&g_tt_phase_cycles[i], (unsigned long long)(tt_ph_t - tt_ph_t0)); \
            tt_ph_t0 = tt_ph_t;                                              \
        }                                                                    \
    } while (0)
#else
#define TT_PH_START() \
    do {              \
    } while (0)
#define TT_PH(i) \
    do {         \
    } while (0)
#endif

namespace tt {
namespace {

constexpr int kFwdThreads = 512;  // forward: 16 warps, at most 128 registers per thread
constexpr int kBwdThreads = 256;  // backward, FP32 variant: 8 warps, up to 255 registers per thread
constexpr int kBwdThreadsTC = 512; // backward, tensor-core kernel: 16 warps (4 per sub-partition), at most 128 registers
constexpr int kNB = kPoolBags;    // bags per pooling task
constexpr int kHChunk = 256;      // sorted lookups per upstream-sum warp
constexpr int kSpinLimit = 1 << 22;
constexpr int kKeyCap = 256;      // distinct rows per chunk whose keys are staged with the chunk
constexpr int kKeyCapB = 512;     // the same for a chunk of the tensor-core backward (not split into
                                  // subtasks, so longer; rows past the cap read their keys directly)

template <int D1_, int D2_, int D3_, int R_>
struct S3 {
    static constexpr int D1 = D1_, D2 = D2_, D3 = D3_, R = R_;
    static constexpr int N = D2 * R;          // columns of B and of C_all
    static constexpr int P = D1 * D2;         // rows of C_p
    static constexpr int D = P * D3;          // embedding width
    // forward: GEMM of MF x N per chunk, 4 x 8 outputs per thread
    static constexpr int MF = 16384 / N;
    static constexpr int MPF = MF / D1;       // prefixes per forward chunk
    static constexpr int TPU = D1 * 2 * (D3 / 4); // threads per distinct row in the suffix step
    static constexpr int NUF = kFwdThreads / TPU;
    static constexpr int SU = R * D3 + 8;     // padded stride of one staged last slice
    static constexpr size_t FWD_FIXED = (size_t)R * N + (size_t)MF * R + (size_t)MF * N;
    static constexpr int FBUF = (FWD_FIXED + 2 * (size_t)NUF * SU) * 4 <= 220 * 1024 ? 2 : 1;
    // backward: MB x N per chunk
    static constexpr int MB = 2048 / R;
    static constexpr int MPB = MB / D1;
    static constexpr int TPUB = (R / 4) * (D3 / 4);   // dS tiles per distinct row
    static constexpr int NUB = kBwdThreads / TPUB;      // distinct rows per backward batch
    static constexpr int SR = D3 + 4;                // padded row of a staged last slice (backward)
    static constexpr int DBR = (R * N) / (kBwdThreads * 4) >= 16 ? 8 : ((R * N) / (kBwdThreads * 4) >= 4 ? 4 : 1);
    static constexpr int DBC = (R * N) / (kBwdThreads * DBR);   // dB columns per thread
    static_assert(D2 == 4, "specialised path needs d_2 = 4");
    static_assert(D1 == 4 || D1 == 8, "specialised path needs d_1 in {4, 8}");
    static_assert(MF % D1 == 0 && MB % D1 == 0, "chunk rows in whole prefixes");
    static_assert(D3 % 4 == 0, "d_3 must be a multiple of 4");
    static_assert(D <= 128, "one warp (4 columns per lane) covers a pooled row");
    static_assert(N >= 32 && N % 32 == 0, "swizzle needs N >= 32");
    static_assert(MF % 4 == 0 && (MF / 4) * (N / 8) == kFwdThreads, "forward GEMM tiling (4 x 8 per thread)");
    static_assert((2048 / R / 4) * (N / 8) == kBwdThreads, "backward GEMM tiling (4 x 8 per thread)");
    static_assert((MF / 4) % 4 == 0 && (MB / 4) % 4 == 0 && (N / 8) % 8 == 0, "warps of 4 x 8 thread tiles");
    static_assert(DBC % 4 == 0, "dB columns in float4 chunks");
    static_assert(NUB >= 1 && NUB * TPUB == kBwdThreads, "backward batch tiling");

    static constexpr size_t fwd_smem_floats() { return FWD_FIXED + (size_t)FBUF * NUF * SU; }
    // tensor-core variants: A and B as NS bf16 terms
    static constexpr size_t fwd_smem_floats_tc(int NS)
    {
        return (size_t)NS * ((size_t)R * N + (size_t)MF * R) / 2 + (size_t)MF * N + (size_t)FBUF * NUF * SU;
    }
    static constexpr size_t bwd_smem_floats()
    {
        return (size_t)R * N + 2 * (size_t)MB * R + 2 * (size_t)MB * N + 2 * (size_t)NUB * P * D3 +
               2 * (size_t)NUB * R * SR;
    }
};

// float4 chunks of row `row` are permuted by a row-dependent XOR so that rows
// read in the same column by different lanes land in different banks.
template <int W>
__device__ __forceinline__ int swz_b(int row, int col)  // key: (row / 4) mod 8
{
    return row * W + ((((col >> 2) ^ ((row >> 2) & 7))) << 2) + (col & 3);
}
template <int W>
__device__ __forceinline__ int swz_m(int row, int col)  // key: row mod 8
{
    return row * W + ((((col >> 2) ^ (row & 7))) << 2) + (col & 3);
}
template <int W>
__device__ __forceinline__ int swz_a(int row, int col)  // key: (row / 4) mod (W / 4)
{
    return row * W + ((((col >> 2) ^ ((row >> 2) & (W / 4 - 1)))) << 2) + (col & 3);
}

__device__ __forceinline__ void red_add_v4(float* p, float4 v)
{
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v.x), "f"(v.y),
                 "f"(v.z), "f"(v.w)
                 : "memory");
}

__device__ __forceinline__ float4 f4add(float4 a, float4 b)
{
    return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

__device__ __forceinline__ float f4get(const float4& v, int i)
{
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// Thread tile coordinates of a register-tiled GEMM with TN tiles across N: each warp
// covers 4 tile rows x 8 tile columns, so one fragment load of A touches 4 rows and one
// of B 8 consecutive 16-byte chunks (one shared-memory wavefront each) instead of 32.
template <int TN>
__device__ __forceinline__ void warp_tile_2d(int tid, int& tm, int& tn)
{
    static_assert(TN % 8 == 0, "tile columns in groups of 8");
    const int warp = tid >> 5, lane = tid & 31;
    tm = (warp / (TN / 8)) * 4 + (lane >> 3);
    tn = (warp % (TN / 8)) * 8 + (lane & 7);
}

// 16-byte asynchronous global -> shared copies (L2 only), grouped and awaited
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem)
{
    const unsigned a = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(a), "l"(gmem) : "memory");
}
template <typename K>
__device__ __forceinline__ void cp_async_key(K* smem, const K* gmem)   // 4- or 8-byte copy (L1 path)
{
    const unsigned a = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(a), "l"(gmem), "n"(sizeof(K)) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <typename K>
__device__ __forceinline__ uint32_t key_row(K key, int ibits)
{
    return (uint32_t)((uint64_t)key & ((uint64_t(1) << ibits) - 1));
}

// Persistent task fetch: dynamic (atomic queue head) or static round robin.
__device__ __forceinline__ int next_task(int sched, int* head, int iter)
{
    return sched == TT_SCHED_STATIC ? (int)blockIdx.x + iter * (int)gridDim.x : atomicAdd(head, 1);
}

// ---------------------------------------------------------------------------
// fifth-generation tensor cores: tensor memory, mbarrier, tcgen05.mma (bf16 x bf16 -> f32)
// ---------------------------------------------------------------------------
constexpr int kMbarSpin = 1 << 20;   // bounded wait for an MMA completion (tens of ms at most)

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Shared-memory matrix descriptor for a K-major operand without swizzle.  The operand is
// stored as 8-row x 16-byte core matrices (8 rows of 8 bf16 along K, 128 contiguous bytes);
// lbo = bytes between the two K-adjacent core matrices one MMA (K = 16) reads, sbo = bytes
// between consecutive 8-row groups.  Bits: start >> 4 [0,14), lbo >> 4 [16,30),
// sbo >> 4 [32,46), descriptor version 1 [46,48), base offset 0, layout 0 (no swizzle).
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
}

// Instruction descriptor of kind::f16: f32 accumulator [4,6) = 1, A = bf16 [7,10) = 1,
// B = bf16 [10,13) = 1, A / B major at bits 15 / 16 (0 = K-major, 1 = MN-major),
// N >> 3 at [17,23), M >> 4 at [24,29).
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N, bool a_mn = false, bool b_mn = false)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// Descriptor of an MN-major operand without swizzle over the same 8 x 16-byte core matrices:
// each core matrix holds 8 K-rows of 8 contiguous MN-elements; sbo = bytes between
// MN-adjacent core matrices, lbo = bytes between K-adjacent ones.
__device__ __forceinline__ uint64_t umma_desc_mn(uint32_t saddr, uint32_t sbo, uint32_t lbo)
{
    return umma_desc(saddr, lbo, sbo);
}

__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols)   // one warp
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)   // the same warp
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// makes this thread's generic-proxy shared-memory writes visible to the tensor cores
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tc_mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0)
        : "memory");
}
// arrives once on the mbarrier when every MMA this thread issued so far has completed
__device__ __forceinline__ void tc_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// bounded wait for the completion of phase `parity`; false when the bound ran out
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity)
{
    const uint32_t a = smem_u32(bar);
    for (int it = 0; it < kMbarSpin; ++it) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.b32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(a), "r"(parity)
            : "memory");
        if (done) return true;
        if (it >= 8) __nanosleep(64);
    }
    return false;
}
// eight fp32 values as two bf16 terms: hi = bf16(x), lo = bf16(x - hi); |x - hi - lo| <= 2^-18 |x|
__device__ __forceinline__ void split_bf16x8(const float (&v)[8], uint4& hi, uint4& lo)
{
    uint32_t h[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        // two values per conversion; a bf16 widens to fp32 exactly by a 16-bit shift
        const __nv_bfloat162 hh = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        const uint32_t hb = *reinterpret_cast<const uint32_t*>(&hh);
        const float r0 = v[2 * i] - __uint_as_float(hb << 16);
        const float r1 = v[2 * i + 1] - __uint_as_float(hb & 0xffff0000u);
        const __nv_bfloat162 ll = __floats2bfloat162_rn(r0, r1);
        h[i] = hb;
        l[i] = *reinterpret_cast<const uint32_t*>(&ll);
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// 32 lanes x 32 consecutive 32-bit columns of tensor memory: lane i of the warp gets row
// (taddr lane + i), columns taddr column .. +31
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32])
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// ---------------------------------------------------------------------------
// forward
// ---------------------------------------------------------------------------
template <class S>
struct FwdSmem {
    float* Bs;   // [R][N]        B = G_2[:, i_2], swizzled
    float* As;   // [MF][R]       A_j = G_1[0, i1_j] rows, swizzled
    uint16_t* Bb;   // tensor-core variant: B as N x R bf16 core matrices (K-major)
    uint16_t* Ab;   // tensor-core variant: A as MF x R bf16 core matrices (K-major)
    float* Cn;   // [MF][N]       C_all, swizzled
    float* Ss;   // [FBUF][NUF][SU] last slices of a batch of distinct rows
};

// Per chunk buffer, for the chunk's first CAP distinct rows: row id, prefix slot, last digit.
template <int CAP>
struct RowTableT {
    int u[2][CAP], p[2][CAP], i3[2][CAP];
};
using RowTable = RowTableT<kKeyCap>;

template <class S>
struct FwdMeta {   // shared-memory metadata of a subtask (double buffered)
    int u0[2][S::MPF];
    int ucum[2][S::MPF + 1];
    int i1[2][S::MPF];
    int cnt[2], t[2], i2[2];
    int cid[2], rb[2], re[2], slot[2];   // chunk, its distinct rows [rb, re), checkpoint slot
    int task[2];
    int flag;
    int ck;                              // checkpoint decision of the current subtask
    RowTable rows;
};

// Index of the prefix (0..cnt-1) holding the chunk's distinct row number kq. Every prefix has at
// least one row, so the first rows ucum[0..cnt) strictly increase and the index is the number of
// prefixes after the first that start at or before kq: counted with independent loads (ucum has
// N1 = slots + 1 entries).
template <int N1>
__device__ __forceinline__ int prefix_of(const int (&ucum)[N1], int cnt, int kq)
{
    int j = 0;
#pragma unroll
    for (int i = 1; i < N1 - 1; ++i) j += (i < cnt && ucum[i] <= kq) ? 1 : 0;
    return j;
}

// The row table of distinct rows base .. base + kKeyCap of a chunk (at most `total`): the row
// id, the prefix slot and the last digit, computed once by all threads from the staged keys
// (which must have landed and be visible).  Batches inside the table then need no per-batch
// metadata pass.
template <typename K, int N1, int CAP>
__device__ __forceinline__ void build_rows(RowTableT<CAP>& rt, int mb, const int (&ucum)[N1], const int* u0, int cnt, int total,
                                           const K* keys, int ibits, uint32_t n3, int nthreads, int base = 0)
{
    const int n = min(total - base, CAP);
    for (int i = threadIdx.x; i < n; i += nthreads) {
        const int kq = base + i;
        const int j = prefix_of(ucum, cnt, kq);
        rt.u[mb][i] = u0[j] + (kq - ucum[j]);
        rt.p[mb][i] = j;
        rt.i3[mb][i] = (int)(key_row(keys[mb * CAP + i], ibits) % n3);
    }
}
// Rows k0 .. k0 + nb of chunk buffer mb: the row table when it covers them, else the batch's own
// metadata (filled by the batch issue)
struct RowRef {
    const int* u;
    const int* p;
    const int* i3;
};
__device__ __forceinline__ RowRef batch_rows(const RowTable& rt, int mb, int k0, int nb, const int* bu,
                                             const int* bp, const int* bi3)
{
    if (k0 + nb <= kKeyCap) return RowRef{rt.u[mb] + k0, rt.p[mb] + k0, rt.i3[mb] + k0};
    return RowRef{bu, bp, bi3};
}

// Metadata of subtask `sub` = (chunk, first row, end row, slot) into buffer mb (all threads
// call; ends with a barrier), and asynchronous copies of the keys of its distinct rows (at most
// kKeyCap) into keys[mb]; those join the caller's next commit group (the chunk's A/B copies).
template <class S, typename K>
__device__ __forceinline__ void fwd_meta(const CoreParams& cp, int4 sub, int mb, const K* __restrict__ uniq_keys,
                                         const int4* __restrict__ grec, const int4* __restrict__ chunks,
                                         FwdMeta<S>& M, K* keys)
{
    const int tid = threadIdx.x;
    const int4 ch = chunks[sub.x];
    if (tid < S::MPF) {
        const int4 g = tid < ch.y ? grec[ch.x + tid] : make_int4(0, 0, 0, 0);
        M.u0[mb][tid] = g.x;
        M.ucum[mb][tid] = g.y;
        M.i1[mb][tid] = g.z;
    }
    if (tid == 0) {
        M.cnt[mb] = ch.y;
        M.t[mb] = ch.z;
        M.i2[mb] = ch.w;
        M.cid[mb] = sub.x;
        M.rb[mb] = sub.y;
        M.re[mb] = sub.z;
        M.slot[mb] = sub.w;
    }
    __syncthreads();
    if (tid == 0) {
        int run = 0;
        for (int j = 0; j < S::MPF; ++j) {
            const int v = M.ucum[mb][j];
            M.ucum[mb][j] = run;
            run += v;
        }
        M.ucum[mb][S::MPF] = run;
    }
    __syncthreads();
    const int nk = min(sub.z - sub.y, kKeyCap);
    for (int i = tid; i < nk; i += kFwdThreads) {
        const int kq = sub.y + i;
        const int j = prefix_of(M.ucum[mb], M.cnt[mb], kq);
        cp_async_key(keys + mb * kKeyCap + i, uniq_keys + M.u0[mb][j] + (kq - M.ucum[mb][j]));
    }
}

// asynchronous copies of the chunk's A rows (and B when its column changes); one commit group
template <class S>
__device__ __forceinline__ void fwd_issue_ab(const CoreParams& cp, int mb, const FwdMeta<S>& M,
                                             const FwdSmem<S>& sm, int& cur_t, int& cur_i2)
{
    constexpr int R = S::R, N = S::N, MF = S::MF, D1 = S::D1;
    const int tid = threadIdx.x;
    const int t = M.t[mb], i2 = M.i2[mb], cnt = M.cnt[mb];
    if (t != cur_t || i2 != cur_i2) {
        const float* G2 = cp.cores[t][1] + (int64_t)i2 * N;
        const int64_t rs = (int64_t)cp.n[t][1] * N;
        for (int q = tid; q < R * N / 4; q += kFwdThreads) {
            const int rho = q / (N / 4), c4 = q % (N / 4);
            cp_async16(&sm.Bs[swz_b<N>(rho, c4 * 4)], G2 + rho * rs + c4 * 4);
        }
        cur_t = t;
        cur_i2 = i2;
    }
    const float* G1 = cp.cores[t][0];
    for (int q = tid; q < MF * (R / 4); q += kFwdThreads) {
        const int m = q / (R / 4), c4 = q % (R / 4);
        const int j = m / D1, a1 = m % D1;
        float* dst = &sm.As[swz_a<R>(m, c4 * 4)];
        if (j < cnt) cp_async16(dst, G1 + ((int64_t)M.i1[mb][j] * D1 + a1) * R + c4 * 4);
        else *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    cp_async_commit();
}

// C_all = A . B into Cn; thread tile rows {4tm+i} x cols {4tn+j, N/2+4tn+j}
template <class S>
__device__ __forceinline__ void fwd_gemm(const FwdSmem<S>& sm)
{
    constexpr int R = S::R, N = S::N;
    constexpr int TN = N / 8;
    int tm, tn;
    warp_tile_2d<TN>(threadIdx.x, tm, tn);
    int rows[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) rows[i] = tm * 4 + i;
    float acc[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
#pragma unroll 1
    for (int rho = 0; rho < R; rho += 4) {
        float4 a[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = *reinterpret_cast<const float4*>(&sm.As[swz_a<R>(rows[i], rho)]);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const float4 b0 = *reinterpret_cast<const float4*>(&sm.Bs[swz_b<N>(rho + r, tn * 4)]);
            const float4 b1 = *reinterpret_cast<const float4*>(&sm.Bs[swz_b<N>(rho + r, N / 2 + tn * 4)]);
            const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float av = f4get(a[i], r);
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av, b[j], acc[i][j]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        *reinterpret_cast<float4*>(&sm.Cn[swz_m<N>(rows[i], tn * 4)]) =
            make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
        *reinterpret_cast<float4*>(&sm.Cn[swz_m<N>(rows[i], N / 2 + tn * 4)]) =
            make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
    }
}

// Tensor-core variant of fwd_issue_ab: the bf16 B tile (already in operand order, one flat
// copy) and the chunk's A rows placed into 8 x 16-byte core matrices; one commit group.
// NS = 2 stores each operand as two bf16 terms (hi tile, then lo tile).
template <class S, int NS>
__device__ __forceinline__ void fwd_issue_ab_tc(const CoreParams& cp, int mb, const FwdMeta<S>& M,
                                                const FwdSmem<S>& sm, int& cur_t, int& cur_i2)
{
    constexpr int R = S::R, N = S::N, MF = S::MF, D1 = S::D1;
    constexpr int KC = R / 8;   // 16-byte K chunks per operand row
    const int tid = threadIdx.x;
    const int t = M.t[mb], i2 = M.i2[mb], cnt = M.cnt[mb];
    if (t != cur_t || i2 != cur_i2) {
        const uint16_t* src = cp.bf2[t] + (int64_t)i2 * (NS * R * N);
        for (int q = tid; q < NS * R * N / 8; q += kFwdThreads) cp_async16(sm.Bb + q * 8, src + q * 8);
        cur_t = t;
        cur_i2 = i2;
    }
    const uint16_t* G1 = cp.bf1[t];
    for (int q = tid; q < NS * MF * KC; q += kFwdThreads) {
        // 8 consecutive threads fill one 128-byte core matrix (rows m % 8), so shared-memory
        // writes of a warp are contiguous
        const int term = q / (MF * KC), r = q % (MF * KC);
        const int m = (r / (8 * KC)) * 8 + (r & 7), kc = (r >> 3) % KC;
        const int j = m / D1, a1 = m % D1;
        uint16_t* dst = sm.Ab + term * (MF * R) + ((m >> 3) * KC + kc) * 64 + (m & 7) * 8;
        if (j < cnt) cp_async16(dst, G1 + ((int64_t)M.i1[mb][j] * D1 + a1) * (NS * R) + term * R + kc * 8);
        else *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
    }
    cp_async_commit();
}

// The MMAs of one K = 16 step of a product whose operands are stored as NT = 1 term
// (bf16) or as two terms hi + lo (NT = 3 products: hi.hi + hi.lo + lo.hi).  a_lo / b_lo
// are the byte distances from the hi tiles to the lo tiles.
template <int NT>
__device__ __forceinline__ void tc_mma_terms(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t a_lo,
                                             uint32_t b_lo, uint32_t idesc, bool accumulate)
{
    tc_mma_bf16(tmem_d, adesc, bdesc, idesc, accumulate ? 1u : 0u);
    if constexpr (NT == 3) {
        tc_mma_bf16(tmem_d, adesc, bdesc + (b_lo >> 4), idesc, 1u);
        tc_mma_bf16(tmem_d, adesc + (a_lo >> 4), bdesc, idesc, 1u);
    }
}

// C_all = A . B on the tensor cores: one thread issues R / 16 MMAs (M = MF, N, K = 16)
// into tensor memory and commits them to the mbarrier; after the bounded wait every warp
// moves its share of the fp32 accumulator (sub-partition warp % 4, a quarter of the
// columns) into Cn.  The caller has waited for the A/B copies; returns false (all
// threads) when the completion wait ran out.
template <class S, int NT>
__device__ __forceinline__ bool fwd_gemm_tc(const FwdSmem<S>& sm, uint32_t tmem, uint64_t* bar, uint32_t& parity,
                                            int* s_ok, bool inject_fail)
{
    constexpr int R = S::R, N = S::N, MF = S::MF;
    static_assert(MF == 64 || MF == 128, "tensor-core M is 64 or 128");
    static_assert(kFwdThreads == 512, "16 warps: 4 sub-partitions x 4 column blocks");
    const int tid = threadIdx.x;
    if (tid == 0) {
        tc_fence_after();
        constexpr uint32_t SBO = (R / 8) * 128;
        constexpr uint32_t idesc = umma_idesc_bf16(MF, N);
        const uint32_t a0 = smem_u32(sm.Ab), b0 = smem_u32(sm.Bb);
#pragma unroll
        for (int k = 0; k < R / 16; ++k)
            tc_mma_terms<NT>(tmem, umma_desc(a0 + k * 256, 128, SBO), umma_desc(b0 + k * 256, 128, SBO),
                             MF * R * 2, R * N * 2, idesc, k > 0);
        tc_commit(bar);
        // an injected failure (test hook) is reported only after the products completed
        *s_ok = (mbar_wait(bar, parity) && !inject_fail) ? 1 : 0;
    }
    __syncthreads();
    parity ^= 1u;
    if (!*s_ok) return false;
    tc_fence_after();
    const int warp = tid >> 5, lane = tid & 31;
    const int sub = warp & 3, cb = warp >> 2;
    constexpr int CPB = N / 4;   // accumulator columns per warp
    // M = 128: row m in lane m; M = 64: rows 16 s .. 16 s + 15 in lanes 32 s .. 32 s + 15
    const int m = MF == 128 ? 32 * sub + lane : 16 * sub + lane;
    const bool valid = MF == 128 || lane < 16;
#pragma unroll 1
    for (int g = 0; g < CPB / 32; ++g) {
        const int c0 = cb * CPB + g * 32;
        float v[32];
        tmem_ld32(tmem + ((uint32_t)(32 * sub) << 16) + (uint32_t)c0, v);
        if (valid) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<float4*>(&sm.Cn[swz_m<N>(m, c0 + 4 * j)]) =
                    make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        }
    }
    tc_fence_before();
    return true;
}

// Distinct rows i0 .. i0 + NUF of the subtask in buffer mb (indices local to the subtask, inside
// its row table) into batch buffer bb: issues their last slices (one commit group).
template <class S>
__device__ __forceinline__ void fwd_issue_batch(const CoreParams& cp, int mb, int i0, int bb, const FwdMeta<S>& M,
                                                const FwdSmem<S>& sm)
{
    constexpr int R = S::R, D3 = S::D3;
    const int tid = threadIdx.x;
    const int nb = min(S::NUF, M.re[mb] - M.rb[mb] - i0);
    const int* i3 = M.rows.i3[mb] + i0;
    const float* G3t = cp.last_t[M.t[mb]];   // [n3][R][D3]: one row's slice is contiguous
    float* Ss = sm.Ss + (size_t)bb * S::NUF * S::SU;
    for (int q = tid; q < nb * R * (D3 / 4); q += kFwdThreads) {
        const int uu = q / (R * (D3 / 4)), rem = q % (R * (D3 / 4));
        cp_async16(&Ss[uu * S::SU + rem * 4], G3t + (int64_t)i3[uu] * (R * D3) + rem * 4);
    }
    cp_async_commit();
}

// As fwd_issue_batch for the subtask's first batch, with each row's last digit taken from the
// staged keys instead of the row table (which is built while these copies run)
template <class S, typename K>
__device__ __forceinline__ void fwd_issue_batch_keys(const CoreParams& cp, int mb, const FwdMeta<S>& M,
                                                     const FwdSmem<S>& sm, const K* keys)
{
    constexpr int R = S::R, D3 = S::D3;
    const int tid = threadIdx.x;
    const int nb = min(S::NUF, M.re[mb] - M.rb[mb]);
    const uint32_t n3 = cp.n[M.t[mb]][2];
    const float* G3t = cp.last_t[M.t[mb]];   // [n3][R][D3]: one row's slice is contiguous
    float* Ss = sm.Ss;
    for (int q = tid; q < nb * R * (D3 / 4); q += kFwdThreads) {
        const int uu = q / (R * (D3 / 4)), rem = q % (R * (D3 / 4));
        const uint32_t i3 = key_row(keys[mb * kKeyCap + uu], cp.ibits) % n3;
        cp_async16(&Ss[uu * S::SU + rem * 4], G3t + (int64_t)i3 * (R * D3) + rem * 4);
    }
    cp_async_commit();
}

// E_u = C_p . S_u for the batch in buffer bb; tile: rows (a1, a2 = 2h, 2h+1) x 4 columns of a3
template <class S>
__device__ __forceinline__ void fwd_batch_compute(int mb, int i0, int nb, int bb, const FwdMeta<S>& M,
                                                  const FwdSmem<S>& sm, float* __restrict__ rowbuf)
{
    constexpr int R = S::R, N = S::N, D1 = S::D1, D2 = S::D2, D3 = S::D3;
    const int tid = threadIdx.x;
    const int uu = tid / S::TPU;
    if (uu >= nb) return;
    const RowRef rr{M.rows.u[mb] + i0, M.rows.p[mb] + i0, M.rows.i3[mb] + i0};
    const int rem = tid % S::TPU;
    const int a1 = rem / (2 * (D3 / 4)), h = (rem / (D3 / 4)) % 2, cg = rem % (D3 / 4);
    const int m = rr.p[uu] * D1 + a1;
    const float* srow = sm.Ss + (size_t)bb * S::NUF * S::SU + uu * S::SU + cg * 4;
    float4 e[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) e[q] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
    for (int rho = 0; rho < R; rho += 4) {
        float4 c[2], s4[4];
#pragma unroll
        for (int q = 0; q < 2; ++q) c[q] = *reinterpret_cast<const float4*>(&sm.Cn[swz_m<N>(m, (2 * h + q) * R + rho)]);
#pragma unroll
        for (int r = 0; r < 4; ++r) s4[r] = *reinterpret_cast<const float4*>(srow + (rho + r) * D3);
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const float cv = f4get(c[q], r);
                e[q].x = fmaf(cv, s4[r].x, e[q].x);
                e[q].y = fmaf(cv, s4[r].y, e[q].y);
                e[q].z = fmaf(cv, s4[r].z, e[q].z);
                e[q].w = fmaf(cv, s4[r].w, e[q].w);
            }
    }
    float* dst = rowbuf + (int64_t)rr.u[uu] * S::D + cg * 4;
#pragma unroll
    for (int q = 0; q < 2; ++q) *reinterpret_cast<float4*>(dst + (a1 * D2 + 2 * h + q) * D3) = e[q];
}

template <class S>
__device__ void fwd_pool(const CoreParams& cp, int ptask, int nP, const int32_t* __restrict__ uid_at_pos,
                         const int64_t* __restrict__ offsets, PlanHeader* hdr,
                         const float* __restrict__ rowbuf, float* __restrict__ out, int32_t* status,
                         int* s_flag, unsigned long long* wait_ns)
{
    constexpr int D = S::D, LB = D / 4, BPW = 32 / LB;
    // row gathers in flight per lane (measured: 24 is best at rank 32, 16 at rank 64)
    constexpr int kPoolLoads = S::R == 32 ? 24 : 16;
    const int t = ptask / nP, jb = ptask % nP;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    TT_PH_START();
    if (tid == 0) {
        // injected failure (test hook): wait for one subtask more than the table has
        const unsigned long long w0 = cp.probe ? global_ns() : 0ull;
        const int want = hdr->nC[t] + (cp.inj_pool ? 1 : 0);
        const int limit = cp.inj_spin > 0 ? cp.inj_spin : kSpinLimit;
        int it = 0, ok = 1;
        while (*reinterpret_cast<volatile int*>(&hdr->done[t]) < want) {
            if (++it > limit) {
                raise_error(status, TT_ERR_TIMEOUT, t);
                ok = 0;
                break;
            }
            if ((it & 63) == 0 && has_error(status)) {   // another block failed: stop waiting
                ok = 0;
                break;
            }
            __nanosleep(256);
        }
        __threadfence();
        s_flag[0] = ok;
        if (cp.probe) *wait_ns += global_ns() - w0;
    }
    __syncthreads();
    TT_PH(4);
    if (!s_flag[0]) return;
    const int64_t B = cp.B, TD = (int64_t)cp.T * D;
    const int sub = lane / LB, sl = lane % LB, col = sl * 4;
    const unsigned smask = LB >= 32 ? kFull : (((1u << (LB & 31)) - 1u) << (sub * LB));
    const int b_lo = jb * kNB, b_hi = (int)min64((int64_t)b_lo + kNB, B);
    const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
    // one sub-warp of LB lanes per bag; every lane owns 4 columns
    for (int b = b_lo + wid * BPW + sub; b < b_hi; b += (kFwdThreads / 32) * BPW) {
        const int64_t g = (int64_t)t * B + b;
        const int64_t l0 = offsets[g], l1 = offsets[g + 1];
        float4 acc = zero;
        for (int64_t base = l0; base < l1; base += LB) {
            const int n = (int)min64(LB, l1 - base);
            const int myu = sl < n ? uid_at_pos[base + sl] : 0;   // row ids of up to LB lookups
            for (int k = 0; k < n; k += kPoolLoads) {
                float4 v[kPoolLoads];
#pragma unroll
                for (int q = 0; q < kPoolLoads; ++q) {
                    const int u = __shfl_sync(smask, myu, (k + q) & (LB - 1), LB);
                    v[q] = (k + q < n) ? __ldcg(reinterpret_cast<const float4*>(rowbuf + (int64_t)u * D + col))
                                       : zero;
                }
#pragma unroll
                for (int q = 0; q < kPoolLoads; ++q)   // lookup order: the sum is the same for every schedule
                    if (k + q < n) acc = f4add(acc, v[q]);
            }
        }
        *reinterpret_cast<float4*>(out + (int64_t)b * TD + (int64_t)t * D + col) = acc;
    }
    __syncthreads();
    TT_PH(5);
}

// ---------------------------------------------------------------------------
// Forward scheduler (FlowTT section 3.4).  Subtasks (row ranges of chunks, in column order)
// are split into one contiguous owner range per persistent block.  A block takes its own
// subtasks front to back; in the stealing modes it then takes subtasks of other blocks that
// have not started, from the back of their ranges, and finally pooling tasks from a shared
// queue.  Each block's remaining range is one 64-bit word, (head + kDequeBias) << 32 |
// (tail + kDequeBias): the owner takes `head` by adding 1 << 32, a thief takes `tail - 1` by
// adding -1, and the one atomic of each tells whether the range still held a subtask, so every
// subtask runs exactly once.  The bias keeps both halves positive: tails fall at most once per
// failed steal per block below the range start.
// One thread only (lane 0 of warp 1: thread 0 issues the tensor-core products, and a queue
// atomic on it would delay them).  Returns a subtask index, -2 - p for pooling task p, or -1
// when done.
// ---------------------------------------------------------------------------
struct FwdSched {
    const int4* subs;
    unsigned long long* deque;   // [grid] (head, tail) of each block's owner range
    int32_t* exhausted;          // [grid] hint: the range has no subtask left
    int32_t* slot_flag;
    float* ckpt;
};

__device__ __forceinline__ int fwd_next(const FwdSched& fs, PlanHeader* hdr, int sched, int npool, int& phase,
                                        int& vk)
{
    const int G = (int)gridDim.x, b = (int)blockIdx.x;
    if (phase == 0) {
        const unsigned long long old = atomicAdd(&fs.deque[b], 1ull << 32);
        const int h = (int)(old >> 32) - kDequeBias, t = (int)(old & 0xffffffffull) - kDequeBias;
        if (h < t) return h;
        phase = sched == TT_SCHED_STATIC ? 2 : 1;
        vk = 1;
    }
    if (phase == 1) {
        while (vk < G) {
            const int v = b + vk < G ? b + vk : b + vk - G;
            if (*reinterpret_cast<volatile int*>(&fs.exhausted[v]) == 0) {
                const unsigned long long old = atomicAdd(&fs.deque[v], ~0ull);   // tail - 1
                const int h = (int)(old >> 32) - kDequeBias, t = (int)(old & 0xffffffffull) - kDequeBias;
                if (t - 1 >= h) return t - 1;   // again from v next time
                *reinterpret_cast<volatile int*>(&fs.exhausted[v]) = 1;
            }
            ++vk;
        }
        phase = 2;
    }
    const int p = atomicAdd(&hdr->pool_head, 1);
    return p < npool ? -2 - p : -1;
}

// L2 checkpoint of a split chunk's C tile (TT_SCHED_STEAL_L2; FlowTT section 3.2 / 3.4: shared
// intermediates kept in L2 for reuse between blocks).  Flag protocol per slot: 0 empty, 1 being
// written (the block that won the compare-and-swap), 2 ready (release after a device fence).
constexpr int kCkptPolls = 64;   // bounded wait for a slot another block is writing; then recompute

__device__ __forceinline__ int ld_acquire(const int32_t* p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(int32_t* p, int v)
{
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint64_t l2_evict_last_policy()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ void st_v4_hint(float* p, float4 v, uint64_t pol)
{
    asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "f"(v.x), "f"(v.y),
                 "f"(v.z), "f"(v.w), "l"(pol)
                 : "memory");
}

// Thread 0: 1 when slot `slot` holds a ready C tile (waiting a bounded number of polls while
// another block writes it), else 0.
__device__ __forceinline__ int ckpt_ready(const FwdSched& fs, int slot)
{
    int f = ld_acquire(&fs.slot_flag[slot]);
    for (int it = 0; f == 1 && it < kCkptPolls; ++it) {
        __nanosleep(200);
        f = ld_acquire(&fs.slot_flag[slot]);
    }
    return f == 2;
}

// All threads: the tile (MF x N floats, the shared-memory layout as is) from / to the slot.
template <class S>
__device__ __forceinline__ void ckpt_load(const FwdSched& fs, int slot, float* Cn)
{
    static_assert(S::MF * S::N == kCkptFloats, "checkpoint slot holds one C tile");
    const float4* src = reinterpret_cast<const float4*>(fs.ckpt + (size_t)slot * (S::MF * S::N));
    float4* dst = reinterpret_cast<float4*>(Cn);
    for (int q = threadIdx.x; q < S::MF * S::N / 4; q += kFwdThreads) dst[q] = __ldcg(src + q);
}
template <class S>
__device__ __forceinline__ void ckpt_store(const FwdSched& fs, int slot, const float* Cn)
{
    static_assert(S::MF * S::N == kCkptFloats, "checkpoint slot holds one C tile");
    float4* dst = reinterpret_cast<float4*>(fs.ckpt + (size_t)slot * (S::MF * S::N));
    const float4* src = reinterpret_cast<const float4*>(Cn);
    const uint64_t pol = l2_evict_last_policy();
    for (int q = threadIdx.x; q < S::MF * S::N / 4; q += kFwdThreads) st_v4_hint(reinterpret_cast<float*>(dst + q), src[q], pol);
}

// Persistent forward.  Software pipeline per subtask: wait for its A/B copies (none when the
// previous subtask was of the same chunk: its C is still in shared memory), the chunk's C
// (GEMM, or the L2 checkpoint a block published), then fetch the next task and, if it is a
// subtask, prefetch its metadata and A/B rows while this subtask's distinct rows are contracted
// batch by batch (double-buffered last slices when shared memory allows).
template <class S, typename K, int NT>
__global__ void __launch_bounds__(kFwdThreads, 1)
k3_fwd_kernel(CoreParams cp, int sched, const K* __restrict__ uniq_keys,
              const int4* __restrict__ grec, const int32_t* __restrict__ uid_at_pos,
              const int64_t* __restrict__ offsets, const int4* __restrict__ chunks,
              FwdSched fs, PlanHeader* hdr,
              float* __restrict__ rowbuf, float* __restrict__ out, int32_t* status)
{
    extern __shared__ __align__(16) float smem_f[];
    __shared__ FwdMeta<S> M;
    __shared__ __align__(16) K s_keys[2 * kKeyCap];   // keys of each buffer's distinct rows
    __shared__ __align__(8) uint64_t s_mbar;
    __shared__ uint32_t s_tmem;
    __shared__ int s_ok;
    if (has_error(status)) return;
    constexpr bool TC = NT > 0;
    constexpr int NS = NT == 3 ? 2 : 1;   // bf16 terms stored per operand element
    FwdSmem<S> sm;
    const int tid = threadIdx.x;
    const unsigned long long pr_t0 = cp.probe ? global_ns() : 0ull;
    unsigned long long pr_wait = 0;
    int pr_tasks = 0, pr_ckpt = 0;
    uint32_t tmem = 0, parity = 0;
    if constexpr (TC) {
        // one bf16 term takes half the room of an fp32 operand, two terms the same room
        sm.Bs = sm.As = nullptr;
        sm.Bb = reinterpret_cast<uint16_t*>(smem_f);
        sm.Ab = sm.Bb + NS * S::R * S::N;
        sm.Cn = smem_f + NS * (S::R * S::N + S::MF * S::R) / 2;
        if (tid < 32) tmem_alloc(&s_tmem, (uint32_t)S::N);
        if (tid == 0) mbar_init(&s_mbar, 1);
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        tmem = s_tmem;
    } else {
        sm.Bs = smem_f;
        sm.As = sm.Bs + S::R * S::N;
        sm.Bb = sm.Ab = nullptr;
        sm.Cn = sm.As + S::MF * S::R;
    }
    sm.Ss = sm.Cn + S::MF * S::N;
    const int nP = hdr->nP, npool = cp.T * nP;
    const bool use_ckpt = sched == TT_SCHED_STEAL_L2;
    int phase = 0, vk = 1;   // scheduler state (the scheduling thread, kSchedTid)
    int cur_t = -1, cur_i2 = -1;   // column of the B now in (or on its way to) the B tile
    int cur_cid = -1;              // chunk whose C tile is in shared memory
    int mb = 0;
    bool staged = false;
    constexpr int kSchedTid = 32;   // the thread that runs the scheduler (state in its registers)
    if (tid == kSchedTid) M.task[0] = fwd_next(fs, hdr, sched, npool, phase, vk);
    __syncthreads();
    int q = M.task[0];
    while (q != -1) {
        if (q <= -2) {
            fwd_pool<S>(cp, -2 - q, nP, uid_at_pos, offsets, hdr, rowbuf, out, status, &M.flag, &pr_wait);
            ++pr_tasks;
            __syncthreads();
            if (tid == kSchedTid) M.task[0] = fwd_next(fs, hdr, sched, npool, phase, vk);
            __syncthreads();
            q = M.task[0];
            staged = false;
            continue;
        }
        TT_PH_START();
        ++pr_tasks;
        if (!staged) {
            const int4 sub = fs.subs[q];
            fwd_meta<S, K>(cp, sub, mb, uniq_keys, grec, chunks, M, s_keys);
            if (sub.x != cur_cid) {
                if constexpr (TC) fwd_issue_ab_tc<S, NS>(cp, mb, M, sm, cur_t, cur_i2);
                else fwd_issue_ab<S>(cp, mb, M, sm, cur_t, cur_i2);
            } else {
                cp_async_commit();   // the row keys alone
            }
        }
        cp_async_wait_all();   // the subtask's A/B rows and row keys (usually prefetched long ago)
        fence_async_smem();    // A/B tiles: read by the tensor cores after the barrier
        __syncthreads();
        const int nrows = M.re[mb] - M.rb[mb];
        // the next task, read after the C step's barriers (the queue atomic runs during the C step)
        if (tid == kSchedTid) M.task[1] = fwd_next(fs, hdr, sched, npool, phase, vk);
        // the first batch of last slices is in flight during the C step (last digits from the keys)
        if (nrows > 0) fwd_issue_batch_keys<S, K>(cp, mb, M, sm, s_keys);
        // the row table; read by the batches, which come after the C step's barriers
        build_rows(M.rows, mb, M.ucum[mb], M.u0[mb], M.cnt[mb], M.re[mb], s_keys, cp.ibits, cp.n[M.t[mb]][2],
                   kFwdThreads, M.rb[mb]);
        TT_PH(0);
        const int cid = M.cid[mb], slot = M.slot[mb];
        if (cid != cur_cid) {
            // C of this chunk: the checkpoint when another block has published it, else the GEMM
            const bool ck_slot = use_ckpt && slot >= 0;   // uniform: slot comes from shared memory
            if (ck_slot) {
                if (tid == 0) M.ck = ckpt_ready(fs, slot);
                __syncthreads();
            }
            if (ck_slot && M.ck) {
                ckpt_load<S>(fs, slot, sm.Cn);
                ++pr_ckpt;
            } else {
                if constexpr (TC) {
                    if (!fwd_gemm_tc<S, NT>(sm, tmem, &s_mbar, parity, &s_ok, cp.inj_mma != 0)) {
                        if (tid == 0) raise_error(status, TT_ERR_TIMEOUT, 100);
                        break;
                    }
                } else {
                    fwd_gemm<S>(sm);
                }
                if (ck_slot) {   // publish once: the block that wins the slot writes it
                    __syncthreads();
                    if (tid == 0) M.ck = atomicCAS(&fs.slot_flag[slot], 0, 1) == 0;
                    __syncthreads();
                    if (M.ck) {
                        ckpt_store<S>(fs, slot, sm.Cn);
                        __syncthreads();
                        if (tid == 0) {
                            __threadfence();
                            st_release(&fs.slot_flag[slot], 2);
                        }
                    }
                }
            }
            cur_cid = cid;
        }
        __syncthreads();
        TT_PH(1);
        const int qn = M.task[1];
        const bool next_sub = qn >= 0;
        if (next_sub) {
            const int4 nsub = fs.subs[qn];
            fwd_meta<S, K>(cp, nsub, mb ^ 1, uniq_keys, grec, chunks, M, s_keys);
            if (nsub.x != cur_cid) {
                if constexpr (TC) fwd_issue_ab_tc<S, NS>(cp, mb ^ 1, M, sm, cur_t, cur_i2);
                else fwd_issue_ab<S>(cp, mb ^ 1, M, sm, cur_t, cur_i2);
            } else {
                cp_async_commit();
            }
        }
        // distinct rows of this subtask, in batches of NUF (commit groups in flight: the batch,
        // then possibly the next subtask's A/B, then possibly the next batch)
        if (S::FBUF == 2) {
            for (int i0 = 0, b = 0; i0 < nrows; i0 += S::NUF, b ^= 1) {
                const bool more = i0 + S::NUF < nrows;
                if (more) {
                    fwd_issue_batch<S>(cp, mb, i0 + S::NUF, b ^ 1, M, sm);
                    cp_async_wait<1>();
                } else if (i0 == 0 && next_sub) {
                    cp_async_wait<1>();
                } else {
                    cp_async_wait_all();
                }
                __syncthreads();
                TT_PH(2);
                fwd_batch_compute<S>(mb, i0, min(S::NUF, nrows - i0), b, M, sm, rowbuf);
                __syncthreads();
                TT_PH(3);
            }
        } else {
            for (int i0 = 0; i0 < nrows; i0 += S::NUF) {
                if (i0 > 0) fwd_issue_batch<S>(cp, mb, i0, 0, M, sm);
                if (i0 == 0 && next_sub) cp_async_wait<1>();
                else cp_async_wait_all();
                __syncthreads();
                TT_PH(2);
                fwd_batch_compute<S>(mb, i0, min(S::NUF, nrows - i0), 0, M, sm, rowbuf);
                __syncthreads();
                TT_PH(3);
            }
        }
        // publish the subtask's rows: the barrier orders every thread's row stores before thread
        // 0's release reduction (cumulative at device scope), which the pooling tasks acquire
        __syncthreads();
        if (tid == 0)
            asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(&hdr->done[M.t[mb]]) : "memory");
        TT_PH(6);
        q = qn;
        staged = next_sub;
        if (next_sub) mb ^= 1;
    }
    cp_async_wait_all();
    if constexpr (TC) {
        tc_fence_before();
        __syncthreads();
        if (tid < 32) {
            tc_fence_after();
            tmem_dealloc(tmem, (uint32_t)S::N);
        }
    }
    probe_write(cp, pr_t0, pr_tasks, pr_wait, pr_ckpt);
}

// ---------------------------------------------------------------------------
// upstream sums H_u = sum over the row's lookups of grad_out[bag] (balanced:
// each warp takes kHChunk consecutive sorted lookups; rows cut by a chunk
// boundary are zeroed first and receive vector reductions)
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) k3_hzero(const int32_t* __restrict__ uid_sorted, int64_t L,
                                                float* __restrict__ rowbuf, const int32_t* status)
{
    if (has_error(status)) return;
    const int64_t nb = ceil_div(L, kHChunk);
    for (int64_t q = 1 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < nb;
         q += (int64_t)gridDim.x * blockDim.x) {
        const int64_t c0 = q * kHChunk;
        const int u = uid_sorted[c0];
        if (u == uid_sorted[c0 - 1]) {
            float4* dst = reinterpret_cast<float4*>(rowbuf + (int64_t)u * D);
            for (int i = 0; i < D / 4; ++i) dst[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
}

// grad_out row of global bag g = t B + b (table t < 64): row b T + t, in units of D floats (B T
// rows of D >= 64 floats fit in device memory, so the row number fits in 32 bits); the quotient
// t comes from a float estimate corrected to the exact value
__device__ __forceinline__ uint32_t grad_row_of_bag(int g, int64_t B, float inv_b, int T)
{
    int t = __float2int_rz(__int2float_rz(g) * inv_b);
    if ((int64_t)t * B > g) --t;
    else if ((int64_t)(t + 1) * B <= g) ++t;
    return (uint32_t)((g - (int64_t)t * B) * T + t);
}

template <int D>
__global__ void __launch_bounds__(256) k3_hsum(const int32_t* __restrict__ uid_sorted,
                                               const int32_t* __restrict__ bag_sorted,
                                               const float* __restrict__ grad_out, int64_t L, int64_t B,
                                               float inv_b, int T, float* __restrict__ rowbuf,
                                               const int32_t* status)
{
    if (has_error(status)) return;
    constexpr int LB = D / 4;
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t c0 = warp * kHChunk;
    if (c0 >= L) return;
    const int64_t c1 = min64(L, c0 + kHChunk);
    const bool active = lane < LB;
    const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
    const float4* g4 = reinterpret_cast<const float4*>(grad_out) + (active ? lane : 0);
    // only the segment's first and last rows can continue past its edges: those (zeroed by
    // k3_hzero) receive vector reductions, every other row one plain store
    const int first_u = uid_sorted[c0], last_u = uid_sorted[c1 - 1];
    const bool cut_lo = c0 > 0 && uid_sorted[c0 - 1] == first_u;
    const bool cut_hi = c1 < L && uid_sorted[c1] == last_u;
    int cur = first_u;
    float4 acc = zero;
    auto flush = [&](int u, float4 a) {
        if (!active) return;
        float* dst = rowbuf + (int64_t)u * D + lane * 4;
        if ((u == first_u && cut_lo) || (u == last_u && cut_hi)) red_add_v4(dst, a);
        else *reinterpret_cast<float4*>(dst) = a;
    };
    // each lane owns one of the next 32 lookups: its row id and its grad_out row, computed once
    // (lane-parallel) one group ahead of the gathers, which then broadcast them
    int myu = -1;
    uint32_t myr = 0;
    if (c0 + lane < c1) {
        myu = uid_sorted[c0 + lane];
        myr = grad_row_of_bag(bag_sorted[c0 + lane], B, inv_b, T);
    }
    for (int64_t base = c0; base < c1; base += 32) {
        const int n = (int)min64(32, c1 - base);
        const int64_t nx = base + 32 + lane;
        int nu = -1, nbag = 0;
        if (nx < c1) {
            nu = uid_sorted[nx];
            nbag = bag_sorted[nx];
        }
        for (int k = 0; k < n; k += 8) {
            float4 v[8];
            int uq[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                uq[q] = __shfl_sync(kFull, myu, k + q);
                const uint32_t r = __shfl_sync(kFull, myr, k + q);
                v[q] = (active && k + q < n) ? __ldg(g4 + (size_t)r * (D / 4)) : zero;
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                if (k + q >= n) break;
                if (uq[q] != cur) {
                    flush(cur, acc);
                    cur = uq[q];
                    acc = zero;
                }
                acc = f4add(acc, v[q]);
            }
        }
        myu = nu;
        myr = nx < c1 ? grad_row_of_bag(nbag, B, inv_b, T) : 0u;
    }
    flush(cur, acc);
}

// ---------------------------------------------------------------------------
// backward over column groups
// ---------------------------------------------------------------------------
template <class S>
struct BwdMeta {
    int u0[2][S::MPB];
    int ucum[2][S::MPB + 1];
    int i1[2][S::MPB];
    int cnt[2];
    int bu[2][S::NUB], bp[2][S::NUB], bi3[2][S::NUB];
    int task;
    RowTable rows;
    int4 rec[2][S::MPB];   // the next chunk's per-group records, prefetched
};

// chunk metadata (groups cfirst+j0 .. +MPB of the column, from the plan's per-group records)
// into buffer mb, ending with a barrier; then asynchronous copies of the keys of its first
// kKeyCap distinct rows into keys[mb], which join the caller's next commit group
template <class S, typename K>
__device__ __forceinline__ void bwd_meta(const int4* recs, int j0, int ccount, int mb, const K* __restrict__ uniq_keys,
                                         BwdMeta<S>& M, K* keys)
{
    // recs: the chunk's per-group records (global memory, or the prefetched shared copy)
    const int tid = threadIdx.x;
    const int cnt = min(S::MPB, ccount - j0);
    if (tid < S::MPB) {
        const int4 g = tid < cnt ? recs[tid] : make_int4(0, 0, 0, 0);
        M.u0[mb][tid] = g.x;
        M.ucum[mb][tid] = g.y;
        M.i1[mb][tid] = g.z;
    }
    if (tid == 0) M.cnt[mb] = cnt;
    __syncthreads();
    if (tid == 0) {
        int run = 0;
        for (int j = 0; j < S::MPB; ++j) {
            const int v = M.ucum[mb][j];
            M.ucum[mb][j] = run;
            run += v;
        }
        M.ucum[mb][S::MPB] = run;
    }
    __syncthreads();
    const int nk = min(M.ucum[mb][S::MPB], kKeyCap);
    for (int kq = tid; kq < nk; kq += (int)blockDim.x) {
        const int j = prefix_of(M.ucum[mb], cnt, kq);
        cp_async_key(keys + mb * kKeyCap + kq, uniq_keys + M.u0[mb][j] + (kq - M.ucum[mb][j]));
    }
}

template <class S>
__device__ __forceinline__ void bwd_issue_a(const CoreParams& cp, int t, int mb, const BwdMeta<S>& M, float* As)
{
    constexpr int R = S::R, MB = S::MB, D1 = S::D1;
    const float* G1 = cp.cores[t][0];
    const int cnt = M.cnt[mb];
    for (int q = threadIdx.x; q < MB * (R / 4); q += (int)blockDim.x) {
        const int m = q / (R / 4), c4 = q % (R / 4);
        const int j = m / D1, a1 = m % D1;
        float* dst = &As[swz_a<R>(m, c4 * 4)];
        if (j < cnt) cp_async16(dst, G1 + ((int64_t)M.i1[mb][j] * D1 + a1) * R + c4 * 4);
        else *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    cp_async_commit();
}

// batch of distinct rows k0.. of chunk buffer mb into batch buffer bb: H rows and last slices (one group)
template <class S, typename K>
__device__ __forceinline__ void bwd_issue_batch(const CoreParams& cp, int t, int mb, int k0, int bb,
                                                const K* __restrict__ uniq_keys, const float* __restrict__ rowbuf,
                                                BwdMeta<S>& M, float* Hs, float* Ss, const K* keys)
{
    constexpr int R = S::R, D3 = S::D3, P = S::P, SR = S::SR;
    const int tid = threadIdx.x;
    const int total = M.ucum[mb][S::MPB];
    const int nb = min(S::NUB, total - k0);
    const uint32_t n3 = cp.n[t][2];
    if (k0 + nb > kKeyCap) {   // beyond the row table: this batch's metadata
        if (tid < nb) {
            const int kq = k0 + tid;
            const int j = prefix_of(M.ucum[mb], M.cnt[mb], kq);
            const int u = M.u0[mb][j] + (kq - M.ucum[mb][j]);
            const K key = kq < kKeyCap ? keys[mb * kKeyCap + kq] : uniq_keys[u];
            M.bu[bb][tid] = u;
            M.bp[bb][tid] = j;
            M.bi3[bb][tid] = (int)(key_row(key, cp.ibits) % n3);
        }
        __syncthreads();
    }
    const RowRef rr = batch_rows(M.rows, mb, k0, nb, M.bu[bb], M.bp[bb], M.bi3[bb]);
    float* H = Hs + (size_t)bb * S::NUB * P * D3;
    float* Sb = Ss + (size_t)bb * S::NUB * R * SR;
    for (int q = tid; q < nb * (P * D3 / 4); q += (int)blockDim.x) {
        const int uu = q / (P * D3 / 4), c4 = q % (P * D3 / 4);
        cp_async16(&H[uu * P * D3 + c4 * 4], rowbuf + (int64_t)rr.u[uu] * S::D + c4 * 4);
    }
    const float* G3t = cp.last_t[t];   // [n3][R][D3]
    for (int q = tid; q < nb * R * (D3 / 4); q += (int)blockDim.x) {
        const int uu = q / (R * (D3 / 4)), rem = q % (R * (D3 / 4));
        const int rho = rem / (D3 / 4), c4 = rem % (D3 / 4);
        cp_async16(&Sb[(uu * R + rho) * SR + c4 * 4], G3t + (int64_t)rr.i3[uu] * (R * D3) + rem * 4);
    }
    cp_async_commit();
}

// Per-row backward of a chunk with one warp per contiguous range of its distinct rows (rank 64,
// d = (4, 4, 8)); lane l owns rho_2 in {2l, 2l + 1}.  For each row u of prefix p:
//   dS_u[rho][a3] = sum_r C_p[r][rho] H_u[r][a3]    -> dG_3[rho, i3(u), a3] (vector reductions into
//                                                      the transposed copy [i3][rho][a3]: one row's
//                                                      2 KB contribution is contiguous)
//   dC_p[r][rho] += sum_a3 H_u[r][a3] S_u[rho][a3]   (registers; into dCn when the prefix ends:
//                                                      a plain store when the prefix lies inside
//                                                      this warp's range, shared atomics if not)
// C_p for the lane's columns sits in registers, H_u is broadcast through a per-warp slot, and the
// lane's two rows of S_u with its quarter-row of H_u are loaded two rows ahead.  No block
// barrier is taken between rows.
struct WarpRow {
    float4 s[4];   // S_u rows 2l, 2l + 1 (8 values each)
    float4 h;      // H_u[4 l .. 4 l + 3]
    int u, j, i3;
};

template <class S, typename K>
__device__ __forceinline__ void warp_row_load(const CoreParams& cp, int t, int mb, int kq, int cnt, const BwdMeta<S>& M,
                                              const K* __restrict__ uniq_keys, const float* __restrict__ rowbuf,
                                              uint32_t n3, WarpRow& w)
{
    constexpr int R = S::R, D3 = S::D3, D = S::D;
    const int lane = threadIdx.x & 31;
    if (kq < kKeyCap) {
        w.u = M.rows.u[mb][kq];
        w.j = M.rows.p[mb][kq];
        w.i3 = M.rows.i3[mb][kq];
    } else {
        w.j = prefix_of(M.ucum[mb], cnt, kq);
        w.u = M.u0[mb][w.j] + (kq - M.ucum[mb][w.j]);
        w.i3 = (int)(key_row(uniq_keys[w.u], cp.ibits) % n3);
    }
    const float4* sp = reinterpret_cast<const float4*>(cp.last_t[t] + (int64_t)w.i3 * (R * D3) + lane * 2 * D3);
    w.s[0] = __ldg(sp);
    w.s[1] = __ldg(sp + 1);
    w.s[2] = __ldg(sp + 2);
    w.s[3] = __ldg(sp + 3);
    w.h = __ldcg(reinterpret_cast<const float4*>(rowbuf + (int64_t)w.u * D) + lane);
}

template <class S, typename K>
__device__ __forceinline__ void bwd_rows_warp(const CoreParams& cp, int t, int mb, int total, int cnt,
                                              const BwdMeta<S>& M, const K* __restrict__ uniq_keys,
                                              const float* __restrict__ rowbuf, const float* Cn, float* dCn,
                                              float* __restrict__ dG3, uint32_t n3, float* hslots)
{
    constexpr int R = S::R, N = S::N, D1 = S::D1, D2 = S::D2, D3 = S::D3, P = S::P;
    static_assert(R == 64 && D3 == 8 && P == 16 && S::D == 128, "warp row path: rank 64, d = (4, 4, 8)");
    constexpr int NW = kBwdThreads / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int lo = (int)((int64_t)total * warp / NW), hi = (int)((int64_t)total * (warp + 1) / NW);
    if (lo >= hi) return;
    float* hs = hslots + warp * 2 * P * D3;   // two slots of one row's H (P x D3 floats each)
    float c[P][2], o[P][2];
    int cur = -1;
    auto flush = [&]() {
        const bool whole = M.ucum[mb][cur] >= lo && M.ucum[mb][cur + 1] <= hi;
#pragma unroll
        for (int r = 0; r < P; ++r) {
            float* d = &dCn[swz_m<N>(cur * D1 + r / D2, (r % D2) * R + 2 * lane)];
            if (whole) {
                *reinterpret_cast<float2*>(d) = make_float2(o[r][0], o[r][1]);
            } else {
                atomicAdd(d, o[r][0]);
                atomicAdd(d + 1, o[r][1]);
            }
        }
    };
    WarpRow a, b;
    warp_row_load<S, K>(cp, t, mb, lo, cnt, M, uniq_keys, rowbuf, n3, a);
    if (lo + 1 < hi) warp_row_load<S, K>(cp, t, mb, lo + 1, cnt, M, uniq_keys, rowbuf, n3, b);
#pragma unroll 1
    for (int kq = lo; kq < hi; ++kq) {
        const WarpRow w = a;
        a = b;
        if (kq + 2 < hi) warp_row_load<S, K>(cp, t, mb, kq + 2, cnt, M, uniq_keys, rowbuf, n3, b);
        if (w.j != cur) {
            if (cur >= 0) flush();
            cur = w.j;
#pragma unroll
            for (int r = 0; r < P; ++r) {
                const float2 cv = *reinterpret_cast<const float2*>(&Cn[swz_m<N>(cur * D1 + r / D2, (r % D2) * R + 2 * lane)]);
                c[r][0] = cv.x;
                c[r][1] = cv.y;
                o[r][0] = o[r][1] = 0.f;
            }
        }
        float* hb = hs + (kq & 1) * (P * D3);
        reinterpret_cast<float4*>(hb)[lane] = w.h;
        __syncwarp();
        const float sv[2][8] = {{w.s[0].x, w.s[0].y, w.s[0].z, w.s[0].w, w.s[1].x, w.s[1].y, w.s[1].z, w.s[1].w},
                                {w.s[2].x, w.s[2].y, w.s[2].z, w.s[2].w, w.s[3].x, w.s[3].y, w.s[3].z, w.s[3].w}};
        float ds[2][8];
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int a3 = 0; a3 < 8; ++a3) ds[q][a3] = 0.f;
#pragma unroll
        for (int r = 0; r < P; ++r) {
            const float4 h0 = *reinterpret_cast<const float4*>(hb + r * D3);
            const float4 h1 = *reinterpret_cast<const float4*>(hb + r * D3 + 4);
            const float hv[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                float acc = o[r][q];
#pragma unroll
                for (int a3 = 0; a3 < 8; ++a3) {
                    ds[q][a3] = fmaf(c[r][q], hv[a3], ds[q][a3]);
                    acc = fmaf(hv[a3], sv[q][a3], acc);
                }
                o[r][q] = acc;
            }
        }
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            float* dst = dG3 + ((int64_t)w.i3 * R + 2 * lane + q) * D3;
            red_add_v4(dst, make_float4(ds[q][0], ds[q][1], ds[q][2], ds[q][3]));
            red_add_v4(dst + 4, make_float4(ds[q][4], ds[q][5], ds[q][6], ds[q][7]));
        }
    }
    flush();
}

// One lane's share of a distinct row in the tensor-core backward (rank 64): its row of the last
// slice and a quarter-row of H_u
struct WarpRow1 {
    float4 s[2];   // S_u row rho (8 values)
    float4 h;      // H_u[4 lane .. 4 lane + 3]
    int u, j, i3;
};

// one thread issues, the others wait at the barrier; false (all threads) when the wait ran out
// (or, with inject_fail, a test hook, once the products have completed)
__device__ __forceinline__ bool tc_commit_wait(uint64_t* bar, uint32_t& parity, int* s_ok, bool inject_fail = false)
{
    if (threadIdx.x == 0) {
        tc_commit(bar);
        *s_ok = (mbar_wait(bar, parity) && !inject_fail) ? 1 : 0;
    }
    __syncthreads();
    parity ^= 1u;
    return *s_ok != 0;
}

// as tc_commit_wait, and when wait2 also the completion of phase parity2 of bar2, and with bar3 the
// completion of phase *parity3 of bar3 (products other threads committed there); the parities of
// the barriers waited for flip
__device__ __forceinline__ bool tc_commit_wait2(uint64_t* bar, uint32_t& parity, uint64_t* bar2, uint32_t& parity2,
                                                bool wait2, int* s_ok, bool inject_fail = false,
                                                uint64_t* bar3 = nullptr, uint32_t* parity3 = nullptr)
{
    if (threadIdx.x == 0) {
        tc_commit(bar);
        const bool ok = mbar_wait(bar, parity) && (!wait2 || mbar_wait(bar2, parity2)) &&
                        (bar3 == nullptr || mbar_wait(bar3, *parity3));
        *s_ok = (ok && !inject_fail) ? 1 : 0;
    }
    __syncthreads();
    parity ^= 1u;
    if (wait2) parity2 ^= 1u;
    if (bar3) *parity3 ^= 1u;
    return *s_ok != 0;
}

template <class S, typename K>
__global__ void __launch_bounds__(kBwdThreads, 1)
k3_bwd_kernel(CoreParams cp, GradPtrs gp, PlanParams pp, const K* __restrict__ uniq_keys,
              const int4* __restrict__ grec, const int32_t* __restrict__ col_count,
              const int32_t* __restrict__ col_start, const int32_t* __restrict__ col_order, PlanHeader* hdr,
              const float* __restrict__ rowbuf, int32_t* status)
{
    constexpr int R = S::R, N = S::N, MB = S::MB, MPB = S::MPB, D1 = S::D1, D2 = S::D2, D3 = S::D3,
                  P = S::P, NUB = S::NUB, DBR = S::DBR, DBC = S::DBC, SR = S::SR;
    extern __shared__ __align__(16) float smem_f[];
    __shared__ BwdMeta<S> M;
    __shared__ __align__(16) K s_keys[2 * kKeyCap];   // keys of each chunk buffer's first rows
    constexpr int BT = kBwdThreads;
    // per-row backward by warps over contiguous row ranges (rank 64, d = (4, 4, 8)); other
    // shapes use barrier-synchronised batches of NUB rows
    constexpr bool WARP_ROWS = R == 64 && D1 == 4 && D2 == 4 && D3 == 8;
    float* Bs = smem_f;                    // [R][N] swizzled (key row/4)
    float* As = smem_f + R * N;            // [2][MB][R] swizzled
    float* Cn = As + 2 * MB * R;           // [MB][N] swizzled (key row)
    float* dCn = Cn + MB * N;              // [MB][N] swizzled (key row)
    float* Hs = dCn + MB * N;              // [2][NUB][P][D3]
    float* Ss = Hs + 2 * NUB * P * D3;     // [2][NUB][R][SR]
    if (has_error(status)) return;
    const int tid = threadIdx.x;

    const unsigned long long pr_t0 = cp.probe ? global_ns() : 0ull;
    int pr_tasks = 0;
    const int ncols_busy = hdr->ncols_busy;   // the column queue (see k_plan_order)
    for (int iter = 0;; ++iter) {
        TT_PH_START();
        if (tid == 0) M.task = next_task(pp.sched, &hdr->col_head, iter);
        __syncthreads();
        if (M.task >= ncols_busy) break;
        const int c = col_order[M.task];
        ++pr_tasks;
        const int ccount = col_count[c];
        if (ccount == 0) {
            __syncthreads();
            continue;
        }
        int t = 0;
        while (t + 1 < cp.T && pp.col_base[t + 1] <= c) ++t;
        const int i2 = c - pp.col_base[t];
        const int cfirst = col_start[c];
        const uint32_t n2 = cp.n[t][1], n3 = cp.n[t][2];
        float* __restrict__ dG1 = gp.g[t][0];
        float* __restrict__ dG2 = gp.g[t][1];
        float* __restrict__ dG3 = gp.g[t][2];   // transposed layout [n3][R][D3]
        TT_PH(17);

        // B for the whole column group, and the first chunk's A
        {
            const float* G2 = cp.cores[t][1] + (int64_t)i2 * N;
            const int64_t rs = (int64_t)n2 * N;
            for (int q = tid; q < R * N / 4; q += BT) {
                const int rho = q / (N / 4), c4 = q % (N / 4);
                cp_async16(&Bs[swz_b<N>(rho, c4 * 4)], G2 + rho * rs + c4 * 4);
            }
        }
        bwd_meta<S, K>(grec + cfirst, 0, ccount, 0, uniq_keys, M, s_keys);
        bwd_issue_a<S>(cp, t, 0, M, As);
        TT_PH(8);

        // dB of the column group in registers: DBR rows x DBC columns per thread
        constexpr int NCH = DBC / 4;
        constexpr int TNB = N / DBC;
        const int tnb = tid % TNB, trb = tid / TNB;
        float dB[DBR][DBC];
#pragma unroll
        for (int i = 0; i < DBR; ++i)
#pragma unroll
            for (int j = 0; j < DBC; ++j) dB[i][j] = 0.f;

        int mb = 0;
        for (int j0 = 0; j0 < ccount; j0 += MPB, mb ^= 1) {
            const int cnt = M.cnt[mb];
            const float* Ab = As + mb * MB * R;
            cp_async_wait_all();   // B, this chunk's A rows and row keys (usually prefetched long ago)
            __syncthreads();
            const int total = M.ucum[mb][MPB];
            const bool more = j0 + MPB < ccount;
            build_rows(M.rows, mb, M.ucum[mb], M.u0[mb], cnt, total, s_keys, cp.ibits, n3, BT);
            // the next chunk's group records travel with this chunk's first batch
            if (more && tid < min(MPB, ccount - j0 - MPB)) cp_async16(&M.rec[mb ^ 1][tid], grec + cfirst + j0 + MPB + tid);
            __syncthreads();
            // the first batch of distinct rows is in flight during the C GEMM
            if (!WARP_ROWS && total > 0) bwd_issue_batch<S, K>(cp, t, mb, 0, 0, uniq_keys, rowbuf, M, Hs, Ss, s_keys);
            else cp_async_commit();
            for (int q = tid; q < MB * N / 4; q += BT)
                reinterpret_cast<float4*>(dCn)[q] = make_float4(0.f, 0.f, 0.f, 0.f);
            __syncthreads();
            TT_PH(9);

            {
                // C_all = A . B  (MB x N): thread tile 4 rows x 8 cols
                constexpr int TN = N / 8;
                int tm, tn;   // tm < MB / 4
                warp_tile_2d<TN>(tid, tm, tn);
                float acc[4][8];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
#pragma unroll 1
                for (int rho = 0; rho < R; rho += 4) {
                    float4 a[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) a[i] = *reinterpret_cast<const float4*>(&Ab[swz_a<R>(tm * 4 + i, rho)]);
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const float4 b0 = *reinterpret_cast<const float4*>(&Bs[swz_b<N>(rho + r, tn * 4)]);
                        const float4 b1 = *reinterpret_cast<const float4*>(&Bs[swz_b<N>(rho + r, N / 2 + tn * 4)]);
                        const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float av = f4get(a[i], r);
#pragma unroll
                            for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av, b[j], acc[i][j]);
                        }
                    }
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int m = tm * 4 + i;
                    *reinterpret_cast<float4*>(&Cn[swz_m<N>(m, tn * 4)]) =
                        make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
                    *reinterpret_cast<float4*>(&Cn[swz_m<N>(m, N / 2 + tn * 4)]) =
                        make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
                }
            }
            __syncthreads();
            TT_PH(10);

            // next chunk's metadata and A rows go in flight while this chunk's rows are processed
            if (more) {
                cp_async_wait_all();   // its group records (and this chunk's first batch)
                __syncthreads();
                bwd_meta<S, K>(M.rec[mb ^ 1], j0 + MPB, ccount, mb ^ 1, uniq_keys, M, s_keys);
                bwd_issue_a<S>(cp, t, mb ^ 1, M, As + (mb ^ 1) * MB * R);
            }
            TT_PH(16);

            if constexpr (WARP_ROWS) {
                bwd_rows_warp<S, K>(cp, t, mb, total, cnt, M, uniq_keys, rowbuf, Cn, dCn, dG3, n3, Hs);
                __syncthreads();
                TT_PH(12);
            }
            // distinct rows in double-buffered batches: dS_u -> dG_3 (vector reductions), dC_p += H_u S_u^T
            // (commit groups in flight: the batch, then possibly the next chunk's A, then possibly the next batch)
            for (int k0 = 0, bb = 0; !WARP_ROWS && k0 < total; k0 += NUB, bb ^= 1) {
                const int nb = min(NUB, total - k0);
                if (k0 + NUB < total) {
                    bwd_issue_batch<S, K>(cp, t, mb, k0 + NUB, bb ^ 1, uniq_keys, rowbuf, M, Hs, Ss, s_keys);
                    TT_PH(7);
                    cp_async_wait<1>();
                } else if (k0 == 0 && more) {
                    cp_async_wait<1>();
                } else {
                    cp_async_wait_all();
                }
                __syncthreads();
                TT_PH(11);
                const float* H = Hs + (size_t)bb * NUB * P * D3;
                const float* Sb = Ss + (size_t)bb * NUB * R * SR;
                // dS_u[rho2][a3]: tile 4 consecutive rho2 x 4 a3, one tile per thread
                {
                    const int uu = tid / S::TPUB, rem = tid % S::TPUB;
                    const int rc = rem / (D3 / 4), cg = rem % (D3 / 4);
                    if (uu < nb) {
                        const RowRef rr = batch_rows(M.rows, mb, k0, nb, M.bu[bb], M.bp[bb], M.bi3[bb]);
                        const int p = rr.p[uu];
                        float4 o[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) o[i] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
                        for (int row = 0; row < P; ++row) {
                            const int m = p * D1 + row / D2, a2 = row % D2;
                            const float4 cv = *reinterpret_cast<const float4*>(&Cn[swz_m<N>(m, a2 * R + rc * 4)]);
                            const float4 h = *reinterpret_cast<const float4*>(&H[uu * P * D3 + row * D3 + cg * 4]);
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const float cr = f4get(cv, i);
                                o[i].x = fmaf(cr, h.x, o[i].x);
                                o[i].y = fmaf(cr, h.y, o[i].y);
                                o[i].z = fmaf(cr, h.z, o[i].z);
                                o[i].w = fmaf(cr, h.w, o[i].w);
                            }
                        }
                        const int i3 = rr.i3[uu];
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            red_add_v4(dG3 + ((int64_t)i3 * R + rc * 4 + i) * D3 + cg * 4, o[i]);
                    }
                }
#ifdef TT_PROFILE_PHASES
                __syncthreads();   // profiling builds only: separates the dS and dC times
#endif
                TT_PH(6);
                // dC_p[row][rho2] += sum_{u in p, a3} H_u[row][a3] S_u[rho2][a3]: each tile (prefix p,
                // rows (a1, a2 = 0..3), rho2 in {rc, rc+R/4, rc+R/2, rc+3R/4}) is owned by one thread, which
                // adds the batch's rows of its prefix in order (plain read-modify-write, deterministic)
                {
                    constexpr int TPD = D1 * (R / 4);
                    for (int w = tid; w < cnt * TPD; w += kBwdThreads) {
                        const int p = w / TPD, rem = w % TPD;
                        const int a1 = rem / (R / 4), rc = rem % (R / 4);
                        const int ulo = max(M.ucum[mb][p], k0) - k0, uhi = min(M.ucum[mb][p + 1], k0 + nb) - k0;
                        if (ulo >= uhi) continue;
                        float o[4][4];
#pragma unroll
                        for (int i = 0; i < 4; ++i)
#pragma unroll
                            for (int j = 0; j < 4; ++j) o[i][j] = 0.f;
                        for (int uu = ulo; uu < uhi; ++uu) {
#pragma unroll
                            for (int ac = 0; ac < D3; ac += 4) {
                                float4 h[4], sv[4];
#pragma unroll
                                for (int i = 0; i < 4; ++i)
                                    h[i] = *reinterpret_cast<const float4*>(&H[uu * P * D3 + (a1 * D2 + i) * D3 + ac]);
#pragma unroll
                                for (int j = 0; j < 4; ++j)
                                    sv[j] = *reinterpret_cast<const float4*>(&Sb[(uu * R + rc + j * (R / 4)) * SR + ac]);
#pragma unroll
                                for (int i = 0; i < 4; ++i)
#pragma unroll
                                    for (int j = 0; j < 4; ++j) {
                                        o[i][j] = fmaf(h[i].x, sv[j].x, o[i][j]);
                                        o[i][j] = fmaf(h[i].y, sv[j].y, o[i][j]);
                                        o[i][j] = fmaf(h[i].z, sv[j].z, o[i][j]);
                                        o[i][j] = fmaf(h[i].w, sv[j].w, o[i][j]);
                                    }
                            }
                        }
                        const int m = p * D1 + a1;
#pragma unroll
                        for (int i = 0; i < 4; ++i)
#pragma unroll
                            for (int j = 0; j < 4; ++j) dCn[swz_m<N>(m, i * R + rc + j * (R / 4))] += o[i][j];
                    }
                }
                __syncthreads();
                TT_PH(12);
            }

            // dA[m][rho1] = sum_n dC[m][n] B[rho1][n] -> dG_1; tiles 4 m x 4 rho1, the n range split
            // between the two halves of the block and combined through shared memory
            {
                constexpr int TRH = R / 4;
                const int kh = tid / 128, tl = tid % 128;
                float* part = Hs;   // batch buffers are free here: 128 tiles x 16 partial sums
                float o[4][4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) o[i][j] = 0.f;
                const bool act = tl < (MB / 4) * TRH;
                const int tr = tl % TRH, tm = tl / TRH;
                if (act) {
#pragma unroll 2
                    for (int n = kh * (N / 2); n < (kh + 1) * (N / 2); n += 4) {
                        float4 dc[4], b[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dc[i] = *reinterpret_cast<const float4*>(&dCn[swz_m<N>(tm * 4 + i, n)]);
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            b[j] = *reinterpret_cast<const float4*>(&Bs[swz_b<N>(tr * 4 + j, n)]);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                o[i][j] += dc[i].x * b[j].x + dc[i].y * b[j].y + dc[i].z * b[j].z + dc[i].w * b[j].w;
                    }
                }
                if (kh == 1 && act) {
#pragma unroll
                    for (int i = 0; i < 4; ++i)
#pragma unroll
                        for (int j = 0; j < 4; ++j) part[tl * 16 + i * 4 + j] = o[i][j];
                }
                __syncthreads();
                if (kh == 0 && act) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int m = tm * 4 + i, p = m / D1, a1 = m % D1;
                        if (p < cnt)
                            red_add_v4(dG1 + ((int64_t)M.i1[mb][p] * D1 + a1) * R + tr * 4,
                                       make_float4(o[i][0] + part[tl * 16 + i * 4 + 0],
                                                   o[i][1] + part[tl * 16 + i * 4 + 1],
                                                   o[i][2] + part[tl * 16 + i * 4 + 2],
                                                   o[i][3] + part[tl * 16 + i * 4 + 3]));
                    }
                }
            }
            TT_PH(13);
            // dB[rho1][n] += sum_m A[m][rho1] dC[m][n]
            {
#pragma unroll 2
                for (int m = 0; m < MB; ++m) {
                    float a[DBR];
                    if constexpr (DBR >= 4) {
                        const float4 a0 = *reinterpret_cast<const float4*>(&Ab[swz_a<R>(m, trb * 4)]);
                        a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w;
                        if constexpr (DBR == 8) {
                            const float4 a1v = *reinterpret_cast<const float4*>(&Ab[swz_a<R>(m, R / 2 + trb * 4)]);
                            a[4] = a1v.x; a[5] = a1v.y; a[6] = a1v.z; a[7] = a1v.w;
                        }
                    } else {
                        a[0] = Ab[swz_a<R>(m, trb)];
                    }
                    float bv[DBC];
#pragma unroll
                    for (int ch = 0; ch < NCH; ++ch) {
                        const float4 v = *reinterpret_cast<const float4*>(&dCn[swz_m<N>(m, ch * (N / NCH) + tnb * 4)]);
                        bv[ch * 4 + 0] = v.x; bv[ch * 4 + 1] = v.y; bv[ch * 4 + 2] = v.z; bv[ch * 4 + 3] = v.w;
                    }
#pragma unroll
                    for (int i = 0; i < DBR; ++i)
#pragma unroll
                        for (int j = 0; j < DBC; ++j) dB[i][j] = fmaf(a[i], bv[j], dB[i][j]);
                }
            }
            __syncthreads();   // dCn, Ab and the partial buffer are reused by the next chunk
            TT_PH(14);
        }
        // the column group is complete: dG_2[:, i_2] = dB (this block owns the slice)
#pragma unroll
        for (int i = 0; i < DBR; ++i) {
            int rho1;
            if constexpr (DBR == 8) rho1 = (i < 4) ? trb * 4 + i : R / 2 + trb * 4 + (i - 4);
            else if constexpr (DBR == 4) rho1 = trb * 4 + i;
            else rho1 = trb;
            if (gp.fused) {   // sparse fused SGD: G_2[:, i_2] -= lr dB
                float* g2 = gp.upd1[t] + ((int64_t)rho1 * n2 + i2) * N;
#pragma unroll
                for (int ch = 0; ch < NCH; ++ch) {
                    float4* q = reinterpret_cast<float4*>(g2 + ch * (N / NCH) + tnb * 4);
                    const float4 x = *q;
                    *q = make_float4(x.x - gp.lr * dB[i][ch * 4], x.y - gp.lr * dB[i][ch * 4 + 1],
                                     x.z - gp.lr * dB[i][ch * 4 + 2], x.w - gp.lr * dB[i][ch * 4 + 3]);
                }
            } else {
                float* dst = dG2 + ((int64_t)rho1 * n2 + i2) * N;
#pragma unroll
                for (int ch = 0; ch < NCH; ++ch)
                    *reinterpret_cast<float4*>(dst + ch * (N / NCH) + tnb * 4) =
                        make_float4(dB[i][ch * 4], dB[i][ch * 4 + 1], dB[i][ch * 4 + 2], dB[i][ch * 4 + 3]);
            }
        }
        __syncthreads();
        TT_PH(15);
    }
    cp_async_wait_all();
    probe_write(cp, pr_t0, pr_tasks, 0ull);
}

// ---------------------------------------------------------------------------
// Tensor-core backward with transposed prefix products (rank 64, d = (4, 4, 8)).
//
// A chunk is kMPB2 = 16 prefixes of a column group, i.e. 64 rows m = (prefix, a_1) of A.
//   C^T = B^T A^T   two M = 128 products (n = (a_2, rho_2) in [0, 128) and [128, 256)), N = 64,
//                   K = R, left in tensor memory: lane n holds column n of C for every chunk row.
//                   The warp of sub-partition s reads rho_2 = 32 (s mod 2) + l for a_2 in
//                   {s / 2, s / 2 + 2} with one tcgen05.ld per prefix -- no copy of C through
//                   shared memory.
//   rows            the four warps of a quad (one per sub-partition) share each distinct row u of
//                   prefix p; a lane holds C_p for its rho_2 and two a_2 (8 values) and adds
//                     dS_u[rho][a3] += sum_{a1, its a2} C_p[(a1, a2)][rho] H_u[(a1, a2)][a3]
//                                      (vector reductions into dG_3^T [i3][rho][a3])
//                     dC_p[(a1, a2)][rho] += sum_a3 H_u[(a1, a2)][a3] S_u[rho][a3]
//                   with the quads on contiguous row ranges and no block barrier between rows.
//   dA = dC . B^T (M = 64, every row a chunk row), dB += A^T . dC over the column group; the
//                   two dA accumulators and dB are issued by three threads of different warps.
// ---------------------------------------------------------------------------
constexpr int kMPB2 = 16;   // prefixes per chunk
constexpr int kMB2 = 64;    // rows of A per chunk

struct BwdMeta2 {
    int u0[2][kMPB2];
    int ucum[2][kMPB2 + 1];
    int i1[2][kMPB2];
    int cnt[2];
    int task;
    RowTableT<kKeyCapB> rows;
    int4 rec[2][kMPB2];   // the next chunk's per-group records, prefetched
};

// chunk metadata into buffer mb (ends with a barrier), then asynchronous copies of the keys of
// its first kKeyCapB distinct rows into keys[mb] (they join the caller's next commit group)
template <typename K>
__device__ __forceinline__ void bwd2_meta(const int4* recs, int j0, int ccount, int mb, const K* __restrict__ uniq_keys,
                                          BwdMeta2& M, K* keys)
{
    const int tid = threadIdx.x;
    const int cnt = min(kMPB2, ccount - j0);
    if (tid < 32) {
        // one warp: records, exclusive scan of the row counts
        const int4 g = tid < cnt ? recs[tid] : make_int4(0, 0, 0, 0);
        int x = tid < kMPB2 ? g.y : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, x, o);
            if (tid >= o) x += y;
        }
        if (tid < kMPB2) {
            M.u0[mb][tid] = g.x;
            M.ucum[mb][tid] = x - g.y;
            M.i1[mb][tid] = g.z;
        }
        if (tid == kMPB2 - 1) M.ucum[mb][kMPB2] = x;
        if (tid == 0) M.cnt[mb] = cnt;
    }
    __syncthreads();
    const int nk = min(M.ucum[mb][kMPB2], kKeyCapB);
    for (int kq = tid; kq < nk; kq += (int)blockDim.x) {
        const int j = prefix_of(M.ucum[mb], cnt, kq);
        cp_async_key(keys + mb * kKeyCapB + kq, uniq_keys + M.u0[mb][j] + (kq - M.ucum[mb][j]));
    }
}

// the chunk's G_1 rows (NS bf16 terms) into 8 x 16-byte core matrices of kMB2 rows; one commit group
template <int NS>
__device__ __forceinline__ void bwd2_issue_a(const CoreParams& cp, int t, int mb, const BwdMeta2& M, uint16_t* Ab)
{
    constexpr int R = 64, MB = kMB2, D1 = 4, KC = R / 8;
    const uint16_t* G1 = cp.bf1[t];
    const int cnt = M.cnt[mb];
    for (int q = threadIdx.x; q < NS * MB * KC; q += (int)blockDim.x) {
        const int term = q / (MB * KC), r = q % (MB * KC);
        const int m = (r / (8 * KC)) * 8 + (r & 7), kc = (r >> 3) % KC;   // 8 threads per core matrix
        const int j = m / D1, a1 = m % D1;
        uint16_t* dst = Ab + term * (MB * R) + ((m >> 3) * KC + kc) * 64 + (m & 7) * 8;
        if (j < cnt) cp_async16(dst, G1 + ((int64_t)M.i1[mb][j] * D1 + a1) * (NS * R) + term * R + kc * 8);
        else *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
    }
    cp_async_commit();
}

// two 32 x 4 reads of tensor memory (lane i of the warp: row taddr lane + i, 4 columns each), and
// the wait for both, in one statement so no use of the values can move above the wait
__device__ __forceinline__ void tmem_ld4x2(uint32_t ta, uint32_t tb, float (&v)[8])
{
    uint32_t r[8];
    asm volatile(
        "{\n\ttcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%8];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%4, %5, %6, %7}, [%9];\n\t"
        "tcgen05.wait::ld.sync.aligned;\n\t}"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
        : "r"(ta), "r"(tb)
        : "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}
// 32 lanes x 16 consecutive columns, with the wait
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile(
        "{\n\ttcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16];\n\ttcgen05.wait::ld.sync.aligned;\n\t}"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

template <typename K>
__device__ __forceinline__ void warp_row_load2(const CoreParams& cp, int t, int mb, int kq, int cnt, int rho,
                                               const BwdMeta2& M, const K* __restrict__ uniq_keys,
                                               const float* __restrict__ rowbuf, uint32_t n3, WarpRow1& w)
{
    constexpr int R = 64, D3 = 8, D = 128;
    const int lane = threadIdx.x & 31;
    if (kq < kKeyCapB) {
        w.u = M.rows.u[mb][kq];
        w.j = M.rows.p[mb][kq];
        w.i3 = M.rows.i3[mb][kq];
    } else {
        w.j = prefix_of(M.ucum[mb], cnt, kq);
        w.u = M.u0[mb][w.j] + (kq - M.ucum[mb][w.j]);
        w.i3 = (int)(key_row(uniq_keys[w.u], cp.ibits) % n3);
    }
    const float4* sp = reinterpret_cast<const float4*>(cp.last_t[t] + (int64_t)w.i3 * (R * D3) + rho * D3);
    w.s[0] = __ldg(sp);
    w.s[1] = __ldg(sp + 1);
    // the four warps of the quad read the same row: through L1
    w.h = __ldg(reinterpret_cast<const float4*>(rowbuf + (int64_t)w.u * D) + lane);
}

// two fp32 fused multiply-adds in one instruction (fma.rn.f32x2): d.lo += a.lo * b.lo,
// d.hi += a.hi * b.hi, each rounded as an fp32 fmaf
__device__ __forceinline__ uint64_t pack2(float lo, float hi)
{
    return ((uint64_t)__float_as_uint(hi) << 32) | __float_as_uint(lo);
}
__device__ __forceinline__ void ffma2(uint64_t& d, uint64_t a, uint64_t b)
{
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(d) : "l"(a), "l"(b));
}

// the chunk's distinct rows by quads of warps (see above); tmem_c = the C^T accumulators
template <typename K>
__device__ __forceinline__ void bwd2_rows(const CoreParams& cp, int t, int mb, int total, int cnt, const BwdMeta2& M,
                                          const K* __restrict__ uniq_keys, const float* __restrict__ rowbuf,
                                          uint32_t tmem_c, float* dCn, float* __restrict__ dG3, uint32_t n3,
                                          float* hslots)
{
    constexpr int R = 64, N = 256, D1 = 4, D2 = 4, D3 = 8, P = 16, MB = kMB2, NQ = kBwdThreadsTC / 128;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, sub = warp & 3, quad = warp >> 2;
    const int rho = (sub & 1) * 32 + lane, a2a = sub >> 1;   // this warp's a_2: a2a and a2a + 2
    const int lo = (int)((int64_t)total * quad / NQ), hi = (int)((int64_t)total * (quad + 1) / NQ);
    if (lo >= hi) return;
    const uint32_t tl = tmem_c + ((uint32_t)(32 * sub) << 16);
    float* hs = hslots + warp * 2 * P * D3;
    WarpRow1 a, b;
    warp_row_load2<K>(cp, t, mb, lo, cnt, rho, M, uniq_keys, rowbuf, n3, a);
    if (lo + 1 < hi) warp_row_load2<K>(cp, t, mb, lo + 1, cnt, rho, M, uniq_keys, rowbuf, n3, b);
    float c[8], o[8];   // entry 2 a1 + g: a_2 = a2a + 2 g
    int cur = -1;
    auto flush = [&]() {
        const bool whole = M.ucum[mb][cur] >= lo && M.ucum[mb][cur + 1] <= hi;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float* d = &dCn[swz_m<N>(cur * D1 + (i >> 1), (a2a + 2 * (i & 1)) * R + rho)];
            if (whole) *d = o[i];
            else atomicAdd(d, o[i]);
        }
    };
#pragma unroll 1
    for (int kq = lo; kq < hi; ++kq) {
        const WarpRow1 w = a;
        a = b;
        if (kq + 2 < hi) warp_row_load2<K>(cp, t, mb, kq + 2, cnt, rho, M, uniq_keys, rowbuf, n3, b);
        if (w.j != cur) {
            if (cur >= 0) flush();
            cur = w.j;
            float v[8];   // columns m = 4 cur + a1 of the two accumulators
            tmem_ld4x2(tl + (uint32_t)(cur * D1), tl + (uint32_t)(MB + cur * D1), v);
#pragma unroll
            for (int a1 = 0; a1 < 4; ++a1) {
                c[2 * a1] = v[a1];
                c[2 * a1 + 1] = v[4 + a1];
                o[2 * a1] = 0.f;
                o[2 * a1 + 1] = 0.f;
            }
        }
        float* hb = hs + (kq & 1) * (P * D3);
        reinterpret_cast<float4*>(hb)[lane] = w.h;
        __syncwarp();
        const float sv[8] = {w.s[0].x, w.s[0].y, w.s[0].z, w.s[0].w, w.s[1].x, w.s[1].y, w.s[1].z, w.s[1].w};
        uint64_t ds2[4] = {0ull, 0ull, 0ull, 0ull};   // dS_u[rho][a3] as (even, odd) a3 pairs
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int r = (i >> 1) * D2 + a2a + 2 * (i & 1);   // row (a1, a2) of H_u
            const float4 h0 = *reinterpret_cast<const float4*>(hb + r * D3);
            const float4 h1 = *reinterpret_cast<const float4*>(hb + r * D3 + 4);
            const float hv[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
            const uint64_t cc = pack2(c[i], c[i]);
#pragma unroll
            for (int k = 0; k < 4; ++k) ffma2(ds2[k], cc, pack2(hv[2 * k], hv[2 * k + 1]));
            float acc = o[i];
#pragma unroll
            for (int a3 = 0; a3 < 8; ++a3) acc = fmaf(hv[a3], sv[a3], acc);
            o[i] = acc;
        }
        float ds[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            ds[2 * k] = __uint_as_float((uint32_t)ds2[k]);
            ds[2 * k + 1] = __uint_as_float((uint32_t)(ds2[k] >> 32));
        }
        float* dst = dG3 + ((int64_t)w.i3 * R + rho) * D3;
        red_add_v4(dst, make_float4(ds[0], ds[1], ds[2], ds[3]));
        red_add_v4(dst + 4, make_float4(ds[4], ds[5], ds[6], ds[7]));
    }
    flush();
}

template <typename K, int NT>
__global__ void __launch_bounds__(kBwdThreadsTC, 1)
k3_bwd_tc2_kernel(CoreParams cp, GradPtrs gp, PlanParams pp, const K* __restrict__ uniq_keys,
                  const int4* __restrict__ grec, const int32_t* __restrict__ col_count,
                  const int32_t* __restrict__ col_start, const int32_t* __restrict__ col_order, PlanHeader* hdr,
                  const float* __restrict__ rowbuf, int32_t* status)
{
    constexpr int R = 64, N = 256, D1 = 4, MPB = kMPB2, MB = kMB2, BT = kBwdThreadsTC;
    constexpr int NS = NT == 3 ? 2 : 1;
    constexpr int CB = BT / 128;   // column blocks per tensor-memory sub-partition
    constexpr int DAQ = 2;         // dA accumulators in tensor-memory columns [N + 2 MB, N + 2 MB + DAQ R)
    constexpr uint32_t TDA = N + 2 * MB;
    static_assert(NT == 1 || NT == 3, "tensor-core variants");
    static_assert(TDA + DAQ * R <= 2 * N, "tensor-memory columns");
    extern __shared__ __align__(16) float smem_f[];
    __shared__ BwdMeta2 M;
    __shared__ __align__(16) K s_keys[2 * kKeyCapB];
    __shared__ __align__(8) uint64_t s_mbar;
    __shared__ __align__(8) uint64_t s_mbar2;   // a chunk's dA and dB products, committed by three threads
    __shared__ __align__(8) uint64_t s_mbar3;   // the second half of a chunk's C^T product
    __shared__ uint32_t s_tmem;
    __shared__ int s_ok;
    uint16_t* Bb = reinterpret_cast<uint16_t*>(smem_f);            // NS x (N x R): [n/8][rho/8][8][8]
    uint16_t* Abt = Bb + NS * R * N;                                // [2][NS][MB x R]: [m/8][rho/8][8][8]
    float* dCn = reinterpret_cast<float*>(Abt + 2 * NS * MB * R);   // [MB][N] swizzled; then NS x (MB x N) bf16
    uint16_t* dCb = reinterpret_cast<uint16_t*>(dCn);
    float* hslots = dCn + MB * N;                                   // [warps][2][P D3]
    if (has_error(status)) return;
    const int tid = threadIdx.x;
    uint32_t parity = 0;
    bool failed = false;
    // tensor memory: columns [0, N) dB of the column group, [N, N + 2 MB) C^T, [TDA, TDA + DAQ R) dA.
    // A chunk's dA and dB products are waited for with the next chunk's C^T product (or at the end
    // of the column): they run while the next chunk's row table is built. They are issued by
    // three threads in different warps (two dA accumulators and dB), because one thread issuing
    // all sixty small products in a row holds the block at its next barrier; each of the three
    // commits to s_mbar2.
    if (tid < 32) tmem_alloc(&s_tmem, 2 * N);
    if (tid == 0) {
        mbar_init(&s_mbar, 1);
        mbar_init(&s_mbar2, 3);
        mbar_init(&s_mbar3, 1);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    uint32_t parity2 = 0, parity3 = 0;
    bool pend2 = false;   // a chunk's dA / dB products committed to s_mbar2 and not yet waited for

    const unsigned long long pr_t0 = cp.probe ? global_ns() : 0ull;
    int pr_tasks = 0;
    const int ncols_busy = hdr->ncols_busy;   // the column queue (see k_plan_order)
    for (int iter = 0;; ++iter) {
        TT_PH_START();
        if (tid == 0) M.task = next_task(pp.sched, &hdr->col_head, iter);
        __syncthreads();
        if (M.task >= ncols_busy) break;
        const int c = col_order[M.task];
        ++pr_tasks;
        const int ccount = col_count[c];
        if (ccount == 0) {
            __syncthreads();
            continue;
        }
        int t = 0;
        while (t + 1 < cp.T && pp.col_base[t + 1] <= c) ++t;
        const int i2 = c - pp.col_base[t];
        const int cfirst = col_start[c];
        const uint32_t n2 = cp.n[t][1], n3 = cp.n[t][2];
        float* __restrict__ dG1 = gp.g[t][0];
        float* __restrict__ dG2 = gp.g[t][1];
        float* __restrict__ dG3 = gp.g[t][2];   // transposed layout [n3][R][D3]
        TT_PH(17);
        {
            const uint16_t* src = cp.bf2[t] + (int64_t)i2 * (NS * R * N);
            for (int q = tid; q < NS * R * N / 8; q += BT) cp_async16(Bb + q * 8, src + q * 8);
        }
        bwd2_meta<K>(grec + cfirst, 0, ccount, 0, uniq_keys, M, s_keys);
        bwd2_issue_a<NS>(cp, t, 0, M, Abt);
        TT_PH(8);
        // dA of a chunk whose products are complete -> dG_1: rows m = 16 sub + lane (lane < 16),
        // columns 16 qtr .. 16 qtr + 15, summed over the accumulators
        auto read_dA = [&](int pmb, int pcnt) {
            const int warp = tid >> 5, lane = tid & 31, sub = warp & 3, qtr = warp >> 2;
            const int m = 16 * sub + lane, p = m / D1, a1 = m % D1;
            const uint32_t ta = tmem + ((uint32_t)(32 * sub) << 16) + (uint32_t)(TDA + qtr * 16);
            float v[16];
            tmem_ld16(ta, v);
#pragma unroll 1
            for (int q = 1; q < DAQ; ++q) {
                float x[16];
                tmem_ld16(ta + (uint32_t)(q * R), x);
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] += x[i];
            }
            if (lane < 16 && p < pcnt) {
                float* dst = dG1 + ((int64_t)M.i1[pmb][p] * D1 + a1) * R + qtr * 16;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    red_add_v4(dst + 4 * j, make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
            }
        };
        int pmb = -1, pcnt = 0;   // the chunk whose dA / dB products are in flight

        int mb = 0;
        for (int j0 = 0; j0 < ccount; j0 += MPB, mb ^= 1) {
            const int cnt = M.cnt[mb];
            const uint16_t* Ab16 = Abt + mb * NS * MB * R;
            cp_async_wait_all();   // B, this chunk's A rows and row keys
            __syncthreads();
            const int total = M.ucum[mb][MPB];
            const bool more = j0 + MPB < ccount;
            build_rows(M.rows, mb, M.ucum[mb], M.u0[mb], cnt, total, s_keys, cp.ibits, n3, BT);
            if (more && tid < min(MPB, ccount - j0 - MPB)) cp_async16(&M.rec[mb ^ 1][tid], grec + cfirst + j0 + MPB + tid);
            cp_async_commit();
            fence_async_smem();
            __syncthreads();
            TT_PH(9);

            // C^T = B^T A^T: A operand = the B tile read as M = n (K-major), B operand = the A tile
            // half h = 0 by thread 0 (committed by tc_commit_wait2), h = 1 by lane 0 of warp 2 (s_mbar3)
            if (tid == 0 || tid == 64) {
                tc_fence_after();
                constexpr uint32_t SBO = (R / 8) * 128;
                const uint32_t a0 = smem_u32(Bb), b0 = smem_u32(Ab16);
                const int h = tid == 0 ? 0 : 1;
#pragma unroll
                for (int k = 0; k < R / 16; ++k)
                    tc_mma_terms<NT>(tmem + (uint32_t)(N + h * MB), umma_desc(a0 + h * 16 * SBO + k * 256, 128, SBO),
                                     umma_desc(b0 + k * 256, 128, SBO), R * N * 2, MB * R * 2,
                                     umma_idesc_bf16(128, MB), k > 0);
                if (h == 1) tc_commit(&s_mbar3);
            }
            if (!tc_commit_wait2(&s_mbar, parity, &s_mbar2, parity2, pend2, &s_ok, cp.inj_mma != 0, &s_mbar3,
                                 &parity3)) {
                failed = true;   // (the wait also covers the previous chunk's dA and dB)
                break;
            }
            pend2 = false;
            tc_fence_after();
            if (pmb >= 0) read_dA(pmb, pcnt);
            for (int q = tid; q < MB * N / 4; q += BT)   // the previous chunk's dC tile is no longer read
                reinterpret_cast<float4*>(dCn)[q] = make_float4(0.f, 0.f, 0.f, 0.f);
            tc_fence_before();
            __syncthreads();
            TT_PH(10);

            // next chunk's metadata and A rows go in flight while this chunk's rows are processed
            if (more) {
                // its group records: copied by the warp-0 threads that read them in bwd2_meta, so
                // each thread's own wait suffices
                cp_async_wait_all();
                bwd2_meta<K>(M.rec[mb ^ 1], j0 + MPB, ccount, mb ^ 1, uniq_keys, M, s_keys);
                bwd2_issue_a<NS>(cp, t, mb ^ 1, M, Abt + (mb ^ 1) * NS * MB * R);
            }
            TT_PH(16);

            bwd2_rows<K>(cp, t, mb, total, cnt, M, uniq_keys, rowbuf, tmem + (uint32_t)N, dCn, dG3, n3, hslots);
            tc_fence_before();
            __syncthreads();
            TT_PH(12);

            // dC -> NS bf16 terms in core matrices (MB rows, K = N), written over dCn once
            {
                constexpr int CPT = MB * N / 8 / BT;   // 16-byte chunks per thread
                static_assert(CPT * BT * 8 == MB * N, "dC conversion tiling");
                float v[CPT][8];
#pragma unroll
                for (int i = 0; i < CPT; ++i) {
                    const int q = tid + i * BT;
                    const int m = (q / (8 * (N / 8))) * 8 + (q & 7), nc = (q >> 3) % (N / 8);
                    const float4 x0 = *reinterpret_cast<const float4*>(&dCn[swz_m<N>(m, nc * 8)]);
                    const float4 x1 = *reinterpret_cast<const float4*>(&dCn[swz_m<N>(m, nc * 8 + 4)]);
                    v[i][0] = x0.x; v[i][1] = x0.y; v[i][2] = x0.z; v[i][3] = x0.w;
                    v[i][4] = x1.x; v[i][5] = x1.y; v[i][6] = x1.z; v[i][7] = x1.w;
                }
                __syncthreads();
                TT_PH(18);
#pragma unroll
                for (int i = 0; i < CPT; ++i) {
                    const int q = tid + i * BT;
                    const int m = (q / (8 * (N / 8))) * 8 + (q & 7), nc = (q >> 3) % (N / 8);
                    uint16_t* dst = dCb + ((m >> 3) * (N / 8) + nc) * 64 + (m & 7) * 8;
                    uint4 hi, lo;
                    split_bf16x8(v[i], hi, lo);
                    *reinterpret_cast<uint4*>(dst) = hi;
                    if constexpr (NS == 2) *reinterpret_cast<uint4*>(dst + MB * N) = lo;
                }
            }
            fence_async_smem();
            __syncthreads();
            TT_PH(19);
            // lane 0 of warps 0 .. DAQ - 1 issues dA accumulator q = warp, lane 0 of warp DAQ issues
            // dB; each commits its products to s_mbar2 (count DAQ + 1)
            static_assert(DAQ == 2, "three issuing threads");
            if ((tid & 31) == 0 && (tid >> 5) <= DAQ) {
                tc_fence_after();
                const int q = tid >> 5;
                const uint32_t c0 = smem_u32(dCb), b0 = smem_u32(Bb), a0 = smem_u32(Ab16);
                if (q < DAQ) {
                    // dA = dC . B^T: A = dC (K-major), B = the B tile viewed MN-major; accumulator q
                    // takes the K range [q N / DAQ, (q + 1) N / DAQ)
#pragma unroll 1
                    for (int kk = 0; kk < N / 16 / DAQ; ++kk) {
                        const int k = q * (N / 16 / DAQ) + kk;
                        tc_mma_terms<NT>(tmem + (uint32_t)(TDA + q * R), umma_desc(c0 + k * 256, 128, (N / 8) * 128),
                                         umma_desc_mn(b0 + k * 2 * (R / 8) * 128, 128, (R / 8) * 128),
                                         MB * N * 2, R * N * 2, umma_idesc_bf16(MB, R, false, true), kk > 0);
                    }
                } else {
                    // dB += A^T . dC: A = the A tile viewed MN-major, B = dC viewed MN-major
#pragma unroll
                    for (int k = 0; k < MB / 16; ++k)
                        tc_mma_terms<NT>(tmem, umma_desc_mn(a0 + k * 2 * (R / 8) * 128, 128, (R / 8) * 128),
                                         umma_desc_mn(c0 + k * 2 * (N / 8) * 128, 128, (N / 8) * 128),
                                         MB * R * 2, MB * N * 2, umma_idesc_bf16(R, N, true, true),
                                         j0 > 0 || k > 0);
                }
                tc_commit(&s_mbar2);
            }
            pend2 = true;
            pmb = mb;
            pcnt = cnt;
            TT_PH(13);
        }
        if (failed) break;
        if (!tc_commit_wait2(&s_mbar, parity, &s_mbar2, parity2, pend2, &s_ok)) {   // the column's last dA and dB
            failed = true;
            break;
        }
        pend2 = false;
        tc_fence_after();
        read_dA(pmb, pcnt);
        TT_PH(14);
        {
            // dG_2[:, i_2] = dB from tensor memory: rows rho_1 = 16 sub + lane (lane < 16)
            tc_fence_after();
            const int warp = tid >> 5, lane = tid & 31, sub = warp & 3, cblk = warp >> 2;
            const int rho1 = 16 * sub + lane;
#pragma unroll 1
            for (int g = 0; g < N / CB / 32; ++g) {
                const int c0 = cblk * (N / CB) + g * 32;
                float v[32];
                tmem_ld32(tmem + ((uint32_t)(32 * sub) << 16) + (uint32_t)c0, v);
                if (lane < 16) {
                    if (gp.fused) {   // sparse fused SGD: G_2[:, i_2] -= lr dB
                        float* g2 = gp.upd1[t] + ((int64_t)rho1 * n2 + i2) * N + c0;
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const float4 x = *reinterpret_cast<const float4*>(g2 + 4 * j);
                            *reinterpret_cast<float4*>(g2 + 4 * j) =
                                make_float4(x.x - gp.lr * v[4 * j], x.y - gp.lr * v[4 * j + 1],
                                            x.z - gp.lr * v[4 * j + 2], x.w - gp.lr * v[4 * j + 3]);
                        }
                    } else {
                        float* dst = dG2 + ((int64_t)rho1 * n2 + i2) * N + c0;
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            *reinterpret_cast<float4*>(dst + 4 * j) =
                                make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                    }
                }
            }
            tc_fence_before();
        }
        __syncthreads();
        TT_PH(15);
    }
    cp_async_wait_all();
    if (failed && tid == 0) raise_error(status, TT_ERR_TIMEOUT, 103);
    tc_fence_before();
    __syncthreads();
    if (tid < 32) {
        tc_fence_after();
        tmem_dealloc(tmem, 2 * N);
    }
    probe_write(cp, pr_t0, pr_tasks, 0ull);
}

// ---------------------------------------------------------------------------
// last core [R][n3][D3] -> [n3][R][D3]; one thread per (table, i3, rho) row of D3 floats
// ---------------------------------------------------------------------------
// bf16 operand copies for the tensor-core forward.  Items are 16-byte output chunks:
// first every table's G_1 (a plain [n_1][d_1][r_1] copy), then every table's G_2 tiles,
// one per i_2, in the operand order of fwd_issue_ab_tc: element (n, k) of the tile
// (n = a_2 r_2 + rho_2, k = rho_1) at ((n / 8) (R / 8) + k / 8) 64 + (n % 8) 8 + k % 8.
struct Bf16Job {
    int32_t T, R, N, NS;   // NS = 2: every value as two bf16 terms (hi, lo), stored as two tiles / row halves
    int64_t base1[kMaxT + 1], base2[kMaxT + 1];   // prefix sums of chunk counts
    uint32_t n2[kMaxT];
    const float* src1[kMaxT];
    const float* src2[kMaxT];
    uint16_t* dst1[kMaxT];
    uint16_t* dst2[kMaxT];
};

__device__ __forceinline__ int table_of(const int64_t* base, int T, int64_t q)
{
    int lo = 0, hi = T - 1;   // last t with base[t] <= q
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (base[mid] <= q) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

__global__ void __launch_bounds__(256) k3_bf16_kernel(Bf16Job j)
{
    const int64_t tot1 = j.base1[j.T], tot2 = j.base2[j.T];
    const int KC = j.R / 8;
    const int64_t per_tile = (int64_t)j.R * j.N / 8;
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < tot1 + tot2;
         q += (int64_t)gridDim.x * blockDim.x) {
        float v[8];
        uint4 hi, lo;
        if (q < tot1) {
            const int t = table_of(j.base1, j.T, q);
            const int64_t off = (q - j.base1[t]) * 8;
            const float4 x0 = __ldg(reinterpret_cast<const float4*>(j.src1[t] + off));
            const float4 x1 = __ldg(reinterpret_cast<const float4*>(j.src1[t] + off + 4));
            v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w;
            v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
            // row (i_1, a_1) of R values -> NS halves of R bf16 values
            const int64_t row = off / j.R, e = off % j.R;
            uint16_t* dst = j.dst1[t] + row * (j.NS * j.R) + e;
            split_bf16x8(v, hi, lo);
            *reinterpret_cast<uint4*>(dst) = hi;
            if (j.NS == 2) *reinterpret_cast<uint4*>(dst + j.R) = lo;
        } else {
            const int64_t q2 = q - tot1;
            const int t = table_of(j.base2, j.T, q2);
            const int64_t r = q2 - j.base2[t];
            const int64_t i2 = r / per_tile;
            const int c = (int)(r % per_tile);          // chunk ((n / 8) KC + kc) 8 + n % 8
            const int n = (c / (8 * KC)) * 8 + (c % 8), kc = (c / 8) % KC;
            const int64_t rs = (int64_t)j.n2[t] * j.N;  // stride between rho_1 rows of G_2
            const float* src = j.src2[t] + i2 * j.N + n + (int64_t)kc * 8 * rs;
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = __ldg(src + e * rs);
            uint16_t* dst = j.dst2[t] + i2 * ((int64_t)j.NS * j.R * j.N) + (int64_t)c * 8;
            split_bf16x8(v, hi, lo);
            *reinterpret_cast<uint4*>(dst) = hi;
            if (j.NS == 2) *reinterpret_cast<uint4*>(dst + (int64_t)j.R * j.N) = lo;
        }
    }
}

struct TransposeJob {
    int32_t T, R, D3, back;   // back: src [n3][R][D3] -> dst [R][n3][D3]
    int64_t row_base[kMaxT + 1];   // prefix sums of n3 * R
    uint32_t n3[kMaxT];
    const float* src[kMaxT];
    float* dst[kMaxT];
};

__global__ void __launch_bounds__(256) k3_transpose_last_kernel(TransposeJob tj, const int32_t* status)
{
    if (status && has_error(status)) return;
    const int64_t total = tj.row_base[tj.T];
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < total;
         q += (int64_t)gridDim.x * blockDim.x) {
        int t = 0;
        while (t + 1 < tj.T && tj.row_base[t + 1] <= q) ++t;
        const int64_t rq = q - tj.row_base[t];
        const int64_t i3 = rq / tj.R, rho = rq % tj.R;
        const int64_t core = (rho * tj.n3[t] + i3) * tj.D3, trans = (i3 * tj.R + rho) * tj.D3;
        const float4* src = reinterpret_cast<const float4*>(tj.src[t] + (tj.back ? trans : core));
        float4* dst = reinterpret_cast<float4*>(tj.dst[t] + (tj.back ? core : trans));
        for (int c = 0; c < tj.D3 / 4; ++c) dst[c] = __ldg(src + c);
    }
}

// ---------------------------------------------------------------------------
// host launchers
// ---------------------------------------------------------------------------
// NT: 0 = FP32 pipes, 1 = bf16 tensor-core products, 3 = fp32-accurate split-bf16 products
template <class S, int NT>
constexpr size_t fwd_smem_bytes()
{
    return sizeof(float) * (NT == 0 ? S::fwd_smem_floats() : S::fwd_smem_floats_tc(NT == 3 ? 2 : 1));
}
template <class S>
constexpr size_t bwd_smem_bytes()
{
    return sizeof(float) * S::bwd_smem_floats();
}

template <class S, typename K, int NT>
cudaError_t fwd_launch(const K3Args& a, float* out, cudaStream_t s, int* nl)
{
    const size_t smem = fwd_smem_bytes<S, NT>();
    cudaError_t e = cudaFuncSetAttribute(k3_fwd_kernel<S, K, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const PlanBuffers& pb = *a.pb;
    if (a.grid != a.pp->grid || a.grid > kMaxGrid) return cudaErrorInvalidConfiguration;
    const FwdSched fs{pb.subs, pb.deque, pb.exhausted, pb.slot_flag, pb.ckpt};
    k3_fwd_kernel<S, K, NT><<<a.grid, kFwdThreads, smem, s>>>(
        *a.cp, a.pp->sched, (const K*)a.uniq_keys, a.grec, a.uid_at_pos, a.offsets,
        pb.chunks, fs, pb.hdr, a.rowbuf, out, a.status);
    *nl += 1;
    return cudaGetLastError();
}

template <int D>
cudaError_t rowsum_launch(const K3Args& a, const float* grad_out, cudaStream_t s, int* nl)
{
    const int64_t L = a.L;
    const int64_t nwarps = ceil_div(L, kHChunk);
    k3_hzero<D><<<148, 256, 0, s>>>(a.uid_sorted, L, a.rowbuf, a.status);
    k3_hsum<D><<<(unsigned)ceil_div(nwarps * 32, 256), 256, 0, s>>>(
        a.uid_sorted, a.bag_sorted, grad_out, L, a.cp->B, (float)(1.0 / (double)a.cp->B), a.cp->T,
        a.rowbuf, a.status);
    *nl += 2;
    return cudaGetLastError();
}

template <class S, typename K>
cudaError_t bwd_launch(const K3Args& a, const GradPtrs& gp, const float* grad_out, cudaStream_t s, int* nl)
{
    (void)grad_out;
    const size_t smem = bwd_smem_bytes<S>();
    cudaError_t e = cudaFuncSetAttribute(k3_bwd_kernel<S, K>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const PlanBuffers& pb = *a.pb;
    k3_bwd_kernel<S, K><<<a.grid, kBwdThreads, smem, s>>>(
        *a.cp, gp, *a.pp, (const K*)a.uniq_keys, a.grec, pb.col_count, pb.col_start, pb.col_order, pb.hdr,
        a.rowbuf, a.status);
    *nl += 1;
    return cudaGetLastError();
}

template <class S>
cudaError_t fwd_dispatch(const K3Args& a, float* out, cudaStream_t s, int* nl)
{
    return a.key64 ? fwd_launch<S, uint64_t, 0>(a, out, s, nl) : fwd_launch<S, uint32_t, 0>(a, out, s, nl);
}
template <class S>
cudaError_t fwd_dispatch_tc(const K3Args& a, float* out, cudaStream_t s, int* nl)
{
    if (a.tc == 3)
        return a.key64 ? fwd_launch<S, uint64_t, 3>(a, out, s, nl) : fwd_launch<S, uint32_t, 3>(a, out, s, nl);
    return a.key64 ? fwd_launch<S, uint64_t, 1>(a, out, s, nl) : fwd_launch<S, uint32_t, 1>(a, out, s, nl);
}
template <class S>
cudaError_t bwd_dispatch(const K3Args& a, const GradPtrs& gp, const float* g, cudaStream_t s, int* nl)
{
    return a.key64 ? bwd_launch<S, uint64_t>(a, gp, g, s, nl) : bwd_launch<S, uint32_t>(a, gp, g, s, nl);
}
// shared memory of the transposed-product backward: B tile, two A tiles, dC, per-warp H slots
template <int NT>
constexpr size_t bwd2_smem_bytes()
{
    constexpr size_t NS = NT == 3 ? 2 : 1;
    return NS * 64 * 256 * 2 + 2 * NS * kMB2 * 64 * 2 + (size_t)kMB2 * 256 * 4 + (kBwdThreadsTC / 32) * 2 * 128 * 4;
}

template <typename K, int NT>
cudaError_t bwd2_launch(const K3Args& a, const GradPtrs& gp, cudaStream_t s, int* nl)
{
    const size_t smem = bwd2_smem_bytes<NT>();
    cudaError_t e = cudaFuncSetAttribute(k3_bwd_tc2_kernel<K, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const PlanBuffers& pb = *a.pb;
    k3_bwd_tc2_kernel<K, NT><<<a.grid, kBwdThreadsTC, smem, s>>>(
        *a.cp, gp, *a.pp, (const K*)a.uniq_keys, a.grec, pb.col_count, pb.col_start, pb.col_order, pb.hdr,
        a.rowbuf, a.status);
    *nl += 1;
    return cudaGetLastError();
}

// tensor-core backward (rank 64, d = (4, 4, 8)): the transposed-product kernel
cudaError_t bwd_dispatch_tc(const K3Args& a, const GradPtrs& gp, cudaStream_t s, int* nl)
{
    if (a.tc == 3) return a.key64 ? bwd2_launch<uint64_t, 3>(a, gp, s, nl) : bwd2_launch<uint32_t, 3>(a, gp, s, nl);
    return a.key64 ? bwd2_launch<uint64_t, 1>(a, gp, s, nl) : bwd2_launch<uint32_t, 1>(a, gp, s, nl);
}

template <class S, int NT>
int occ_fwd()
{
    const size_t smem = fwd_smem_bytes<S, NT>();
    cudaFuncSetAttribute(k3_fwd_kernel<S, uint32_t, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k3_fwd_kernel<S, uint32_t, NT>, kFwdThreads, smem) != cudaSuccess)
        return 1;
    return n > 0 ? n : 1;
}
template <class S>
int occ_bwd()
{
    const size_t smem = sizeof(float) * S::bwd_smem_floats();
    cudaFuncSetAttribute(k3_bwd_kernel<S, uint32_t>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k3_bwd_kernel<S, uint32_t>, kBwdThreads, smem) !=
        cudaSuccess)
        return 1;
    return n > 0 ? n : 1;
}

}  // namespace

int k3_blocks_per_sm(const CoreParams& cp, bool backward, bool tc)
{
    if (tc) return 1;   // tensor-core variants hold tensor memory: one block per SM
#define TT_OCC_CASE(Q1, Q2, Q3, QR) \
    if (cp.d[0] == Q1 && cp.d[2] == Q3 && cp.r[1] == QR) return backward ? occ_bwd<S3<Q1, Q2, Q3, QR>>() : occ_fwd<S3<Q1, Q2, Q3, QR>, 0>();
    TT_K3_CASES_INNER(TT_OCC_CASE)
#undef TT_OCC_CASE
    return 1;
}

bool k3_tc_supported(const CoreParams& cp)
{
    return k3_supported(cp) && cp.d[0] == 4 && cp.d[1] == 4 && cp.d[2] == 8 && (cp.r[1] == 64 || cp.r[1] == 32);
}

bool k3_tc_bwd_supported(const CoreParams& cp)
{
    return k3_tc_supported(cp) && cp.r[1] == 64;
}

bool k3_supported(const CoreParams& cp)
{
    if (cp.k != 3 || cp.d[1] != 4 || cp.r[1] != cp.r[2] || cp.d[0] * cp.d[1] * cp.d[2] > 128) return false;
#define TT_SUP_CASE(Q1, Q2, Q3, QR) \
    if (cp.d[0] == Q1 && cp.d[2] == Q3 && cp.r[1] == QR) return true;
    TT_K3_CASES_INNER(TT_SUP_CASE)
#undef TT_SUP_CASE
    return false;
}

int k3_plan_mp(const CoreParams& cp)
{
    const int N = cp.d[1] * cp.r[1];
    return (16384 / N) / cp.d[0];
}

#define TT_K3_CASES(X) TT_K3_CASES_INNER(X)

cudaError_t k3_forward(const K3Args& a, float* out, cudaStream_t s, int* nl)
{
    const CoreParams& cp = *a.cp;
    if (a.tc) {
        if (cp.d[0] == 4 && cp.d[2] == 8 && cp.r[1] == 64) return fwd_dispatch_tc<S3<4, 4, 8, 64>>(a, out, s, nl);
        if (cp.d[0] == 4 && cp.d[2] == 8 && cp.r[1] == 32) return fwd_dispatch_tc<S3<4, 4, 8, 32>>(a, out, s, nl);
        return cudaErrorInvalidValue;
    }
#define TT_FWD_CASE(Q1, Q2, Q3, QR) \
    if (cp.d[0] == Q1 && cp.d[2] == Q3 && cp.r[1] == QR) return fwd_dispatch<S3<Q1, Q2, Q3, QR>>(a, out, s, nl);
    TT_K3_CASES(TT_FWD_CASE)
#undef TT_FWD_CASE
    return cudaErrorInvalidValue;
}

static cudaError_t transpose_last(const CoreParams& cp, const float* const* src, float* const* dst, bool back,
                                  cudaStream_t s, int* nl)
{
    TransposeJob tj;
    memset(&tj, 0, sizeof(tj));
    tj.T = cp.T;
    tj.R = cp.r[2];
    tj.D3 = cp.d[2];
    tj.back = back ? 1 : 0;
    int64_t b = 0;
    for (int t = 0; t < cp.T; ++t) {
        tj.row_base[t] = b;
        b += (int64_t)cp.n[t][2] * tj.R;
        tj.n3[t] = cp.n[t][2];
        tj.src[t] = src[t];
        tj.dst[t] = dst[t];
    }
    tj.row_base[cp.T] = b;
    if (b == 0) return cudaSuccess;
    const int grid = (int)min64(ceil_div(b, 256), 148 * 16);
    k3_transpose_last_kernel<<<grid, 256, 0, s>>>(tj, nullptr);
    *nl += 1;
    return cudaGetLastError();
}

cudaError_t k3_transpose_last(const CoreParams& cp, float* const* dst, cudaStream_t s, int* nl)
{
    const float* src[kMaxT];
    for (int t = 0; t < cp.T; ++t) src[t] = cp.cores[t][2];
    return transpose_last(cp, src, dst, false, s, nl);
}

cudaError_t k3_transpose_last_back(const CoreParams& cp, const float* const* src, float* const* dst, cudaStream_t s,
                                   int* nl)
{
    return transpose_last(cp, src, dst, true, s, nl);
}

cudaError_t k3_to_bf16(const CoreParams& cp, int terms, uint16_t* const* dst1, uint16_t* const* dst2,
                      cudaStream_t s, int* nl)
{
    Bf16Job j;
    memset(&j, 0, sizeof(j));
    j.T = cp.T;
    j.NS = terms;
    j.R = cp.r[1];
    j.N = cp.d[1] * cp.r[2];
    int64_t b1 = 0, b2 = 0;
    for (int t = 0; t < cp.T; ++t) {
        j.base1[t] = b1;
        j.base2[t] = b2;
        b1 += (int64_t)cp.n[t][0] * cp.d[0] * cp.r[1] / 8;
        b2 += (int64_t)cp.n[t][1] * j.R * j.N / 8;
        j.n2[t] = cp.n[t][1];
        j.src1[t] = cp.cores[t][0];
        j.src2[t] = cp.cores[t][1];
        j.dst1[t] = dst1[t];
        j.dst2[t] = dst2[t];
    }
    j.base1[cp.T] = b1;
    j.base2[cp.T] = b2;
    if (b1 + b2 == 0) return cudaSuccess;
    const int grid = (int)min64(ceil_div(b1 + b2, 256), 148 * 16);
    k3_bf16_kernel<<<grid, 256, 0, s>>>(j);
    *nl += 1;
    return cudaGetLastError();
}

cudaError_t k3_rowsum(const K3Args& a, const float* grad_out, cudaStream_t s, int* nl)
{
    const int D = a.cp->D;
    if (D == 128) return rowsum_launch<128>(a, grad_out, s, nl);
    if (D == 64) return rowsum_launch<64>(a, grad_out, s, nl);
    return cudaErrorInvalidValue;
}

cudaError_t k3_backward(const K3Args& a, const GradPtrs& gp, const float* grad_out, cudaStream_t s, int* nl)
{
    const CoreParams& cp = *a.cp;
    if (a.tc) {
        if (k3_tc_bwd_supported(cp)) return bwd_dispatch_tc(a, gp, s, nl);
        return cudaErrorInvalidValue;
    }
#define TT_BWD_CASE(Q1, Q2, Q3, QR) \
    if (cp.d[0] == Q1 && cp.d[2] == Q3 && cp.r[1] == QR) return bwd_dispatch<S3<Q1, Q2, Q3, QR>>(a, gp, grad_out, s, nl);
    TT_K3_CASES(TT_BWD_CASE)
#undef TT_BWD_CASE
    return cudaErrorInvalidValue;
}

}  // namespace tt

#ifdef TT_PROFILE_PHASES
extern "C" int tt_emb_debug_phase_cycles(unsigned long long* out, int n)
{
    if (!out || n < 1 || n > 32) return TT_ERR_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return TT_ERR_CUDA;
    if (cudaMemcpyFromSymbol(out, g_tt_phase_cycles, sizeof(unsigned long long) * n) != cudaSuccess) return TT_ERR_CUDA;
    unsigned long long zero[32] = {};
    if (cudaMemcpyToSymbol(g_tt_phase_cycles, zero, sizeof(zero)) != cudaSuccess) return TT_ERR_CUDA;
    return TT_OK;
}
#endif
