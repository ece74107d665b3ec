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
#include "tt_common.cuh"

#define TT_K3_CASES_INNER(X) \
    X(4, 4, 8, 64)           \
    X(4, 4, 8, 32)           \
    X(4, 4, 8, 16)           \
    X(4, 4, 4, 32)           \
    X(4, 4, 4, 16)

namespace tt {
namespace {

constexpr int kThreads = 256;
constexpr int kNB = kPoolBags;    // bags per pooling task
constexpr int kHChunk = 256;      // sorted lookups per upstream-sum warp
constexpr int kSpinLimit = 1 << 22;

template <int D1_, int D2_, int D3_, int R_>
struct S3 {
    static constexpr int D1 = D1_, D2 = D2_, D3 = D3_, R = R_;
    static constexpr int N = D2 * R;          // columns of B and of C_all
    static constexpr int P = D1 * D2;         // rows of C_p
    static constexpr int D = P * D3;          // embedding width
    // forward: GEMM of MF x N per chunk, 8x8 outputs per thread
    static constexpr int MF = 16384 / N;
    static constexpr int MPF = MF / D1;       // prefixes per forward chunk
    static constexpr int TPU = D1 * (D3 / 4); // threads per distinct row in the suffix step
    static constexpr int NUF = kThreads / TPU;
    static constexpr int SU = R * D3 + 4;     // padded stride of one staged last slice
    // backward: MB x N per chunk
    static constexpr int MB = 2048 / R;
    static constexpr int MPB = MB / D1;
    static constexpr int NUB = 16;            // distinct rows per backward batch
    static constexpr int DBR = (R * N) / (kThreads * 4) >= 16 ? 8 : ((R * N) / (kThreads * 4) >= 4 ? 4 : 1);
    static constexpr int DBC = (R * N) / (kThreads * DBR);   // dB columns per thread
    static_assert(D2 == 4, "specialised path needs d_2 = 4");
    static_assert(D1 == 4, "specialised path needs d_1 = 4");
    static_assert(D3 % 4 == 0, "d_3 must be a multiple of 4");
    static_assert(N >= 32 && N % 32 == 0, "swizzle needs N >= 32");
    static_assert(MF % 8 == 0 && (MF / 8) * (N / 8) == kThreads, "forward GEMM tiling");
    static_assert(DBC % 4 == 0, "dB columns in float4 chunks");

    static constexpr size_t fwd_smem_floats()
    {
        return (size_t)R * N + (size_t)R * MF + (size_t)MF * N + (size_t)NUF * SU;
    }
    static constexpr size_t bwd_smem_floats()
    {
        return (size_t)R * N + 2 * (size_t)MB * R + 2 * (size_t)MB * N + 2 * (size_t)NUB * P * D3 +
               (size_t)NUB * (D3 * R + 4);
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
// forward
// ---------------------------------------------------------------------------
template <class S, typename K>
__device__ void fwd_chunk(const CoreParams& cp, int task, const K* __restrict__ uniq_keys,
                          const int32_t* __restrict__ grp_start, const int32_t* __restrict__ sorted_groups,
                          const int4* __restrict__ chunks, PlanHeader* hdr, float* __restrict__ rowbuf,
                          float* sm, int* si)
{
    constexpr int R = S::R, N = S::N, MF = S::MF, MPF = S::MPF, D1 = S::D1, D2 = S::D2, D3 = S::D3;
    float* Bs = sm;
    float* AsT = Bs + R * N;
    float* Cn = AsT + R * MF;
    float* Ss = Cn + MF * N;
    int* s_u0 = si;
    int* s_ucum = s_u0 + MPF;
    int* s_i1 = s_ucum + MPF + 1;
    int* s_bu = s_i1 + MPF;
    int* s_bp = s_bu + S::NUF;
    int* s_bi3 = s_bp + S::NUF;
    int* s_cur = s_bi3 + S::NUF;   // [0] table, [1] column digit of the staged B, [2] scratch
    const int tid = threadIdx.x;

    const int4 ch = chunks[task];
    const int start = ch.x, cnt = ch.y, t = ch.z, i2 = ch.w;
    const uint32_t n2 = cp.n[t][1], n3 = cp.n[t][2];
    const float* __restrict__ G1 = cp.cores[t][0];
    const float* __restrict__ G2 = cp.cores[t][1];
    const float* __restrict__ G3 = cp.cores[t][2];

    if (tid < MPF) {
        int u0 = 0, nu = 0, i1 = 0;
        if (tid < cnt) {
            const int g = sorted_groups[start + tid];
            u0 = grp_start[g];
            nu = grp_start[g + 1] - u0;
            i1 = (int)(key_row(uniq_keys[u0], cp.ibits) / n3 / n2);
        }
        s_u0[tid] = u0;
        s_ucum[tid] = nu;
        s_i1[tid] = i1;
    }
    const bool need_b = !(s_cur[0] == t && s_cur[1] == i2);
    __syncthreads();
    if (tid == 0) {
        int run = 0;
        for (int j = 0; j < MPF; ++j) {
            const int v = s_ucum[j];
            s_ucum[j] = run;
            run += v;
        }
        s_ucum[MPF] = run;
        s_cur[0] = t;
        s_cur[1] = i2;
    }
    // stage B = G_2[:, i_2] (rows of N floats at stride n_2 * N), swizzled
    if (need_b) {
        for (int q = tid; q < R * N / 4; q += kThreads) {
            const int rho = q / (N / 4), c4 = q % (N / 4);
            const float4 v = __ldg(reinterpret_cast<const float4*>(G2 + ((int64_t)rho * n2 + i2) * N) + c4);
            *reinterpret_cast<float4*>(&Bs[swz_b<N>(rho, c4 * 4)]) = v;
        }
    }
    // stage A^T: AsT[rho][m], m = j * D1 + a1, A_j = G_1[0, i1_j] (D1 x R)
    for (int q = tid; q < R * MF; q += kThreads) {
        const int rho = q / MF, m = q % MF;
        const int j = m / D1, a1 = m % D1;
        float v = 0.f;
        if (j < cnt) v = __ldg(G1 + ((int64_t)s_i1[j] * D1 + a1) * R + rho);
        AsT[rho * MF + m] = v;
    }
    __syncthreads();

    // C_all[m][n] = sum_rho A[m][rho] B[rho][n]; thread: rows {4tm+i, MF/2+4tm+i}, cols {4tn+j, N/2+4tn+j}
    {
        constexpr int TN = N / 8;
        const int tn = tid % TN, tm = tid / TN;
        float acc[8][8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
#pragma unroll 2
        for (int rho = 0; rho < R; ++rho) {
            const float4 a0 = *reinterpret_cast<const float4*>(&AsT[rho * MF + tm * 4]);
            const float4 a1 = *reinterpret_cast<const float4*>(&AsT[rho * MF + MF / 2 + tm * 4]);
            const float4 b0 = *reinterpret_cast<const float4*>(&Bs[swz_b<N>(rho, tn * 4)]);
            const float4 b1 = *reinterpret_cast<const float4*>(&Bs[swz_b<N>(rho, N / 2 + tn * 4)]);
            const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int m = (i < 4) ? tm * 4 + i : MF / 2 + tm * 4 + (i - 4);
            *reinterpret_cast<float4*>(&Cn[swz_m<N>(m, tn * 4)]) =
                make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
            *reinterpret_cast<float4*>(&Cn[swz_m<N>(m, N / 2 + tn * 4)]) =
                make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
        }
    }
    __syncthreads();

    // suffix step: E_u = C_p (P x R) . S_u (R x D3), for the chunk's distinct rows
    const int total = s_ucum[MPF];
    const uint64_t rmask = (uint64_t(1) << cp.ibits) - 1;
    for (int k0 = 0; k0 < total; k0 += S::NUF) {
        const int nb = min(S::NUF, total - k0);
        if (tid < nb) {
            const int kq = k0 + tid;
            int j = 0;
            while (j + 1 < cnt && s_ucum[j + 1] <= kq) ++j;
            const int u = s_u0[j] + (kq - s_ucum[j]);
            s_bu[tid] = u;
            s_bp[tid] = j;
            s_bi3[tid] = (int)((uint32_t)((uint64_t)uniq_keys[u] & rmask) % n3);
        }
        __syncthreads();
        for (int q = tid; q < nb * R * (D3 / 4); q += kThreads) {
            const int uu = q / (R * (D3 / 4)), rem = q % (R * (D3 / 4));
            const int rho = rem / (D3 / 4), c4 = rem % (D3 / 4);
            const float4 v = __ldg(reinterpret_cast<const float4*>(
                G3 + ((int64_t)rho * n3 + s_bi3[uu]) * D3) + c4);
            *reinterpret_cast<float4*>(&Ss[uu * S::SU + rho * D3 + c4 * 4]) = v;
        }
        __syncthreads();
        {
            const int uu = tid / S::TPU;
            const int a1 = (tid % S::TPU) / (D3 / 4), cg = tid % (D3 / 4);
            if (uu < nb) {
                const int p = s_bp[uu];
                const int m = p * D1 + a1;
                const float* srow = &Ss[uu * S::SU + cg * 4];
                float4 e[4];
#pragma unroll
                for (int a2 = 0; a2 < 4; ++a2) e[a2] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
                for (int rho = 0; rho < R; rho += 4) {
                    float4 c[4];
#pragma unroll
                    for (int a2 = 0; a2 < 4; ++a2)
                        c[a2] = *reinterpret_cast<const float4*>(&Cn[swz_m<N>(m, a2 * R + rho)]);
                    float4 s[4];
#pragma unroll
                    for (int r = 0; r < 4; ++r) s[r] = *reinterpret_cast<const float4*>(srow + (rho + r) * D3);
#pragma unroll
                    for (int a2 = 0; a2 < 4; ++a2) {
                        const float cv[4] = {c[a2].x, c[a2].y, c[a2].z, c[a2].w};
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            e[a2].x = fmaf(cv[r], s[r].x, e[a2].x);
                            e[a2].y = fmaf(cv[r], s[r].y, e[a2].y);
                            e[a2].z = fmaf(cv[r], s[r].z, e[a2].z);
                            e[a2].w = fmaf(cv[r], s[r].w, e[a2].w);
                        }
                    }
                }
                float* dst = rowbuf + (int64_t)s_bu[uu] * S::D + cg * 4;
#pragma unroll
                for (int a2 = 0; a2 < 4; ++a2)
                    *reinterpret_cast<float4*>(dst + (a1 * D2 + a2) * D3) = e[a2];
            }
        }
        __syncthreads();
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) atomicAdd(&hdr->done[t], 1);
}

template <class S>
__device__ void fwd_pool(const CoreParams& cp, int ptask, int nP, const int32_t* __restrict__ uid_at_pos,
                         const int64_t* __restrict__ offsets, PlanHeader* hdr,
                         const float* __restrict__ rowbuf, float* __restrict__ out, int32_t* status,
                         int* s_flag)
{
    constexpr int D = S::D, LB = D / 4, BPW = 32 / LB;
    const int t = ptask / nP, jb = ptask % nP;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    if (tid == 0) {
        const int want = hdr->nC[t];
        int it = 0, ok = 1;
        while (*reinterpret_cast<volatile int*>(&hdr->done[t]) < want) {
            if (++it > kSpinLimit) {
                raise_error(status, TT_ERR_TIMEOUT, t);
                ok = 0;
                break;
            }
            __nanosleep(256);
        }
        __threadfence();
        s_flag[0] = ok;
    }
    __syncthreads();
    if (!s_flag[0]) return;
    const int64_t B = cp.B, TD = (int64_t)cp.T * D;
    const int sub = lane / LB, col = (lane % LB) * 4;
    const int b_lo = jb * kNB, b_hi = (int)min64((int64_t)b_lo + kNB, B);
    for (int b = b_lo + wid * BPW + sub; b < b_hi; b += (kThreads / 32) * BPW) {
        const int64_t g = (int64_t)t * B + b;
        const int64_t l0 = offsets[g], l1 = offsets[g + 1];
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int64_t l = l0; l < l1; ++l) {
            const int u = uid_at_pos[l];
            acc = f4add(acc, __ldcg(reinterpret_cast<const float4*>(rowbuf + (int64_t)u * D + col)));
        }
        *reinterpret_cast<float4*>(out + (int64_t)b * TD + (int64_t)t * D + col) = acc;
    }
}

template <class S, typename K>
__global__ void __launch_bounds__(kThreads, 1)
k3_fwd_kernel(CoreParams cp, int sched, const K* __restrict__ uniq_keys,
              const int32_t* __restrict__ grp_start, const int32_t* __restrict__ uid_at_pos,
              const int64_t* __restrict__ offsets, const int32_t* __restrict__ sorted_groups,
              const int4* __restrict__ chunks, const int32_t* __restrict__ tasks, PlanHeader* hdr,
              float* __restrict__ rowbuf, float* __restrict__ out, int32_t* status)
{
    extern __shared__ __align__(16) float sm[];
    int* si = reinterpret_cast<int*>(sm + S::fwd_smem_floats());
    __shared__ int s_task[2];
    if (has_error(status)) return;
    int* s_cur = si + S::MPF * 3 + 1 + S::NUF * 3;
    if (threadIdx.x == 0) {
        s_cur[0] = -1;
        s_cur[1] = -1;
    }
    const int ntasks = hdr->ntasks, nP = hdr->nP;
    __syncthreads();
    for (int iter = 0;; ++iter) {
        if (threadIdx.x == 0) s_task[0] = next_task(sched, &hdr->queue_head, iter);
        __syncthreads();
        const int q = s_task[0];
        if (q >= ntasks) break;
        const int task = tasks[q];
        if (task >= 0)
            fwd_chunk<S, K>(cp, task, uniq_keys, grp_start, sorted_groups, chunks, hdr, rowbuf, sm, si);
        else
            fwd_pool<S>(cp, -1 - task, nP, uid_at_pos, offsets, hdr, rowbuf, out, status, &s_task[1]);
        __syncthreads();
    }
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

template <int D>
__global__ void __launch_bounds__(256) k3_hsum(const int32_t* __restrict__ uid_sorted,
                                               const int32_t* __restrict__ bag_sorted,
                                               const int32_t* __restrict__ uniq_start,
                                               const float* __restrict__ grad_out, int64_t L, int64_t B,
                                               int T, float* __restrict__ rowbuf, const int32_t* status)
{
    if (has_error(status)) return;
    constexpr int LB = D / 4;
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t c0 = warp * kHChunk;
    if (c0 >= L || lane >= LB) return;
    const int64_t c1 = min64(L, c0 + kHChunk);
    const int64_t TD = (int64_t)T * D;
    int cur = uid_sorted[c0];
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t l = c0; l <= c1; ++l) {
        const int u = l < c1 ? uid_sorted[l] : -1;
        if (u != cur) {
            float* dst = rowbuf + (int64_t)cur * D + lane * 4;
            const bool whole = uniq_start[cur] >= c0 && uniq_start[cur + 1] <= c1;
            if (whole) *reinterpret_cast<float4*>(dst) = acc;
            else red_add_v4(dst, acc);
            if (l == c1) break;
            cur = u;
            acc = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        const int bag = bag_sorted[l];
        const int t = (int)(bag / B);
        const int64_t b = bag - (int64_t)t * B;
        acc = f4add(acc, __ldg(reinterpret_cast<const float4*>(grad_out + b * TD + (int64_t)t * D) + lane));
    }
}

// ---------------------------------------------------------------------------
// backward over column groups
// ---------------------------------------------------------------------------
template <class S, typename K>
__global__ void __launch_bounds__(kThreads, 1)
k3_bwd_kernel(CoreParams cp, GradPtrs gp, PlanParams pp, const K* __restrict__ uniq_keys,
              const int32_t* __restrict__ grp_start, const int32_t* __restrict__ sorted_groups,
              const int32_t* __restrict__ col_count, const int32_t* __restrict__ col_start,
              PlanHeader* hdr, const float* __restrict__ rowbuf, int32_t* status)
{
    constexpr int R = S::R, N = S::N, MB = S::MB, MPB = S::MPB, D1 = S::D1, D2 = S::D2, D3 = S::D3,
                  P = S::P, NUB = S::NUB, DBR = S::DBR, DBC = S::DBC;
    extern __shared__ __align__(16) float sm[];
    float* Bs = sm;                       // [R][N] swizzled (key row/4)
    float* As = Bs + R * N;               // [MB][R]
    float* AsT = As + MB * R;             // [R][MB]
    float* Cn = AsT + R * MB;             // [MB][N] swizzled (key row)
    float* dCn = Cn + MB * N;             // [MB][N] swizzled (key row)
    float* Hs = dCn + MB * N;             // [NUB][P][D3]
    float* HsT = Hs + NUB * P * D3;       // [NUB][D3][P]
    float* SsT = HsT + NUB * P * D3;      // [NUB][D3][R] (+4 pad per row block)
    __shared__ int s_u0[MPB], s_ucum[MPB + 1], s_i1[MPB];
    __shared__ int s_bu[NUB], s_bp[NUB], s_bi3[NUB];
    __shared__ int s_task;
    constexpr int SST = D3 * R + 4;
    if (has_error(status)) return;
    const int tid = threadIdx.x, lane = tid & 31;
    const uint64_t rmask = (uint64_t(1) << cp.ibits) - 1;
    (void)lane;

    for (int iter = 0;; ++iter) {
        if (tid == 0) s_task = next_task(pp.sched, &hdr->col_head, iter);
        __syncthreads();
        const int c = s_task;
        if (c >= pp.ncols) break;
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
        const float* __restrict__ G1 = cp.cores[t][0];
        const float* __restrict__ G2 = cp.cores[t][1];
        const float* __restrict__ G3 = cp.cores[t][2];
        float* __restrict__ dG1 = gp.g[t][0];
        float* __restrict__ dG2 = gp.g[t][1];
        float* __restrict__ dG3 = gp.g[t][2];

        for (int q = tid; q < R * N / 4; q += kThreads) {
            const int rho = q / (N / 4), c4 = q % (N / 4);
            const float4 v = __ldg(reinterpret_cast<const float4*>(G2 + ((int64_t)rho * n2 + i2) * N) + c4);
            *reinterpret_cast<float4*>(&Bs[swz_b<N>(rho, c4 * 4)]) = v;
        }
        // dB accumulators: rows {tr*(DBR/2)+i, R/2 + tr*(DBR/2)+i} (DBR >= 4) or {tr} (DBR == 1),
        // cols: DBC/4 float4 chunks {tn*4, N/(DBC/4) + tn*4, ...}
        constexpr int NCH = DBC / 4;
        constexpr int TNB = N / DBC;  // column tiles
        const int tnb = tid % TNB, trb = tid / TNB;
        float dB[DBR][DBC];
#pragma unroll
        for (int i = 0; i < DBR; ++i)
#pragma unroll
            for (int j = 0; j < DBC; ++j) dB[i][j] = 0.f;

        for (int j0 = 0; j0 < ccount; j0 += MPB) {
            const int cnt = min(MPB, ccount - j0);
            __syncthreads();   // previous chunk finished with As / dCn
            if (tid < MPB) {
                int u0 = 0, nu = 0, i1 = 0;
                if (tid < cnt) {
                    const int g = sorted_groups[cfirst + j0 + tid];
                    u0 = grp_start[g];
                    nu = grp_start[g + 1] - u0;
                    i1 = (int)(key_row(uniq_keys[u0], cp.ibits) / n3 / n2);
                }
                s_u0[tid] = u0;
                s_ucum[tid] = nu;
                s_i1[tid] = i1;
            }
            __syncthreads();
            if (tid == 0) {
                int run = 0;
                for (int j = 0; j < MPB; ++j) {
                    const int v = s_ucum[j];
                    s_ucum[j] = run;
                    run += v;
                }
                s_ucum[MPB] = run;
            }
            for (int q = tid; q < MB * R; q += kThreads) {
                const int m = q / R, rho = q % R;
                const int j = m / D1, a1 = m % D1;
                const float v = j < cnt ? __ldg(G1 + ((int64_t)s_i1[j] * D1 + a1) * R + rho) : 0.f;
                As[m * R + rho] = v;
                AsT[rho * MB + m] = v;
            }
            for (int q = tid; q < MB * N / 4; q += kThreads)
                reinterpret_cast<float4*>(dCn)[q] = make_float4(0.f, 0.f, 0.f, 0.f);
            __syncthreads();

            // C_all = A . B  (MB x N): thread tile 4 rows x 8 cols
            {
                constexpr int TN = N / 8;
                const int tn = tid % TN, tm = tid / TN;   // tm < MB / 4
                float acc[4][8];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
#pragma unroll 2
                for (int rho = 0; rho < R; ++rho) {
                    const float4 a0 = *reinterpret_cast<const float4*>(&AsT[rho * MB + tm * 4]);
                    const float4 b0 = *reinterpret_cast<const float4*>(&Bs[swz_b<N>(rho, tn * 4)]);
                    const float4 b1 = *reinterpret_cast<const float4*>(&Bs[swz_b<N>(rho, N / 2 + tn * 4)]);
                    const float a[4] = {a0.x, a0.y, a0.z, a0.w};
                    const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i)
#pragma unroll
                        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
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

            // distinct rows in batches: dS_u -> dG3 (vector reductions), dC_p accumulated in dCn
            const int total = s_ucum[MPB];
            for (int k0 = 0; k0 < total; k0 += NUB) {
                const int nb = min(NUB, total - k0);
                if (tid < nb) {
                    const int kq = k0 + tid;
                    int j = 0;
                    while (j + 1 < cnt && s_ucum[j + 1] <= kq) ++j;
                    const int u = s_u0[j] + (kq - s_ucum[j]);
                    s_bu[tid] = u;
                    s_bp[tid] = j;
                    s_bi3[tid] = (int)((uint32_t)((uint64_t)uniq_keys[u] & rmask) % n3);
                }
                __syncthreads();
                // stage H (both layouts) and S^T
                for (int q = tid; q < nb * P * D3; q += kThreads) {
                    const int uu = q / (P * D3), rem = q % (P * D3);
                    const int row = rem / D3, a3 = rem % D3;
                    const float v = __ldcg(rowbuf + (int64_t)s_bu[uu] * S::D + rem);
                    Hs[uu * P * D3 + rem] = v;
                    HsT[uu * P * D3 + a3 * P + row] = v;
                }
                for (int q = tid; q < nb * R * D3; q += kThreads) {
                    const int uu = q / (R * D3), rem = q % (R * D3);
                    const int rho = rem / D3, a3 = rem % D3;
                    SsT[uu * SST + a3 * R + rho] = __ldg(G3 + ((int64_t)rho * n3 + s_bi3[uu]) * D3 + a3);
                }
                __syncthreads();
                // dS_u[rho2][a3] = sum_row C_p[row][rho2] H_u[row][a3]; tile 4 rho2 x 4 a3
                {
                    constexpr int TPU = (R / 4) * (D3 / 4);
                    for (int w = tid; w < nb * TPU; w += kThreads) {
                        const int uu = w / TPU, rem = w % TPU;
                        const int rc = rem / (D3 / 4), cg = rem % (D3 / 4);
                        const int p = s_bp[uu];
                        float4 o[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) o[i] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
                        for (int row = 0; row < P; ++row) {
                            const int m = p * D1 + row / D2, a2 = row % D2;
                            const float4 cv = *reinterpret_cast<const float4*>(&Cn[swz_m<N>(m, a2 * R + rc * 4)]);
                            const float4 h = *reinterpret_cast<const float4*>(&Hs[uu * P * D3 + row * D3 + cg * 4]);
                            const float cr[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                o[i].x = fmaf(cr[i], h.x, o[i].x);
                                o[i].y = fmaf(cr[i], h.y, o[i].y);
                                o[i].z = fmaf(cr[i], h.z, o[i].z);
                                o[i].w = fmaf(cr[i], h.w, o[i].w);
                            }
                        }
                        const int i3 = s_bi3[uu];
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            red_add_v4(dG3 + ((int64_t)(rc * 4 + i) * n3 + i3) * D3 + cg * 4, o[i]);
                    }
                }
                // dC_p[row][rho2] += sum_{u in p, a3} H_u[row][a3] S_u[rho2][a3]; tile rows (a1, a2=0..3) x 4 rho2
                {
                    constexpr int TPP = D1 * (R / 4);
                    for (int w = tid; w < cnt * TPP; w += kThreads) {
                        const int p = w / TPP, rem = w % TPP;
                        const int a1 = rem / (R / 4), rc = rem % (R / 4);
                        const int ulo = max(s_ucum[p], k0) - k0, uhi = min(s_ucum[p + 1], k0 + nb) - k0;
                        if (ulo >= uhi) continue;
                        float4 o[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) o[i] = make_float4(0.f, 0.f, 0.f, 0.f);
                        for (int uu = ulo; uu < uhi; ++uu) {
#pragma unroll
                            for (int a3 = 0; a3 < D3; ++a3) {
                                const float4 h = *reinterpret_cast<const float4*>(&HsT[uu * P * D3 + a3 * P + a1 * D2]);
                                const float4 sv = *reinterpret_cast<const float4*>(&SsT[uu * SST + a3 * R + rc * 4]);
                                const float hr[4] = {h.x, h.y, h.z, h.w};
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    o[i].x = fmaf(hr[i], sv.x, o[i].x);
                                    o[i].y = fmaf(hr[i], sv.y, o[i].y);
                                    o[i].z = fmaf(hr[i], sv.z, o[i].z);
                                    o[i].w = fmaf(hr[i], sv.w, o[i].w);
                                }
                            }
                        }
                        const int m = p * D1 + a1;
#pragma unroll
                        for (int a2 = 0; a2 < 4; ++a2) {
                            float4* d = reinterpret_cast<float4*>(&dCn[swz_m<N>(m, a2 * R + rc * 4)]);
                            *d = f4add(*d, o[a2]);
                        }
                    }
                }
                __syncthreads();
            }

            // dA[m][rho1] = sum_n dC[m][n] B[rho1][n] -> dG_1 (vector reductions); tile 2 m x 4 rho1
            {
                constexpr int TRH = R / 4;
                const int tr = tid % TRH, tm = tid / TRH;   // tm < MB / 2
                float o[2][4];
#pragma unroll
                for (int i = 0; i < 2; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) o[i][j] = 0.f;
#pragma unroll 2
                for (int n = 0; n < N; n += 4) {
                    float4 dc[2], b[4];
#pragma unroll
                    for (int i = 0; i < 2; ++i)
                        dc[i] = *reinterpret_cast<const float4*>(&dCn[swz_m<N>(tm * 2 + i, n)]);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        b[j] = *reinterpret_cast<const float4*>(&Bs[swz_b<N>(tr * 4 + j, n)]);
#pragma unroll
                    for (int i = 0; i < 2; ++i)
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            o[i][j] = fmaf(dc[i].x, b[j].x, o[i][j]);
                            o[i][j] = fmaf(dc[i].y, b[j].y, o[i][j]);
                            o[i][j] = fmaf(dc[i].z, b[j].z, o[i][j]);
                            o[i][j] = fmaf(dc[i].w, b[j].w, o[i][j]);
                        }
                }
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int m = tm * 2 + i, p = m / D1, a1 = m % D1;
                    if (p < cnt)
                        red_add_v4(dG1 + ((int64_t)s_i1[p] * D1 + a1) * R + tr * 4,
                                   make_float4(o[i][0], o[i][1], o[i][2], o[i][3]));
                }
            }
            // dB[rho1][n] += sum_m A[m][rho1] dC[m][n]
            {
#pragma unroll 2
                for (int m = 0; m < MB; ++m) {
                    float a[DBR];
                    if constexpr (DBR >= 4) {
                        const float4 a0 = *reinterpret_cast<const float4*>(&As[m * R + trb * 4]);
                        a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w;
                        if constexpr (DBR == 8) {
                            const float4 a1v = *reinterpret_cast<const float4*>(&As[m * R + R / 2 + trb * 4]);
                            a[4] = a1v.x; a[5] = a1v.y; a[6] = a1v.z; a[7] = a1v.w;
                        }
                    } else {
                        a[0] = As[m * R + trb];
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
        }
        // the column group is complete: dG_2[:, i_2] = dB (this block owns the slice)
#pragma unroll
        for (int i = 0; i < DBR; ++i) {
            int rho1;
            if constexpr (DBR == 8) rho1 = (i < 4) ? trb * 4 + i : R / 2 + trb * 4 + (i - 4);
            else if constexpr (DBR == 4) rho1 = trb * 4 + i;
            else rho1 = trb;
            float* dst = dG2 + ((int64_t)rho1 * n2 + i2) * N;
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch)
                *reinterpret_cast<float4*>(dst + ch * (N / NCH) + tnb * 4) =
                    make_float4(dB[i][ch * 4], dB[i][ch * 4 + 1], dB[i][ch * 4 + 2], dB[i][ch * 4 + 3]);
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// host launchers
// ---------------------------------------------------------------------------
template <class S, typename K>
cudaError_t fwd_launch(const K3Args& a, float* out, cudaStream_t s, int* nl)
{
    const size_t smem = sizeof(float) * S::fwd_smem_floats() + sizeof(int) * (S::MPF * 3 + 1 + S::NUF * 3 + 4);
    cudaError_t e = cudaFuncSetAttribute(k3_fwd_kernel<S, K>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const PlanBuffers& pb = *a.pb;
    k3_fwd_kernel<S, K><<<a.grid, kThreads, smem, s>>>(
        *a.cp, a.pp->sched, (const K*)a.uniq_keys, a.grp_start, a.uid_at_pos, a.offsets,
        pb.sorted_groups, pb.chunks, pb.tasks, pb.hdr, a.rowbuf, out, a.status);
    *nl += 1;
    return cudaGetLastError();
}

template <class S, typename K>
cudaError_t bwd_launch(const K3Args& a, const GradPtrs& gp, const float* grad_out, cudaStream_t s, int* nl)
{
    const int64_t L = a.L;
    const int64_t nwarps = ceil_div(L, kHChunk);
    k3_hzero<S::D><<<148, 256, 0, s>>>(a.uid_sorted, L, a.rowbuf, a.status);
    k3_hsum<S::D><<<(unsigned)ceil_div(nwarps * 32, 256), 256, 0, s>>>(
        a.uid_sorted, a.bag_sorted, a.uniq_start, grad_out, L, a.cp->B, a.cp->T, a.rowbuf, a.status);
    *nl += 2;
    const size_t smem = sizeof(float) * S::bwd_smem_floats();
    cudaError_t e = cudaFuncSetAttribute(k3_bwd_kernel<S, K>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const PlanBuffers& pb = *a.pb;
    k3_bwd_kernel<S, K><<<a.grid, kThreads, smem, s>>>(
        *a.cp, gp, *a.pp, (const K*)a.uniq_keys, a.grp_start, pb.sorted_groups, pb.col_count,
        pb.col_start, pb.hdr, a.rowbuf, a.status);
    *nl += 1;
    return cudaGetLastError();
}

template <class S>
cudaError_t fwd_dispatch(const K3Args& a, float* out, cudaStream_t s, int* nl)
{
    return a.key64 ? fwd_launch<S, uint64_t>(a, out, s, nl) : fwd_launch<S, uint32_t>(a, out, s, nl);
}
template <class S>
cudaError_t bwd_dispatch(const K3Args& a, const GradPtrs& gp, const float* g, cudaStream_t s, int* nl)
{
    return a.key64 ? bwd_launch<S, uint64_t>(a, gp, g, s, nl) : bwd_launch<S, uint32_t>(a, gp, g, s, nl);
}

template <class S>
int occ_fwd()
{
    const size_t smem = sizeof(float) * S::fwd_smem_floats() + sizeof(int) * (S::MPF * 3 + 1 + S::NUF * 3 + 4);
    cudaFuncSetAttribute(k3_fwd_kernel<S, uint32_t>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k3_fwd_kernel<S, uint32_t>, kThreads, smem) != cudaSuccess) return 1;
    return n > 0 ? n : 1;
}
template <class S>
int occ_bwd()
{
    const size_t smem = sizeof(float) * S::bwd_smem_floats();
    cudaFuncSetAttribute(k3_bwd_kernel<S, uint32_t>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k3_bwd_kernel<S, uint32_t>, kThreads, smem) != cudaSuccess) return 1;
    return n > 0 ? n : 1;
}

}  // namespace

int k3_blocks_per_sm(const CoreParams& cp, bool backward)
{
#define TT_OCC_CASE(Q1, Q2, Q3, QR) \
    if (cp.d[2] == Q3 && cp.r[1] == QR) return backward ? occ_bwd<S3<Q1, Q2, Q3, QR>>() : occ_fwd<S3<Q1, Q2, Q3, QR>>();
    TT_K3_CASES_INNER(TT_OCC_CASE)
#undef TT_OCC_CASE
    return 1;
}

bool k3_supported(const CoreParams& cp)
{
    if (cp.k != 3 || cp.d[0] != 4 || cp.d[1] != 4 || cp.r[1] != cp.r[2]) return false;
    const int R = cp.r[1], d3 = cp.d[2];
    return (R == 64 && d3 == 8) || (R == 32 && d3 == 8) || (R == 16 && d3 == 4) || (R == 32 && d3 == 4) ||
           (R == 16 && d3 == 8);
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
#define TT_FWD_CASE(Q1, Q2, Q3, QR) \
    if (cp.d[2] == Q3 && cp.r[1] == QR) return fwd_dispatch<S3<Q1, Q2, Q3, QR>>(a, out, s, nl);
    TT_K3_CASES(TT_FWD_CASE)
#undef TT_FWD_CASE
    return cudaErrorInvalidValue;
}

cudaError_t k3_backward(const K3Args& a, const GradPtrs& gp, const float* grad_out, cudaStream_t s, int* nl)
{
    const CoreParams& cp = *a.cp;
#define TT_BWD_CASE(Q1, Q2, Q3, QR) \
    if (cp.d[2] == Q3 && cp.r[1] == QR) return bwd_dispatch<S3<Q1, Q2, Q3, QR>>(a, gp, grad_out, s, nl);
    TT_K3_CASES(TT_BWD_CASE)
#undef TT_BWD_CASE
    return cudaErrorInvalidValue;
}

}  // namespace tt
