// Generic fused TT gather kernels: any k <= 4, any d, r the handle accepts.
//
// FlowTT section 3.2 ("Flow-Aware Fused TT Embedding Execution"): per prefix
// group, the shared intermediate C = A.B (the product of the first k-1
// slices) is computed once and kept in shared memory; each distinct row of
// the group then applies its last slice (E = C.D) and E is pooled into the
// row's bags (in-kernel pooling; lookups of one row that fall in the same
// bag are merged first, the batched-aggregation idea of the same section).
// The backward pass walks the same groups in reverse: the upstream gradient
// of a distinct row is the sum of its bags' gradients, it produces the last
// core's gradient slice and the gradient of C, which is then pushed back
// through the prefix slices.
//
// These kernels favour plainness over speed: one block per group (cyclic
// over a fixed grid), one output element per thread, fp32 FMA.  The
// shape-specialised kernels in fused_fast.cu take over for the benchmark
// shapes.  Gradients here are accumulated with global atomics.
#include "tt_common.cuh"

namespace tt {

// Sizes, in floats, of the generic kernels' shared memory.
static void chain_sizes(const CoreParams& cp, int64_t* max_inter, int64_t* sum_left)
{
    int64_t rows = 1, best = 1, sum = 0;
    for (int j = 0; j + 1 < cp.k; ++j) {
        rows *= cp.d[j];
        const int64_t sz = rows * cp.r[j + 1];
        best = sz > best ? sz : best;
        sum += sz;
    }
    *max_inter = best;
    *sum_left = sum;
}

int64_t generic_forward_smem_floats(const CoreParams& cp)
{
    int64_t inter, sum;
    chain_sizes(cp, &inter, &sum);
    return 2 * inter + cp.D;
}

int64_t generic_backward_smem_floats(const CoreParams& cp)
{
    int64_t inter, sum;
    chain_sizes(cp, &inter, &sum);
    const int64_t pk = (int64_t)cp.P * cp.r[cp.k - 1];
    return sum + 1 + 2 * (inter > pk ? inter : pk) + cp.D;
}

__device__ __forceinline__ void row_digits(const CoreParams& cp, int t, uint32_t row, uint32_t* dig)
{
    for (int j = cp.k - 1; j >= 0; --j) {
        const uint32_t nj = cp.n[t][j];
        dig[j] = row % nj;
        row /= nj;
    }
}

// next[(alpha, a), s] = sum_rho cur[alpha, rho] * G_j[rho, i_j, a, s]
__device__ __forceinline__ void chain_step(const float* __restrict__ cur, float* __restrict__ nxt,
                                           int rows, int rj, int dj, int rj1, uint32_t nj, uint32_t ij,
                                           const float* __restrict__ Gj)
{
    const int total = rows * dj * rj1;
    for (int i = threadIdx.x; i < total; i += blockDim.x) {
        const int s = i % rj1;
        const int a = (i / rj1) % dj;
        const int alpha = i / (rj1 * dj);
        float acc = 0.f;
        for (int rho = 0; rho < rj; ++rho)
            acc = fmaf(cur[alpha * rj + rho], __ldg(Gj + (((int64_t)rho * nj + ij) * dj + a) * rj1 + s), acc);
        nxt[i] = acc;
    }
}

template <typename K>
__global__ void __launch_bounds__(256) k_fwd_generic(CoreParams cp, const K* __restrict__ uniq_keys,
                                                     const int32_t* __restrict__ uniq_start,
                                                     const int32_t* __restrict__ grp_start,
                                                     const int32_t* __restrict__ bag_sorted,
                                                     const WsCounters* __restrict__ counters,
                                                     int inter, float* __restrict__ out,
                                                     const int32_t* status)
{
    extern __shared__ float smem[];
    if (has_error(status)) return;
    float* bufA = smem;
    float* bufB = smem + inter;
    float* E = smem + 2 * inter;
    const int64_t G = counters->num_groups;
    const uint64_t rmask = (uint64_t(1) << cp.ibits) - 1;
    const int k = cp.k, D = cp.D, dk = cp.d[k - 1], rk1 = cp.r[k - 1];
    const int64_t TD = (int64_t)cp.T * D;

    for (int64_t g = blockIdx.x; g < G; g += gridDim.x) {
        const int u0 = grp_start[g], u1 = grp_start[g + 1];
        const K key0 = uniq_keys[u0];
        const int t = (int)(key0 >> cp.ibits);
        uint32_t dig[kMaxK];
        row_digits(cp, t, (uint32_t)(key0 & rmask), dig);

        float* cur = bufA;
        float* nxt = bufB;
        int rows = 1;
        if (k == 1) {
            if (threadIdx.x == 0) cur[0] = 1.f;
        } else {
            rows = cp.d[0];
            const float* s0 = cp.cores[t][0] + (int64_t)dig[0] * cp.d[0] * cp.r[1];
            for (int i = threadIdx.x; i < rows * cp.r[1]; i += blockDim.x) cur[i] = __ldg(s0 + i);
            for (int j = 1; j + 1 < k; ++j) {
                __syncthreads();
                chain_step(cur, nxt, rows, cp.r[j], cp.d[j], cp.r[j + 1], cp.n[t][j], dig[j],
                           cp.cores[t][j]);
                float* tmp = cur; cur = nxt; nxt = tmp;
                rows *= cp.d[j];
            }
        }
        __syncthreads();

        const uint32_t nk = cp.n[t][k - 1];
        const float* Gk = cp.cores[t][k - 1];
        for (int u = u0; u < u1; ++u) {
            const uint32_t ik = (uint32_t)(uniq_keys[u] & rmask) % nk;
            for (int c = threadIdx.x; c < D; c += blockDim.x) {
                const int row = c / dk, a = c % dk;
                float acc = 0.f;
                for (int rho = 0; rho < rk1; ++rho)
                    acc = fmaf(cur[row * rk1 + rho], __ldg(Gk + ((int64_t)rho * nk + ik) * dk + a), acc);
                E[c] = acc;
            }
            __syncthreads();
            int l = uniq_start[u];
            const int le = uniq_start[u + 1];
            while (l < le) {
                const int bag = bag_sorted[l];
                int m = 1;
                while (l + m < le && bag_sorted[l + m] == bag) ++m;
                const int64_t b = (int64_t)bag - (int64_t)t * cp.B;
                float* o = out + b * TD + (int64_t)t * D;
                for (int c = threadIdx.x; c < D; c += blockDim.x) atomicAdd(o + c, (float)m * E[c]);
                l += m;
            }
            __syncthreads();
        }
    }
}

cudaError_t launch_forward_generic(const CoreParams& cp, bool key64, const void* uniq_keys,
                                   const int32_t* uniq_start, const int32_t* grp_start,
                                   const int32_t* bag_sorted, const WsCounters* counters,
                                   int64_t max_groups, float* out, int32_t* status,
                                   cudaStream_t s, int grid, int* nl)
{
    int64_t inter, sum;
    chain_sizes(cp, &inter, &sum);
    const size_t smem = sizeof(float) * (size_t)(2 * inter + cp.D);
    const int g = (int)(max_groups < grid ? max_groups : grid);
    if (g <= 0) return cudaSuccess;
    if (key64) {
        const cudaError_t ea = cudaFuncSetAttribute(k_fwd_generic<uint64_t>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (ea != cudaSuccess) return ea;
        k_fwd_generic<uint64_t><<<g, 256, smem, s>>>(cp, (const uint64_t*)uniq_keys, uniq_start,
                                                     grp_start, bag_sorted, counters, (int)inter,
                                                     out, status);
    } else {
        const cudaError_t ea = cudaFuncSetAttribute(k_fwd_generic<uint32_t>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (ea != cudaSuccess) return ea;
        k_fwd_generic<uint32_t><<<g, 256, smem, s>>>(cp, (const uint32_t*)uniq_keys, uniq_start,
                                                     grp_start, bag_sorted, counters, (int)inter,
                                                     out, status);
    }
    *nl += 1;
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Backward.  Shared memory: the left partials L_1..L_{k-1} (L_j is the product
// of the first j slices, (d_1..d_j) x r_j), two ping-pong gradient buffers
// and the distinct row's upstream gradient H.
// ---------------------------------------------------------------------------
template <typename K>
__global__ void __launch_bounds__(256) k_bwd_generic(CoreParams cp, GradPtrs gp,
                                                     const K* __restrict__ uniq_keys,
                                                     const int32_t* __restrict__ uniq_start,
                                                     const int32_t* __restrict__ grp_start,
                                                     const int32_t* __restrict__ bag_sorted,
                                                     const WsCounters* __restrict__ counters,
                                                     int inter, int sum_left,
                                                     const float* __restrict__ grad_out,
                                                     const int32_t* status)
{
    extern __shared__ float smem[];
    if (has_error(status)) return;
    const int k = cp.k, D = cp.D, dk = cp.d[k - 1], rk1 = cp.r[k - 1], P = cp.P;
    float* left[kMaxK];       // left[j] for j = 1..k-1
    {
        float* p = smem;
        int rows = 1;
        left[0] = nullptr;
        for (int j = 0; j + 1 < k; ++j) {
            rows *= cp.d[j];
            left[j + 1] = p;
            p += rows * cp.r[j + 1];
        }
    }
    float* one = smem + sum_left;          // the 1x1 identity L_0
    float* dA = one + 1;
    float* dB = dA + inter;
    float* H = dB + inter;
    if (threadIdx.x == 0) one[0] = 1.f;
    const int64_t G = counters->num_groups;
    const uint64_t rmask = (uint64_t(1) << cp.ibits) - 1;
    const int64_t TD = (int64_t)cp.T * D;

    for (int64_t g = blockIdx.x; g < G; g += gridDim.x) {
        const int u0 = grp_start[g], u1 = grp_start[g + 1];
        const K key0 = uniq_keys[u0];
        const int t = (int)(key0 >> cp.ibits);
        uint32_t dig[kMaxK];
        row_digits(cp, t, (uint32_t)(key0 & rmask), dig);

        // left partials of the prefix
        if (k >= 2) {
            const float* s0 = cp.cores[t][0] + (int64_t)dig[0] * cp.d[0] * cp.r[1];
            for (int i = threadIdx.x; i < cp.d[0] * cp.r[1]; i += blockDim.x) left[1][i] = __ldg(s0 + i);
            int rows = cp.d[0];
            for (int j = 1; j + 1 < k; ++j) {
                __syncthreads();
                chain_step(left[j], left[j + 1], rows, cp.r[j], cp.d[j], cp.r[j + 1], cp.n[t][j],
                           dig[j], cp.cores[t][j]);
                rows *= cp.d[j];
            }
        }
        const float* C = (k >= 2) ? left[k - 1] : one;
        float* dC = dA;
        for (int i = threadIdx.x; i < P * rk1; i += blockDim.x) dC[i] = 0.f;
        __syncthreads();

        const uint32_t nk = cp.n[t][k - 1];
        const float* Gk = cp.cores[t][k - 1];
        float* dGk = gp.g[t][k - 1];
        for (int u = u0; u < u1; ++u) {
            const uint32_t ik = (uint32_t)(uniq_keys[u] & rmask) % nk;
            // H = sum of the upstream gradients of the row's lookups
            const int ls = uniq_start[u], le = uniq_start[u + 1];
            for (int c = threadIdx.x; c < D; c += blockDim.x) {
                float acc = 0.f;
                for (int l = ls; l < le; ++l) {
                    const int64_t b = (int64_t)bag_sorted[l] - (int64_t)t * cp.B;
                    acc += __ldg(grad_out + b * TD + (int64_t)t * D + c);
                }
                H[c] = acc;
            }
            __syncthreads();
            // dG_k[rho, i_k, a, 0] += sum_row C[row, rho] * H[row, a]
            for (int i = threadIdx.x; i < rk1 * dk; i += blockDim.x) {
                const int rho = i / dk, a = i % dk;
                float acc = 0.f;
                for (int row = 0; row < P; ++row) acc = fmaf(C[row * rk1 + rho], H[row * dk + a], acc);
                atomicAdd(dGk + ((int64_t)rho * nk + ik) * dk + a, acc);
            }
            // dC[row, rho] += sum_a H[row, a] * G_k[rho, i_k, a, 0]
            for (int i = threadIdx.x; i < P * rk1; i += blockDim.x) {
                const int row = i / rk1, rho = i % rk1;
                float acc = 0.f;
                for (int a = 0; a < dk; ++a)
                    acc = fmaf(H[row * dk + a], __ldg(Gk + ((int64_t)rho * nk + ik) * dk + a), acc);
                dC[i] += acc;
            }
            __syncthreads();
        }

        // back through the prefix slices j = k-2 .. 0 (0-based)
        float* dcur = dA;
        float* dprev = dB;
        int rows = P;
        for (int j = k - 2; j >= 0; --j) {
            const int rj = cp.r[j], dj = cp.d[j], rj1 = cp.r[j + 1];
            rows /= dj;  // rows of L_j
            const float* Lj = (j == 0) ? one : left[j];
            const uint32_t nj = cp.n[t][j], ij = dig[j];
            const float* Gj = cp.cores[t][j];
            float* dGj = gp.g[t][j];
            // dG_j[rho, i_j, a, s] += sum_alpha L_j[alpha, rho] * dL[alpha, (a, s)]
            for (int i = threadIdx.x; i < rj * dj * rj1; i += blockDim.x) {
                const int s = i % rj1, a = (i / rj1) % dj, rho = i / (rj1 * dj);
                float acc = 0.f;
                for (int alpha = 0; alpha < rows; ++alpha)
                    acc = fmaf(Lj[alpha * rj + rho], dcur[(alpha * dj + a) * rj1 + s], acc);
                atomicAdd(dGj + (((int64_t)rho * nj + ij) * dj + a) * rj1 + s, acc);
            }
            if (j > 0) {
                // dL_j[alpha, rho] = sum_{a, s} dL[alpha, (a, s)] * G_j[rho, i_j, a, s]
                for (int i = threadIdx.x; i < rows * rj; i += blockDim.x) {
                    const int alpha = i / rj, rho = i % rj;
                    float acc = 0.f;
                    for (int a = 0; a < dj; ++a)
                        for (int s = 0; s < rj1; ++s)
                            acc = fmaf(dcur[(alpha * dj + a) * rj1 + s],
                                       __ldg(Gj + (((int64_t)rho * nj + ij) * dj + a) * rj1 + s), acc);
                    dprev[i] = acc;
                }
            }
            __syncthreads();
            float* tmp = dcur; dcur = dprev; dprev = tmp;
        }
        __syncthreads();
    }
}

cudaError_t launch_backward_generic(const CoreParams& cp, const GradPtrs& gp, bool key64,
                                    const void* uniq_keys, const int32_t* uniq_start,
                                    const int32_t* grp_start, const int32_t* bag_sorted,
                                    const WsCounters* counters, int64_t max_groups,
                                    const float* grad_out, int32_t* status, cudaStream_t s,
                                    int grid, int* nl)
{
    int64_t inter, sum;
    chain_sizes(cp, &inter, &sum);
    const int64_t dcap = inter > (int64_t)cp.P * cp.r[cp.k - 1] ? inter : (int64_t)cp.P * cp.r[cp.k - 1];
    const size_t smem = sizeof(float) * (size_t)(sum + 1 + 2 * dcap + cp.D);
    const int g = (int)(max_groups < grid ? max_groups : grid);
    if (g <= 0) return cudaSuccess;
    if (key64) {
        const cudaError_t ea = cudaFuncSetAttribute(k_bwd_generic<uint64_t>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (ea != cudaSuccess) return ea;
        k_bwd_generic<uint64_t><<<g, 256, smem, s>>>(cp, gp, (const uint64_t*)uniq_keys, uniq_start,
                                                     grp_start, bag_sorted, counters, (int)dcap,
                                                     (int)sum, grad_out, status);
    } else {
        const cudaError_t ea = cudaFuncSetAttribute(k_bwd_generic<uint32_t>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (ea != cudaSuccess) return ea;
        k_bwd_generic<uint32_t><<<g, 256, smem, s>>>(cp, gp, (const uint32_t*)uniq_keys, uniq_start,
                                                     grp_start, bag_sorted, counters, (int)dcap,
                                                     (int)sum, grad_out, status);
    }
    *nl += 1;
    return cudaGetLastError();
}

}  // namespace tt
