// Merging the first two cores of a four-core table (forward) and splitting
// the merged gradient back (backward).
//
// A four-core table with factors (n_1, n_2, n_3, n_4) is the same virtual
// table as the three-core table with factors (n_1 n_2, n_3, n_4) whose first
// core is G_12[0, i_1 n_2 + i_2, a_1 d_2 + a_2, :] = G_1[0, i_1, a_1, :] . G_2[:, i_2, a_2, :]:
// the row numbering, the prefixes (row / n_4) and the contraction order are
// unchanged, and the first two levels of the prefix chain are shared by every
// row with the same (i_1, i_2) -- the multi-level prefix reuse of the pages'
// prefix-sharing idea.  G_12 is materialised for every (i_1, i_2) once per
// forward call; after the backward, dG_12 goes back to the two cores:
//   dG_1[0, i_1, a_1, r] = sum_{i_2, a_2, s} dG_12[i_1 n_2 + i_2, (a_1, a_2), s] G_2[r, i_2, a_2, s]
//   dG_2[r, i_2, a_2, s] = sum_{i_1, a_1}    G_1[0, i_1, a_1, r] dG_12[i_1 n_2 + i_2, (a_1, a_2), s]
// One block per (table, i_2): the G_2 slice stays in shared memory while the
// block walks i_1; dG_2[:, i_2] is owned by the block and written once.
#include "tt_common.cuh"

namespace tt {

__global__ void __launch_bounds__(256) k4_merge(MergeParams mp, const int32_t* status)
{
    extern __shared__ __align__(16) float sm[];
    if (has_error(status)) return;
    const int d1 = mp.d1, d2 = mp.d2, r1 = mp.r1, r2 = mp.r2;
    const int W = d2 * r2;                  // row of a G_2 slice: (a_2, s)
    float* G2s = sm;                        // [r1][W]
    float* G1s = G2s + r1 * W;              // [d1][r1]
    // block -> (table, i_2)
    int t = 0;
    while (t + 1 < mp.T && mp.blk_base[t + 1] <= (int)blockIdx.x) ++t;
    const int i2 = blockIdx.x - mp.blk_base[t];
    const uint32_t n1 = mp.n1[t], n2 = mp.n2[t];
    const float* G1 = mp.g1[t];
    const float* G2 = mp.g2[t];
    float* G12 = mp.g12[t];
    for (int q = threadIdx.x; q < r1 * W; q += blockDim.x) {
        const int r = q / W, c = q % W;
        G2s[q] = __ldg(G2 + ((int64_t)r * n2 + i2) * W + c);
    }
    const int outs = d1 * W;                // outputs per (i_1, i_2): (a_1, a_2, s)
    for (uint32_t i1 = 0; i1 < n1; ++i1) {
        __syncthreads();
        for (int q = threadIdx.x; q < d1 * r1; q += blockDim.x) G1s[q] = __ldg(G1 + (int64_t)i1 * d1 * r1 + q);
        __syncthreads();
        float* dst = G12 + ((int64_t)i1 * n2 + i2) * outs;
        for (int o = threadIdx.x; o < outs; o += blockDim.x) {
            const int a1 = o / W, c = o % W;   // c = (a_2, s); G_12 column (a_1 d_2 + a_2), s
            float acc = 0.f;
            for (int r = 0; r < r1; ++r) acc = fmaf(G1s[a1 * r1 + r], G2s[r * W + c], acc);
            dst[o] = acc;
        }
    }
}

__global__ void __launch_bounds__(256) k4_unmerge(MergeParams mp, const int32_t* status)
{
    extern __shared__ __align__(16) float sm[];
    if (has_error(status)) return;
    const int d1 = mp.d1, d2 = mp.d2, r1 = mp.r1, r2 = mp.r2;
    const int W = d2 * r2;
    float* G2s = sm;                        // [r1][W]
    float* dG2s = G2s + r1 * W;             // [r1][W] accumulator of dG_2[:, i_2]
    float* D12 = dG2s + r1 * W;             // [d1][W]  dG_12 of the current (i_1, i_2)
    float* G1s = D12 + d1 * W;              // [d1][r1]
    float* red = G1s + d1 * r1;             // [blockDim] partial sums for dG_1
    int t = 0;
    while (t + 1 < mp.T && mp.blk_base[t + 1] <= (int)blockIdx.x) ++t;
    const int i2 = blockIdx.x - mp.blk_base[t];
    const uint32_t n1 = mp.n1[t], n2 = mp.n2[t];
    const float* G1 = mp.g1[t];
    const float* G2 = mp.g2[t];
    const float* dG12 = mp.dg12[t];
    float* dG1 = mp.dg1[t];
    float* dG2 = mp.dg2[t];
    for (int q = threadIdx.x; q < r1 * W; q += blockDim.x) {
        const int r = q / W, c = q % W;
        G2s[q] = __ldg(G2 + ((int64_t)r * n2 + i2) * W + c);
        dG2s[q] = 0.f;
    }
    const int nout1 = d1 * r1;              // dG_1 outputs of one i_1
    const int split = blockDim.x / nout1;   // threads per dG_1 output (>= 1)
    for (uint32_t i1 = 0; i1 < n1; ++i1) {
        __syncthreads();
        const float* src = dG12 + ((int64_t)i1 * n2 + i2) * d1 * W;
        for (int q = threadIdx.x; q < d1 * W; q += blockDim.x) D12[q] = __ldcg(src + q);
        for (int q = threadIdx.x; q < d1 * r1; q += blockDim.x) G1s[q] = __ldg(G1 + (int64_t)i1 * d1 * r1 + q);
        __syncthreads();
        // dG_2[r, (a_2, s)] += sum_{a_1} G_1[i_1, a_1, r] dG_12[(a_1, a_2), s]
        for (int q = threadIdx.x; q < r1 * W; q += blockDim.x) {
            const int r = q / W, c = q % W;
            float acc = dG2s[q];
            for (int a1 = 0; a1 < d1; ++a1) acc = fmaf(G1s[a1 * r1 + r], D12[a1 * W + c], acc);
            dG2s[q] = acc;
        }
        // dG_1[i_1, a_1, r] += sum_{(a_2, s)} dG_12[(a_1, a_2), s] G_2[r, (a_2, s)]
        float part = 0.f;
        const int o = threadIdx.x / split, sub = threadIdx.x % split;
        if (o < nout1) {
            const int a1 = o / r1, r = o % r1;
            for (int c = sub; c < W; c += split) part = fmaf(D12[a1 * W + c], G2s[r * W + c], part);
        }
        red[threadIdx.x] = part;
        __syncthreads();
        if (sub == 0 && o < nout1) {
            float acc = 0.f;
            for (int k = 0; k < split; ++k) acc += red[threadIdx.x + k];
            if (acc != 0.f) atomicAdd(dG1 + (int64_t)i1 * nout1 + o, acc);
        }
    }
    __syncthreads();
    for (int q = threadIdx.x; q < r1 * W; q += blockDim.x) {
        const int r = q / W, c = q % W;
        dG2[((int64_t)r * n2 + i2) * W + c] = dG2s[q];
    }
}

static size_t merge_smem(const MergeParams& mp) { return sizeof(float) * ((size_t)mp.r1 * mp.d2 * mp.r2 + mp.d1 * mp.r1); }
static size_t unmerge_smem(const MergeParams& mp)
{
    const size_t W = (size_t)mp.d2 * mp.r2;
    return sizeof(float) * (2 * mp.r1 * W + mp.d1 * W + (size_t)mp.d1 * mp.r1 + 256);
}

bool merge_fits(const MergeParams& mp)
{
    return merge_smem(mp) <= 160 * 1024 && unmerge_smem(mp) <= 160 * 1024 && mp.d1 * mp.r1 <= 256;
}

cudaError_t launch_merge(const MergeParams& mp, int32_t* status, cudaStream_t s, int* nl)
{
    const size_t smem = merge_smem(mp);
    cudaError_t e = cudaFuncSetAttribute(k4_merge, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k4_merge<<<mp.blk_base[mp.T], 256, smem, s>>>(mp, status);
    *nl += 1;
    return cudaGetLastError();
}

cudaError_t launch_unmerge(const MergeParams& mp, int32_t* status, cudaStream_t s, int* nl)
{
    const size_t smem = unmerge_smem(mp);
    cudaError_t e = cudaFuncSetAttribute(k4_unmerge, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k4_unmerge<<<mp.blk_base[mp.T], 256, smem, s>>>(mp, status);
    *nl += 1;
    return cudaGetLastError();
}

}  // namespace tt
