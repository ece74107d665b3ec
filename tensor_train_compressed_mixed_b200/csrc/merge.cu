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
// block walks i_1 in tiles of kMergeTile; dG_2[:, i_2] is owned by the block,
// accumulated in registers and written once.
#include "tt_common.cuh"

namespace tt {

namespace {
constexpr int kMergeThreads = 256;
constexpr int kMergeTile = 16;   // values of i_1 per step of the walk
}  // namespace

__global__ void __launch_bounds__(kMergeThreads) k4_merge(MergeParams mp, const int32_t* status)
{
    extern __shared__ __align__(16) float sm[];
    if (has_error(status)) return;
    const int d1 = mp.d1, d2 = mp.d2, r1 = mp.r1, r2 = mp.r2;
    const int W = d2 * r2;                  // row of a G_2 slice: (a_2, s)
    float* G2s = sm;                        // [r1][W]
    float* G1s = G2s + r1 * W;              // [kMergeTile][d1][r1]
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
    for (uint32_t i0 = 0; i0 < n1; i0 += kMergeTile) {
        const int nt = (int)min((uint32_t)kMergeTile, n1 - i0);
        __syncthreads();
        for (int q = threadIdx.x; q < nt * d1 * r1; q += blockDim.x) G1s[q] = __ldg(G1 + (int64_t)i0 * d1 * r1 + q);
        __syncthreads();
        // output o = (ii, a_1, c): G_12[(i0 + ii) n_2 + i_2][a_1 d_2 + a_2][s], c = (a_2, s)
        for (int o = threadIdx.x; o < nt * outs; o += blockDim.x) {
            const int ii = o / outs, rem = o % outs, a1 = rem / W, c = rem % W;
            const float* g1 = G1s + (ii * d1 + a1) * r1;
            float acc = 0.f;
            for (int r = 0; r < r1; ++r) acc = fmaf(g1[r], G2s[r * W + c], acc);
            G12[((int64_t)(i0 + ii) * n2 + i2) * outs + rem] = acc;
        }
    }
}

__global__ void __launch_bounds__(kMergeThreads) k4_unmerge(MergeParams mp, const int32_t* status)
{
    extern __shared__ __align__(16) float sm[];
    if (has_error(status)) return;
    const int d1 = mp.d1, d2 = mp.d2, r1 = mp.r1, r2 = mp.r2;
    const int W = d2 * r2;
    const int RP = r1 + 1;                  // padded row of the transposed slice (no bank conflicts)
    float* G2t = sm;                        // [W][RP]: G_2[:, i_2] transposed (dG_1 reads along r)
    float* D12 = G2t + W * RP;              // [kMergeTile][d1][W]  dG_12 of the tile's (i_1, i_2)
    float* G1s = D12 + kMergeTile * d1 * W; // [kMergeTile][d1][r1]
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
        G2t[c * RP + r] = __ldg(G2 + ((int64_t)r * n2 + i2) * W + c);
    }
    // dG_2[:, i_2] accumulates in registers: thread owns entries tid, tid + 256, ... of [r1][W]
    constexpr int kMaxOwn = 32;
    float acc2[kMaxOwn];
#pragma unroll
    for (int k = 0; k < kMaxOwn; ++k) acc2[k] = 0.f;
    const int own = (r1 * W + (int)blockDim.x - 1) / (int)blockDim.x;
    for (uint32_t i0 = 0; i0 < n1; i0 += kMergeTile) {
        const int nt = (int)min((uint32_t)kMergeTile, n1 - i0);
        __syncthreads();
        for (int q = threadIdx.x; q < nt * d1 * W; q += blockDim.x) {
            const int ii = q / (d1 * W), rem = q % (d1 * W);
            D12[q] = __ldcg(dG12 + ((int64_t)(i0 + ii) * n2 + i2) * d1 * W + rem);
        }
        for (int q = threadIdx.x; q < nt * d1 * r1; q += blockDim.x) G1s[q] = __ldg(G1 + (int64_t)i0 * d1 * r1 + q);
        __syncthreads();
        // dG_2[r, c] += sum_{ii, a_1} G_1[i0 + ii, a_1, r] dG_12[(ii, a_1), c]
#pragma unroll
        for (int k = 0; k < kMaxOwn; ++k) {
            const int q = threadIdx.x + k * (int)blockDim.x;
            if (k < own && q < r1 * W) {
                const int r = q / W, c = q % W;
                float a = acc2[k];
                for (int ii = 0; ii < nt; ++ii)
                    for (int a1 = 0; a1 < d1; ++a1)
                        a = fmaf(G1s[(ii * d1 + a1) * r1 + r], D12[(ii * d1 + a1) * W + c], a);
                acc2[k] = a;
            }
        }
        // dG_1[i0 + ii, a_1, r] += sum_c dG_12[(ii, a_1), c] G_2[r, c]: one owner per output of the
        // tile; consecutive threads take consecutive r (reads of the transposed slice are contiguous,
        // the dG_12 row is the same for the warp)
        for (int o = threadIdx.x; o < nt * d1 * r1; o += blockDim.x) {
            const int row = o / r1, r = o % r1;   // row = (ii, a_1)
            const float* dr = D12 + row * W;
            float a = 0.f;
            for (int c = 0; c < W; ++c) a = fmaf(dr[c], G2t[c * RP + r], a);
            if (a != 0.f) atomicAdd(dG1 + (int64_t)i0 * d1 * r1 + o, a);
        }
    }
#pragma unroll
    for (int k = 0; k < kMaxOwn; ++k) {
        const int q = threadIdx.x + k * (int)blockDim.x;
        if (k < own && q < r1 * W) {
            const int r = q / W, c = q % W;
            dG2[((int64_t)r * n2 + i2) * W + c] = acc2[k];
        }
    }
}

static size_t merge_smem(const MergeParams& mp)
{
    return sizeof(float) * ((size_t)mp.r1 * mp.d2 * mp.r2 + (size_t)kMergeTile * mp.d1 * mp.r1);
}
static size_t unmerge_smem(const MergeParams& mp)
{
    const size_t W = (size_t)mp.d2 * mp.r2;
    return sizeof(float) * ((mp.r1 + 1) * W + (size_t)kMergeTile * mp.d1 * W + (size_t)kMergeTile * mp.d1 * mp.r1);
}

bool merge_fits(const MergeParams& mp)
{
    // dG_2[:, i_2] is held in registers: at most 32 entries per thread
    return merge_smem(mp) <= 160 * 1024 && unmerge_smem(mp) <= 160 * 1024 &&
           (int64_t)mp.r1 * mp.d2 * mp.r2 <= 32 * kMergeThreads;
}

cudaError_t launch_merge(const MergeParams& mp, int32_t* status, cudaStream_t s, int* nl)
{
    const size_t smem = merge_smem(mp);
    cudaError_t e = cudaFuncSetAttribute(k4_merge, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k4_merge<<<mp.blk_base[mp.T], kMergeThreads, smem, s>>>(mp, status);
    *nl += 1;
    return cudaGetLastError();
}

cudaError_t launch_unmerge(const MergeParams& mp, int32_t* status, cudaStream_t s, int* nl)
{
    const size_t smem = unmerge_smem(mp);
    cudaError_t e = cudaFuncSetAttribute(k4_unmerge, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k4_unmerge<<<mp.blk_base[mp.T], kMergeThreads, smem, s>>>(mp, status);
    *nl += 1;
    return cudaGetLastError();
}

}  // namespace tt
