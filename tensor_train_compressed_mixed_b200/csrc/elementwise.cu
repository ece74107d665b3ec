// Elementwise kernels over the T*k core buffers of a handle: zero fill of the
// gradient buffers and the SGD step G <- G - lr * dG (the benchmark's training
// step; the FlowTT pages leave the optimiser open, plain SGD is the reading).
// One launch covers every buffer: block x finds its buffer by binary search
// over the per-buffer chunk prefix sums and handles one 8192-float chunk,
// with 16-byte vector accesses (buffers are 16-byte aligned) and a scalar tail.
#include "tt_common.cuh"

namespace tt {

__device__ __forceinline__ int find_buffer(const BufferList& bl, int64_t chunk)
{
    int a = 0, b = bl.count;  // chunk_start[a] <= chunk < chunk_start[b]
    while (b - a > 1) {
        const int m = (a + b) >> 1;
        if (bl.chunk_start[m] <= chunk) a = m; else b = m;
    }
    return a;
}

__global__ void __launch_bounds__(256) k_fill_zero(BufferList bl, const int32_t* status)
{
    if (has_error(status)) return;
    const int64_t chunk = blockIdx.x;
    const int buf = find_buffer(bl, chunk);
    const int64_t lo = (chunk - bl.chunk_start[buf]) * kElemChunk;
    const int64_t hi = min64(lo + kElemChunk, bl.size[buf]);
    float* p = bl.a[buf];
    const int64_t hi4 = lo + ((hi - lo) & ~int64_t(3));
    for (int64_t i = lo + 4 * threadIdx.x; i < hi4; i += 4 * blockDim.x)
        *reinterpret_cast<float4*>(p + i) = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t i = hi4 + threadIdx.x; i < hi; i += blockDim.x) p[i] = 0.f;
}

__global__ void __launch_bounds__(256) k_sgd(BufferList bl, float lr, const int32_t* status)
{
    if (has_error(status)) return;
    const int64_t chunk = blockIdx.x;
    const int buf = find_buffer(bl, chunk);
    const int64_t lo = (chunk - bl.chunk_start[buf]) * kElemChunk;
    const int64_t hi = min64(lo + kElemChunk, bl.size[buf]);
    float* p = bl.a[buf];
    const float* g = bl.b[buf];
    const int64_t hi4 = lo + ((hi - lo) & ~int64_t(3));
    for (int64_t i = lo + 4 * threadIdx.x; i < hi4; i += 4 * blockDim.x) {
        float4 w = *reinterpret_cast<const float4*>(p + i);
        const float4 d = __ldg(reinterpret_cast<const float4*>(g + i));
        w.x = fmaf(-lr, d.x, w.x);
        w.y = fmaf(-lr, d.y, w.y);
        w.z = fmaf(-lr, d.z, w.z);
        w.w = fmaf(-lr, d.w, w.w);
        *reinterpret_cast<float4*>(p + i) = w;
    }
    for (int64_t i = hi4 + threadIdx.x; i < hi; i += blockDim.x) p[i] = fmaf(-lr, g[i], p[i]);
}

cudaError_t launch_fill_zero(const BufferList& bl, int32_t* status, cudaStream_t s, int* nl)
{
    const int64_t chunks = bl.chunk_start[bl.count];
    if (chunks <= 0) return cudaSuccess;
    k_fill_zero<<<(unsigned)chunks, 256, 0, s>>>(bl, status);
    *nl += 1;
    return cudaGetLastError();
}

cudaError_t launch_sgd(const BufferList& bl, float lr, int32_t* status, cudaStream_t s, int* nl)
{
    const int64_t chunks = bl.chunk_start[bl.count];
    if (chunks <= 0) return cudaSuccess;
    k_sgd<<<(unsigned)chunks, 256, 0, s>>>(bl, lr, status);
    *nl += 1;
    return cudaGetLastError();
}

}  // namespace tt
