// Work planning for the shape-specialised fused kernels.
//
// FlowTT section 3.4 ("Dynamic Load Balancing via Persistent Threads and Work
// Stealing"): prefix groups become block-level work units, long runs are cut
// into chunks, and persistent blocks take chunks dynamically.  Here a work
// unit is a *column group*: all prefix groups of one table that share the
// digit of the largest prefix slice (i_2 for three cores), so that slice is
// staged in shared memory once and reused by every prefix of the unit.  The
// plan
//   1. keys every prefix group by its column (table, i_c) and counts columns,
//   2. stable-sorts the groups by column (so each column's groups stay in
//      canonical order and results do not depend on the schedule),
//   3. scans the column counts into column starts and chunk bases,
//   4. writes one record per chunk (at most MP groups of one column) with its
//      distinct-row total,
//   5. splits chunks of more than kSplitRows distinct rows into row-range
//      subtasks (the stealing granule of FlowTT section 3.4), numbers the
//      split chunks' checkpoint slots (TT_SCHED_STEAL_L2), and gives every
//      persistent block of the forward an owner range: an equal share of the
//      subtasks, contiguous in column order (the static prefix mapping the
//      pages start from).  Pooling tasks (NB bags of one table) follow.
#include "tt_common.cuh"

namespace tt {

__device__ __forceinline__ void group_col(const PlanParams& pp, uint64_t key, int* t_out,
                                          uint32_t* ic_out, uint32_t* i1_out)
{
    const int t = (int)(key >> pp.ibits);
    uint32_t row = (uint32_t)(key & ((uint64_t(1) << pp.ibits) - 1));
    uint32_t dig[kMaxK];
    for (int j = pp.k - 1; j >= 0; --j) {
        const uint32_t nj = pp.n[t][j];
        dig[j] = row % nj;
        row /= nj;
    }
    *t_out = t;
    *ic_out = dig[pp.col_digit];
    *i1_out = dig[0];
}

template <typename K>
__global__ void __launch_bounds__(256) k_plan_keys(PlanParams pp, const K* __restrict__ uniq_keys,
                                                   const int32_t* __restrict__ grp_start,
                                                   const WsCounters* __restrict__ counters,
                                                   uint32_t* __restrict__ pkeys,
                                                   int32_t* __restrict__ pvals,
                                                   int32_t* __restrict__ col_count,
                                                   int32_t* __restrict__ col_rows,
                                                   const int32_t* status)
{
    if (has_error(status)) return;
    const int64_t G = counters->num_groups;
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < G;
         g += (int64_t)gridDim.x * blockDim.x) {
        int t;
        uint32_t ic, i1;
        const int u0 = grp_start[g];
        group_col(pp, (uint64_t)uniq_keys[u0], &t, &ic, &i1);
        const uint32_t col = (uint32_t)pp.col_base[t] + ic;
        pkeys[g] = col;
        pvals[g] = (int32_t)g;
        atomicAdd(&col_count[col], 1);
        atomicAdd(&col_rows[col], grp_start[g + 1] - u0);
    }
}

// One block: the backward's column queue.  TT_SCHED_STATIC: every column in index order (the
// static round robin of the backward).  Stealing modes: the non-empty columns, heavy ones first
// (cost = distinct rows + 4 x prefix groups above twice the mean), each part in index order, so
// the dynamic queue starts the long column groups early while blocks working at the same time
// stay on neighbouring columns of one table (its gradient rows and last slices shared in L2).
// Each thread takes a contiguous range of columns; a block scan of the per-range counts gives
// every column its position (stable).
__global__ void __launch_bounds__(1024) k_plan_order(PlanParams pp, const int32_t* __restrict__ col_count,
                                                    const int32_t* __restrict__ col_rows,
                                                    int32_t* __restrict__ col_order, PlanHeader* __restrict__ hdr,
                                                    const int32_t* status)
{
    __shared__ long long s_sum[32];
    __shared__ int s_w[2][32];
    if (has_error(status)) return;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    if (pp.sched == TT_SCHED_STATIC) {
        for (int c = tid; c < pp.ncols; c += 1024) col_order[c] = c;
        if (tid == 0) hdr->ncols_busy = pp.ncols;
        return;
    }
    const int per = (pp.ncols + 1023) / 1024;
    const int lo = min(pp.ncols, tid * per), hi = min(pp.ncols, lo + per);
    auto cost = [&](int c) { return (long long)col_rows[c] + 4ll * col_count[c]; };
    // mean cost of the non-empty columns
    long long sum = 0;
    int busy = 0;
    for (int c = lo; c < hi; ++c) {
        const long long k = cost(c);
        sum += k;
        busy += k > 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        sum += __shfl_xor_sync(kFull, sum, o);
        busy += __shfl_xor_sync(kFull, busy, o);
    }
    if (lane == 0) {
        s_sum[wid] = sum;
        s_w[0][wid] = busy;
    }
    __syncthreads();
    long long tot = 0;
    int nbusy = 0;
    for (int w = 0; w < 32; ++w) {
        tot += s_sum[w];
        nbusy += s_w[0][w];
    }
    __syncthreads();
    const long long heavy = nbusy > 0 ? 2 * tot / nbusy : 0;   // cost above this: a heavy column
    // stable two-way partition of the non-empty columns: heavy first
    int nh = 0, nl = 0;
    for (int c = lo; c < hi; ++c) {
        const long long k = cost(c);
        nh += k > heavy;
        nl += k > 0 && k <= heavy;
    }
    int x[2] = {nh, nl};
#pragma unroll
    for (int q = 0; q < 2; ++q) {
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, x[q], o);
            if (lane >= o) x[q] += y;
        }
        if (lane == 31) s_w[q][wid] = x[q];
    }
    __syncthreads();
    if (wid == 0) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            int v = s_w[q][lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(kFull, v, o);
                if (lane >= o) v += y;
            }
            s_w[q][lane] = v;
        }
    }
    __syncthreads();
    const int H = s_w[0][31];
    int ph = (wid ? s_w[0][wid - 1] : 0) + x[0] - nh;
    int pl = H + (wid ? s_w[1][wid - 1] : 0) + x[1] - nl;
    for (int c = lo; c < hi; ++c) {
        const long long k = cost(c);
        if (k > heavy) col_order[ph++] = c;
        else if (k > 0) col_order[pl++] = c;
    }
    if (tid == 0) hdr->ncols_busy = H + s_w[1][31];
}

// One block: column starts, chunk bases and the task layout.
__global__ void __launch_bounds__(1024) k_plan_cols(PlanParams pp,
                                                   const int32_t* __restrict__ col_count,
                                                   int32_t* __restrict__ col_start,
                                                   int32_t* __restrict__ chunk_base,
                                                   PlanHeader* __restrict__ hdr,
                                                   const int32_t* status)
{
    __shared__ int32_t s_w[2][32];
    __shared__ int32_t s_carry[2];
    if (has_error(status)) return;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (threadIdx.x == 0) s_carry[0] = s_carry[1] = 0;
    __syncthreads();
    for (int b0 = 0; b0 < pp.ncols; b0 += 1024) {
        const int c = b0 + threadIdx.x;
        const int cnt = c < pp.ncols ? col_count[c] : 0;
        const int v[2] = {cnt, (cnt + pp.MP - 1) / pp.MP};
        int x[2] = {v[0], v[1]};
#pragma unroll
        for (int q = 0; q < 2; ++q) {
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(kFull, x[q], o);
                if (lane >= o) x[q] += y;
            }
            if (lane == 31) s_w[q][wid] = x[q];
        }
        __syncthreads();
        if (wid == 0) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                int w = s_w[q][lane];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(kFull, w, o);
                    if (lane >= o) w += y;
                }
                s_w[q][lane] = w;
            }
        }
        __syncthreads();
        if (c < pp.ncols) {
            col_start[c] = s_carry[0] + (wid ? s_w[0][wid - 1] : 0) + x[0] - v[0];
            chunk_base[c] = s_carry[1] + (wid ? s_w[1][wid - 1] : 0) + x[1] - v[1];
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            s_carry[0] += s_w[0][31];
            s_carry[1] += s_w[1][31];
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        col_start[pp.ncols] = s_carry[0];
        chunk_base[pp.ncols] = s_carry[1];
        hdr->nP = (int)((pp.B + pp.NB - 1) / pp.NB);
        hdr->nchunks = s_carry[1];
        hdr->pool_head = 0;
        hdr->col_head = 0;
    }
    if (threadIdx.x < pp.T) hdr->done[threadIdx.x] = 0;
}

__global__ void __launch_bounds__(256) k_plan_chunks(PlanParams pp, const WsCounters* __restrict__ counters,
                                                     const uint32_t* __restrict__ sorted_cols,
                                                     const int32_t* __restrict__ col_count,
                                                     const int32_t* __restrict__ col_start,
                                                     const int32_t* __restrict__ chunk_base,
                                                     const int4* __restrict__ grec,
                                                     int4* __restrict__ chunks, int32_t* __restrict__ crow,
                                                     const int32_t* status)
{
    if (has_error(status)) return;
    const int64_t G = counters->num_groups;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < G; i += stride) {
        const uint32_t c = sorted_cols[i];
        const int r = (int)(i - col_start[c]);
        if (r % pp.MP != 0) continue;
        // table of column c: last t with col_base[t] <= c
        int t = 0;
        while (t + 1 < pp.T && (uint32_t)pp.col_base[t + 1] <= c) ++t;
        const int cid = chunk_base[c] + r / pp.MP;
        const int cnt = min(pp.MP, col_count[c] - r);
        int rows = 0;
        for (int q = 0; q < cnt; ++q) rows += grec[i + q].y;
        chunks[cid] = make_int4((int)i, cnt, t, (int)(c - (uint32_t)pp.col_base[t]));
        crow[cid] = rows;
    }
}


// One block: subtask bases and checkpoint slots of every chunk (an exclusive scan of the
// subtask counts and of the split flags), subtasks per table, and the owner ranges.
__global__ void __launch_bounds__(1024) k_plan_split(PlanParams pp, const int32_t* __restrict__ crow,
                                                    const int32_t* __restrict__ chunk_base,
                                                    int32_t* __restrict__ sub_base, int32_t* __restrict__ slot_of,
                                                    PlanHeader* __restrict__ hdr,
                                                    unsigned long long* __restrict__ deque,
                                                    int32_t* __restrict__ exhausted, const int32_t* status)
{
    __shared__ int32_t s_w[2][32];
    if (has_error(status)) return;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int nch = hdr->nchunks;
    // a multiple of 4 chunks per thread, so each range starts 16-byte aligned (crow is 256-byte
    // aligned) and is read four row counts per load
    const int per = ((nch + 1023) / 1024 + 3) & ~3;
    const int lo = min(nch, tid * per), hi = min(nch, lo + per);
    auto rows4 = [&](int c, int (&r)[4]) {
        if (c + 4 <= hi) {
            const int4 v = *reinterpret_cast<const int4*>(crow + c);
            r[0] = v.x; r[1] = v.y; r[2] = v.z; r[3] = v.w;
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) r[i] = c + i < hi ? crow[c + i] : 0;
        }
    };
    int ns = 0, np = 0;
    for (int c = lo; c < hi; c += 4) {
        int r[4];
        rows4(c, r);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (c + i >= hi) break;
            const int k = subtasks_of(r[i], pp.split_rows);
            ns += k;
            np += k > 1;
        }
    }
    int x[2] = {ns, np};
#pragma unroll
    for (int q = 0; q < 2; ++q) {
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, x[q], o);
            if (lane >= o) x[q] += y;
        }
        if (lane == 31) s_w[q][wid] = x[q];
    }
    __syncthreads();
    if (wid == 0) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            int w = s_w[q][lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(kFull, w, o);
                if (lane >= o) w += y;
            }
            s_w[q][lane] = w;
        }
    }
    __syncthreads();
    int rs = (wid ? s_w[0][wid - 1] : 0) + x[0] - ns;
    int rp = (wid ? s_w[1][wid - 1] : 0) + x[1] - np;
    const bool ckpt = pp.sched == TT_SCHED_STEAL_L2;
    for (int c = lo; c < hi; c += 4) {
        int r[4];
        rows4(c, r);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (c + i >= hi) break;
            const int k = subtasks_of(r[i], pp.split_rows);
            sub_base[c + i] = rs;
            slot_of[c + i] = (ckpt && k > 1 && rp < pp.slot_cap) ? rp : -1;
            rs += k;
            rp += k > 1;
        }
    }
    const int S = s_w[0][31];
    if (tid == 0) {
        sub_base[nch] = S;
        hdr->nsub = S;
        hdr->nslots = ckpt ? min(s_w[1][31], pp.slot_cap) : 0;
    }
    __syncthreads();
    if (tid < pp.T)
        hdr->nC[tid] = sub_base[chunk_base[pp.col_base[tid + 1]]] - sub_base[chunk_base[pp.col_base[tid]]];
    for (int b = tid; b < pp.grid; b += 1024) {
        const unsigned long long h = (unsigned long long)(owner_start(S, b, pp.grid) + kDequeBias);
        const unsigned long long t = (unsigned long long)(owner_start(S, b + 1, pp.grid) + kDequeBias);
        deque[b] = (h << 32) | t;
        exhausted[b] = 0;
    }
}

// Subtask records: chunk c's rows split into n near-equal row ranges; the checkpoint flags
// start at zero.
__global__ void __launch_bounds__(256) k_plan_subs(const PlanHeader* __restrict__ hdr, const int32_t* __restrict__ crow,
                                                   const int32_t* __restrict__ sub_base,
                                                   const int32_t* __restrict__ slot_of, int4* __restrict__ subs,
                                                   int32_t* __restrict__ slot_flag, const int32_t* status)
{
    if (has_error(status)) return;
    const int nch = hdr->nchunks;
    for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < nch; c += gridDim.x * blockDim.x) {
        const int base = sub_base[c], n = sub_base[c + 1] - base, R = crow[c], slot = slot_of[c];
        for (int q = 0; q < n; ++q)
            subs[base + q] = make_int4(c, (int)((int64_t)R * q / n), (int)((int64_t)R * (q + 1) / n), slot);
        if (slot >= 0) slot_flag[slot] = 0;
    }
}

// Per sorted group position: first distinct row, row count and the first digit of the
// three-core view (i_1 = row / (n_2 n_3)), so that the fused kernels read a chunk's
// metadata with one load per group instead of a chain of three dependent loads.
template <typename K>
__global__ void __launch_bounds__(256) k_plan_grec(PlanParams pp, const WsCounters* __restrict__ counters,
                                                   const int32_t* __restrict__ sorted_groups,
                                                   const int32_t* __restrict__ grp_start,
                                                   const K* __restrict__ uniq_keys, int4* __restrict__ grec,
                                                   const int32_t* status)
{
    if (has_error(status)) return;
    const int64_t G = counters->num_groups;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < G; i += (int64_t)gridDim.x * blockDim.x) {
        const int g = sorted_groups[i];
        const int u0 = grp_start[g];
        const uint64_t key = (uint64_t)uniq_keys[u0];
        const int t = (int)(key >> pp.ibits);
        const uint32_t row = (uint32_t)(key & ((uint64_t(1) << pp.ibits) - 1));
        const uint32_t i1 = row / pp.n[t][pp.k - 1] / pp.n[t][pp.k - 2];
        grec[i] = make_int4(u0, grp_start[g + 1] - u0, (int)i1, 0);
    }
}

cudaError_t launch_plan(const PlanParams& pp, bool key64, const void* uniq_keys,
                        const int32_t* grp_start, const WsCounters* counters, int64_t max_groups,
                        PlanBuffers& pb, int32_t* status, cudaStream_t s, int* nl)
{
    cudaError_t e = cudaMemsetAsync(pb.col_count, 0, sizeof(int32_t) * (size_t)pp.ncols, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(pb.col_rows, 0, sizeof(int32_t) * (size_t)pp.ncols, s);
    if (e != cudaSuccess) return e;
    const int grid = 148 * 4;
    if (key64)
        k_plan_keys<uint64_t><<<grid, 256, 0, s>>>(pp, (const uint64_t*)uniq_keys, grp_start, counters,
                                                   (uint32_t*)pb.sort.keys[0], pb.sort.vals[0],
                                                   pb.col_count, pb.col_rows, status);
    else
        k_plan_keys<uint32_t><<<grid, 256, 0, s>>>(pp, (const uint32_t*)uniq_keys, grp_start, counters,
                                                   (uint32_t*)pb.sort.keys[0], pb.sort.vals[0],
                                                   pb.col_count, pb.col_rows, status);
    *nl += 1;
    int bits = 1;
    while ((1u << bits) < (uint32_t)pp.ncols) ++bits;
    int which = 0;
    e = radix_sort_pairs(false, max_groups, bits, pb.sort, &which, status, s, nl,
                         &counters->num_groups);
    if (e != cudaSuccess) return e;
    pb.sorted_groups = pb.sort.vals[which];
    k_plan_cols<<<1, 1024, 0, s>>>(pp, pb.col_count, pb.col_start, pb.chunk_base, pb.hdr, status);
    k_plan_order<<<1, 1024, 0, s>>>(pp, pb.col_count, pb.col_rows, pb.col_order, pb.hdr, status);
    if (key64)
        k_plan_grec<uint64_t><<<grid, 256, 0, s>>>(pp, counters, pb.sorted_groups, grp_start,
                                                   (const uint64_t*)uniq_keys, pb.grec, status);
    else
        k_plan_grec<uint32_t><<<grid, 256, 0, s>>>(pp, counters, pb.sorted_groups, grp_start,
                                                   (const uint32_t*)uniq_keys, pb.grec, status);
    k_plan_chunks<<<grid, 256, 0, s>>>(pp, counters, (const uint32_t*)pb.sort.keys[which], pb.col_count,
                                       pb.col_start, pb.chunk_base, pb.grec, pb.chunks, pb.crow, status);
    k_plan_split<<<1, 1024, 0, s>>>(pp, pb.crow, pb.chunk_base, pb.sub_base, pb.slot_of, pb.hdr, pb.deque,
                                    pb.exhausted, status);
    k_plan_subs<<<grid, 256, 0, s>>>(pb.hdr, pb.crow, pb.sub_base, pb.slot_of, pb.subs, pb.slot_flag, status);
    *nl += 7;
    return cudaGetLastError();
}

}  // namespace tt
