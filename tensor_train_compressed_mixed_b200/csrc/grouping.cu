// Index grouping for TT gather: key extraction, stable LSD radix sort, and
// unique + prefix run-length segmentation.
//
// FlowTT (Exploiting Computation Flow Reuse in Irregular Tensor-Train
// Embedding), section 3.3 "Flow-Aligned Prefix-Based Index Grouping" and the
// section 4 latency breakdown: the batch is sorted, deduplicated, converted
// to mixed radix, reduced to prefixes and run-length encoded into prefix
// groups.  Here a key is (table << ibits) | row.  Because the mixed-radix
// digits of a row are ordered most-significant first, sorting keys sorts
// lookups by (table, i_1, ..., i_k), so equal rows and equal prefixes
// (row / n_k) are contiguous, and the segmentation is two run-length passes
// over the sorted keys.
#include "tt_common.cuh"

namespace tt {

// ---------------------------------------------------------------------------
// Keys.  One block per 256 bags: the block stages its 257 offsets in shared
// memory (clamped to [0, L], so a broken partition can never index outside
// the arrays), checks that they are a monotone partition, and then walks its
// lookups coalesced, finding each lookup's bag by binary search.
// ---------------------------------------------------------------------------
constexpr int kBagsPerBlock = 256;

template <typename K>
__global__ void __launch_bounds__(256) k_make_keys(KeyParams kp, const int64_t* __restrict__ indices,
                                                   const int64_t* __restrict__ offsets,
                                                   K* __restrict__ keys, int32_t* __restrict__ vals,
                                                   int32_t* __restrict__ bag_of_pos, int32_t* status)
{
    __shared__ int64_t s_off[kBagsPerBlock + 1];
    if (has_error(status)) return;
    const int64_t nbags = (int64_t)kp.T * kp.B;
    const int64_t g0 = (int64_t)blockIdx.x * kBagsPerBlock;
    const int nb = (int)min64(kBagsPerBlock, nbags - g0);
    for (int j = threadIdx.x; j <= nb; j += blockDim.x) {
        int64_t o = offsets[g0 + j];
        if (o < 0 || o > kp.L) {
            raise_error(status, TT_ERR_OFFSETS, (int)min64(g0 + j, INT32_MAX));
            o = o < 0 ? 0 : kp.L;
        }
        s_off[j] = o;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (g0 == 0 && s_off[0] != 0) raise_error(status, TT_ERR_OFFSETS, 0);
        if (g0 + nb == nbags && s_off[nb] != kp.L) raise_error(status, TT_ERR_OFFSETS, (int)min64(nbags, INT32_MAX));
    }
    for (int j = threadIdx.x; j < nb; j += blockDim.x)
        if (s_off[j + 1] < s_off[j]) raise_error(status, TT_ERR_OFFSETS, (int)min64(g0 + j, INT32_MAX));
    const int64_t lo = s_off[0], hi = s_off[nb];
    const uint64_t rmask = (uint64_t(1) << kp.ibits) - 1;
    // the block's bags span at most two tables when B >= 256: one division per block
    const int t0 = (int)(g0 / kp.B);
    const int64_t g_next = (int64_t)(t0 + 1) * kp.B;   // first bag of the next table
    const bool two_max = kp.B >= kBagsPerBlock;
    for (int64_t l = lo + threadIdx.x; l < hi; l += blockDim.x) {
        // bag = last j with s_off[j] <= l (upper bound - 1), clamped to [0, nb)
        int a = 0, b = nb;  // invariant: s_off[a] <= l < s_off[b] when monotone
        while (b - a > 1) {
            const int m = (a + b) >> 1;
            if (s_off[m] <= l) a = m; else b = m;
        }
        const int64_t g = g0 + a;
        const int t = two_max ? t0 + (g >= g_next ? 1 : 0) : (int)(g / kp.B);
        int64_t row = indices[l];
        if (row < 0 || row >= (int64_t)kp.nrows[t]) {
            raise_error(status, TT_ERR_INDEX_RANGE, (int)min64(l, INT32_MAX));
            row = 0;
        }
        keys[l] = (K)(((uint64_t)t << kp.ibits) | ((uint64_t)row & rmask));
        vals[l] = (int32_t)l;
        bag_of_pos[l] = (int32_t)g;
    }
}

cudaError_t launch_make_keys(const KeyParams& kp, bool key64, const int64_t* indices,
                             const int64_t* offsets, void* keys, int32_t* vals,
                             int32_t* bag_of_pos, int32_t* status, cudaStream_t s, int* nl)
{
    const int64_t nbags = (int64_t)kp.T * kp.B;
    const int grid = (int)ceil_div(nbags, kBagsPerBlock);
    if (grid == 0) return cudaSuccess;
    if (key64)
        k_make_keys<uint64_t><<<grid, 256, 0, s>>>(kp, indices, offsets, (uint64_t*)keys, vals,
                                                  bag_of_pos, status);
    else
        k_make_keys<uint32_t><<<grid, 256, 0, s>>>(kp, indices, offsets, (uint32_t*)keys, vals,
                                                  bag_of_pos, status);
    *nl += 1;
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Stable LSD radix sort, 8 bits per pass, three kernels per pass:
//   hist     per-tile digit counts, stored digit-major: hist[d * tiles + tile]
//   colscan  one block per digit: exclusive scan of its row over tiles, and
//            the digit's total
//   scatter  per tile: stable rank of each key among equal digits (warp
//            match + per-warp counters, warps in tile order), staged in
//            shared memory by digit, then written out coalesced at
//            digit base + tile base + rank
// A tile is 256 threads x kSortItems keys; warp w owns keys [w*32*kSortItems, (w+1)*32*kSortItems) of
// the tile, visited in (item, lane) order, which is input order.  The scatter is held to four
// blocks per SM with 32-bit keys (64 registers; three with 64-bit keys), which takes the
// 4-pass sort of 17.9 M keys from 0.705 to 0.627 ms despite a few spilled registers.
// ---------------------------------------------------------------------------
template <typename K>
__global__ void __launch_bounds__(256) k_radix_hist(const K* __restrict__ kin, int64_t n,
                                                    const int64_t* __restrict__ dev_n, int shift,
                                                    uint32_t* __restrict__ hist, int tiles,
                                                    const int32_t* status)
{
    __shared__ uint32_t s_cnt[256];
    if (has_error(status)) return;
    if (dev_n) n = min64(n, *dev_n);
    s_cnt[threadIdx.x] = 0;
    __syncthreads();
    const int64_t base = (int64_t)blockIdx.x * kSortTile;
    const int cnt = (int)min64(kSortTile, n - base);
    for (int e = threadIdx.x; e < cnt; e += 256)
        atomicAdd(&s_cnt[(uint32_t)(kin[base + e] >> shift) & 255u], 1u);
    __syncthreads();
    hist[(int64_t)threadIdx.x * tiles + blockIdx.x] = s_cnt[threadIdx.x];
}

__global__ void __launch_bounds__(1024) k_radix_colscan(uint32_t* __restrict__ hist, int tiles,
                                                       uint32_t* __restrict__ digit_total,
                                                       const int32_t* status)
{
    __shared__ uint32_t s_w[32];
    if (has_error(status)) return;
    uint32_t* row = hist + (int64_t)blockIdx.x * tiles;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    uint32_t carry = 0;
    for (int b0 = 0; b0 < tiles; b0 += 1024) {
        const int i = b0 + threadIdx.x;
        const uint32_t v = i < tiles ? row[i] : 0u;
        uint32_t x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t y = __shfl_up_sync(kFull, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) s_w[wid] = x;
        __syncthreads();
        if (wid == 0) {
            uint32_t w = s_w[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                uint32_t y = __shfl_up_sync(kFull, w, o);
                if (lane >= o) w += y;
            }
            s_w[lane] = w;
        }
        __syncthreads();
        const uint32_t excl = carry + (wid ? s_w[wid - 1] : 0u) + x - v;
        if (i < tiles) row[i] = excl;
        carry += s_w[31];
        __syncthreads();
    }
    if (threadIdx.x == 0) digit_total[blockIdx.x] = carry;
}

template <typename K>
__global__ void __launch_bounds__(256, sizeof(K) == 4 ? 4 : 3) k_radix_scatter(const K* __restrict__ kin,
                                                       const int32_t* __restrict__ vin,
                                                       K* __restrict__ kout, int32_t* __restrict__ vout,
                                                       int64_t n, const int64_t* __restrict__ dev_n,
                                                       int shift,
                                                       const uint32_t* __restrict__ hist,
                                                       const uint32_t* __restrict__ digit_total,
                                                       int tiles, const int32_t* status)
{
    __shared__ uint32_t s_wcnt[8][256];
    __shared__ uint32_t s_tile_start[256];
    __shared__ uint32_t s_gbase[256];
    __shared__ uint32_t s_tmp[8];
    __shared__ K s_keys[kSortTile];
    __shared__ int32_t s_vals[kSortTile];
    if (has_error(status)) return;

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    if (dev_n) n = min64(n, *dev_n);
    const int64_t base = (int64_t)blockIdx.x * kSortTile;
    const int cnt = (int)min64(kSortTile, n - base);
    if (cnt <= 0) return;
    for (int i = tid; i < 8 * 256; i += 256) (&s_wcnt[0][0])[i] = 0;
    {
        uint32_t tot;
        const uint32_t dbase = block256_exclusive_scan<uint32_t>(digit_total[tid], &tot, s_tmp);
        s_gbase[tid] = dbase + hist[(int64_t)tid * tiles + blockIdx.x];
    }
    __syncthreads();

    K key[kSortItems];
    int32_t val[kSortItems];
    uint32_t rank[kSortItems];
    int dig[kSortItems];
    const int sub = wid * 32 * kSortItems;
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll
    for (int j = 0; j < kSortItems; ++j) {
        const int e = sub + j * 32 + lane;
        const bool valid = e < cnt;
        key[j] = valid ? kin[base + e] : K(0);
        val[j] = valid ? vin[base + e] : 0;
        dig[j] = valid ? (int)((uint32_t)(key[j] >> shift) & 255u) : 256;
        const unsigned peers = __match_any_sync(kFull, dig[j]);
        const uint32_t pre = valid ? s_wcnt[wid][dig[j]] : 0u;
        rank[j] = pre + (uint32_t)__popc(peers & lt);
        __syncwarp();
        if (valid && (peers & lt) == 0) s_wcnt[wid][dig[j]] = pre + (uint32_t)__popc(peers);
        __syncwarp();
    }
    __syncthreads();
    {
        uint32_t run = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            const uint32_t c = s_wcnt[w][tid];
            s_wcnt[w][tid] = run;
            run += c;
        }
        uint32_t tot;
        s_tile_start[tid] = block256_exclusive_scan<uint32_t>(run, &tot, s_tmp);
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kSortItems; ++j) {
        if (dig[j] < 256) {
            const uint32_t p = s_tile_start[dig[j]] + s_wcnt[wid][dig[j]] + rank[j];
            s_keys[p] = key[j];
            s_vals[p] = val[j];
        }
    }
    __syncthreads();
    for (int e = tid; e < cnt; e += 256) {
        const K k = s_keys[e];
        const int d = (int)((uint32_t)(k >> shift) & 255u);
        const int64_t o = (int64_t)s_gbase[d] + (e - (int)s_tile_start[d]);
        kout[o] = k;
        vout[o] = s_vals[e];
    }
}

template <typename K>
static cudaError_t radix_sort_t(int64_t n, int bits, SortBuffers& sb, int* which, int32_t* status,
                                cudaStream_t s, int* nl, const int64_t* dev_n)
{
    const int tiles = (int)ceil_div(n, kSortTile);
    int cur = 0;
    for (int shift = 0; shift < bits; shift += 8) {
        const K* kin = (const K*)sb.keys[cur];
        k_radix_hist<K><<<tiles, 256, 0, s>>>(kin, n, dev_n, shift, sb.hist, tiles, status);
        k_radix_colscan<<<256, 1024, 0, s>>>(sb.hist, tiles, sb.digit_total, status);
        k_radix_scatter<K><<<tiles, 256, 0, s>>>(kin, sb.vals[cur], (K*)sb.keys[cur ^ 1],
                                                 sb.vals[cur ^ 1], n, dev_n, shift, sb.hist,
                                                 sb.digit_total, tiles, status);
        cur ^= 1;
        *nl += 3;
    }
    *which = cur;
    return cudaGetLastError();
}

cudaError_t radix_sort_pairs(bool key64, int64_t n, int bits, SortBuffers& sb, int* which,
                             int32_t* status, cudaStream_t s, int* nl, const int64_t* dev_n)
{
    if (n <= 0) {
        *which = 0;
        return cudaSuccess;
    }
    return key64 ? radix_sort_t<uint64_t>(n, bits, sb, which, status, s, nl, dev_n)
                 : radix_sort_t<uint32_t>(n, bits, sb, which, status, s, nl, dev_n);
}

// ---------------------------------------------------------------------------
// Segmentation.  Over sorted keys, flag u marks the first lookup of each
// distinct key and flag g the first lookup of each prefix group (a new
// table, or a new row / n_k).  Both are counted in one uint64 (u in the low
// word, g in the high word) by a reduce / scan-of-partials / write scheme:
//   reduce   per 4096-lookup tile: sum of packed flags
//   partials one block: exclusive scan of tile sums; totals -> U, G
//   write    per tile: block scan; each flagged lookup writes its run start
//            (uniq_start, uniq_keys, grp_start); every lookup writes its bag
// ---------------------------------------------------------------------------
// The 16 consecutive sorted keys of one thread (l = base .. base + 15) and the key before them.
// Runs that lie inside [0, L) are read with 16-byte loads (the key arrays are 256-byte aligned and
// base is a multiple of 16 keys); a ragged last run reads key by key.
template <typename K>
__device__ __forceinline__ void load_run16(const K* __restrict__ keys, int64_t base, int64_t L, K (&k)[16], K& kprev)
{
    if (base + 16 <= L) {
        const uint4* p = reinterpret_cast<const uint4*>(keys + base);
        if constexpr (sizeof(K) == 4) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint4 v = p[i];
                k[4 * i] = v.x;
                k[4 * i + 1] = v.y;
                k[4 * i + 2] = v.z;
                k[4 * i + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint4 v = p[i];
                k[2 * i] = ((uint64_t)v.y << 32) | v.x;
                k[2 * i + 1] = ((uint64_t)v.w << 32) | v.z;
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) k[j] = base + j < L ? keys[base + j] : K(0);
    }
    kprev = base > 0 && base <= L ? keys[base - 1] : K(0);
}

// Segment flags of sorted position l from its key k and the previous key q: bit 0 = first
// lookup of a distinct key, bit 32 = first distinct key of a prefix group (new table, or a new
// row / n_k; every distinct key in unique-only grouping).
template <typename K>
__device__ __forceinline__ uint64_t seg_flags_kq(K k, K q, int64_t l, const KeyParams& kp)
{
    if (l == 0) return 1ull | (1ull << 32);
    if (k == q) return 0ull;
    if (kp.unique_only) return 1ull | (1ull << 32);
    const uint32_t t = (uint32_t)(k >> kp.ibits), tq = (uint32_t)(q >> kp.ibits);
    if (t != tq) return 1ull | (1ull << 32);
    const uint64_t m = (uint64_t(1) << kp.ibits) - 1;
    const uint32_t nl = kp.nlast[t < kMaxT ? t : 0];
    const bool ng = ((uint32_t)(k & m) / nl) != ((uint32_t)(q & m) / nl);
    return 1ull | ((uint64_t)ng << 32);
}

template <typename K>
__global__ void __launch_bounds__(256) k_seg_reduce(KeyParams kp, const K* __restrict__ keys,
                                                    uint64_t* __restrict__ partials,
                                                    const int32_t* status)
{
    __shared__ uint64_t s_tmp[8];
    if (has_error(status)) return;
    const int64_t base = (int64_t)blockIdx.x * kScanTile + (int64_t)threadIdx.x * 16;
    K k[16], kprev;
    load_run16(keys, base, kp.L, k, kprev);
    uint64_t acc = 0;
#pragma unroll
    for (int j = 0; j < 16; ++j)
        if (base + j < kp.L) acc += seg_flags_kq(k[j], j ? k[j - 1] : kprev, base + j, kp);
    uint64_t tot;
    block256_exclusive_scan<uint64_t>(acc, &tot, s_tmp);
    if (threadIdx.x == 0) partials[blockIdx.x] = tot;
}

__global__ void __launch_bounds__(1024) k_seg_partials(uint64_t* __restrict__ partials, int nb,
                                                      WsCounters* counters, const int32_t* status)
{
    __shared__ uint64_t s_w[32];
    if (has_error(status)) return;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    uint64_t carry = 0;
    for (int b0 = 0; b0 < nb; b0 += 1024) {
        const int i = b0 + threadIdx.x;
        const uint64_t v = i < nb ? partials[i] : 0ull;
        uint64_t x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint64_t y = __shfl_up_sync(kFull, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) s_w[wid] = x;
        __syncthreads();
        if (wid == 0) {
            uint64_t w = s_w[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                uint64_t y = __shfl_up_sync(kFull, w, o);
                if (lane >= o) w += y;
            }
            s_w[lane] = w;
        }
        __syncthreads();
        const uint64_t excl = carry + (wid ? s_w[wid - 1] : 0ull) + x - v;
        if (i < nb) partials[i] = excl;
        carry += s_w[31];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        counters->num_unique = (int64_t)(carry & 0xffffffffull);
        counters->num_groups = (int64_t)(carry >> 32);
    }
}

template <typename K>
__global__ void __launch_bounds__(256) k_seg_write(KeyParams kp, const K* __restrict__ keys,
                                                   const int32_t* __restrict__ perm,
                                                   const int32_t* __restrict__ bag_of_pos,
                                                   const uint64_t* __restrict__ partials,
                                                   K* __restrict__ uniq_keys,
                                                   int32_t* __restrict__ uniq_start,
                                                   int32_t* __restrict__ grp_start,
                                                   int32_t* __restrict__ bag_sorted,
                                                   int32_t* __restrict__ uid_at_pos,
                                                   int32_t* __restrict__ uid_sorted,
                                                   const int32_t* status)
{
    __shared__ uint64_t s_tmp[8];
    if (has_error(status)) return;
    const int64_t base = (int64_t)blockIdx.x * kScanTile + (int64_t)threadIdx.x * 16;
    const bool full = base + 16 <= kp.L;
    // every load first (independent, vectorised where the run is whole), then the scan and stores
    K k[16], kprev;
    load_run16(keys, base, kp.L, k, kprev);
    int32_t pv[16], bg[16];
    if (full) {
        const int4* pp = reinterpret_cast<const int4*>(perm + base);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int4 v = pp[i];
            pv[4 * i] = v.x;
            pv[4 * i + 1] = v.y;
            pv[4 * i + 2] = v.z;
            pv[4 * i + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) pv[j] = base + j < kp.L ? perm[base + j] : 0;
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) bg[j] = base + j < kp.L ? bag_of_pos[pv[j]] : 0;
    uint64_t f[16];
    uint64_t acc = 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        f[j] = base + j < kp.L ? seg_flags_kq(k[j], j ? k[j - 1] : kprev, base + j, kp) : 0ull;
        acc += f[j];
    }
    uint64_t tot;
    uint64_t run = partials[blockIdx.x] + block256_exclusive_scan<uint64_t>(acc, &tot, s_tmp);
    int32_t us[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const int64_t l = base + j;
        const bool in = l < kp.L;
        const uint32_t uid = (uint32_t)(run & 0xffffffffull);  // distinct keys before l
        const uint32_t gid = (uint32_t)(run >> 32);
        if (in && (f[j] & 1ull)) {
            uniq_start[uid] = (int32_t)l;
            uniq_keys[uid] = k[j];
            if (f[j] >> 32) grp_start[gid] = (int32_t)uid;
        }
        run += f[j];
        us[j] = (int32_t)(run & 0xffffffffull) - 1;   // inclusive count - 1
        if (in && uid_at_pos) uid_at_pos[pv[j]] = us[j];
        if (l == kp.L - 1) {
            uniq_start[(uint32_t)(run & 0xffffffffull)] = (int32_t)kp.L;
            grp_start[(uint32_t)(run >> 32)] = (int32_t)(run & 0xffffffffull);
        }
    }
    if (full) {
        int4* bs = reinterpret_cast<int4*>(bag_sorted + base);
#pragma unroll
        for (int i = 0; i < 4; ++i) bs[i] = make_int4(bg[4 * i], bg[4 * i + 1], bg[4 * i + 2], bg[4 * i + 3]);
        if (uid_sorted) {
            int4* ps = reinterpret_cast<int4*>(uid_sorted + base);
#pragma unroll
            for (int i = 0; i < 4; ++i) ps[i] = make_int4(us[4 * i], us[4 * i + 1], us[4 * i + 2], us[4 * i + 3]);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            if (base + j >= kp.L) break;
            bag_sorted[base + j] = bg[j];
            if (uid_sorted) uid_sorted[base + j] = us[j];
        }
    }
}

cudaError_t launch_segment(const KeyParams& kp, bool key64, const void* sorted_keys,
                           const int32_t* perm, const int32_t* bag_of_pos, void* uniq_keys,
                           int32_t* uniq_start, int32_t* grp_start, int32_t* bag_sorted,
                           uint64_t* partials, WsCounters* counters, int32_t* uid_at_pos,
                           int32_t* uid_sorted, int32_t* status, cudaStream_t s, int* nl)
{
    const int nb = (int)ceil_div(kp.L, kScanTile);
    if (nb == 0) return cudaSuccess;
    if (key64) {
        k_seg_reduce<uint64_t><<<nb, 256, 0, s>>>(kp, (const uint64_t*)sorted_keys, partials, status);
        k_seg_partials<<<1, 1024, 0, s>>>(partials, nb, counters, status);
        k_seg_write<uint64_t><<<nb, 256, 0, s>>>(kp, (const uint64_t*)sorted_keys, perm, bag_of_pos,
                                                 partials, (uint64_t*)uniq_keys, uniq_start,
                                                 grp_start, bag_sorted, uid_at_pos, uid_sorted,
                                                 status);
    } else {
        k_seg_reduce<uint32_t><<<nb, 256, 0, s>>>(kp, (const uint32_t*)sorted_keys, partials, status);
        k_seg_partials<<<1, 1024, 0, s>>>(partials, nb, counters, status);
        k_seg_write<uint32_t><<<nb, 256, 0, s>>>(kp, (const uint32_t*)sorted_keys, perm, bag_of_pos,
                                                 partials, (uint32_t*)uniq_keys, uniq_start,
                                                 grp_start, bag_sorted, uid_at_pos, uid_sorted,
                                                 status);
    }
    *nl += 3;
    return cudaGetLastError();
}

}  // namespace tt
