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
    for (int64_t l = lo + threadIdx.x; l < hi; l += blockDim.x) {
        // bag = last j with s_off[j] <= l (upper bound - 1), clamped to [0, nb)
        int a = 0, b = nb;  // invariant: s_off[a] <= l < s_off[b] when monotone
        while (b - a > 1) {
            const int m = (a + b) >> 1;
            if (s_off[m] <= l) a = m; else b = m;
        }
        const int64_t g = g0 + a;
        const int t = (int)(g / kp.B);
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
// Stable LSD radix sort, 8 bits per pass: one histogram kernel per sort and
// one kernel per pass.
//   hist_all  the digit counts of every pass in one read of the keys (the
//             count of a digit over the whole array does not depend on the
//             order the earlier passes leave), and the zeroing of the first
//             pass's look-back words
//   onesweep  per tile of kSortTile keys, tiles numbered in the order blocks
//             start (an atomic counter): the stable rank of each key among
//             equal digits (warp match + per-warp counters, warps in tile
//             order); the tile's count of every digit published at once; the
//             count of each digit over all earlier tiles found by decoupled
//             look-back (Merrill and Garland, "Single-pass Parallel Prefix Scan
//             with Decoupled Look-back", NVIDIA technical report NVR-2016-002);
//             keys staged in shared memory by digit, then written out coalesced
//             at digit base + earlier tiles + rank
// A tile is 256 threads x kSortItems keys; warp w owns keys
// [w*32*kSortItems, (w+1)*32*kSortItems) of the tile, visited in (item, lane)
// order, which is input order, so equal digits keep input order.
//
// Look-back words (one per tile and digit, 64 bits): bits 62-63 = 1 when the
// low bits hold the tile's own count, 2 when they hold the inclusive count
// over tiles 0..t, 0 while the tile has published nothing.  A block only
// waits for tiles with smaller numbers, which blocks that started before it
// hold, so the wait always ends; it is bounded all the same (kLookbackLimit
// polls, then TT_ERR_TIMEOUT), and it stops when another block has failed.
// Pass p reads the words of buffer p & 1 and zeroes, for its own tile, the
// words of the other buffer, which pass p + 1 reads.
// ---------------------------------------------------------------------------
constexpr uint64_t kLbOwn = 1ull << 62, kLbIncl = 2ull << 62, kLbCount = (1ull << 62) - 1;
constexpr int kLookbackLimit = 1 << 22;

__device__ __forceinline__ void st_relaxed_u64(uint64_t* p, uint64_t v)
{
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ uint64_t ld_relaxed_u64(const uint64_t* p)
{
    uint64_t v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

template <typename K>
__global__ void __launch_bounds__(256) k_radix_hist_all(const K* __restrict__ kin, int64_t n,
                                                        const int64_t* __restrict__ dev_n, int passes,
                                                        uint32_t* __restrict__ ghist, uint64_t* __restrict__ look0,
                                                        int64_t look_words, const int32_t* status)
{
    __shared__ uint32_t s_cnt[kSortPassMax][256];
    if (has_error(status)) return;
    if (dev_n) n = min64(n, *dev_n);
    const int tid = threadIdx.x, lane = tid & 31;
    const int64_t stride = (int64_t)gridDim.x * 256;
    for (int64_t i = (int64_t)blockIdx.x * 256 + tid; i < look_words; i += stride) look0[i] = 0ull;
    for (int i = tid; i < kSortPassMax * 256; i += 256) (&s_cnt[0][0])[i] = 0u;
    __syncthreads();
    // whole warps walk the keys; a lane past the end counts nothing (digit 256)
    for (int64_t base = (int64_t)blockIdx.x * 256; base < n; base += stride) {
        const int64_t e = base + tid;
        const bool valid = e < n;
        const K k = valid ? kin[e] : K(0);
        for (int p = 0; p < passes; ++p) {
            const int d = valid ? (int)((uint32_t)(k >> (8 * p)) & 255u) : 256;
            const unsigned peers = __match_any_sync(kFull, d);
            // one shared-memory add per distinct digit of the warp, by its lowest lane
            if (valid && (peers & ((1u << lane) - 1u)) == 0) atomicAdd(&s_cnt[p][d], (uint32_t)__popc(peers));
        }
    }
    __syncthreads();
    for (int p = 0; p < passes; ++p)
        if (s_cnt[p][tid]) atomicAdd(&ghist[p * 256 + tid], s_cnt[p][tid]);
}

template <typename K>
__global__ void __launch_bounds__(256) k_radix_onesweep(const K* __restrict__ kin, const int32_t* __restrict__ vin,
                                                        K* __restrict__ kout, int32_t* __restrict__ vout, int64_t n,
                                                        const int64_t* __restrict__ dev_n, int shift,
                                                        const uint32_t* __restrict__ ghist, uint64_t* look,
                                                        uint64_t* __restrict__ look_next, int* tile_counter,
                                                        int inject_spin, int32_t* status)
{
    __shared__ uint32_t s_wcnt[8][256];
    __shared__ uint32_t s_tile_start[256];
    __shared__ uint32_t s_gbase[256];
    __shared__ uint32_t s_tmp[8];
    __shared__ K s_keys[kSortTile];
    __shared__ int32_t s_vals[kSortTile];
    __shared__ int s_tile;

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    if (tid == 0) s_tile = atomicAdd(tile_counter, 1);
    __syncthreads();
    const int tile = s_tile;
    if (look_next) look_next[(int64_t)tile * 256 + tid] = 0ull;
    if (has_error(status)) return;
    if (dev_n) n = min64(n, *dev_n);
    const int64_t base = (int64_t)tile * kSortTile;
    const int cnt = (int)min64(kSortTile, n - base);
    if (cnt <= 0) return;   // only tiles after every tile that holds keys

    // the tile's keys and positions, all loads issued before the ranking
    K key[kSortItems];
    int32_t val[kSortItems];
    const int sub = wid * 32 * kSortItems;
#pragma unroll
    for (int j = 0; j < kSortItems; ++j) {
        const int e = sub + j * 32 + lane;
        key[j] = e < cnt ? kin[base + e] : K(0);
        val[j] = e < cnt ? vin[base + e] : 0;
    }
    for (int i = tid; i < 8 * 256; i += 256) (&s_wcnt[0][0])[i] = 0;
    __syncthreads();

    uint32_t rank[kSortItems];
    int dig[kSortItems];
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll
    for (int j = 0; j < kSortItems; ++j) {
        const bool valid = sub + j * 32 + lane < cnt;
        dig[j] = valid ? (int)((uint32_t)(key[j] >> shift) & 255u) : 256;
        const unsigned peers = __match_any_sync(kFull, dig[j]);
        const uint32_t pre = valid ? s_wcnt[wid][dig[j]] : 0u;
        rank[j] = pre + (uint32_t)__popc(peers & lt);
        __syncwarp();
        if (valid && (peers & lt) == 0) s_wcnt[wid][dig[j]] = pre + (uint32_t)__popc(peers);
        __syncwarp();
    }
    __syncthreads();
    uint32_t own;   // this tile's count of digit tid
    {
        uint32_t run = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            const uint32_t c = s_wcnt[w][tid];
            s_wcnt[w][tid] = run;
            run += c;
        }
        own = run;
    }
    // publish the tile's counts; the first tile's are already inclusive
    uint64_t* my = look + (int64_t)tile * 256 + tid;
    const bool withhold = inject_spin > 0 && tile == 0;   // test hook: the first tile never publishes
    if (!withhold) st_relaxed_u64(my, (tile == 0 ? kLbIncl : kLbOwn) | own);
    {
        uint32_t tot;
        s_tile_start[tid] = block256_exclusive_scan<uint32_t>(own, &tot, s_tmp);
    }
    // decoupled look-back: this digit's count over all earlier tiles
    uint64_t before = 0;
    bool ok = true;
    {
        const int limit = inject_spin > 0 ? inject_spin : kLookbackLimit;
        int polls = 0;
        for (int tp = tile - 1; tp >= 0;) {
            const uint64_t v = ld_relaxed_u64(look + (int64_t)tp * 256 + tid);
            const uint64_t flag = v >> 62;
            if (flag == 0) {
                if (++polls > limit || ((polls & 63) == 0 && has_error(status))) {
                    ok = false;
                    break;
                }
                __nanosleep(32);
                continue;
            }
            before += v & kLbCount;
            if (flag == 2) break;
            --tp;
        }
    }
    if (tile > 0 && ok) st_relaxed_u64(my, kLbIncl | (before + own));
    if (__syncthreads_or(!ok)) {
        if (tid == 0) raise_error(status, TT_ERR_TIMEOUT, 200 + tile);
        return;
    }
    {
        uint32_t tot;
        s_gbase[tid] = block256_exclusive_scan<uint32_t>(ghist[tid], &tot, s_tmp) + (uint32_t)before;
    }
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
    const int passes = (bits + 7) / 8;
    int* counters = reinterpret_cast<int*>(sb.ghist + kSortPassMax * 256);
    cudaError_t e = cudaMemsetAsync(sb.ghist, 0, kSortGhistBytes, s);
    if (e != cudaSuccess) return e;
    const int hgrid = (int)min64(ceil_div(n, 256), 148 * 8);
    k_radix_hist_all<K><<<hgrid, 256, 0, s>>>((const K*)sb.keys[0], n, dev_n, passes, sb.ghist, sb.look[0],
                                              (int64_t)tiles * 256, status);
    *nl += 1;
    int cur = 0;
    for (int p = 0; p < passes; ++p) {
        k_radix_onesweep<K><<<tiles, 256, 0, s>>>((const K*)sb.keys[cur], sb.vals[cur], (K*)sb.keys[cur ^ 1],
                                                  sb.vals[cur ^ 1], n, dev_n, 8 * p, sb.ghist + p * 256,
                                                  sb.look[p & 1], p + 1 < passes ? sb.look[(p + 1) & 1] : nullptr,
                                                  counters + p, p == 0 ? sb.inject_spin : 0, status);
        cur ^= 1;
        *nl += 1;
    }
    *which = cur;
    return cudaGetLastError();
}

cudaError_t radix_sort_pairs(bool key64, int64_t n, int bits, SortBuffers& sb, int* which,
                             int32_t* status, cudaStream_t s, int* nl, const int64_t* dev_n)
{
    if (n <= 0 || bits <= 0) {
        *which = 0;
        return cudaSuccess;
    }
    if (bits > 8 * kSortPassMax) return cudaErrorInvalidValue;
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
