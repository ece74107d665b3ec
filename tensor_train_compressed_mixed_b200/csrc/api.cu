// C ABI of libttemb: handle, argument and shape validation, workspace layout,
// stream-ordered launch sequences and the device status block.
#include <new>
#include <string.h>
#include <vector>

#include "tt_common.cuh"

using namespace tt;

namespace {

struct Layout {
    size_t counters, keys[2], vals[2], bag_of_pos, hist, digit_total, partials, uniq_keys,
        uniq_start, grp_start, bag_sorted;
    // specialised path only (zero when unused)
    size_t uid_at_pos, uid_sorted, rowbuf, pkeys[2], pvals[2], col_count, col_rows, col_order, col_start, chunk_base,
        hdr, chunks, grec, crow, sub_base, slot_of, subs, deque, exhausted, slot_flag,
        ckpt, g12, dg12, g3t, dg3t, bf1, bf2;
    int64_t chunk_cap, sub_cap, slot_cap;
    size_t total;
};

// Sizes the specialised path adds (filled from the handle).
struct FastDims {
    bool on;
    int D, ncols, MP, T;
    int64_t g12_floats;   // merged first cores of four-core tables (0 otherwise)
    int64_t g3t_floats;   // transposed copies of the last cores
    int64_t bf1_elems, bf2_elems;   // bf16 operand copies of G_1 and G_2 (tensor-core forward)
    int split;                      // distinct rows per forward subtask at most
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

Layout make_layout(int key_bytes, int64_t L, int64_t B, const FastDims& f)
{
    Layout y;
    memset(&y, 0, sizeof(y));
    size_t p = 0;
    auto take = [&](size_t bytes) {
        const size_t at = p;
        p = align_up(p + bytes, 256);
        return at;
    };
    const size_t Lz = (size_t)(L > 0 ? L : 1);
    const size_t tiles = (size_t)ceil_div((int64_t)Lz, kSortTile);
    y.counters = take(sizeof(WsCounters));
    y.keys[0] = take(Lz * key_bytes);
    y.keys[1] = take(Lz * key_bytes);
    y.vals[0] = take(Lz * 4);
    y.vals[1] = take(Lz * 4);
    y.bag_of_pos = take(Lz * 4);
    y.hist = take(256 * tiles * 4);
    y.digit_total = take(256 * 4);
    y.partials = take((size_t)ceil_div((int64_t)Lz, kScanTile) * 8);
    y.uniq_keys = take(Lz * key_bytes);
    y.uniq_start = take((Lz + 1) * 4);
    y.grp_start = take((Lz + 1) * 4);
    y.bag_sorted = take(Lz * 4);
    if (f.on) {
        y.uid_at_pos = take(Lz * 4);
        y.uid_sorted = take(Lz * 4);
        y.rowbuf = take(Lz * (size_t)f.D * 4);
        y.pkeys[0] = take(Lz * 4);
        y.pkeys[1] = take(Lz * 4);
        y.pvals[0] = take(Lz * 4);
        y.pvals[1] = take(Lz * 4);
        y.col_count = take(((size_t)f.ncols + 1) * 4);
        y.col_rows = take(((size_t)f.ncols + 1) * 4);
        y.col_order = take(((size_t)f.ncols + 1) * 4);
        y.col_start = take(((size_t)f.ncols + 1) * 4);
        y.chunk_base = take(((size_t)f.ncols + 1) * 4);
        y.hdr = take(sizeof(PlanHeader));
        y.chunk_cap = (int64_t)f.ncols + ceil_div((int64_t)Lz, f.MP) + 1;
        y.chunks = take((size_t)y.chunk_cap * sizeof(int4));
        y.grec = take(Lz * sizeof(int4));
        // forward subtasks: every chunk once, plus one per kSplitRows distinct rows of split chunks
        y.sub_cap = y.chunk_cap + ceil_div((int64_t)Lz, f.split) + 1;
        y.slot_cap = min64(kCkptSlots, ceil_div((int64_t)Lz, f.split) + 1);
        y.crow = take((size_t)y.chunk_cap * 4);
        y.sub_base = take(((size_t)y.chunk_cap + 1) * 4);
        y.slot_of = take((size_t)y.chunk_cap * 4);
        y.subs = take((size_t)y.sub_cap * sizeof(int4));
        y.deque = take((size_t)kMaxGrid * 8);
        y.exhausted = take((size_t)kMaxGrid * 4);
        y.slot_flag = take((size_t)y.slot_cap * 4);
        y.ckpt = take((size_t)y.slot_cap * kCkptFloats * 4);
        if (f.g12_floats > 0) {
            y.g12 = take((size_t)f.g12_floats * 4);
            y.dg12 = take((size_t)f.g12_floats * 4);
        }
        y.g3t = take((size_t)f.g3t_floats * 4);
        y.dg3t = take((size_t)f.g3t_floats * 4);
        if (f.bf1_elems > 0) {
            y.bf1 = take((size_t)f.bf1_elems * 2);
            y.bf2 = take((size_t)f.bf2_elems * 2);
        }
    }
    y.total = p;
    return y;
}

int bits_for(uint64_t v)  // bits needed to hold values 0..v
{
    int b = 0;
    while (b < 64 && (v >> b) != 0) ++b;
    return b;
}

}  // namespace

struct tt_emb_handle {
    int32_t T = 0, k = 0, D = 0, P = 0;
    int64_t n[kMaxT][kMaxK] = {};
    int64_t n_rows[kMaxT] = {};
    int32_t d[kMaxK] = {};
    int32_t r[kMaxK + 1] = {};
    tt_emb_options opt{};
    int ibits = 0, tbits = 0;
    bool key64 = false;
    float* cores[kMaxT * kMaxK] = {};
    float* grads[kMaxT * kMaxK] = {};
    bool have_cores = false, have_grads = false;
    char* ws = nullptr;
    size_t ws_bytes = 0;
    int64_t ws_L = 0, ws_B = 0;
    Layout lay{};
    int32_t* d_status = nullptr;
    cudaStream_t last_stream = nullptr;
    bool used_stream = false;
    bool have_fwd = false;
    int64_t fwd_L = 0, fwd_B = 0;
    int fwd_which = 0;
    int device = 0, num_sms = 148;
    // specialised three-core path (four-core tables through the merged-core view)
    bool fast = false;
    bool merged = false;
    int ncols = 0;
    int col_base[kMaxT + 1] = {};
    int64_t vn[kMaxT][3] = {};      // three-core view: factors (n_1 n_2, n_3, n_4) when merged
    int32_t vd[3] = {}, vr[4] = {};
    int64_t g12_off[kMaxT + 1] = {};  // merged-core offsets (floats) in the workspace
    int64_t g3t_off[kMaxT + 1] = {};  // transposed last-core offsets (floats) in the workspace
    int tc = 0;                       // tensor-core prefix products: 0 none, 1 bf16, 3 split bf16 (two terms)
    int64_t bf1_off[kMaxT + 1] = {};  // bf16 copies of G_1 and G_2 (elements) in the workspace
    int64_t bf2_off[kMaxT + 1] = {};
    // timing and launch accounting
    bool timing = false;
    double phase_ms[TT_EMB_NUM_PHASES] = {};
    int64_t launches = 0;
    int last_error = TT_OK;           // tt_emb_last_error
    int inject = TT_INJECT_NONE, inject_spin = 0;   // tt_emb_debug_inject, armed until consumed
    unsigned long long* probe = nullptr;              // tt_emb_set_probe
    int32_t probe_cap = 0;
    struct Interval { int phase; cudaEvent_t a, b; };
    std::vector<Interval> pending;
    std::vector<cudaEvent_t> pool;
    int open_phase = -1;
    cudaEvent_t open_event = nullptr;

    cudaEvent_t take_event()
    {
        if (!pool.empty()) {
            cudaEvent_t e = pool.back();
            pool.pop_back();
            return e;
        }
        cudaEvent_t e = nullptr;
        if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
        return e;
    }
    void begin(int phase, cudaStream_t s)
    {
        if (!timing) return;
        open_phase = phase;
        open_event = take_event();
        if (open_event) cudaEventRecord(open_event, s);
    }
    void end(cudaStream_t s)
    {
        if (!timing || open_phase < 0) return;
        cudaEvent_t b = take_event();
        if (open_event && b) {
            cudaEventRecord(b, s);
            pending.push_back({open_phase, open_event, b});
        }
        open_phase = -1;
        open_event = nullptr;
    }
    void fold()
    {
        for (const Interval& iv : pending) {
            float ms = 0.f;
            if (cudaEventSynchronize(iv.b) == cudaSuccess && cudaEventElapsedTime(&ms, iv.a, iv.b) == cudaSuccess)
                phase_ms[iv.phase] += ms;
            pool.push_back(iv.a);
            pool.push_back(iv.b);
        }
        pending.clear();
    }

    int key_bytes() const { return key64 ? 8 : 4; }
    FastDims fast_dims() const
    {
        FastDims f;
        f.on = fast;
        f.D = D;
        f.ncols = ncols;
        f.MP = fast ? k3_plan_mp(view_params()) : 1;
        f.T = T;
        f.g12_floats = merged ? g12_off[T] : 0;
        f.g3t_floats = g3t_off[T];
        f.bf1_elems = tc ? bf1_off[T] : 0;
        f.bf2_elems = tc ? bf2_off[T] : 0;
        f.split = opt.chunk > 0 ? opt.chunk : kSplitRows;
        return f;
    }
    // three-core view of the shapes (identity for three-core tables), without core pointers
    CoreParams view_params() const
    {
        CoreParams cp;
        memset(&cp, 0, sizeof(cp));
        cp.T = T; cp.k = 3; cp.D = D;
        for (int j = 0; j < 3; ++j) cp.d[j] = vd[j];
        for (int j = 0; j < 4; ++j) cp.r[j] = vr[j];
        cp.P = vd[0] * vd[1];
        cp.ibits = ibits;
        cp.unique_only = opt.grouping == TT_GROUP_UNIQUE_ONLY;
        cp.B = fwd_B;
        for (int t = 0; t < T; ++t)
            for (int j = 0; j < 3; ++j) cp.n[t][j] = (uint32_t)vn[t][j];
        return cp;
    }
    // view with cores (merged first core from the workspace) and the matching gradient pointers
    CoreParams view_cores(int64_t batch, GradPtrs* gp) const
    {
        CoreParams cp = view_params();
        cp.B = batch;
        if (gp) memset(gp, 0, sizeof(*gp));
        for (int t = 0; t < T; ++t) {
            const int off = merged ? 1 : 0;   // real core j+off is view core j (j >= 1)
            cp.cores[t][0] = merged ? (const float*)at(lay.g12) + g12_off[t] : cores[t * k];
            cp.cores[t][1] = cores[t * k + 1 + off];
            cp.cores[t][2] = cores[t * k + 2 + off];
            cp.last_t[t] = (const float*)at(lay.g3t) + g3t_off[t];
            if (tc) {
                cp.bf1[t] = (const uint16_t*)at(lay.bf1) + bf1_off[t];
                cp.bf2[t] = (const uint16_t*)at(lay.bf2) + bf2_off[t];
            }
            if (gp) {
                gp->g[t][0] = merged ? (float*)at(lay.dg12) + g12_off[t] : grads[t * k];
                gp->g[t][1] = grads[t * k + 1 + off];
                gp->g[t][2] = grads[t * k + 2 + off];
            }
        }
        return cp;
    }
    MergeParams merge_params() const
    {
        MergeParams mp;
        memset(&mp, 0, sizeof(mp));
        mp.T = T;
        mp.d1 = d[0];
        mp.d2 = d[1];
        mp.r1 = r[1];
        mp.r2 = r[2];
        int b = 0;
        for (int t = 0; t < T; ++t) {
            mp.blk_base[t] = b;
            b += (int)n[t][1];
            mp.n1[t] = (uint32_t)n[t][0];
            mp.n2[t] = (uint32_t)n[t][1];
            mp.g1[t] = cores[t * k];
            mp.g2[t] = cores[t * k + 1];
            if (ws) {
                mp.g12[t] = (float*)at(lay.g12) + g12_off[t];
                mp.dg12[t] = (const float*)at(lay.dg12) + g12_off[t];
            }
            mp.dg1[t] = grads[t * k];
            mp.dg2[t] = grads[t * k + 1];
        }
        mp.blk_base[T] = b;
        return mp;
    }
    PlanParams plan_params(int64_t batch) const
    {
        PlanParams pp;
        memset(&pp, 0, sizeof(pp));
        pp.T = T;
        pp.k = 3;
        pp.ibits = ibits;
        pp.col_digit = 1;
        pp.B = batch;
        pp.MP = k3_plan_mp(view_params());
        pp.NB = kPoolBags;
        pp.ncols = ncols;
        pp.sched = opt.sched;
        pp.grid = fwd_grid();
        pp.slot_cap = (int32_t)lay.slot_cap;
        pp.split_rows = opt.chunk > 0 ? opt.chunk : kSplitRows;
        for (int t = 0; t < T; ++t)
            for (int j = 0; j < 3; ++j) pp.n[t][j] = (uint32_t)vn[t][j];
        for (int t = 0; t <= T; ++t) pp.col_base[t] = col_base[t];
        return pp;
    }
    // persistent blocks of the fused forward: the option, else one wave (owner ranges need it at plan time)
    mutable int fwd_grid_cache = 0;
    int fwd_grid() const
    {
        if (fwd_grid_cache == 0) {
            // at most one resident wave: a pooling task waits for subtasks owned by other blocks,
            // which must all be running
            const int wave = num_sms * k3_blocks_per_sm(view_params(), false, tc != 0);
            const int g = opt.grid > 0 && opt.grid < wave ? opt.grid : wave;
            fwd_grid_cache = g < kMaxGrid ? g : kMaxGrid;
        }
        return fwd_grid_cache;
    }
    int64_t core_floats(int t, int j) const { return (int64_t)r[j] * n[t][j] * d[j] * r[j + 1]; }

    CoreParams core_params() const
    {
        CoreParams cp;
        memset(&cp, 0, sizeof(cp));
        cp.T = T; cp.k = k; cp.D = D; cp.P = P;
        for (int j = 0; j < k; ++j) cp.d[j] = d[j];
        for (int j = 0; j <= k; ++j) cp.r[j] = r[j];
        cp.ibits = ibits;
        cp.unique_only = opt.grouping == TT_GROUP_UNIQUE_ONLY;
        cp.B = fwd_B;
        for (int t = 0; t < T; ++t)
            for (int j = 0; j < k; ++j) {
                cp.n[t][j] = (uint32_t)n[t][j];
                cp.cores[t][j] = cores[t * k + j];
            }
        return cp;
    }

    // every core (or its gradient); skip_middle leaves out core 1 of every table (size 0)
    BufferList buffers(bool with_grads_as_b, bool grads_as_a, bool skip_middle = false) const
    {
        BufferList bl;
        memset(&bl, 0, sizeof(bl));
        bl.count = T * k;
        int64_t c = 0;
        for (int q = 0; q < T * k; ++q) {
            const int64_t sz = (skip_middle && q % k == 1) ? 0 : core_floats(q / k, q % k);
            bl.chunk_start[q] = c;
            bl.size[q] = sz;
            bl.a[q] = grads_as_a ? grads[q] : cores[q];
            bl.b[q] = with_grads_as_b ? grads[q] : nullptr;
            c += ceil_div(sz, kElemChunk);
        }
        bl.chunk_start[T * k] = c;
        return bl;
    }

    char* at(size_t off) const { return ws + off; }

    int32_t* plan_sorted_groups = nullptr;  // set by the last forward's plan

    PlanBuffers plan_buffers(const SortBuffers& lookup_sort)
    {
        PlanBuffers pb;
        memset(&pb, 0, sizeof(pb));
        pb.sort.keys[0] = at(lay.pkeys[0]);
        pb.sort.keys[1] = at(lay.pkeys[1]);
        pb.sort.vals[0] = (int32_t*)at(lay.pvals[0]);
        pb.sort.vals[1] = (int32_t*)at(lay.pvals[1]);
        pb.sort.hist = lookup_sort.hist ? lookup_sort.hist : (uint32_t*)at(lay.hist);
        pb.sort.digit_total = lookup_sort.digit_total ? lookup_sort.digit_total : (uint32_t*)at(lay.digit_total);
        pb.col_count = (int32_t*)at(lay.col_count);
        pb.col_rows = (int32_t*)at(lay.col_rows);
        pb.col_order = (int32_t*)at(lay.col_order);
        pb.col_start = (int32_t*)at(lay.col_start);
        pb.chunk_base = (int32_t*)at(lay.chunk_base);
        pb.hdr = (PlanHeader*)at(lay.hdr);
        pb.chunks = (int4*)at(lay.chunks);
        pb.grec = (int4*)at(lay.grec);
        pb.crow = (int32_t*)at(lay.crow);
        pb.sub_base = (int32_t*)at(lay.sub_base);
        pb.slot_of = (int32_t*)at(lay.slot_of);
        pb.subs = (int4*)at(lay.subs);
        pb.deque = (unsigned long long*)at(lay.deque);
        pb.exhausted = (int32_t*)at(lay.exhausted);
        pb.slot_flag = (int32_t*)at(lay.slot_flag);
        pb.ckpt = (float*)at(lay.ckpt);
        return pb;
    }

    K3Args k3_args(const CoreParams* cp, const PlanParams* pp, const PlanBuffers* pb,
                   const int64_t* offsets, int64_t L, bool backward) const
    {
        K3Args a;
        memset(&a, 0, sizeof(a));
        a.cp = cp;
        a.pp = pp;
        a.key64 = key64;
        a.uniq_keys = at(lay.uniq_keys);
        a.uniq_start = (const int32_t*)at(lay.uniq_start);
        a.grp_start = (const int32_t*)at(lay.grp_start);
        a.bag_sorted = (const int32_t*)at(lay.bag_sorted);
        a.uid_at_pos = (const int32_t*)at(lay.uid_at_pos);
        a.uid_sorted = (const int32_t*)at(lay.uid_sorted);
        a.counters = (const WsCounters*)at(lay.counters);
        a.pb = pb;
        a.grec = pb ? pb->grec : nullptr;
        a.offsets = offsets;
        a.rowbuf = (float*)at(lay.rowbuf);
        a.L = L;
        a.tc = (tc && (!backward || k3_tc_bwd_supported(*cp))) ? tc : 0;
        a.grid = backward ? (opt.grid > 0 ? opt.grid : num_sms * k3_blocks_per_sm(*cp, true, a.tc != 0))
                          : fwd_grid();
        a.status = d_status;
        return a;
    }
};

static int cuda_status(cudaError_t e) { return e == cudaSuccess ? TT_OK : TT_ERR_CUDA; }

// records a failed call on the handle for tt_emb_last_error
static int note(tt_emb_t h, int rc)
{
    if (h && rc != TT_OK) h->last_error = rc;
    return rc;
}

namespace tt {
// device the handle was created on (tt_emb_forward_noalloc checks it is current)
int handle_device(tt_emb_t h) { return h ? h->device : -1; }
// records a failed call of an entry point defined in another file
int record_error(tt_emb_t h, int rc) { return note(h, rc); }
}  // namespace tt

extern "C" {

int tt_emb_abi_version(void) { return TT_EMB_ABI_VERSION; }

void tt_emb_default_options(tt_emb_options* opt)
{
    if (!opt) return;
    memset(opt, 0, sizeof(*opt));
    opt->sched = TT_SCHED_STEAL_L2;
    opt->grouping = TT_GROUP_PREFIX;
    opt->chunk = 0;
    opt->grid = 0;
}

const char* tt_emb_error_string(int code)
{
    switch (code) {
    case TT_OK: return "ok";
    case TT_ERR_ARG: return "invalid argument";
    case TT_ERR_SHAPE: return "unsupported table or core shape";
    case TT_ERR_INDEX_RANGE: return "an index is outside [0, N) of its table";
    case TT_ERR_OFFSETS: return "offsets are not a monotone partition of [0, num_lookups)";
    case TT_ERR_WORKSPACE: return "workspace missing or too small";
    case TT_ERR_STATE: return "call out of order (cores, gradients or forward missing)";
    case TT_ERR_CUDA: return "a CUDA runtime call failed";
    case TT_ERR_TIMEOUT: return "a bounded device wait ran out";
    case TT_ERR_UNSUPPORTED: return "not supported by this build";
    default: return "unknown status code";
    }
}

int tt_emb_create(int32_t num_tables, int32_t num_cores, const int64_t* n_factors,
                  const int64_t* n_rows, const int32_t* d_factors, const int32_t* ranks,
                  const tt_emb_options* opt, tt_emb_t* out)
{
    if (!out || !n_factors || !n_rows || !d_factors || !ranks) return TT_ERR_ARG;
    *out = nullptr;
    if (num_tables < 1 || num_tables > kMaxT || num_cores < 1 || num_cores > kMaxK) return TT_ERR_SHAPE;
    tt_emb_options o;
    tt_emb_default_options(&o);
    if (opt) {
        o = *opt;
        for (int i = 0; i < 10; ++i)
            if (o.reserved[i] != 0) return TT_ERR_ARG;
        if (o.force_generic != 0 && o.force_generic != 1) return TT_ERR_ARG;
        if (o.precision != TT_PREC_FP32 && o.precision != TT_PREC_BF16_TC && o.precision != TT_PREC_FP32_SPLIT_TC)
            return TT_ERR_ARG;
        if (o.sched < TT_SCHED_STATIC || o.sched > TT_SCHED_STEAL_L2) return TT_ERR_ARG;
        if (o.grouping < TT_GROUP_PREFIX || o.grouping > TT_GROUP_UNIQUE_ONLY) return TT_ERR_ARG;
        if (o.chunk < 0 || o.chunk > kSplitRows || o.grid < 0) return TT_ERR_ARG;
    }
    const int k = num_cores;
    if (ranks[0] != 1 || ranks[k] != 1) return TT_ERR_SHAPE;
    int64_t D = 1;
    for (int j = 0; j < k; ++j) {
        if (d_factors[j] < 1 || ranks[j] < 1 || ranks[j] > 128) return TT_ERR_SHAPE;
        D *= d_factors[j];
    }
    if (D > 1024) return TT_ERR_SHAPE;
    uint64_t max_rows = 1;
    for (int t = 0; t < num_tables; ++t) {
        long double prod = 1;
        for (int j = 0; j < k; ++j) {
            const int64_t nj = n_factors[(int64_t)t * k + j];
            if (nj < 1 || nj > 0xffffffffLL) return TT_ERR_SHAPE;
            prod *= (long double)nj;
        }
        if (prod >= (long double)(1ULL << 40)) return TT_ERR_SHAPE;
        if (n_rows[t] < 1 || (long double)n_rows[t] > prod || n_rows[t] > 0xffffffffLL) return TT_ERR_SHAPE;
        if ((uint64_t)n_rows[t] > max_rows) max_rows = (uint64_t)n_rows[t];
    }

    tt_emb_handle* h = new (std::nothrow) tt_emb_handle();
    if (!h) return TT_ERR_ARG;
    h->T = num_tables;
    h->k = k;
    h->D = (int32_t)D;
    h->P = (int32_t)(D / d_factors[k - 1]);
    for (int j = 0; j < k; ++j) h->d[j] = d_factors[j];
    for (int j = 0; j <= k; ++j) h->r[j] = ranks[j];
    for (int t = 0; t < num_tables; ++t) {
        h->n_rows[t] = n_rows[t];
        for (int j = 0; j < k; ++j) h->n[t][j] = n_factors[(int64_t)t * k + j];
    }
    h->opt = o;
    h->ibits = bits_for(max_rows - 1);
    if (h->ibits < 1) h->ibits = 1;
    h->tbits = bits_for((uint64_t)num_tables - 1);
    h->key64 = h->ibits + h->tbits > 32;

    const CoreParams cp = h->core_params();
    // three-core view: the shapes themselves, or (n_1 n_2, n_3, n_4) with the merged first core
    if (k == 3 || k == 4) {
        const bool m4 = k == 4;
        h->vd[0] = m4 ? d_factors[0] * d_factors[1] : d_factors[0];
        h->vd[1] = d_factors[m4 ? 2 : 1];
        h->vd[2] = d_factors[m4 ? 3 : 2];
        h->vr[0] = 1;
        h->vr[1] = ranks[m4 ? 2 : 1];
        h->vr[2] = ranks[m4 ? 3 : 2];
        h->vr[3] = 1;
        bool ok = true;
        int64_t g12 = 0;
        for (int t = 0; t < num_tables; ++t) {
            const int64_t a = m4 ? h->n[t][0] * h->n[t][1] : h->n[t][0];
            if (a > 0xffffffffLL) ok = false;
            h->vn[t][0] = a;
            h->vn[t][1] = h->n[t][m4 ? 2 : 1];
            h->vn[t][2] = h->n[t][m4 ? 3 : 2];
            h->g12_off[t] = g12;
            if (m4) g12 += a * h->vd[0] * h->vr[1];
        }
        h->g12_off[num_tables] = g12;
        int64_t g3t = 0;
        for (int t = 0; t < num_tables; ++t) {
            h->g3t_off[t] = g3t;
            g3t += h->vn[t][2] * h->vr[2] * h->vd[2];
        }
        h->g3t_off[num_tables] = g3t;
        h->merged = m4;
        h->fast = ok && !o.force_generic && k3_supported(h->view_params());
        if (h->fast && m4) {
            MergeParams mp = h->merge_params();
            if (!merge_fits(mp) || g12 * 4 > (int64_t)2 << 30) h->fast = false;
        }
        if (!h->fast) h->merged = false;
    }
    if (h->fast) {
        int64_t nc = 0;
        for (int t = 0; t < num_tables; ++t) {
            h->col_base[t] = (int)nc;
            nc += h->vn[t][1];
        }
        h->col_base[num_tables] = (int)nc;
        if (nc >= (1LL << 24)) h->fast = h->merged = false;
        h->ncols = (int)nc;
    }
    if (o.precision == TT_PREC_BF16_TC || o.precision == TT_PREC_FP32_SPLIT_TC) {
        // the tensor-core prefix GEMM exists for three-core tables of the listed shapes only
        if (!h->fast || h->merged || !k3_tc_supported(h->view_params())) {
            delete h;
            return TT_ERR_SHAPE;
        }
        h->tc = o.precision == TT_PREC_FP32_SPLIT_TC ? 3 : 1;
        const int terms = h->tc == 3 ? 2 : 1;
        int64_t b1 = 0, b2 = 0;
        for (int t = 0; t < num_tables; ++t) {
            h->bf1_off[t] = b1;
            h->bf2_off[t] = b2;
            b1 += terms * h->vn[t][0] * h->vd[0] * h->vr[1];
            b2 += terms * h->vn[t][1] * h->vr[1] * h->vd[1] * h->vr[2];
        }
        h->bf1_off[num_tables] = b1;
        h->bf2_off[num_tables] = b2;
    }
    if (generic_backward_smem_floats(cp) * 4 > 200 * 1024 ||
        generic_forward_smem_floats(cp) * 4 > 200 * 1024) {
        delete h;
        return TT_ERR_SHAPE;
    }
    if (cudaGetDevice(&h->device) != cudaSuccess ||
        cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device) != cudaSuccess ||
        cudaMalloc((void**)&h->d_status, 256) != cudaSuccess) {
        delete h;
        return TT_ERR_CUDA;
    }
    if (cudaMemset(h->d_status, 0, 256) != cudaSuccess) {
        cudaFree(h->d_status);
        delete h;
        return TT_ERR_CUDA;
    }
    *out = h;
    return TT_OK;
}

static int tt_emb_set_cores_impl(tt_emb_t h, float* const* cores, float* const* core_grads)
{
    if (!h || !cores) return TT_ERR_ARG;
    const int n = h->T * h->k;
    for (int q = 0; q < n; ++q) {
        if (!cores[q] || ((uintptr_t)cores[q] & 15)) return TT_ERR_ARG;
        if (core_grads && (!core_grads[q] || ((uintptr_t)core_grads[q] & 15))) return TT_ERR_ARG;
    }
    for (int q = 0; q < n; ++q) {
        h->cores[q] = cores[q];
        h->grads[q] = core_grads ? core_grads[q] : nullptr;
    }
    h->have_cores = true;
    h->have_grads = core_grads != nullptr;
    return TT_OK;
}

static int tt_emb_workspace_size_impl(tt_emb_t h, int64_t max_lookups, int64_t batch, size_t* bytes)
{
    if (!h || !bytes || max_lookups < 0 || batch < 1) return TT_ERR_ARG;
    if (max_lookups >= (int64_t)INT32_MAX) return TT_ERR_ARG;
    *bytes = make_layout(h->key_bytes(), max_lookups, batch, h->fast_dims()).total;
    return TT_OK;
}

static int tt_emb_set_workspace_impl(tt_emb_t h, void* workspace, size_t bytes, int64_t max_lookups,
                         int64_t batch)
{
    if (!h || !workspace || max_lookups < 0 || batch < 1) return TT_ERR_ARG;
    if (((uintptr_t)workspace & 255) != 0) return TT_ERR_ARG;
    if (max_lookups >= (int64_t)INT32_MAX) return TT_ERR_ARG;
    const Layout lay = make_layout(h->key_bytes(), max_lookups, batch, h->fast_dims());
    if (bytes < lay.total) return TT_ERR_WORKSPACE;
    h->ws = (char*)workspace;
    h->ws_bytes = bytes;
    h->ws_L = max_lookups;
    h->ws_B = batch;
    h->lay = lay;
    h->have_fwd = false;
    return TT_OK;
}

static int tt_emb_forward_impl(tt_emb_t h, const int64_t* indices, const int64_t* offsets, int64_t num_lookups,
                   int64_t batch, float* out, tt_stream_t stream)
{
    if (!h || !offsets || !out || num_lookups < 0 || batch < 1) return TT_ERR_ARG;
    if (num_lookups > 0 && !indices) return TT_ERR_ARG;
    if (!h->have_cores) return TT_ERR_STATE;
    if (!h->ws || num_lookups > h->ws_L || batch > h->ws_B) return TT_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    h->last_stream = s;
    h->used_stream = true;
    h->have_fwd = false;
    const Layout& y = h->lay;
    WsCounters* counters = (WsCounters*)h->at(y.counters);
    const int64_t L = num_lookups;

    cudaError_t e = cudaSuccess;
    if (!h->fast || L == 0) e = cudaMemsetAsync(out, 0, sizeof(float) * (size_t)batch * h->T * h->D, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(counters, 0, sizeof(WsCounters), s);
    if (e != cudaSuccess) return TT_ERR_CUDA;

    KeyParams kp;
    memset(&kp, 0, sizeof(kp));
    kp.T = h->T;
    kp.ibits = h->ibits;
    kp.B = batch;
    kp.L = L;
    kp.unique_only = h->opt.grouping == TT_GROUP_UNIQUE_ONLY;
    for (int t = 0; t < h->T; ++t) {
        kp.nrows[t] = (uint32_t)h->n_rows[t];
        kp.nlast[t] = (uint32_t)h->n[t][h->k - 1];
    }
    int32_t* bag_of_pos = (int32_t*)h->at(y.bag_of_pos);
    SortBuffers sb;
    sb.keys[0] = h->at(y.keys[0]);
    sb.keys[1] = h->at(y.keys[1]);
    sb.vals[0] = (int32_t*)h->at(y.vals[0]);
    sb.vals[1] = (int32_t*)h->at(y.vals[1]);
    sb.hist = (uint32_t*)h->at(y.hist);
    sb.digit_total = (uint32_t*)h->at(y.digit_total);

    int nl = 0;
    h->begin(TT_PHASE_FWD_KEYS, s);
    e = launch_make_keys(kp, h->key64, indices, offsets, sb.keys[0], sb.vals[0], bag_of_pos,
                         h->d_status, s, &nl);
    h->end(s);
    h->launches += nl;
    if (e != cudaSuccess) return TT_ERR_CUDA;
    h->fwd_L = L;
    h->fwd_B = batch;
    if (L == 0) {
        h->fwd_which = 0;
        h->have_fwd = true;
        return TT_OK;
    }
    int which = 0;
    nl = 0;
    h->begin(TT_PHASE_FWD_SORT, s);
    e = radix_sort_pairs(h->key64, L, h->ibits + h->tbits, sb, &which, h->d_status, s, &nl);
    h->end(s);
    if (e != cudaSuccess) return TT_ERR_CUDA;
    h->begin(TT_PHASE_FWD_SEGMENT, s);
    e = launch_segment(kp, h->key64, sb.keys[which], sb.vals[which], bag_of_pos,
                       h->at(y.uniq_keys), (int32_t*)h->at(y.uniq_start),
                       (int32_t*)h->at(y.grp_start), (int32_t*)h->at(y.bag_sorted),
                       (uint64_t*)h->at(y.partials), counters,
                       h->fast ? (int32_t*)h->at(y.uid_at_pos) : nullptr,
                       h->fast ? (int32_t*)h->at(y.uid_sorted) : nullptr, h->d_status, s, &nl);
    PlanBuffers pb;
    PlanParams pp;
    CoreParams cp = h->fast ? h->view_cores(batch, nullptr) : h->core_params();
    cp.B = batch;
    if (e == cudaSuccess && h->fast) {
        pp = h->plan_params(batch);
        pb = h->plan_buffers(sb);
        e = launch_plan(pp, h->key64, h->at(y.uniq_keys), (const int32_t*)h->at(y.grp_start), counters, L,
                        pb, h->d_status, s, &nl);
        h->plan_sorted_groups = pb.sorted_groups;
    }
    h->end(s);
    if (e != cudaSuccess) return TT_ERR_CUDA;
    h->begin(TT_PHASE_FWD_FUSED, s);
    if (h->fast) {
        if (h->merged) e = launch_merge(h->merge_params(), h->d_status, s, &nl);
        if (e == cudaSuccess) {
            float* dst[kMaxT];
            for (int t = 0; t < h->T; ++t) dst[t] = (float*)h->at(y.g3t) + h->g3t_off[t];
            e = k3_transpose_last(cp, dst, s, &nl);
        }
        if (e == cudaSuccess && h->tc) {
            uint16_t* d1[kMaxT];
            uint16_t* d2[kMaxT];
            for (int t = 0; t < h->T; ++t) {
                d1[t] = (uint16_t*)h->at(y.bf1) + h->bf1_off[t];
                d2[t] = (uint16_t*)h->at(y.bf2) + h->bf2_off[t];
            }
            e = k3_to_bf16(cp, h->tc == 3 ? 2 : 1, d1, d2, s, &nl);
        }
        cp.probe = h->probe;
        cp.probe_slot = 0;
        cp.probe_cap = h->probe_cap;
        if (h->inject == TT_INJECT_POOL_WAIT || (h->inject == TT_INJECT_MMA_WAIT_FWD && h->tc)) {
            cp.inj_pool = h->inject == TT_INJECT_POOL_WAIT;
            cp.inj_mma = h->inject == TT_INJECT_MMA_WAIT_FWD;
            cp.inj_spin = h->inject_spin;
            h->inject = TT_INJECT_NONE;
        }
        K3Args a = h->k3_args(&cp, &pp, &pb, offsets, L, false);
        if (e == cudaSuccess) e = k3_forward(a, out, s, &nl);
    } else {
        const int grid = h->opt.grid > 0 ? h->opt.grid : h->num_sms * 8;
        e = launch_forward_generic(cp, h->key64, h->at(y.uniq_keys), (const int32_t*)h->at(y.uniq_start),
                                   (const int32_t*)h->at(y.grp_start), (const int32_t*)h->at(y.bag_sorted),
                                   counters, L, out, h->d_status, s, grid, &nl);
    }
    h->end(s);
    h->launches += nl;
    if (e != cudaSuccess) return TT_ERR_CUDA;
    h->fwd_which = which;
    h->have_fwd = true;
    return TT_OK;
}

// Backward of the last forward; fused: the middle cores take their SGD step inside the
// column-group kernel (the caller checked that the handle qualifies) and their gradient
// buffers are skipped by the zero fill.
static int backward_impl(tt_emb_t h, const float* grad_out, tt_stream_t stream, bool fused, float lr)
{
    cudaStream_t s = (cudaStream_t)stream;
    h->last_stream = s;
    h->used_stream = true;
    int nl = 0;
    h->begin(TT_PHASE_BWD_REDUCE, s);
    // fused: dG_2 is never materialised, so it is not zero-filled either
    cudaError_t e = launch_fill_zero(h->buffers(false, true, fused), h->d_status, s, &nl);
    h->end(s);
    h->launches += nl;
    if (e != cudaSuccess) return TT_ERR_CUDA;
    if (h->fwd_L == 0) return TT_OK;
    const Layout& y = h->lay;
    GradPtrs gp;
    memset(&gp, 0, sizeof(gp));
    for (int t = 0; t < h->T; ++t)
        for (int j = 0; j < h->k; ++j) gp.g[t][j] = h->grads[t * h->k + j];
    const CoreParams cp = h->core_params();
    nl = 0;
    if (h->fast) {
        PlanParams pp = h->plan_params(h->fwd_B);
        SortBuffers sb;
        memset(&sb, 0, sizeof(sb));
        PlanBuffers pb = h->plan_buffers(sb);
        pb.sorted_groups = h->plan_sorted_groups;
        GradPtrs vgp;
        CoreParams vcp = h->view_cores(h->fwd_B, &vgp);
        if (h->inject == TT_INJECT_MMA_WAIT_BWD) {
            vcp.inj_mma = 1;
            h->inject = TT_INJECT_NONE;
        }
        vcp.probe = h->probe;
        vcp.probe_slot = 1;
        vcp.probe_cap = h->probe_cap;
        if (fused) {
            vgp.fused = 1;
            vgp.lr = lr;
            for (int t = 0; t < h->T; ++t) vgp.upd1[t] = h->cores[t * h->k + 1];
        }
        K3Args a = h->k3_args(&vcp, &pp, &pb, nullptr, h->fwd_L, true);
        h->begin(TT_PHASE_BWD_ROWSUM, s);
        e = k3_rowsum(a, grad_out, s, &nl);
        h->end(s);
        e = e == cudaSuccess ? cudaMemsetAsync(&pb.hdr->col_head, 0, sizeof(int32_t), s) : e;
        if (e == cudaSuccess && h->merged)
            e = cudaMemsetAsync(h->at(y.dg12), 0, sizeof(float) * (size_t)h->g12_off[h->T], s);
        // the last cores' gradients accumulate in the transposed layout [n_3][r_2][d_3] (one
        // row's contribution is one contiguous block) and are transposed back afterwards
        float* dg3[kMaxT];
        for (int t = 0; t < h->T; ++t) {
            dg3[t] = vgp.g[t][2];
            vgp.g[t][2] = (float*)h->at(y.dg3t) + h->g3t_off[t];
        }
        if (e == cudaSuccess) e = cudaMemsetAsync(h->at(y.dg3t), 0, sizeof(float) * (size_t)h->g3t_off[h->T], s);
        h->begin(TT_PHASE_BWD_FUSED, s);
        if (e == cudaSuccess) e = k3_backward(a, vgp, grad_out, s, &nl);
        h->end(s);
        h->begin(TT_PHASE_BWD_REDUCE, s);
        if (e == cudaSuccess) {
            const float* src[kMaxT];
            for (int t = 0; t < h->T; ++t) src[t] = vgp.g[t][2];
            e = k3_transpose_last_back(vcp, src, dg3, s, &nl);
        }
        if (e == cudaSuccess && h->merged) e = launch_unmerge(h->merge_params(), h->d_status, s, &nl);
    } else {
        h->begin(TT_PHASE_BWD_FUSED, s);
        const int grid = h->opt.grid > 0 ? h->opt.grid : h->num_sms * 8;
        e = launch_backward_generic(cp, gp, h->key64, h->at(y.uniq_keys),
                                    (const int32_t*)h->at(y.uniq_start), (const int32_t*)h->at(y.grp_start),
                                    (const int32_t*)h->at(y.bag_sorted), (const WsCounters*)h->at(y.counters),
                                    h->fwd_L, grad_out, h->d_status, s, grid, &nl);
    }
    h->end(s);
    h->launches += nl;
    return cuda_status(e);
}

static int tt_emb_backward_impl(tt_emb_t h, const float* grad_out, tt_stream_t stream)
{
    if (!h || !grad_out) return TT_ERR_ARG;
    if (!h->have_fwd || !h->have_grads || !h->have_cores) return TT_ERR_STATE;
    return backward_impl(h, grad_out, stream, false, 0.f);
}

static int tt_emb_backward_sgd_impl(tt_emb_t h, const float* grad_out, float lr, tt_stream_t stream)
{
    if (!h || !grad_out) return TT_ERR_ARG;
    if (!h->have_fwd || !h->have_grads || !h->have_cores) return TT_ERR_STATE;
    // the middle core's column groups are reduced on chip only by the three-core specialised kernel
    const bool fused = h->fast && !h->merged && h->k == 3;
    int rc = backward_impl(h, grad_out, stream, fused, lr);
    if (rc != TT_OK) return rc;
    if (!fused) return tt_emb_sgd_update(h, lr, stream);
    cudaStream_t s = (cudaStream_t)stream;
    int nl = 0;
    h->begin(TT_PHASE_SGD, s);
    const cudaError_t e = launch_sgd(h->buffers(true, false, true), lr, h->d_status, s, &nl);
    h->end(s);
    h->launches += nl;
    return cuda_status(e);
}

static int tt_emb_sgd_update_impl(tt_emb_t h, float lr, tt_stream_t stream)
{
    if (!h) return TT_ERR_ARG;
    if (!h->have_cores || !h->have_grads) return TT_ERR_STATE;
    cudaStream_t s = (cudaStream_t)stream;
    h->last_stream = s;
    h->used_stream = true;
    int nl = 0;
    h->begin(TT_PHASE_SGD, s);
    const cudaError_t e = launch_sgd(h->buffers(true, false), lr, h->d_status, s, &nl);
    h->end(s);
    h->launches += nl;
    return cuda_status(e);
}

int tt_emb_sync(tt_emb_t h)
{
    if (!h) return TT_ERR_ARG;
    cudaStream_t s = h->used_stream ? h->last_stream : (cudaStream_t)0;
    if (cudaStreamSynchronize(s) != cudaSuccess) return note(h, TT_ERR_CUDA);
    h->fold();
    int32_t st[2] = {0, 0};
    if (cudaMemcpyAsync(st, h->d_status, sizeof(st), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return note(h, TT_ERR_CUDA);
    if (st[0] != 0) {
        if (cudaMemsetAsync(h->d_status, 0, 256, s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess)
            return note(h, TT_ERR_CUDA);
        return note(h, st[0]);
    }
    return TT_OK;
}

static int tt_emb_get_segmentation_impl(tt_emb_t h, tt_seg_view* v)
{
    if (!h || !v) return TT_ERR_ARG;
    if (!h->have_fwd) return TT_ERR_STATE;
    cudaStream_t s = h->used_stream ? h->last_stream : (cudaStream_t)0;
    WsCounters c;
    if (cudaMemcpyAsync(&c, h->at(h->lay.counters), sizeof(c), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return TT_ERR_CUDA;
    const Layout& y = h->lay;
    v->num_lookups = h->fwd_L;
    v->num_unique = c.num_unique;
    v->num_groups = c.num_groups;
    v->key_bits = h->ibits;
    v->key_bytes = h->key_bytes();
    v->sorted_keys = h->at(y.keys[h->fwd_which]);
    v->perm = (const int32_t*)h->at(y.vals[h->fwd_which]);
    v->uniq_keys = h->at(y.uniq_keys);
    v->uniq_start = (const int32_t*)h->at(y.uniq_start);
    v->grp_start = (const int32_t*)h->at(y.grp_start);
    v->bag_sorted = (const int32_t*)h->at(y.bag_sorted);
    return TT_OK;
}

static int tt_emb_copy_segmentation_impl(tt_emb_t h, void* sorted_keys, int32_t* perm, void* uniq_keys,
                             int32_t* uniq_start, int32_t* grp_start, int32_t* bag_sorted)
{
    tt_seg_view v;
    int rc = tt_emb_get_segmentation(h, &v);
    if (rc != TT_OK) return rc;
    const size_t L = (size_t)v.num_lookups, U = (size_t)v.num_unique, G = (size_t)v.num_groups;
    const size_t kb = (size_t)v.key_bytes;
    cudaError_t e = cudaSuccess;
    if (sorted_keys && L) e = cudaMemcpy(sorted_keys, v.sorted_keys, L * kb, cudaMemcpyDefault);
    if (e == cudaSuccess && perm && L) e = cudaMemcpy(perm, v.perm, L * 4, cudaMemcpyDefault);
    if (e == cudaSuccess && uniq_keys && U) e = cudaMemcpy(uniq_keys, v.uniq_keys, U * kb, cudaMemcpyDefault);
    if (e == cudaSuccess && uniq_start && U) e = cudaMemcpy(uniq_start, v.uniq_start, (U + 1) * 4, cudaMemcpyDefault);
    if (e == cudaSuccess && grp_start && G) e = cudaMemcpy(grp_start, v.grp_start, (G + 1) * 4, cudaMemcpyDefault);
    if (e == cudaSuccess && bag_sorted && L) e = cudaMemcpy(bag_sorted, v.bag_sorted, L * 4, cudaMemcpyDefault);
    return cuda_status(e);
}

static int tt_emb_enable_timing_impl(tt_emb_t h, int enable)
{
    if (!h) return TT_ERR_ARG;
    h->fold();
    h->timing = enable != 0;
    for (int i = 0; i < TT_EMB_NUM_PHASES; ++i) h->phase_ms[i] = 0.0;
    h->launches = 0;
    return TT_OK;
}

static int tt_emb_phase_times_impl(tt_emb_t h, double* ms, int64_t* launches)
{
    if (!h || !ms) return TT_ERR_ARG;
    for (int i = 0; i < TT_EMB_NUM_PHASES; ++i) ms[i] = h->phase_ms[i];
    if (launches) *launches = h->launches;
    return TT_OK;
}

// Public entry points: the implementations above, with failures recorded for tt_emb_last_error.
int tt_emb_set_cores(tt_emb_t h, float* const* cores, float* const* core_grads)
{
    return note(h, tt_emb_set_cores_impl(h, cores, core_grads));
}
int tt_emb_workspace_size(tt_emb_t h, int64_t max_lookups, int64_t batch, size_t* bytes)
{
    return note(h, tt_emb_workspace_size_impl(h, max_lookups, batch, bytes));
}
int tt_emb_set_workspace(tt_emb_t h, void* workspace, size_t bytes, int64_t max_lookups, int64_t batch)
{
    return note(h, tt_emb_set_workspace_impl(h, workspace, bytes, max_lookups, batch));
}
int tt_emb_forward(tt_emb_t h, const int64_t* indices, const int64_t* offsets, int64_t num_lookups,
                   int64_t batch, float* out, tt_stream_t stream)
{
    return note(h, tt_emb_forward_impl(h, indices, offsets, num_lookups, batch, out, stream));
}
int tt_emb_backward(tt_emb_t h, const float* grad_out, tt_stream_t stream)
{
    return note(h, tt_emb_backward_impl(h, grad_out, stream));
}
int tt_emb_backward_sgd(tt_emb_t h, const float* grad_out, float lr, tt_stream_t stream)
{
    return note(h, tt_emb_backward_sgd_impl(h, grad_out, lr, stream));
}
int tt_emb_sgd_update(tt_emb_t h, float lr, tt_stream_t stream)
{
    return note(h, tt_emb_sgd_update_impl(h, lr, stream));
}
int tt_emb_get_segmentation(tt_emb_t h, tt_seg_view* v)
{
    return note(h, tt_emb_get_segmentation_impl(h, v));
}
int tt_emb_copy_segmentation(tt_emb_t h, void* sorted_keys, int32_t* perm, void* uniq_keys,
                             int32_t* uniq_start, int32_t* grp_start, int32_t* bag_sorted)
{
    return note(h, tt_emb_copy_segmentation_impl(h, sorted_keys, perm, uniq_keys, uniq_start, grp_start,
                                                 bag_sorted));
}
int tt_emb_enable_timing(tt_emb_t h, int enable) { return note(h, tt_emb_enable_timing_impl(h, enable)); }
int tt_emb_phase_times(tt_emb_t h, double* ms, int64_t* launches)
{
    return note(h, tt_emb_phase_times_impl(h, ms, launches));
}

int tt_emb_last_error(tt_emb_t h)
{
    if (!h) return TT_ERR_ARG;
    const int rc = h->last_error;
    h->last_error = TT_OK;
    return rc;
}

int tt_emb_set_probe(tt_emb_t h, uint64_t* records, int32_t max_blocks)
{
    if (!h || max_blocks < 0 || (records && max_blocks == 0)) return note(h, TT_ERR_ARG);
    if (records && ((uintptr_t)records & 7)) return note(h, TT_ERR_ARG);
    h->probe = (unsigned long long*)records;
    h->probe_cap = records ? max_blocks : 0;
    return TT_OK;
}

int tt_emb_debug_inject(tt_emb_t h, int32_t what, int32_t spin_limit)
{
    if (!h || spin_limit < 0) return note(h, TT_ERR_ARG);
    switch (what) {
    case TT_INJECT_NONE: break;
    case TT_INJECT_POOL_WAIT:
        if (!h->fast) return note(h, TT_ERR_UNSUPPORTED);
        break;
    case TT_INJECT_MMA_WAIT_FWD:
        if (!h->tc) return note(h, TT_ERR_UNSUPPORTED);
        break;
    case TT_INJECT_MMA_WAIT_BWD:
        if (!h->tc || !k3_tc_bwd_supported(h->view_params())) return note(h, TT_ERR_UNSUPPORTED);
        break;
    default: return note(h, TT_ERR_ARG);
    }
    h->inject = what;
    h->inject_spin = spin_limit;
    return TT_OK;
}

void tt_emb_destroy(tt_emb_t h)
{
    if (!h) return;
    h->fold();
    for (cudaEvent_t e : h->pool) cudaEventDestroy(e);
    if (h->d_status) cudaFree(h->d_status);
    delete h;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Forward into caller-provided scratch (used by tt_emb_forward_noalloc in
// noalloc.cu).  Same launch sequence as tt_emb_forward, laid out for exactly
// num_lookups in `scratch`; no event recording, no allocation, and the
// segmentation is not kept for a backward pass.
// ---------------------------------------------------------------------------
namespace tt {

size_t scratch_bytes_for(tt_emb_t h, int64_t num_lookups)
{
    FastDims off;
    memset(&off, 0, sizeof(off));
    return make_layout(h->key_bytes(), num_lookups, 1, off).total;
}

int forward_with_scratch(tt_emb_t h, char* scratch, size_t scratch_bytes, const int64_t* indices,
                         const int64_t* offsets, int64_t num_lookups, int64_t batch, float* out,
                         cudaStream_t s)
{
    if (!h || !scratch || !offsets || !out || num_lookups < 0 || batch < 1) return TT_ERR_ARG;
    if (num_lookups > 0 && !indices) return TT_ERR_ARG;
    if (!h->have_cores) return TT_ERR_STATE;
    FastDims off;
    memset(&off, 0, sizeof(off));
    const Layout y = make_layout(h->key_bytes(), num_lookups, batch, off);
    if (y.total > scratch_bytes) return TT_ERR_WORKSPACE;
    h->last_stream = s;
    h->used_stream = true;
    h->have_fwd = false;
    auto at = [&](size_t off) { return scratch + off; };
    WsCounters* counters = (WsCounters*)at(y.counters);
    const int64_t L = num_lookups;
    cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float) * (size_t)batch * h->T * h->D, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(counters, 0, sizeof(WsCounters), s);
    if (e != cudaSuccess) return TT_ERR_CUDA;
    KeyParams kp;
    memset(&kp, 0, sizeof(kp));
    kp.T = h->T;
    kp.ibits = h->ibits;
    kp.B = batch;
    kp.L = L;
    kp.unique_only = h->opt.grouping == TT_GROUP_UNIQUE_ONLY;
    for (int t = 0; t < h->T; ++t) {
        kp.nrows[t] = (uint32_t)h->n_rows[t];
        kp.nlast[t] = (uint32_t)h->n[t][h->k - 1];
    }
    int32_t* bag_of_pos = (int32_t*)at(y.bag_of_pos);
    SortBuffers sb;
    sb.keys[0] = at(y.keys[0]);
    sb.keys[1] = at(y.keys[1]);
    sb.vals[0] = (int32_t*)at(y.vals[0]);
    sb.vals[1] = (int32_t*)at(y.vals[1]);
    sb.hist = (uint32_t*)at(y.hist);
    sb.digit_total = (uint32_t*)at(y.digit_total);
    int nl = 0;
    e = launch_make_keys(kp, h->key64, indices, offsets, sb.keys[0], sb.vals[0], bag_of_pos,
                         h->d_status, s, &nl);
    if (e == cudaSuccess && L > 0) {
        int which = 0;
        e = radix_sort_pairs(h->key64, L, h->ibits + h->tbits, sb, &which, h->d_status, s, &nl);
        if (e == cudaSuccess)
            e = launch_segment(kp, h->key64, sb.keys[which], sb.vals[which], bag_of_pos,
                               at(y.uniq_keys), (int32_t*)at(y.uniq_start), (int32_t*)at(y.grp_start),
                               (int32_t*)at(y.bag_sorted), (uint64_t*)at(y.partials), counters,
                               nullptr, nullptr, h->d_status, s, &nl);
        if (e == cudaSuccess) {
            CoreParams cp = h->core_params();
            cp.B = batch;
            const int grid = h->opt.grid > 0 ? h->opt.grid : h->num_sms * 8;
            e = launch_forward_generic(cp, h->key64, at(y.uniq_keys), (const int32_t*)at(y.uniq_start),
                                       (const int32_t*)at(y.grp_start), (const int32_t*)at(y.bag_sorted),
                                       counters, L, out, h->d_status, s, grid, &nl);
        }
    }
    h->launches += nl;
    return cuda_status(e);
}

}  // namespace tt
