// moe_sparse.cu -- the C ABI (include/moe_sparse.h): argument checking,
// weight repacking, workspace ownership and path dispatch.
#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <set>

#include "../../include/moe_sparse.h"
#include "internal.h"

namespace moe {
}

namespace {

constexpr unsigned kMagic = 0x4d6f4553u;   // "MoES"
constexpr int kDefaultTStar = 16;       // AUTO: sparse iff T <= this, when the dense branch exists

struct Block {   // bump allocator over one cudaMalloc
    char *base = nullptr;
    size_t used = 0, cap = 0;
    void *take(size_t bytes)
    {
        size_t off = (used + 255) & ~size_t(255);
        if (off + bytes > cap) return nullptr;
        used = off + bytes;
        return base + off;
    }
};

}  // namespace

struct moe_sparse_s {
    unsigned magic;
    int device;
    int n_sm;
    moe::Dims dm;
    moe::DeviceWeights w;
    moe::Workspace ws;
    unsigned long long *stats_dev;
    void *weight_mem;
    void *ws_mem;
    int path;
    int t_star;
    // the last forward
    int last_T, last_path, last_masked;
    cudaStream_t last_stream;
    moe::DenseState dense;   // tensor maps of the dense branch (dense.ok: available)
    cudaEvent_t ev[3];   // optional launch events (moe_set_launch_events)
    int n_ev;
    float *scores;       // calibration buffer, allocated by the first moe_calibrate_tau
    unsigned *hist;      // 256 bins, inside the workspace
    int inject_next;     // test-only fault for the next sparse forward (moe_debug_inject)
    int fused_router;    // route decode batches inside the expert kernel (moe_set_fused_router)
    float tau_shared;    // the shared experts' threshold on masked forwards (moe_set_shared_tau)
    int last_fused;      // the last forward routed inside the expert kernel
    // rank budget (moe_set_rank_budget): < 0 off; else each routed pair keeps
    // its rank_r highest-scoring neurons on masked forwards
    int rank_r;
    float *rank_a;       // [max_tokens * k][f] silu(g) of the first pass
    float *rank_v;       // [max_tokens * k] cut values
    int *rank_j;         // [max_tokens * k] last tied index kept
    float cap_gamma;     // capacity factor of the token drop (moe_set_capacity); <= 0: none
    int last_cap;        // the capacity the last forward applied (-1: none)
    float *det_rows;     // deterministic combine's rows (moe_set_deterministic), allocated on first use
    int det;             // later forwards combine in a fixed order (ws.ypart = det_rows)
    int last_det;
};

static bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// Host-side fault injection for tests: MOE_INJECT_ALLOC_FAIL=<what> makes the
// named device allocation ("weights", "workspace", "scores", "rank" or
// "deterministic") report failure
// without being attempted, so the error paths can be exercised on a live GPU.
static bool inject_alloc_fail(const char *what)
{
    const char *v = std::getenv("MOE_INJECT_ALLOC_FAIL");
    return v && std::strcmp(v, what) == 0;
}

// Live handles, so that a NULL, foreign or destroyed handle is an error code
// rather than a dereference of freed memory.
static std::mutex g_live_mu;
static std::set<moe_handle> g_live;

static bool is_live(moe_handle h)
{
    std::lock_guard<std::mutex> lk(g_live_mu);
    return h && g_live.count(h) && h->magic == kMagic;
}

static int check_handle(moe_handle h)
{
    if (!is_live(h)) return MOE_EHANDLE;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ECUDA;
    if (dev != h->device) return MOE_EINVAL;
    return MOE_OK;
}

static void free_handle(moe_handle h)
{
    if (!h) return;
    {
        std::lock_guard<std::mutex> lk(g_live_mu);
        g_live.erase(h);
    }
    cudaDeviceSynchronize();
    if (h->weight_mem) cudaFree(h->weight_mem);
    if (h->ws_mem) cudaFree(h->ws_mem);
    if (h->scores) cudaFree(h->scores);
    if (h->rank_a) cudaFree(h->rank_a);
    if (h->det_rows) cudaFree(h->det_rows);
    h->magic = 0;
    delete h;
}


extern "C" int moe_sparse_create(const moe_weights *w, int E, int top_k, int d_model, int d_ff,
                                 int n_shared, int max_tokens, moe_handle *out)
{
    if (!out) return MOE_EINVAL;
    *out = nullptr;
    if (!w) return MOE_EINVAL;
    if (max_tokens == 0) max_tokens = 4096;
    if (E < 1 || E > moe::kMaxExperts || top_k < 1 || top_k > E) return MOE_EINVAL;
    if (d_model < 8 || d_model % 8 != 0 || d_model > 4096) return MOE_EINVAL;
    if (d_ff < 32 || d_ff % 32 != 0 || d_ff > 65535) return MOE_EINVAL;
    if (n_shared < 0 || n_shared > 8 || max_tokens < 1 || max_tokens > 65536) return MOE_EINVAL;
    if (!w->w_router || !w->w_gate || !w->w_up || !w->w_down) return MOE_EINVAL;
    const bool any_shared = w->ws_gate || w->ws_up || w->ws_down;
    const bool all_shared = w->ws_gate && w->ws_up && w->ws_down;
    if (n_shared > 0 ? !all_shared : any_shared) return MOE_EINVAL;
    const void *ptrs[7] = {w->w_router, w->w_gate, w->w_up, w->w_down, w->ws_gate, w->ws_up, w->ws_down};
    for (const void *p : ptrs)
        if (!aligned16(p)) return MOE_EALIGN;

    moe_handle h = new (std::nothrow) moe_sparse_s();
    if (!h) return MOE_ENOMEM;
    h->magic = kMagic;
    h->path = MOE_PATH_AUTO;
    h->t_star = INT_MAX;   // set below once the dense branch is known to be available
    if (cudaGetDevice(&h->device) != cudaSuccess ||
        cudaDeviceGetAttribute(&h->n_sm, cudaDevAttrMultiProcessorCount, h->device) != cudaSuccess) {
        delete h;
        return MOE_ECUDA;
    }
    moe::Dims &dm = h->dm;
    dm.E = E; dm.k = top_k; dm.d = d_model; dm.f = d_ff; dm.S = n_shared; dm.max_tokens = max_tokens;
    dm.dp = (d_model + 127) & ~127;
    dm.fp = (d_ff + 127) & ~127;
    dm.n_kb = dm.dp / 64;
    dm.n_blk = dm.fp / 128;

    const size_t fd = (size_t)d_ff * d_model;
    const bool dense = moe::dense_supported(dm);
    const size_t gd = (size_t)dm.fp * dm.dp;   // gate tiles per expert (elements)
    const size_t wbytes = 2 * ((size_t)E * d_model + E * (gd + 2 * fd) + (size_t)n_shared * (gd + 2 * fd)) +
                          (dense ? 2 * ((size_t)E + n_shared) * fd : 0) + 16 * 256;
    const size_t T = max_tokens, P = T * top_k;
    const size_t wsbytes = 4 * T * E + 4 * P + 4 * P + 4 * P + 8 * P + 4 * P * (d_ff / 32) + 4 * T * d_model +
                           4 * T + 4 * ((T + 7) / 8) + 64 + sizeof(moe::Plan) + 2 * (P + T) * d_model +
                           2 * (P + n_shared * T) * d_ff + 2 * 2 * T * d_model + 32 * (size_t)dm.dp + 64 + 1024 +
                           64 + 4 * moe::kMaxExperts + 40 * 256;
    // gate split workspace (batches of one or two tokens): items of such a batch
    // number at most (min(2k, E) + S) x blocks
    const long long split_items = (long long)((2 * top_k < E ? 2 * top_k : E) + n_shared) * dm.n_blk;
    const bool split_ok = split_items <= 4096;
    const size_t part_floats = (size_t)(moe::kMaxParts - 1) * moe::kBlk * moe::kSplitCols;   // per item
    const size_t split_bytes =
        split_ok ? (size_t)split_items * (part_floats * sizeof(float) + sizeof(int) + sizeof(moe::SplitShare)) + 3 * 256
                 : 0;
    if (inject_alloc_fail("weights") || cudaMalloc(&h->weight_mem, wbytes) != cudaSuccess) {
        cudaGetLastError();
        h->weight_mem = nullptr;
        free_handle(h);
        return MOE_ENOMEM;
    }
    if (inject_alloc_fail("workspace") || cudaMalloc(&h->ws_mem, wsbytes + split_bytes) != cudaSuccess) {
        cudaGetLastError();
        h->ws_mem = nullptr;
        free_handle(h);
        return MOE_ENOMEM;
    }

    Block wb{(char *)h->weight_mem, 0, wbytes};
    uint16_t *wr = (uint16_t *)wb.take(2 * (size_t)E * d_model);
    uint16_t *wg = (uint16_t *)wb.take(2 * E * gd), *wud = (uint16_t *)wb.take(4 * E * fd);
    uint16_t *wsg = nullptr, *wsud = nullptr;
    if (n_shared) {
        wsg = (uint16_t *)wb.take(2 * n_shared * gd);
        wsud = (uint16_t *)wb.take(4 * n_shared * fd);
    }
    uint16_t *wdt = nullptr, *wsdt = nullptr;
    if (dense) {
        wdt = (uint16_t *)wb.take(2 * E * fd);
        if (n_shared) wsdt = (uint16_t *)wb.take(2 * n_shared * fd);
    }
    if (!wr || !wg || !wud || (n_shared && (!wsg || !wsud)) || (dense && (!wdt || (n_shared && !wsdt)))) {
        free_handle(h);
        return MOE_ENOMEM;
    }
    h->w = {wr, wg, wud, wsg, wsud, wdt, wsdt};

    Block sb{(char *)h->ws_mem, 0, wsbytes + split_bytes};
    moe::Workspace &ws = h->ws;
    ws.logits = (float *)sb.take(4 * T * E);
    ws.topk_idx = (int *)sb.take(4 * P);
    ws.topk_w = (float *)sb.take(4 * P);
    ws.perm = (int *)sb.take(4 * P);
    ws.perm_tok = (int *)sb.take(4 * P);
    ws.perm_w = (float *)sb.take(4 * P);
    ws.mask = (uint32_t *)sb.take(4 * P * (d_ff / 32));
    ws.y_acc = (float *)sb.take(4 * T * d_model);
    ws.tok_cnt = (int *)sb.take(4 * T);
    ws.tile_ticket = (int *)sb.take(4 * ((T + 7) / 8));
    ws.done_ticket = (int *)sb.take(4);
    ws.error_word = (int *)sb.take(4);
    ws.error_sticky = (int *)sb.take(4);
    ws.route_count = (int *)sb.take(4);
    ws.tail = (int *)sb.take(8);
    ws.cursor = (int *)sb.take(4 * moe::kMaxExperts);
    ws.ecount = (int *)sb.take(4 * moe::kMaxExperts);
    if (split_ok) {
        ws.gpart = (float *)sb.take((size_t)split_items * part_floats * sizeof(float));
        ws.gcnt = (int *)sb.take((size_t)split_items * sizeof(int));
        ws.gshare = (moe::SplitShare *)sb.take((size_t)split_items * sizeof(moe::SplitShare));
        ws.gcnt_n = ws.gpart && ws.gcnt && ws.gshare ? (int)split_items : 0;
        if (!ws.gcnt_n) ws.gpart = nullptr, ws.gcnt = nullptr;
    }
    ws.plan = (moe::Plan *)sb.take(sizeof(moe::Plan));
    ws.x_perm = (uint16_t *)sb.take(2 * (P + T) * d_model);
    ws.h_perm = (uint16_t *)sb.take(2 * (P + n_shared * T) * d_ff);
    ws.x_stage = (uint16_t *)sb.take(2 * T * d_model);
    ws.out_stage = (uint16_t *)sb.take(2 * T * d_model);
    ws.x_tiles = (uint16_t *)sb.take(32 * (size_t)dm.dp);
    h->stats_dev = (unsigned long long *)sb.take(64);
    h->hist = (unsigned *)sb.take(256 * sizeof(unsigned));
    if (!h->stats_dev || !h->hist || !ws.x_tiles || !ws.error_sticky || !ws.route_count || !ws.tail || !ws.cursor || !ws.ecount) {
        free_handle(h);
        return MOE_ENOMEM;
    }

    cudaStream_t st = nullptr;
    bool ok = cudaMemsetAsync(h->ws_mem, 0, wsbytes + split_bytes, st) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(wr, w->w_router, 2 * (size_t)E * d_model, cudaMemcpyDeviceToDevice, st) == cudaSuccess;
    const int d = d_model;
    ok = ok && moe::launch_repack_gate_tiles((const uint16_t *)w->w_gate, wg, E, dm, st) == cudaSuccess;
    ok = ok && moe::launch_repack_transpose((const uint16_t *)w->w_up, wud, E, d, d_ff, 2 * d, 0, st) == cudaSuccess;
    ok = ok && moe::launch_repack_rows((const uint16_t *)w->w_down, wud, E, d_ff, d, 2 * d, d, st) == cudaSuccess;
    if (dense) {
        ok = ok && moe::launch_repack_transpose((const uint16_t *)w->w_down, wdt, E, d_ff, d, d_ff, 0, st) == cudaSuccess;
        if (n_shared)
            ok = ok && moe::launch_repack_transpose((const uint16_t *)w->ws_down, wsdt, n_shared, d_ff, d, d_ff, 0, st) == cudaSuccess;
    }
    if (n_shared) {
        ok = ok && moe::launch_repack_gate_tiles((const uint16_t *)w->ws_gate, wsg, n_shared, dm, st) == cudaSuccess;
        ok = ok && moe::launch_repack_transpose((const uint16_t *)w->ws_up, wsud, n_shared, d, d_ff, 2 * d, 0, st) == cudaSuccess;
        ok = ok && moe::launch_repack_rows((const uint16_t *)w->ws_down, wsud, n_shared, d_ff, d, 2 * d, d, st) == cudaSuccess;
    }
    ok = ok && cudaDeviceSynchronize() == cudaSuccess;
    ok = ok && moe::dense_setup(h->dm, h->w, h->ws, &h->dense);
    // measured on B200 at the OLMoE shape, 90 % sparsity: the sparse branch
    // is faster through T = 16 tokens, the dense branch from T = 32 on
    if (h->dense.ok) h->t_star = kDefaultTStar;
    if (!ok) {
        cudaGetLastError();
        free_handle(h);
        return MOE_ECUDA;
    }
    h->fused_router = 1;
    h->rank_r = -1;
    h->last_cap = -1;
    h->last_T = 0;
    h->last_path = MOE_PATH_SPARSE;
    h->last_masked = 1;
    h->last_stream = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_live_mu);
        g_live.insert(h);
    }
    *out = h;
    return MOE_OK;
}

extern "C" void moe_sparse_destroy(moe_handle h)
{
    if (!is_live(h)) return;
    free_handle(h);
}

// The router for a batch: from 1024 tokens on (when the layer has the dense
// branch) the logits are one tcgen05 GEMM and the router kernel only selects
// and buckets; smaller batches keep the router kernel's own logits, which
// are spread over more CTAs and cost one launch less.
constexpr int kTcLogitsMinT = 1024;
static cudaError_t route(moe_handle h, const uint16_t *xb, int T, int tile_tokens, cudaStream_t st, int cap = -1)
{
    if (T >= kTcLogitsMinT && h->dense.ok) {
        cudaError_t e = moe::launch_logits_tc(h->dm, h->ws, h->dense, xb, T, h->n_sm, st);
        if (e != cudaSuccess) return e;
        return moe::launch_router(h->dm, h->w, h->ws, xb, T, tile_tokens, st, cap, true);
    }
    return moe::launch_router(h->dm, h->w, h->ws, xb, T, tile_tokens, st, cap);
}

static int run_forward(moe_handle h, const void *x, int T, float tau, bool masked, void *out,
                       void *stream, int forced_path)
{
    int rc = check_handle(h);
    if (rc) return rc;
    if (!x || !out) return MOE_EINVAL;
    if (T < 1 || T > h->dm.max_tokens) return MOE_EINVAL;
    if (std::isnan(tau)) return MOE_EINVAL;
    if (!aligned16(x) || !aligned16(out)) return MOE_EALIGN;
    if (x == out) return MOE_EINVAL;
    int path = forced_path;
    if (path == MOE_PATH_AUTO) path = h->path;
    if (path == MOE_PATH_AUTO) path = (T <= h->t_star) ? MOE_PATH_SPARSE : MOE_PATH_DENSE;
    const bool rank = masked && h->rank_r >= 0;
    // capacity-aware token drop: C = ceil(gamma * T * k / E) pairs per expert;
    // an expert holds at most T pairs, so C >= T drops nothing
    int cap = -1;
    if (h->cap_gamma > 0.f) {
        const double c = std::ceil((double)h->cap_gamma * ((double)T * h->dm.k) / h->dm.E);
        if (c < (double)T) {
            if ((long long)T * h->dm.k > 4096) return MOE_ENOTSUP;
            cap = (int)c;
        }
    }
    if (rank) {   // the rank budget is built on the sparse path only
        if (forced_path == MOE_PATH_DENSE || (forced_path == MOE_PATH_AUTO && h->path == MOE_PATH_DENSE))
            return MOE_ENOTSUP;
        path = MOE_PATH_SPARSE;
    }
    if (path == MOE_PATH_DENSE && !h->dense.ok) {
        if (forced_path == MOE_PATH_DENSE || h->path == MOE_PATH_DENSE) return MOE_ENOTSUP;
        path = MOE_PATH_SPARSE;   // AUTO on a shape the dense branch does not cover
    }
    cudaStream_t st = (cudaStream_t)stream;
    const uint16_t *xb = (const uint16_t *)x;
    uint16_t *ob = (uint16_t *)out;
    cudaError_t e = cudaSuccess;
    // inside a stream capture the launch events must be external nodes, so that
    // every replay records them; outside a capture a plain record
    cudaStreamCaptureStatus capst = cudaStreamCaptureStatusNone;
    if (h->n_ev && cudaStreamIsCapturing(st, &capst) != cudaSuccess) capst = cudaStreamCaptureStatusNone;
    const unsigned ev_flags =
        capst == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : cudaEventRecordDefault;
    if (h->n_ev) e = cudaEventRecordWithFlags(h->ev[0], st, ev_flags);
    bool fused = false;
    if (path == MOE_PATH_SPARSE) {
        const moe::SparseTiling til = moe::sparse_tiling(T, h->dm.d, h->dm.S);
        // decode batches route inside the expert kernel: no router launch
        fused = !rank && cap < 0 && h->fused_router && moe::fused_possible(h->dm, T);
        if (e == cudaSuccess && !fused) e = route(h, xb, T, til.nt, st, cap);
        if (e == cudaSuccess && h->n_ev) e = cudaEventRecordWithFlags(h->ev[1], st, ev_flags);
        if (rank) {   // silu(g) of the routed pairs, each pair's cut, then the masked layer
            moe::RankPass r1{h->rank_a, nullptr, nullptr, false};
            moe::RankPass r2{h->rank_a, h->rank_v, h->rank_j, true};
            if (e == cudaSuccess)
                e = moe::launch_expert_sparse(h->dm, h->w, h->ws, xb, T, tau, masked, ob, til, h->n_sm, st, nullptr,
                                              0, false, h->tau_shared, false, &r1);
            if (e == cudaSuccess)
                e = moe::launch_rank_select(h->rank_a, T * h->dm.k, h->dm.f, h->rank_r, h->rank_v, h->rank_j, st);
            if (e == cudaSuccess)
                e = moe::launch_expert_sparse(h->dm, h->w, h->ws, xb, T, tau, masked, ob, til, h->n_sm, st, nullptr,
                                              h->inject_next, false, h->tau_shared, false, &r2);
        } else if (e == cudaSuccess) {
            e = moe::launch_expert_sparse(h->dm, h->w, h->ws, xb, T, tau, masked, ob, til, h->n_sm, st, nullptr,
                                          h->inject_next, fused, h->tau_shared, false, nullptr,
                                          fused && h->fused_router == 2);
        }
        h->inject_next = 0;
    } else {
        if (e == cudaSuccess) e = route(h, xb, T, 8, st, cap);
        if (e == cudaSuccess && h->n_ev) e = cudaEventRecordWithFlags(h->ev[1], st, ev_flags);
        if (e == cudaSuccess)
            e = moe::launch_dense(h->dm, h->ws, h->dense, xb, T, tau, masked, ob, st, h->tau_shared, h->n_sm);
    }
    if (e == cudaSuccess && h->n_ev) e = cudaEventRecordWithFlags(h->ev[2], st, ev_flags);
    h->last_T = T;
    h->last_path = path;
    h->last_masked = masked;
    h->last_fused = fused ? h->fused_router : 0;
    h->last_cap = cap;
    h->last_det = h->det;
    h->last_stream = st;
    return e == cudaSuccess ? MOE_OK : MOE_ECUDA;
}

extern "C" int moe_sparse_forward(moe_handle h, const void *x, int T, float tau, void *out, void *stream)
{
    return run_forward(h, x, T, tau, true, out, stream, MOE_PATH_AUTO);
}

extern "C" int moe_dense_forward(moe_handle h, const void *x, int T, void *out, void *stream)
{
    return run_forward(h, x, T, 0.0f, false, out, stream, MOE_PATH_DENSE);
}

extern "C" int moe_sparse_forward_host(moe_handle h, const void *x_host, int T, float tau,
                                       void *out_host, void *stream)
{
    int rc = check_handle(h);
    if (rc) return rc;
    if (!x_host || !out_host || T < 1 || T > h->dm.max_tokens) return MOE_EINVAL;
    cudaStream_t st = (cudaStream_t)stream;
    const size_t bytes = (size_t)T * h->dm.d * 2;
    if (cudaMemcpyAsync(h->ws.x_stage, x_host, bytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
        return MOE_ECUDA;
    rc = moe_sparse_forward(h, h->ws.x_stage, T, tau, h->ws.out_stage, stream);
    if (rc) return rc;
    if (cudaMemcpyAsync(out_host, h->ws.out_stage, bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return MOE_ECUDA;
    return cudaStreamSynchronize(st) == cudaSuccess ? MOE_OK : MOE_ECUDA;
}

extern "C" int moe_set_path(moe_handle h, int path)
{
    if (!is_live(h)) return MOE_EHANDLE;
    if (path != MOE_PATH_AUTO && path != MOE_PATH_SPARSE && path != MOE_PATH_DENSE) return MOE_EINVAL;
    if (path == MOE_PATH_DENSE && !h->dense.ok) return MOE_ENOTSUP;
    h->path = path;
    return MOE_OK;
}

extern "C" int moe_set_t_star(moe_handle h, int t_star)
{
    if (!is_live(h)) return MOE_EHANDLE;
    if (t_star < 0) return MOE_EINVAL;
    h->t_star = t_star;
    return MOE_OK;
}

extern "C" int moe_tune_t_star(moe_handle h, const void *x, int T_max, float tau, int *t_star_out, void *stream)
{
    int rc = check_handle(h);
    if (rc) return rc;
    if (!x || !t_star_out || T_max < 1 || T_max > h->dm.max_tokens || std::isnan(tau)) return MOE_EINVAL;
    if (!aligned16(x)) return MOE_EALIGN;
    if (!h->dense.ok) {   // no dense branch: AUTO always takes the sparse one
        h->t_star = INT_MAX;
        *t_star_out = INT_MAX;
        return MOE_OK;
    }
    // the caller's earlier work (x) is complete, then everything runs on a
    // private stream, where each forward can be captured into a graph
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MOE_ECUDA;
    int l2 = 0;
    if (cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, h->device) != cudaSuccess) return MOE_ECUDA;
    const size_t flush_bytes = 2 * (size_t)(l2 > 0 ? l2 : (64 << 20));
    void *flush = nullptr;
    if (cudaMalloc(&flush, flush_bytes) != cudaSuccess) { cudaGetLastError(); return MOE_ENOMEM; }
    cudaStream_t st = nullptr;
    cudaEvent_t e0 = nullptr, e1 = nullptr;
    if (cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) != cudaSuccess || cudaEventCreate(&e0) != cudaSuccess ||
        cudaEventCreate(&e1) != cudaSuccess) {
        if (e0) cudaEventDestroy(e0);
        if (st) cudaStreamDestroy(st);
        cudaFree(flush);
        cudaGetLastError();
        return MOE_ECUDA;
    }
    const int saved_ev = h->n_ev;
    h->n_ev = 0;   // the caller's launch events stay out of the tuning runs
    // the median of five device-timed forwards of the first T rows of x, L2
    // flushed before each; the forward is captured into a graph and launched
    // whole, so neither branch pays for host-side gaps between its launches
    auto time_path = [&](int T, int path, int row0, float *us) -> int {
        cudaGraph_t g = nullptr;
        cudaGraphExec_t ge = nullptr;
        const void *xs = (const uint16_t *)x + (size_t)row0 * h->dm.d;
        if (cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal) != cudaSuccess) return MOE_ECUDA;
        const int frc = run_forward(h, xs, T, tau, true, h->ws.out_stage, st, path);
        const cudaError_t ce = cudaStreamEndCapture(st, &g);
        if (frc || ce != cudaSuccess || cudaGraphInstantiate(&ge, g, 0) != cudaSuccess) {
            if (g) cudaGraphDestroy(g);
            cudaGetLastError();
            return frc ? frc : MOE_ECUDA;
        }
        float t[5];
        int rc2 = MOE_OK;
        for (int r = -1; r < 5 && rc2 == MOE_OK; ++r) {   // one untimed run first
            if (cudaMemsetAsync(flush, r & 0xff, flush_bytes, st) != cudaSuccess ||
                moe::launch_read_all(flush, flush_bytes, h->hist, h->n_sm, st) != cudaSuccess ||
                cudaEventRecord(e0, st) != cudaSuccess || cudaGraphLaunch(ge, st) != cudaSuccess ||
                cudaEventRecord(e1, st) != cudaSuccess || cudaEventSynchronize(e1) != cudaSuccess ||
                (r >= 0 && cudaEventElapsedTime(&t[r], e0, e1) != cudaSuccess))
                rc2 = MOE_ECUDA;
        }
        cudaGraphExecDestroy(ge);
        cudaGraphDestroy(g);
        if (rc2 != MOE_OK) return rc2;
        std::sort(t, t + 5);
        *us = 1000.f * t[2];
        return MOE_OK;
    };
    // batch sizes 1, 2, 3, 4, 6, 8, 12, 16, 24, ... (steps of about 1.5x) up to T_max
    int best = 0;
    rc = MOE_OK;
    for (int T = 1, last = 0; T <= T_max && rc == MOE_OK;) {
        float us_s = 0.f, us_d = 0.f, us_s2 = 0.f;
        rc = time_path(T, MOE_PATH_SPARSE, 0, &us_s);
        // the sparse branch's cost depends on how the batch routes (its load
        // balance over the experts): where x holds them, a second, disjoint
        // batch of the same size is timed too and the two averaged.  The
        // dense branch's cost is nearly the same for every batch of a size.
        if (rc == MOE_OK && 2 * T <= T_max) {
            rc = time_path(T, MOE_PATH_SPARSE, T_max - T, &us_s2);
            us_s = 0.5f * (us_s + us_s2);
        }
        if (rc == MOE_OK) rc = time_path(T, MOE_PATH_DENSE, 0, &us_d);
        if (rc != MOE_OK) break;
        // the dense branch is faster from here on; a sparse time within 5 %
        // of the dense one counts as slower (the batches only sample routing)
        if (us_s > 0.95f * us_d) break;
        best = T;
        last = T;
        T = T < 4 ? T + 1 : (T % 3 == 0 ? T * 4 / 3 : T * 3 / 2);
        if (T > T_max && last < T_max) T = T_max;
    }
    h->n_ev = saved_ev;
    // the timing forwards ran on the private stream, which is about to go:
    // moe_query_stats (which describes the last of them) synchronises the
    // caller's stream instead; all of that work is complete already
    if (cudaStreamSynchronize(st) != cudaSuccess && rc == MOE_OK) rc = MOE_ECUDA;
    h->last_stream = (cudaStream_t)stream;
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    cudaStreamDestroy(st);
    cudaFree(flush);
    if (rc != MOE_OK) return rc;
    h->t_star = best;
    *t_star_out = best;
    return MOE_OK;
}

extern "C" int moe_debug_router(moe_handle h, const void *x, int T, int *idx_out, float *w_out, void *stream)
{
    int rc = check_handle(h);
    if (rc) return rc;
    if (!x || !idx_out || !w_out || T < 1 || T > h->dm.max_tokens) return MOE_EINVAL;
    if (!aligned16(x)) return MOE_EALIGN;
    cudaStream_t st = (cudaStream_t)stream;
    const size_t n = (size_t)T * h->dm.k;
    cudaError_t e = route(h, (const uint16_t *)x, T, 1, st);
    if (e == cudaSuccess) e = cudaMemcpyAsync(idx_out, h->ws.topk_idx, 4 * n, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess) e = cudaMemcpyAsync(w_out, h->ws.topk_w, 4 * n, cudaMemcpyDeviceToDevice, st);
    return e == cudaSuccess ? MOE_OK : MOE_ECUDA;
}

extern "C" int moe_debug_active(moe_handle h, const void *x, int T, float tau, uint16_t *idx_out,
                                int *cnt_out, void *out, void *stream)
{
    int rc = check_handle(h);
    if (rc) return rc;
    if (!idx_out || !cnt_out) return MOE_EINVAL;
    if (T < 1 || T > h->dm.max_tokens) return MOE_EINVAL;
    rc = run_forward(h, x, T, tau, true, out ? out : (void *)h->ws.out_stage, stream, MOE_PATH_SPARSE);
    if (rc) return rc;
    cudaError_t e = moe::launch_mask_compact(h->ws, T * h->dm.k, h->dm.f, idx_out, cnt_out,
                                             (cudaStream_t)stream);
    return e == cudaSuccess ? MOE_OK : MOE_ECUDA;
}

// The floor(q N)-th smallest score of a population: the routed pairs' (N = T k
// d_ff) or the shared experts' neurons (N = T S d_ff).
static int calibrate(moe_handle h, const void *x, int T, double sparsity, float *tau_out, void *stream, bool shared)
{
    int rc = check_handle(h);
    if (rc) return rc;
    if (!x || !tau_out || T < 1 || T > h->dm.max_tokens || std::isnan(sparsity)) return MOE_EINVAL;
    if (shared && h->dm.S == 0) return MOE_EINVAL;
    if (!aligned16(x)) return MOE_EALIGN;
    const moe::Dims &dm = h->dm;
    const size_t n = (size_t)T * (shared ? dm.S : dm.k) * dm.f;
    if (sparsity <= 0.0) { *tau_out = 0.0f; return MOE_OK; }
    const double kq = std::floor(sparsity * (double)n);
    if (kq >= (double)n) { *tau_out = INFINITY; return MOE_OK; }
    if (!h->scores) {
        const size_t cap = (size_t)dm.max_tokens * (dm.k > dm.S ? dm.k : dm.S) * dm.f * sizeof(float);
        if (inject_alloc_fail("scores") || cudaMalloc(&h->scores, cap) != cudaSuccess) {
            cudaGetLastError();
            h->scores = nullptr;
            return MOE_ENOMEM;
        }
    }
    cudaStream_t st = (cudaStream_t)stream;
    const uint16_t *xb = (const uint16_t *)x;
    const moe::SparseTiling til = moe::sparse_tiling(T, dm.d, dm.S);
    cudaError_t e = route(h, xb, T, til.nt, st);
    if (e == cudaSuccess)
        e = moe::launch_expert_sparse(dm, h->w, h->ws, xb, T, 0.0f, false, h->ws.out_stage, til, h->n_sm, st,
                                      h->scores, 0, false, 0.0f, shared);
    // exact selection of the kq-th smallest, 8 bits per pass, most significant first
    unsigned long long want = (unsigned long long)kq;
    uint32_t prefix = 0, pmask = 0;
    for (int shift = 24; shift >= 0 && e == cudaSuccess; shift -= 8) {
        unsigned hist[256];
        e = moe::launch_radix_hist((const uint32_t *)h->scores, n, prefix, pmask, shift, h->hist, h->n_sm, st);
        if (e == cudaSuccess) e = cudaMemcpyAsync(hist, h->hist, sizeof hist, cudaMemcpyDeviceToHost, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) break;
        unsigned long long below = 0;
        int b = 0;
        for (; b < 256; ++b) {
            if (below + hist[b] > want) break;
            below += hist[b];
        }
        if (b == 256) return MOE_ECUDA;   // counts do not add up: cannot happen for a consistent buffer
        want -= below;
        prefix |= (uint32_t)b << shift;
        pmask |= 255u << shift;
    }
    if (e != cudaSuccess) return MOE_ECUDA;
    float tau;
    std::memcpy(&tau, &prefix, sizeof tau);
    *tau_out = tau;
    return MOE_OK;
}

extern "C" int moe_calibrate_tau(moe_handle h, const void *x, int T, double sparsity, float *tau_out,
                                 void *stream)
{
    return calibrate(h, x, T, sparsity, tau_out, stream, false);
}

extern "C" int moe_calibrate_tau_shared(moe_handle h, const void *x, int T, double sparsity, float *tau_out,
                                        void *stream)
{
    return calibrate(h, x, T, sparsity, tau_out, stream, true);
}

extern "C" int moe_set_shared_tau(moe_handle h, float tau_shared)
{
    if (!is_live(h)) return MOE_EHANDLE;
    if (std::isnan(tau_shared)) return MOE_EINVAL;
    h->tau_shared = tau_shared;
    return MOE_OK;
}

extern "C" int moe_set_rank_budget(moe_handle h, int r)
{
    if (!is_live(h)) return MOE_EHANDLE;
    if (r >= 0 && !h->rank_a) {
        const size_t pairs = (size_t)h->dm.max_tokens * h->dm.k;
        const size_t bytes = pairs * h->dm.f * sizeof(float) + 2 * ((pairs * 4 + 255) & ~size_t(255));
        void *mem = nullptr;
        if (inject_alloc_fail("rank") || cudaMalloc(&mem, bytes) != cudaSuccess) {
            cudaGetLastError();
            return MOE_ENOMEM;
        }
        h->rank_a = (float *)mem;
        uint8_t *tail = (uint8_t *)mem + pairs * h->dm.f * sizeof(float);
        h->rank_v = (float *)tail;
        h->rank_j = (int *)(tail + ((pairs * 4 + 255) & ~size_t(255)));
    }
    h->rank_r = r < 0 ? -1 : r;
    return MOE_OK;
}

extern "C" int moe_set_capacity(moe_handle h, float gamma)
{
    if (!is_live(h)) return MOE_EHANDLE;
    if (std::isnan(gamma)) return MOE_EINVAL;
    h->cap_gamma = gamma > 0.f ? gamma : 0.f;
    return MOE_OK;
}

extern "C" int moe_set_deterministic(moe_handle h, int enable)
{
    if (!is_live(h)) return MOE_EHANDLE;
    if (enable) {
        const size_t bytes =
            (size_t)h->dm.max_tokens * (h->dm.k + h->dm.S) * h->dm.n_blk * h->dm.d * sizeof(float);
        if (!h->det_rows) {
            void *mem = nullptr;
            if (inject_alloc_fail("deterministic") || cudaMalloc(&mem, bytes) != cudaSuccess) {
                cudaGetLastError();
                return MOE_ENOMEM;
            }
            h->det_rows = (float *)mem;
        }
        // all-zero before the first forward that uses the rows (and again after
        // any earlier forward that a device error cut short)
        if (cudaMemset(h->det_rows, 0, bytes) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess)
            return MOE_ECUDA;
    }
    h->det = enable ? 1 : 0;
    h->ws.ypart = h->det ? h->det_rows : nullptr;
    return MOE_OK;
}

extern "C" int moe_set_launch_events(moe_handle h, void *const *events, int n)
{
    if (!is_live(h)) return MOE_EHANDLE;
    if (!events || n == 0) { h->n_ev = 0; return MOE_OK; }
    if (n != 3 || !events[0] || !events[1] || !events[2]) return MOE_EINVAL;
    for (int i = 0; i < 3; ++i) h->ev[i] = (cudaEvent_t)events[i];
    h->n_ev = 3;
    return MOE_OK;
}

extern "C" int moe_set_trace(moe_handle h, void *buf, long long bytes)
{
    if (!is_live(h)) return MOE_EHANDLE;
    if (!buf || bytes <= 0) {
        h->ws.trace_router = h->ws.trace_expert = nullptr;
        h->ws.trace_router_ctas = h->ws.trace_expert_ctas = 0;
        return MOE_OK;
    }
    if (((uintptr_t)buf & 7u) != 0) return MOE_EALIGN;
    const long long words = bytes / 8;
    const long long router = words / 2;   // first half: router CTAs x 8 stamps
    h->ws.trace_router = (unsigned long long *)buf;
    h->ws.trace_router_ctas = (int)(router / 8);
    h->ws.trace_expert = (unsigned long long *)buf + router;
    h->ws.trace_expert_ctas = (int)((words - router) / 64);
    return MOE_OK;
}

extern "C" int moe_query_stats(moe_handle h, moe_stats *st)
{
    int rc = check_handle(h);
    if (rc) return rc;
    if (!st) return MOE_EINVAL;
    std::memset(st, 0, sizeof *st);
    const moe::Dims &dm = h->dm;
    st->path = h->last_path;
    st->n_tokens = h->last_T;
    st->t_star = h->t_star;
    st->fused_router = h->last_fused;
    st->capacity = h->last_cap;
    st->deterministic = h->last_det;
    if (cudaStreamSynchronize(h->last_stream) != cudaSuccess) return MOE_ECUDA;
    // the first error code since the previous call: an earlier forward's (kept
    // in the sticky word by the router of the next forward), else the last
    // forward's own; both are cleared
    int words[2] = {0, 0};
    if (cudaMemcpy(&words[0], h->ws.error_sticky, 4, cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(&words[1], h->ws.error_word, 4, cudaMemcpyDeviceToHost) != cudaSuccess)
        return MOE_ECUDA;
    const int err = words[0] != 0 ? words[0] : words[1];
    if (err != 0 && (cudaMemset(h->ws.error_sticky, 0, 4) != cudaSuccess ||
                     cudaMemset(h->ws.error_word, 0, 4) != cudaSuccess))
        return MOE_ECUDA;
    st->device_error = err;
    if (h->last_T > 0) {
        unsigned long long v[3] = {0, 0, 0};
        if (moe::launch_stats(dm, h->ws, h->last_T, h->stats_dev, h->last_stream) != cudaSuccess ||
            cudaMemcpyAsync(v, h->stats_dev, sizeof v, cudaMemcpyDeviceToHost, h->last_stream) != cudaSuccess ||
            cudaStreamSynchronize(h->last_stream) != cudaSuccess)
            return MOE_ECUDA;
        const double d = dm.d, f = dm.f;
        const bool masked = h->last_masked && h->last_path == MOE_PATH_SPARSE;
        st->n_touched = (int)v[2];
        st->n_active = masked ? (long long)v[0] : (long long)h->last_T * dm.k * dm.f;
        st->n_union = masked ? (long long)v[1] : (long long)v[2] * dm.f;
        const double fixed = dm.S * 3.0 * d * f * 2 + (double)dm.E * d * 2 + 2.0 * h->last_T * d * 2;
        st->alg_bytes = st->n_touched * d * f * 2 + 2.0 * d * 2 * (double)st->n_union + fixed;
        st->dense_bytes = st->n_touched * 3.0 * d * f * 2 + fixed;
    }
    return err ? MOE_EDEVICE : MOE_OK;
}

extern "C" int moe_set_fused_router(moe_handle h, int mode)
{
    if (!is_live(h)) return MOE_EHANDLE;
    if (mode < 0 || mode > 2) return MOE_EINVAL;
    h->fused_router = mode;
    return MOE_OK;
}

extern "C" int moe_debug_inject(moe_handle h, int kind)
{
    if (!is_live(h)) return MOE_EHANDLE;
    if (kind != MOE_INJECT_NONE && kind != MOE_INJECT_WITHHOLD_ITEMS) return MOE_EINVAL;
    h->inject_next = kind;
    return MOE_OK;
}

extern "C" const char *moe_strerror(int code)
{
    switch (code) {
    case MOE_OK: return "success";
    case MOE_EINVAL: return "invalid argument";
    case MOE_ENOMEM: return "out of memory";
    case MOE_ECUDA: return "CUDA runtime error";
    case MOE_EALIGN: return "pointer not 16-byte aligned";
    case MOE_EHANDLE: return "invalid or destroyed handle";
    case MOE_EDEVICE: return "a kernel reported a device-side error";
    case MOE_ENOTSUP: return "not supported by this build";
    default: return "unknown error code";
    }
}
