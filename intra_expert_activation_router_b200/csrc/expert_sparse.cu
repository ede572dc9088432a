// expert_sparse.cu -- fused gate projection, threshold mask, compaction and
// gathered up/down projection for the routed experts (and the dense shared
// experts): a persistent, warp-specialised kernel fed by bulk copies (TMA).
//
// "Uncovering Intra-expert Activation Sparsity for Efficient Mixture-of-Expert
// Model Execution" (technical summary, Methodology item 3):
//   - gate projection, dense ("Gate projection" bullet): g = x Wg[e] for every
//     neuron of the selected expert;
//   - activation mask in one O(n) pass, no sort ("Activation masking"):
//     active iff |silu(g)| >= tau -- a warp ballot over 32 neurons;
//   - fused up-down projection over the active neurons only ("Fused up-down
//     projection"): the active rows of Wu and Wd are gathered and packed
//     densely in shared memory, h = silu(g) * (x Wu[:,j]) and y += w h Wd[j][:]
//     (Hindi summary, "The skip": inactive neurons' weights are never loaded).
//   - shared experts: the same code with the mask off and weight 1 (their
//     execution is unchanged and always dense).
//
// Work items are (expert, token tile of up to MT of that expert's tokens,
// chunk of 32 neurons), ordered expert, tile, chunk.  Each CTA (one per SM)
// takes a contiguous range of items.  Warp 8 is the producer: one thread
// issues, as cp.async.bulk copies completed on mbarriers,
//   x(i)   the tile's token rows                          -> xbuf[i % 3]
//   G(i)   the chunk's 32 gate rows, stages of <= 16 KB  -> ring
//   U(i)   once the mask of item i is known, the union-active rows of Wu and
//          Wd, packed in batches of GB neurons           -> gather buffer
// from a polling loop: U(i) as soon as the mask of item i is known, x(i) at
// most one item ahead of the gate cursor once item i-3 has released its
// buffer, and G(i) stages whenever ring slots are free (only after x(i), so a
// ring smaller than a chunk cannot deadlock against the consumers).
// Warps 0-7 consume in the order G(0) M(0) | G(1) M(1) UD(0) | ..., so the
// gather of item i is in flight while the gate rows of item i+1 are reduced.
//   G   each warp owns a slice of d; per stage it dots the stage's rows with
//       the tile's tokens (fp32) and keeps one partial per (row, token) after
//       a transposed warp reduction;
//   M   the 8 slice partials are summed, silu and the threshold evaluated, a
//       32-bit mask word balloted per token (written out as the pair's mask),
//       and the union of the tile's words compacted into an ascending list;
//   UD  up rows: the same slice dots give u, then h = bit ? silu(g) u : 0;
//       down rows: each thread owns 8 output dims per pass and accumulates
//       sum_j h_j Wd[j][:] in registers across consecutive items of the same
//       (expert, tile); when that changes the partial goes to the fp32
//       accumulator y_acc[token] with vector atomics and a per-token ticket
//       counts the chunks; the token's last chunk converts y_acc to bf16 into
//       `out` and re-zeroes its row and ticket.
#include "common.cuh"
#include "internal.h"
#include "tma.cuh"

namespace moe {

constexpr int kConsumerThreads = 256;
constexpr int kSparseThreads = kConsumerThreads + 32;
constexpr int kSparseSmemBudget = 220 * 1024;

struct SparseLayout {   // byte offsets into dynamic shared memory
    int ring_off, stage_bytes, rows_per_stage, n_stages, stages_per_chunk;
    int gather_off, gather_rows;
    int xbuf_off, xbuf_bytes;
    int meta_off, meta_bytes;
    int part_off, h_off, last_off, plan_off, bar_off;
    int total;
};

struct SparseArgs {
    const uint16_t *x;
    uint16_t *out;
    DeviceWeights w;
    Workspace ws;
    int T, d, f, k, S;
    float tau;
    int use_mask;
    int n_chunks;
    int n_tok_tiles;      // ceil(T / MT), for the shared experts
    int n_shared_items;   // S * n_tok_tiles * n_chunks
    int target;           // chunk contributions per token: (k + S) * n_chunks
    int max_touched;      // plan cache capacity
    float *score_out;     // score mode: write |silu(g)| [pair][f], no up/down
    SparseLayout L;
};

template <int MT>
struct ItemMeta {
    const uint16_t *wg, *wu, *wd;
    long long key;           // (expert or shared index, token tile): items that may share y
    int tok[MT];
    int pair[MT];
    float w[MT];
    unsigned word[MT];
    float a[kChunk][MT];     // silu(g) of the chunk's neurons
    int uni[kChunk];         // union-active neuron offsets, ascending
    int m, chunk, masked, n_uni;
};

// Partial dot products over this warp's slice of d for up to 4 rows:
// acc[q][r] = sum_{i in slice} row_q[i] * x_r[i]; the transposed reduction
// leaves the warp-wide sum for (q, r) in one lane, which stores it.
template <int MT, int NP>
__device__ __forceinline__ void slice_dot4(const uint8_t *rows, int row_bytes, int nrows, const uint16_t *xb,
                                           int d, int m, float *part_w, int row_off, int lane, int warp)
{
    constexpr int NV = 4 * MT;
    constexpr int SH = 5 - Log2<NV>::value;
    const int d8 = d >> 3;
    float acc[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) acc[i] = 0.f;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        const int v = warp * 32 + lane + 256 * p;
        if (v < d8) {
            float xf[MT][8];
#pragma unroll
            for (int r = 0; r < MT; ++r)
                if (r < m) unpack8(*reinterpret_cast<const uint4 *>(xb + (size_t)r * d + v * 8), xf[r]);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (q < nrows) {
                    float wf[8];
                    unpack8(*reinterpret_cast<const uint4 *>(rows + (size_t)q * row_bytes + v * 16), wf);
#pragma unroll
                    for (int r = 0; r < MT; ++r) {
                        if (r < m) {
                            float s = acc[q * MT + r];
#pragma unroll
                            for (int e = 0; e < 8; ++e) s = fmaf(wf[e], xf[r][e], s);
                            acc[q * MT + r] = s;
                        }
                    }
                }
            }
        }
    }
    const float val = transpose_reduce<NV>(acc, lane);
    const int vi = lane >> SH, q = vi / MT, r = vi % MT;
    if ((lane & ((1 << SH) - 1)) == 0 && q < nrows) part_w[(row_off + q) * MT + r] = val;
}

template <int MT, int NP>
__global__ void __launch_bounds__(kSparseThreads, 1) k_expert_sparse(SparseArgs a)
{
    extern __shared__ __align__(128) uint8_t smem[];
    const SparseLayout &L = a.L;
    uint8_t *ring = smem + L.ring_off;
    uint8_t *gather = smem + L.gather_off;
    ItemMeta<MT> *meta = reinterpret_cast<ItemMeta<MT> *>(smem + L.meta_off);
    float *part = reinterpret_cast<float *>(smem + L.part_off);   // [8][32][MT]
    float *hs = reinterpret_cast<float *>(smem + L.h_off);        // [GB][MT]
    int *s_last = reinterpret_cast<int *>(smem + L.last_off);     // [MT]
    int *s_prefix = reinterpret_cast<int *>(smem + L.plan_off);
    int *s_expert = s_prefix + a.max_touched + 1;
    int *s_off = s_expert + a.max_touched;
    int *s_cnt = s_off + a.max_touched;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    const int NS = L.n_stages;
    uint64_t *full_g = bars, *empty_g = bars + NS;
    uint64_t *xfull = bars + 2 * NS, *xempty = xfull + 3;
    uint64_t *full_u = xempty + 3, *empty_u = full_u + 1;
    // items whose mask and union list are final (written by consumer thread 0,
    // polled by the producer); a counter, so it cannot be read two items stale
    volatile int *mask_done = reinterpret_cast<volatile int *>(s_last + 8);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const Plan *plan = a.ws.plan;
    int *err = a.ws.error_word;
    const int d = a.d, row_bytes = 2 * d;
    const bool score_mode = a.score_out != nullptr;

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full_g[s], 1);
            mbar_init(&empty_g[s], 8);
        }
        for (int p = 0; p < 3; ++p) {
            mbar_init(&xfull[p], 1);
            mbar_init(&xempty[p], 1);
        }
        *mask_done = 0;
        mbar_init(full_u, 1);
        mbar_init(empty_u, 1);
        fence_mbar_init();
    }
    // everything above overlaps the router's tail (programmatic dependent
    // launch); the routing plan is read only after the router grid is done
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // plan cache
    const int n_touched = plan->n_touched;
    for (int i = tid; i <= n_touched; i += blockDim.x) {
        s_prefix[i] = plan->item_prefix[i];
        if (i < n_touched) {
            const int e = plan->touched[i];
            s_expert[i] = e;
            s_off[i] = plan->offsets[e];
            s_cnt[i] = plan->offsets[e + 1] - plan->offsets[e];
        }
    }
    __syncthreads();

    const int n_items = a.n_shared_items + plan->n_routed_items;
    const int G = gridDim.x, b = blockIdx.x;
    const int per = n_items / G, rem = n_items % G;
    const int first = b * per + min(b, rem);
    const int n_my = per + (b < rem ? 1 : 0);
    const size_t fd = (size_t)a.f * d;

    if (warp == 8) {
        // ------------------------------------------------------------ producer
        // A polling loop over three queues, so no queue can block another:
        //   gather U(ui)  as soon as the mask of item ui is known (critical path)
        //   x(xi)         the tile rows, at most one item ahead of the gate cursor,
        //                 once item xi-3 has released its buffer
        //   G(gi) stage   whenever a ring slot is free, only for items whose x is issued
        // Every index read back from shared memory is clamped, so even after a
        // timed-out wait no copy can leave its buffers.
        if (lane == 0 && n_my > 0) {
            const uint64_t pol = policy_evict_first();
            uint32_t g = 0, ub = 0, idle = 0;
            int xi = 0, gi = 0, gs = 0, ui = 0, ub0 = 0, u_n = -1;
            while (score_mode ? gi < n_my : ui < n_my) {
                bool prog = false;
                // gather of item ui (needs its gate issued and its mask computed)
                if (!score_mode && ui < gi) {
                    ItemMeta<MT> &M = meta[ui % 3];
                    if (u_n < 0 && *mask_done > ui) {
                        __threadfence_block();
                        u_n = min(max(M.n_uni, 0), kChunk);
                        ub0 = 0;
                        prog = true;
                    }
                    if (u_n >= 0) {
                        if (ub0 >= u_n) {
                            ++ui;
                            u_n = -1;
                            prog = true;
                        } else if (mbar_test(empty_u, (ub & 1) ^ 1)) {
                            const int nb = min(L.gather_rows, u_n - ub0);
                            const size_t j0 = (size_t)min(max(M.chunk, 0), a.n_chunks - 1) * kChunk;
                            mbar_arrive_expect_tx(full_u, (uint32_t)(nb * 2 * row_bytes));
                            for (int q = 0; q < nb; ++q) {
                                const size_t j = j0 + (M.uni[ub0 + q] & (kChunk - 1));
                                bulk_g2s_hint(gather + (size_t)(2 * q) * row_bytes, M.wu + j * d,
                                              (uint32_t)row_bytes, full_u, pol);
                                bulk_g2s_hint(gather + (size_t)(2 * q + 1) * row_bytes, M.wd + j * d,
                                              (uint32_t)row_bytes, full_u, pol);
                            }
                            ub0 += nb;
                            ++ub;
                            prog = true;
                        }
                    }
                }
                // x rows and metadata of item xi
                if (xi < n_my && xi <= gi + 1 && mbar_test(&xempty[xi % 3], ((xi / 3) & 1) ^ 1)) {
                    ItemMeta<MT> &M = meta[xi % 3];
                    const int item = first + xi;
                    int m, chunk, tok0 = -1, off = 0;
                    if (item < a.n_shared_items) {
                        const int per_s = a.n_tok_tiles * a.n_chunks;
                        const int s = item / per_s, r0 = item % per_s;
                        const int tile = r0 / a.n_chunks;
                        chunk = r0 % a.n_chunks;
                        tok0 = tile * MT;
                        m = min(MT, a.T - tok0);
                        M.wg = a.w.wsg_n + s * fd;
                        M.wu = a.w.wsu_n + s * fd;
                        M.wd = a.w.wsd + s * fd;
                        M.masked = 0;
                        M.key = ((long long)(-1 - s) << 32) | (unsigned)tile;
                    } else {
                        const int ir = item - a.n_shared_items;
                        int lo = 0, hi = n_touched - 1;   // last slot with prefix <= ir
                        while (lo < hi) {
                            const int mid = (lo + hi + 1) >> 1;
                            if (s_prefix[mid] <= ir) lo = mid; else hi = mid - 1;
                        }
                        const int e = s_expert[lo], cnt = s_cnt[lo];
                        const int local = ir - s_prefix[lo];
                        const int tile = local / a.n_chunks;
                        chunk = local % a.n_chunks;
                        const int base = tile * MT;
                        m = min(MT, cnt - base);
                        M.wg = a.w.wg_n + e * fd;
                        M.wu = a.w.wu_n + e * fd;
                        M.wd = a.w.wd + e * fd;
                        M.masked = a.use_mask;
                        M.key = ((long long)(e + 1) << 32) | (unsigned)tile;
                        off = s_off[lo] + base;
                    }
                    m = min(max(m, 1), MT);
                    M.m = m;
                    M.chunk = chunk;
                    for (int r = 0; r < m; ++r) {
                        if (tok0 >= 0) {
                            M.tok[r] = tok0 + r;
                            M.pair[r] = -1;
                            M.w[r] = 1.f;
                        } else {
                            M.pair[r] = min(max(a.ws.perm[off + r], 0), a.T * a.k - 1);
                            M.tok[r] = min(max(a.ws.perm_tok[off + r], 0), a.T - 1);
                            M.w[r] = a.ws.perm_w[off + r];
                        }
                    }
                    uint16_t *xb = reinterpret_cast<uint16_t *>(smem + L.xbuf_off + (xi % 3) * L.xbuf_bytes);
                    mbar_arrive_expect_tx(&xfull[xi % 3], (uint32_t)(m * row_bytes));
                    if (tok0 >= 0) {
                        bulk_g2s(xb, a.x + (size_t)tok0 * d, (uint32_t)(m * row_bytes), &xfull[xi % 3]);
                    } else {
                        for (int r = 0; r < m; ++r)
                            bulk_g2s(xb + (size_t)r * d, a.x + (size_t)M.tok[r] * d, (uint32_t)row_bytes,
                                     &xfull[xi % 3]);
                    }
                    ++xi;
                    prog = true;
                }
                // one gate stage of item gi
                if (gi < n_my && gi < xi) {
                    const int slot = g % NS;
                    if (mbar_test(&empty_g[slot], ((g / NS) & 1) ^ 1)) {
                        const ItemMeta<MT> &M = meta[gi % 3];
                        const uint16_t *src = M.wg + ((size_t)M.chunk * kChunk + (size_t)gs * L.rows_per_stage) * d;
                        mbar_arrive_expect_tx(&full_g[slot], (uint32_t)L.stage_bytes);
                        bulk_g2s_hint(ring + (size_t)slot * L.stage_bytes, src, (uint32_t)L.stage_bytes,
                                      &full_g[slot], pol);
                        ++g;
                        if (++gs == L.stages_per_chunk) {
                            gs = 0;
                            ++gi;
                        }
                        prog = true;
                    }
                }
                if (prog) {
                    idle = 0;
                } else if (++idle > kSpinLimit) {
                    atomicCAS(err, 0, 12);
                    break;
                }
            }
            // drain: every copy issued has landed before the CTA may exit
            for (int s = 0; s < NS && (uint32_t)s < g; ++s) {
                const uint32_t uses = (g - s + NS - 1) / NS;
                mbar_wait(&full_g[s], (uses - 1) & 1, err, 15);
            }
            if (ub > 0) mbar_wait(full_u, (ub - 1) & 1, err, 16);
            for (int p = 0; p < 3 && p < xi; ++p) {
                const uint32_t uses = (xi - p + 2) / 3;
                mbar_wait(&xfull[p], (uses - 1) & 1, err, 17);
            }
        }
        __syncwarp();
    } else if (n_my > 0) {
        // ------------------------------------------------------------ consumers
        const int ct = tid;   // 0..255
        const int d8 = d >> 3;
        float acc_y[NP][8][MT];
#pragma unroll
        for (int p = 0; p < NP; ++p)
#pragma unroll
            for (int e = 0; e < 8; ++e)
#pragma unroll
                for (int r = 0; r < MT; ++r) acc_y[p][e][r] = 0.f;
        uint32_t g = 0, ub = 0;
        int n_acc = 0;
        for (int ii = 0; ii <= n_my; ++ii) {
            if (ii < n_my) {
                // G(ii): slice partials of the chunk's 32 gate rows
                const int par = ii % 3;
                ItemMeta<MT> &M = meta[par];
                mbar_wait(&xfull[par], (ii / 3) & 1, err, 21);
                const int m = M.m;
                const uint16_t *xb = reinterpret_cast<const uint16_t *>(smem + L.xbuf_off + par * L.xbuf_bytes);
                for (int s = 0; s < L.stages_per_chunk; ++s, ++g) {
                    const int slot = g % NS;
                    mbar_wait(&full_g[slot], (g / NS) & 1, err, 22);
                    const uint8_t *stg = ring + (size_t)slot * L.stage_bytes;
                    for (int q0 = 0; q0 < L.rows_per_stage; q0 += 4)
                        slice_dot4<MT, NP>(stg + (size_t)q0 * row_bytes, row_bytes, min(4, L.rows_per_stage - q0),
                                           xb, d, m, part + warp * kChunk * MT, s * L.rows_per_stage + q0, lane,
                                           warp);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty_g[slot]);
                }
                consumer_sync(kConsumerThreads);
                // M(ii): sum the slices, silu, threshold, ballot
                for (int r = warp; r < MT; r += 8) {
                    float gsum = 0.f;
#pragma unroll
                    for (int w8 = 0; w8 < 8; ++w8) gsum += part[(w8 * kChunk + lane) * MT + r];
                    const float av = silu_f(gsum);
                    const bool on = (r < m) && (!M.masked || fabsf(av) >= a.tau);
                    const unsigned word = __ballot_sync(kFull, on);
                    M.a[lane][r] = av;
                    if (lane == 0) {
                        M.word[r] = word;
                        if (M.masked && r < m) a.ws.mask[(size_t)M.pair[r] * a.n_chunks + M.chunk] = word;
                    }
                    if (score_mode && r < m && M.pair[r] >= 0)
                        a.score_out[(size_t)M.pair[r] * a.f + M.chunk * kChunk + lane] = fabsf(av);
                }
                consumer_sync(kConsumerThreads);
                if (ct == 0) {
                    unsigned uw = 0;
                    for (int r = 0; r < m; ++r) uw |= M.word[r];
                    int n = 0;
                    for (unsigned bits = uw; bits; bits &= bits - 1) M.uni[n++] = __ffs(bits) - 1;
                    M.n_uni = n;
                    __threadfence_block();
                    *mask_done = ii + 1;
                    if (score_mode) mbar_arrive(&xempty[par]);
                }
            }
            if (ii >= 1 && !score_mode) {
                // UD(ii-1): gathered up rows -> h, gathered down rows -> y
                const int jj = ii - 1, pj = jj % 3;
                ItemMeta<MT> &M = meta[pj];
                consumer_sync(kConsumerThreads);
                const int m = M.m, n_uni = min(max(M.n_uni, 0), kChunk);
                const uint16_t *xb = reinterpret_cast<const uint16_t *>(smem + L.xbuf_off + pj * L.xbuf_bytes);
                for (int b0 = 0; b0 < n_uni; b0 += L.gather_rows, ++ub) {
                    const int nb = min(L.gather_rows, n_uni - b0);
                    mbar_wait(full_u, ub & 1, err, 23);
                    for (int q0 = 0; q0 < nb; q0 += 4)
                        slice_dot4<MT, NP>(gather + (size_t)(2 * q0) * row_bytes, 2 * row_bytes, min(4, nb - q0),
                                           xb, d, m, part + warp * kChunk * MT, q0, lane, warp);
                    consumer_sync(kConsumerThreads);
                    for (int i = ct; i < nb * MT; i += kConsumerThreads) {
                        const int q = i / MT, r = i % MT;
                        float u = 0.f;
#pragma unroll
                        for (int w8 = 0; w8 < 8; ++w8) u += part[(w8 * kChunk + q) * MT + r];
                        const int jl = M.uni[b0 + q] & (kChunk - 1);
                        const bool bit = (r < m) && ((M.word[r] >> jl) & 1u);
                        hs[q * MT + r] = bit ? M.a[jl][r] * u : 0.f;
                    }
                    consumer_sync(kConsumerThreads);
#pragma unroll
                    for (int p = 0; p < NP; ++p) {
                        const int v = ct + 256 * p;
                        if (v < d8) {
                            for (int q = 0; q < nb; ++q) {
                                float wf[8];
                                unpack8(*reinterpret_cast<const uint4 *>(gather + (size_t)(2 * q + 1) * row_bytes +
                                                                         v * 16),
                                        wf);
#pragma unroll
                                for (int r = 0; r < MT; ++r) {
                                    const float hv = hs[q * MT + r];
#pragma unroll
                                    for (int e = 0; e < 8; ++e) acc_y[p][e][r] = fmaf(hv, wf[e], acc_y[p][e][r]);
                                }
                            }
                        }
                    }
                    consumer_sync(kConsumerThreads);
                    if (ct == 0) mbar_arrive(empty_u);
                }
                ++n_acc;
                const bool flush = (jj == n_my - 1) || (meta[(jj + 1) % 3].key != M.key);
                if (flush) {
#pragma unroll
                    for (int p = 0; p < NP; ++p) {
                        const int v = ct + 256 * p;
#pragma unroll
                        for (int r = 0; r < MT; ++r) {
                            if (v < d8 && r < m) {
                                const float wt = M.w[r];
                                float4 *dst = reinterpret_cast<float4 *>(a.ws.y_acc + (size_t)M.tok[r] * d + v * 8);
                                atomicAdd(dst, make_float4(wt * acc_y[p][0][r], wt * acc_y[p][1][r],
                                                           wt * acc_y[p][2][r], wt * acc_y[p][3][r]));
                                atomicAdd(dst + 1, make_float4(wt * acc_y[p][4][r], wt * acc_y[p][5][r],
                                                               wt * acc_y[p][6][r], wt * acc_y[p][7][r]));
                            }
#pragma unroll
                            for (int e = 0; e < 8; ++e) acc_y[p][e][r] = 0.f;
                        }
                    }
                    __threadfence();
                    consumer_sync(kConsumerThreads);
                    if (ct < m) {
                        const int old = atomicAdd(&a.ws.tok_cnt[M.tok[ct]], n_acc);
                        s_last[ct] = (old + n_acc == a.target);
                    }
                    consumer_sync(kConsumerThreads);
                    for (int r = 0; r < m; ++r) {
                        if (!s_last[r]) continue;
                        __threadfence();
                        const int t = M.tok[r];
                        float *yrow = a.ws.y_acc + (size_t)t * d;
                        uint16_t *orow = a.out + (size_t)t * d;
                        for (int i = ct * 4; i < d; i += kConsumerThreads * 4) {
                            const float4 v4 = __ldcg(reinterpret_cast<const float4 *>(yrow + i));
                            uint2 packed;
                            packed.x = (uint32_t)f2bf_bits(v4.x) | ((uint32_t)f2bf_bits(v4.y) << 16);
                            packed.y = (uint32_t)f2bf_bits(v4.z) | ((uint32_t)f2bf_bits(v4.w) << 16);
                            *reinterpret_cast<uint2 *>(orow + i) = packed;
                            __stcg(reinterpret_cast<float4 *>(yrow + i), make_float4(0.f, 0.f, 0.f, 0.f));
                        }
                        if (ct == 0) a.ws.tok_cnt[t] = 0;
                    }
                    n_acc = 0;
                }
                consumer_sync(kConsumerThreads);
                if (ct == 0) mbar_arrive(&xempty[pj]);
            }
        }
    }
    __syncthreads();
}

// tokens per work item for a batch of T tokens and a model width d
int sparse_tile_tokens(int T, int d)
{
    int mt = T <= 1 ? 1 : T <= 2 ? 2 : 4;
    const int np = (d / 8 + 255) / 256;
    while (mt > 1 && mt * np > 4) mt >>= 1;
    return mt;
}

static int meta_size(int mt)
{
    switch (mt) {
    case 1: return (int)sizeof(ItemMeta<1>);
    case 2: return (int)sizeof(ItemMeta<2>);
    default: return (int)sizeof(ItemMeta<4>);
    }
}

static bool make_layout(int d, int mt, int max_touched, SparseLayout &L)
{
    const int row_bytes = 2 * d;
    auto up = [](int v) { return (v + 127) & ~127; };
    int rs = 4;
    while (rs > 1 && rs * row_bytes > 16384) rs >>= 1;
    L.rows_per_stage = rs;
    L.stage_bytes = rs * row_bytes;
    L.stages_per_chunk = kChunk / rs;
    int gb = 65536 / (2 * row_bytes);
    if (gb > kChunk) gb = kChunk;
    if (gb < 1) gb = 1;
    L.gather_rows = gb;
    const int gather_bytes = up(gb * 2 * row_bytes);
    L.xbuf_bytes = up(mt * row_bytes);
    L.meta_bytes = up(3 * meta_size(mt));
    const int part_bytes = up(8 * kChunk * mt * 4);
    const int h_bytes = up(kChunk * mt * 4);
    const int last_bytes = 128;
    const int plan_bytes = up(4 * (4 * max_touched + 1));
    const int fixed = gather_bytes + 3 * L.xbuf_bytes + L.meta_bytes + part_bytes + h_bytes + last_bytes +
                      plan_bytes + 1024;
    int ns = (kSparseSmemBudget - fixed) / L.stage_bytes;
    if (ns > 16) ns = 16;
    if (ns < 2) return false;
    L.n_stages = ns;
    int off = 0;
    L.ring_off = off; off += up(ns * L.stage_bytes);
    L.gather_off = off; off += gather_bytes;
    L.xbuf_off = off; off += 3 * L.xbuf_bytes;
    L.meta_off = off; off += L.meta_bytes;
    L.part_off = off; off += part_bytes;
    L.h_off = off; off += h_bytes;
    L.last_off = off; off += last_bytes;
    L.plan_off = off; off += plan_bytes;
    L.bar_off = off; off += up((2 * ns + 8) * 8);
    L.total = off;
    return L.total <= 227 * 1024;
}

template <int MT, int NP>
static cudaError_t launch_mt(const SparseArgs &a, int grid, cudaStream_t st)
{
    auto kern = k_expert_sparse<MT, NP>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, a.L.total);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kSparseThreads);
    cfg.dynamicSmemBytes = a.L.total;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_expert_sparse(const Dims &dm, const DeviceWeights &w, const Workspace &ws,
                                 const uint16_t *x, int T, float tau, bool use_mask,
                                 uint16_t *out, int mt, int grid_cap, cudaStream_t st,
                                 float *score_out)
{
    SparseArgs a;
    a.x = x;
    a.out = out;
    a.w = w;
    a.ws = ws;
    a.T = T;
    a.d = dm.d;
    a.f = dm.f;
    a.k = dm.k;
    a.S = dm.S;
    a.tau = tau;
    a.use_mask = use_mask ? 1 : 0;
    a.score_out = score_out;
    a.n_chunks = dm.f / kChunk;
    a.n_tok_tiles = (T + mt - 1) / mt;
    a.n_shared_items = score_out ? 0 : dm.S * a.n_tok_tiles * a.n_chunks;
    a.target = (dm.k + dm.S) * a.n_chunks;
    const int pairs = T * dm.k;
    a.max_touched = pairs < dm.E ? pairs : dm.E;
    if (!make_layout(dm.d, mt, a.max_touched, a.L)) return cudaErrorInvalidValue;
    const int np = (dm.d / 8 + 255) / 256;
    const int bound = a.n_shared_items + (a.max_touched + pairs / mt) * a.n_chunks;
    int grid = bound < grid_cap ? bound : grid_cap;
    if (grid < 1) grid = 1;
    switch (np * 8 + mt) {
    case 8 + 1: return launch_mt<1, 1>(a, grid, st);
    case 8 + 2: return launch_mt<2, 1>(a, grid, st);
    case 8 + 4: return launch_mt<4, 1>(a, grid, st);
    case 16 + 1: return launch_mt<1, 2>(a, grid, st);
    case 16 + 2: return launch_mt<2, 2>(a, grid, st);
    case 24 + 1:
    case 32 + 1: return launch_mt<1, 4>(a, grid, st);
    default: return cudaErrorInvalidValue;
    }
}

int sparse_blocks_per_sm(int) { return 1; }

}  // namespace moe
