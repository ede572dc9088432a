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
// takes a contiguous range of items and runs three agents:
//   gate/x lane (warp 8)  item metadata and the tile's token rows (copied only
//                         when the (expert, tile) changes, into one of two
//                         slots), and the chunk's gate rows in 32 KB stages
//                         into a ring -- few, large bulk copies, since each
//                         copy costs the issuing thread a fixed time;
//   gather warp (warp 9)  once an item's mask is final, its union-active
//                         neurons' [up | down] records (4d bytes each), in
//                         batches, copies split over four lanes;
//   consumers (warps 0-7) in the order G(0) M(0) | G(1) M(1) UD(0) | ..., so
//                         the gather of item i lands while the gate rows of
//                         item i+1 are reduced:
//   G   each warp owns a slice of d, holds the tile's tokens for that slice in
//       registers and, per group of 8 gate rows, accumulates fp32 dot
//       products, then one transposed warp reduction leaves a partial per
//       (row, token);
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
// The agents meet on mbarriers (copies, buffer reuse) and on monotonic
// progress counters in shared memory; every wait is bounded.
#include "common.cuh"
#include "internal.h"
#include "tma.cuh"

namespace moe {

constexpr int kConsumerThreads = 256;
constexpr int kSparseThreads = kConsumerThreads + 64;   // + gate/x producer warp + gather warp
constexpr int kSparseSmemBudget = 220 * 1024;
constexpr int kPrefetchStages = 1;   // next-item gate stages allowed before the previous gather starts
constexpr int kGatherLanes = 4;      // lanes of the gather warp that issue copies

struct SparseLayout {   // byte offsets into dynamic shared memory
    int ring_off, stage_bytes, rows_per_stage, n_stages, stages_per_chunk;
    int gather_off, gather_rows, gpitch;   // neuron records [Wu row | Wd row] + 16-byte skew
    int xbuf_off, xbuf_bytes, xpitch;      // token rows + 16-byte skew
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
    const uint16_t *wud;     // the expert's [f][2d] up/down records
    long long key;           // (expert or shared index, token tile): items that share tokens
    int xslot, xseq, xfirst; // token rows: slot, load sequence number, first item using them
    int tok[MT];
    int pair[MT];
    float w[MT];
    unsigned word[MT];
    float a[kChunk][MT];     // silu(g) of the chunk's neurons
    int uni[kChunk];         // union-active neuron offsets, ascending
    int m, chunk, masked, n_uni;
};

// The tile's token rows, this lane's slice of d, widened to fp32 once per
// phase: xf[p][r][e] = x_r[8 v + e] with v = warp*32 + lane + 256 p.
template <int MT, int NP>
__device__ __forceinline__ void load_x(const uint8_t *xb, int xpitch, int m, int d8, int warp, int lane,
                                       float (&xf)[NP][MT][8])
{
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        const int v = warp * 32 + lane + 256 * p;
#pragma unroll
        for (int r = 0; r < MT; ++r) {
            if (r < m && v < d8) {
                unpack8(*reinterpret_cast<const uint4 *>(xb + (size_t)r * xpitch + 16 * v), xf[p][r]);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) xf[p][r][e] = 0.f;
            }
        }
    }
}

// Partial projections of a group of 8 weight rows over this warp's slice of
// d: acc[q][r] = sum_{k in slice} w_q[k] x_r[k].  Row q lives at
// lo + q * stride for q < split and at hi + (q - split) * stride after (a
// group may straddle two ring stages).  When swz, the row's 16-byte blocks
// are permuted b -> b ^ (q & 7) inside complete 128-byte groups (gate rows,
// see gate_pos), otherwise stored in order.  All eight 16-byte loads are
// issued before the math.  After one transposed warp reduction the warp-wide
// sum for (q, r) sits in one lane, which stores it to
// part_w[(row_off + q) * MT + r].
template <int MT, int NP>
__device__ __forceinline__ void group8(const uint8_t *lo, const uint8_t *hi, int split, int stride, bool swz,
                                       int nrows, const float (&xf)[NP][MT][8], int d8, int warp, int lane,
                                       float *part_w, int row_off)
{
    constexpr int NV = 8 * MT;
    constexpr int SH = 5 - Log2<NV>::value;
    const int full = (d8 >> 3) << 3;   // blocks in complete 128-byte groups
    float acc[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) acc[i] = 0.f;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        const int v = warp * 32 + lane + 256 * p;
        if (v < d8) {
            const bool sw = swz && v < full;
            uint4 wv[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint8_t *row = q < split ? lo + q * stride : hi + (q - split) * stride;
                const int pb = sw ? (v ^ q) : v;
                wv[q] = q < nrows ? *reinterpret_cast<const uint4 *>(row + 16 * pb) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                float wf[8];
                unpack8(wv[q], wf);
#pragma unroll
                for (int r = 0; r < MT; ++r) {
                    float s = acc[q * MT + r];
#pragma unroll
                    for (int e = 0; e < 8; ++e) s = fmaf(wf[e], xf[p][r][e], s);
                    acc[q * MT + r] = s;
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
    // progress counters shared between the three agents (monotonic, so a
    // reader can never mistake an old value for a new one):
    //   mask_done   items whose mask and union list are final   (consumers)
    //   pub_gi/xi   items whose gate stages / metadata are issued (gate lane)
    //   pub_gstart  items whose gather has started                (gather warp)
    volatile int *mask_done = reinterpret_cast<volatile int *>(s_last + 8);
    volatile int *pub_gi = mask_done + 1, *pub_xi = mask_done + 2, *pub_gstart = mask_done + 3;
    int *s_prefix = reinterpret_cast<int *>(smem + L.plan_off);
    int *s_expert = s_prefix + a.max_touched + 1;
    int *s_off = s_expert + a.max_touched;
    int *s_cnt = s_off + a.max_touched;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    const int NS = L.n_stages;
    uint64_t *full_g = bars, *empty_g = bars + NS;
    uint64_t *mfull = bars + 2 * NS, *mempty = mfull + 3;      // item metadata, 3 deep
    uint64_t *xfull = mempty + 3, *xempty = xfull + 2;         // token-row slots, by key
    uint64_t *full_u = xempty + 2, *empty_u = full_u + 1;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const Plan *plan = a.ws.plan;
    int *err = a.ws.error_word;
    const int d = a.d, row_bytes = 2 * d;
    const bool score_mode = a.score_out != nullptr;
    unsigned long long *tr = (a.ws.trace_expert && (int)blockIdx.x < a.ws.trace_expert_ctas)
                                 ? a.ws.trace_expert + blockIdx.x * 64 : nullptr;
    if (tr && tid == 0) tr[0] = global_ns();

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full_g[s], 1);
            mbar_init(&empty_g[s], 8);
        }
        for (int p = 0; p < 3; ++p) {
            mbar_init(&mfull[p], 1);
            mbar_init(&mempty[p], 1);
        }
        for (int p = 0; p < 2; ++p) {
            mbar_init(&xfull[p], 1);
            mbar_init(&xempty[p], 1);
        }
        mbar_init(full_u, 1);
        mbar_init(empty_u, 1);
        *mask_done = 0;
        *pub_gi = 0;
        *pub_xi = 0;
        *pub_gstart = 0;
        fence_mbar_init();
    }
    // everything above overlaps the router's tail (programmatic dependent
    // launch); the routing plan is read only after the router grid is done
    asm volatile("griddepcontrol.wait;" ::: "memory");

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
    if (tr && tid == 0) tr[1] = global_ns();

    const int n_items = a.n_shared_items + plan->n_routed_items;
    const int G = gridDim.x, b = blockIdx.x;
    const int per = n_items / G, rem = n_items % G;
    const int first = b * per + min(b, rem);
    const int n_my = per + (b < rem ? 1 : 0);
    const size_t fd = (size_t)a.f * d;

    // item -> (expert slot or shared index, tile, chunk); routed slot found by
    // binary search over the plan's per-slot item prefix
    auto locate = [&](int item, int &slot, int &tile, int &chunk) {
        if (item < a.n_shared_items) {
            const int per_s = a.n_tok_tiles * a.n_chunks;
            slot = -1 - item / per_s;
            const int r0 = item % per_s;
            tile = r0 / a.n_chunks;
            chunk = r0 % a.n_chunks;
        } else {
            const int ir = item - a.n_shared_items;
            int lo = 0, hi = n_touched - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (s_prefix[mid] <= ir) lo = mid; else hi = mid - 1;
            }
            const int local = ir - s_prefix[lo];
            slot = lo;
            tile = local / a.n_chunks;
            chunk = local % a.n_chunks;
        }
    };

    if (warp == 8) {
        // ------------------------------------------------------- gate/x producer
        // One lane polls two queues, so neither blocks the other:
        //   metadata + token rows of item xi (at most one item ahead of the gate
        //     cursor) once item xi-3 has released its metadata buffer; the token
        //     rows are copied only when the (expert, tile) changes, into the slot
        //     the tile before last has released
        //   gate stages of item gi into free ring slots; at most
        //     kPrefetchStages of an item before the previous item's gather has
        //     started, so that gather is not queued behind them
        if (lane == 0 && n_my > 0) {
            const uint64_t pol = policy_evict_first();
            uint32_t g = 0, idle = 0;
            int xi = 0, gi = 0, gs = 0, kseq = -1, cur_slot = 0;
            long long prev_key = 0;
            const uint16_t *g_src = nullptr;
            while (gi < n_my || xi < n_my) {
                bool prog = false;
                if (xi < n_my && xi <= gi + 1 && mbar_test(&mempty[xi % 3], ((xi / 3) & 1) ^ 1)) {
                    int slot, tile, chunk;
                    locate(first + xi, slot, tile, chunk);
                    const long long key = slot < 0 ? (((long long)slot << 32) | (unsigned)tile)
                                                   : (((long long)(s_expert[slot] + 1) << 32) | (unsigned)tile);
                    const bool newkey = score_mode || xi == 0 || key != prev_key;
                    const int nslot = (kseq + 1) & 1;
                    if (!newkey || mbar_test(&xempty[nslot], (((kseq + 1) >> 1) & 1) ^ 1)) {
                        ItemMeta<MT> &M = meta[xi % 3];
                        int m, tok0 = -1, off = 0;
                        if (slot < 0) {
                            const int s = -1 - slot;
                            tok0 = tile * MT;
                            m = min(MT, a.T - tok0);
                            M.wud = a.w.wsud + 2 * s * fd;
                            M.masked = 0;
                        } else {
                            m = min(MT, s_cnt[slot] - tile * MT);
                            M.wud = a.w.wud + 2 * s_expert[slot] * fd;
                            M.masked = a.use_mask;
                            off = s_off[slot] + tile * MT;
                        }
                        m = min(max(m, 1), MT);
                        M.key = key;
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
                        if (newkey) {
                            ++kseq;
                            cur_slot = kseq & 1;
                            uint8_t *xb = smem + L.xbuf_off + cur_slot * L.xbuf_bytes;
                            if (tr && xi < 4) tr[60 + xi] = global_ns();
                            mbar_arrive_expect_tx(&xfull[cur_slot], (uint32_t)(m * row_bytes));
                            for (int r = 0; r < m; ++r)
                                bulk_g2s(xb + (size_t)r * L.xpitch, a.x + (size_t)M.tok[r] * d, (uint32_t)row_bytes,
                                         &xfull[cur_slot]);
                        }
                        M.xslot = cur_slot;
                        M.xseq = kseq;
                        M.xfirst = newkey ? 1 : 0;
                        prev_key = key;
                        mbar_arrive(&mfull[xi % 3]);
                        ++xi;
                        *pub_xi = xi;
                        prog = true;
                    }
                }
                if (gi < n_my && (score_mode || *pub_gstart >= gi || gs < kPrefetchStages)) {
                    const int rslot = g % NS;
                    if (mbar_test(&empty_g[rslot], ((g / NS) & 1) ^ 1)) {
                        if (gs == 0) {
                            int slot, tile, chunk;
                            locate(first + gi, slot, tile, chunk);
                            const uint16_t *wg = slot < 0 ? a.w.wsg_n + (-1 - slot) * fd
                                                          : a.w.wg_n + s_expert[slot] * fd;
                            g_src = wg + (size_t)chunk * kChunk * d;
                        }
                        if (tr && gi < 4 && (gs == 0 || gs == L.stages_per_chunk - 1))
                            tr[52 + 2 * gi + (gs != 0)] = global_ns();
                        mbar_arrive_expect_tx(&full_g[rslot], (uint32_t)L.stage_bytes);
                        bulk_g2s_hint(ring + (size_t)rslot * L.stage_bytes,
                                      g_src + (size_t)gs * L.rows_per_stage * d, (uint32_t)L.stage_bytes,
                                      &full_g[rslot], pol);
                        ++g;
                        if (++gs == L.stages_per_chunk) {
                            gs = 0;
                            ++gi;
                            *pub_gi = gi;
                        }
                        prog = true;
                    }
                }
                if (prog) {
                    idle = 0;
                } else {
                    if (++idle > kSpinLimit) {
                        atomicCAS(err, 0, 12);
                        break;
                    }
                    __nanosleep(32);
                }
            }
            // drain: every copy issued has landed before the CTA may exit
            for (int s = 0; s < NS && (uint32_t)s < g; ++s) {
                const uint32_t uses = (g - s + NS - 1) / NS;
                mbar_wait(&full_g[s], (uses - 1) & 1, err, 15);
            }
            for (int p = 0; p < 2 && p <= kseq; ++p) {
                const uint32_t uses = (kseq - p + 2) / 2;
                mbar_wait(&xfull[p], (uses - 1) & 1, err, 17);
            }
        }
        __syncwarp();
    } else if (warp == 9) {
        // ------------------------------------------------------- gather producer
        // Lanes 0..3: once the mask of item ui is final, its union-active up/down
        // records are copied in batches of GB; lane 0 decides and waits for the
        // buffer, the four lanes split each batch's copies.
        if (lane < kGatherLanes && n_my > 0 && !score_mode) {
            const uint64_t pol = policy_evict_first();
            const unsigned lanes = (1u << kGatherLanes) - 1u;
            uint32_t ub = 0, idle = 0;
            int ui = 0;
            while (ui < n_my) {
                int go = 0;
                if (lane == 0) go = ui < *pub_gi && ui < *pub_xi && *mask_done > ui;
                go = __shfl_sync(lanes, go, 0);
                if (!go) {
                    if (++idle > kSpinLimit) {
                        if (lane == 0) atomicCAS(err, 0, 14);
                        break;
                    }
                    __nanosleep(64);
                    continue;
                }
                idle = 0;
                __threadfence_block();
                const ItemMeta<MT> &M = meta[ui % 3];
                const int n = min(max(M.n_uni, 0), kChunk);
                const size_t j0 = (size_t)min(max(M.chunk, 0), a.n_chunks - 1) * kChunk;
                if (n == 0 && lane == 0) *pub_gstart = ui + 1;
                for (int b0 = 0; b0 < n; b0 += L.gather_rows, ++ub) {
                    const int nb = min(L.gather_rows, n - b0);
                    if (lane == 0) {
                        mbar_wait(empty_u, (ub & 1) ^ 1, err, 14);
                        if (tr && b0 == 0 && ui < 4) tr[9 + 12 * ui] = global_ns();
                        mbar_arrive_expect_tx(full_u, (uint32_t)(nb * 2 * row_bytes));
                    }
                    __syncwarp(lanes);
                    for (int q = lane; q < nb; q += kGatherLanes) {
                        const size_t j = j0 + (M.uni[b0 + q] & (kChunk - 1));
                        bulk_g2s_hint(gather + (size_t)q * L.gpitch, M.wud + j * 2 * d, (uint32_t)(2 * row_bytes),
                                      full_u, pol);
                    }
                    __syncwarp(lanes);
                    if (b0 == 0 && lane == 0) *pub_gstart = ui + 1;
                }
                ++ui;
            }
            if (lane == 0 && ub > 0) mbar_wait(full_u, (ub - 1) & 1, err, 16);
        }
        if (tr && lane == 31 && n_my > 0) {
            // trace observer: arrival time of the first ring-full of gate stages
            const int n_obs = min(NS, min(8, n_my * L.stages_per_chunk));
            for (int gg = 0; gg < n_obs; ++gg) {
                mbar_wait(&full_g[gg], 0, err, 0x7f);
                tr[40 + gg] = global_ns();
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
        const int spg = 8 / L.rows_per_stage;   // stages per group of 8 rows
        for (int ii = 0; ii <= n_my; ++ii) {
            if (ii < n_my) {
                // G(ii): slice partials of the chunk's 32 gate rows, 8 at a time
                const int par = ii % 3;
                ItemMeta<MT> &M = meta[par];
                mbar_wait(&mfull[par], (ii / 3) & 1, err, 20);
                if (M.xfirst) mbar_wait(&xfull[M.xslot & 1], (M.xseq >> 1) & 1, err, 21);
                if (tr && ct == 0 && ii < 4) tr[2 + 12 * ii] = global_ns();
                const int m = M.m;
                float xf[NP][MT][8];
                load_x<MT, NP>(smem + L.xbuf_off + (M.xslot & 1) * L.xbuf_bytes, L.xpitch, m, d8, warp, lane, xf);
                const int rs = L.rows_per_stage;   // a power of two; groups of 8 rows span spg stages
                for (int grp = 0; grp < kChunk / 8; ++grp) {
                    const uint32_t g0 = g + grp * spg;
                    for (int j = 0; j < spg; ++j) {
                        const uint32_t gg = g0 + j;
                        mbar_wait(&full_g[gg % NS], (gg / NS) & 1, err, 22);
                    }
                    if (tr && ct == 0 && ii < 4) tr[3 + 12 * ii + grp] = global_ns();
                    // rows 8*grp .. 8*grp+7: within one stage when rs >= 8, else spg stages of rs rows
                    const int q0 = (8 * grp) & (rs - 1);
                    const uint8_t *lo = ring + (size_t)(g0 % NS) * L.stage_bytes + (size_t)q0 * row_bytes;
                    const uint8_t *hi = ring + (size_t)((g0 + 1) % NS) * L.stage_bytes;
                    group8<MT, NP>(lo, hi, rs >= 8 ? 8 : rs, row_bytes, true, 8, xf, d8, warp, lane,
                                   part + warp * kChunk * MT, 8 * grp);
                    __syncwarp();
                    if (lane == 0)
                        for (int j = 0; j < spg; ++j) mbar_arrive(&empty_g[(g0 + j) % NS]);
                }
                g += L.stages_per_chunk;
                consumer_sync(kConsumerThreads);
                if (tr && ct == 0 && ii < 4) tr[7 + 12 * ii] = global_ns();
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
                    if (tr && ii < 4) tr[8 + 12 * ii] = global_ns();
                    if (score_mode) {
                        mbar_arrive(&mempty[par]);
                        mbar_arrive(&xempty[M.xslot & 1]);
                    }
                }
            }
            if (ii >= 1 && !score_mode) {
                // UD(ii-1): gathered up rows -> h, gathered down rows -> y
                const int jj = ii - 1, pj = jj % 3;
                ItemMeta<MT> &M = meta[pj];
                consumer_sync(kConsumerThreads);
                const int m = M.m, n_uni = min(max(M.n_uni, 0), kChunk);
                float xf[NP][MT][8];
                load_x<MT, NP>(smem + L.xbuf_off + (M.xslot & 1) * L.xbuf_bytes, L.xpitch, m, d8, warp, lane, xf);
                for (int b0 = 0; b0 < n_uni; b0 += L.gather_rows, ++ub) {
                    const int nb = min(L.gather_rows, n_uni - b0);
                    mbar_wait(full_u, ub & 1, err, 23);
                    if (tr && ct == 0 && jj < 4 && b0 == 0) tr[10 + 12 * jj] = global_ns();
                    for (int grp = 0; grp * 8 < nb; ++grp) {
                        const uint8_t *lo = gather + (size_t)(8 * grp) * L.gpitch;
                        group8<MT, NP>(lo, lo, 8, L.gpitch, false, min(8, nb - 8 * grp), xf, d8, warp, lane,
                                       part + warp * kChunk * MT, 8 * grp);
                    }
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
                                unpack8(*reinterpret_cast<const uint4 *>(gather + (size_t)q * L.gpitch + row_bytes +
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
                    if (tr && ct == 0 && jj < 4) tr[12 + 12 * jj] = global_ns();
                }
                consumer_sync(kConsumerThreads);
                if (ct == 0) {
                    mbar_arrive(&mempty[pj]);
                    if (flush) mbar_arrive(&xempty[M.xslot & 1]);
                }
                if (tr && ct == 0 && jj < 4) tr[11 + 12 * jj] = global_ns();
            }
        }
    }
    __syncthreads();
    if (tr && tid == 0) {
        tr[50] = global_ns();
        tr[51] = (unsigned long long)n_my;
    }
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
    int rs = 8;   // rows per ring stage: 8 or 4 (d <= 4096), one copy of <= 32 KB
    while (rs > 4 && rs * row_bytes > 32 * 1024) rs >>= 1;
    L.rows_per_stage = rs;
    L.stage_bytes = rs * row_bytes;
    L.stages_per_chunk = kChunk / rs;
    L.gpitch = 2 * row_bytes + 16;
    int gb = 65536 / (2 * row_bytes);
    if (gb > kChunk) gb = kChunk;
    if (gb < 1) gb = 1;
    L.gather_rows = gb;
    const int gather_bytes = up(gb * L.gpitch);
    L.xpitch = row_bytes + 16;
    L.xbuf_bytes = up(mt * L.xpitch);
    L.meta_bytes = up(3 * meta_size(mt));
    const int part_bytes = up(8 * kChunk * mt * 4);
    const int h_bytes = up(kChunk * mt * 4);
    const int last_bytes = 128;
    const int plan_bytes = up(4 * (4 * max_touched + 1));
    const int fixed = gather_bytes + 2 * L.xbuf_bytes + L.meta_bytes + part_bytes + h_bytes + last_bytes +
                      plan_bytes + 1024;
    int ns = (kSparseSmemBudget - fixed) / L.stage_bytes;
    if (ns > 32) ns = 32;
    if (ns < (rs >= 8 ? 1 : 8 / rs) + kPrefetchStages) return false;   // a group of 8 rows plus the prefetch
    L.n_stages = ns;
    int off = 0;
    L.ring_off = off; off += up(ns * L.stage_bytes);
    L.gather_off = off; off += gather_bytes;
    L.xbuf_off = off; off += 2 * L.xbuf_bytes;
    L.meta_off = off; off += L.meta_bytes;
    L.part_off = off; off += part_bytes;
    L.h_off = off; off += h_bytes;
    L.last_off = off; off += last_bytes;
    L.plan_off = off; off += plan_bytes;
    L.bar_off = off; off += up((2 * ns + 12) * 8);
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
    default: return cudaErrorInvalidValue;
    }
}

int sparse_blocks_per_sm(int) { return 1; }

}  // namespace moe
