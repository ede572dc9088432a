// router.cu -- softmax top-k router and token-to-expert bucketing.
//
// "Uncovering Intra-expert Activation Sparsity for Efficient Mixture-of-Expert
// Model Execution" (technical summary, Methodology item 3): the router is kept
// unchanged -- logits = x Wr^T, p = softmax over all E experts, the top_k
// experts by p are selected and weighted by p.  Ties go to the lower index.
//
// One launch does three things:
//   1. logits: CTA (2 experts, 8 tokens), four warps per expert each taking a
//      quarter of d, fp32 accumulation of bf16 products; the tile's x rows are
//      staged in shared memory and the router rows loaded before the math, so
//      the phase costs about one memory round trip on E/2 CTAs per tile.
//   2. the last CTA of each token tile (atomic ticket; no waiting) runs the
//      softmax and the ordered top-k of its tokens, one warp per token: for
//      E <= 256 every logit's rank is counted directly, above that k rounds of
//      a warp arg-max select them.
//   3. the last token tile builds the routing plan for the expert kernels:
//      per-expert counts, offsets, a permutation of the pairs (t*k + rank)
//      ordered by expert (then by token up to kSmallPlan pairs; above that
//      the order inside an expert is arbitrary), the ascending list of
//      touched experts and the work-item prefix sums of both paths.
// Tickets reset themselves, so the launch can be replayed (graphs) without
// host-side clears.
#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kRtTok = 8;   // tokens per router CTA
constexpr int kRtExp = 2;   // experts per router CTA (four warps each)
constexpr int kStagePairs = 4096;   // plan built from shared memory up to this many pairs ...
constexpr int kSmallPlan = 256;     // ... when there are at most this many, or a capacity applies;
                                    // else from the token tiles' counts and k_plan_scatter (one CTA
                                    // placing pairs one warp-step at a time took 30 us at 2048 pairs)

__host__ __device__ __forceinline__ bool plan_staged(long long P, int cap)
{
    return P <= kStagePairs && (cap >= 0 || P <= kSmallPlan);
}
constexpr int kRankTopk = 256;      // up to this many experts, top-k by ranking all logits

struct RouterArgs {
    const uint16_t *x, *wr;
    int T, d, E, k;
    int mt, n_chunks;   // sparse work items per expert: ceil(tokens / mt) * n_chunks
    int dp;             // d rounded up to 128
    int xtile;          // T <= xtile <= 16: also write x into ws.x_tiles with xtile rows; else 0
    int epc;            // experts per CTA (even): gridDim.x = ceil(E / epc)
    int logits_ready;   // ws.logits already holds the batch's logits (a tensor-core GEMM): no phase 1
    int cap;            // capacity-aware token drop: pairs an expert keeps (-1: no capacity)
    int mask_words;     // 32-neuron mask words per pair (cleared for dropped pairs)
    Workspace ws;
};

__device__ __forceinline__ bool better(float v1, int i1, float v0, int i0)
{
    return v1 > v0 || (v1 == v0 && i1 < i0);
}

// Build the routing plan from topk_idx; executed by one whole CTA.
__device__ void build_plan(const RouterArgs &a, int *s_cnt, int *s_cur, int *s_idx, float *s_w, int *s_seg)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int E = a.E, P = a.T * a.k;
    const bool staged = s_idx != nullptr;   // top-k of all pairs held in shared memory
    Plan *plan = a.ws.plan;
    // large batches: the token tiles counted their pairs per expert (ecount);
    // staged ones count here, from exactly the indices the scatter places.
    // Either way ecount is left zero for the next call.
    for (int e = tid; e < E; e += blockDim.x) {
        s_cnt[e] = staged ? 0 : __ldcg(&a.ws.ecount[e]);
        a.ws.ecount[e] = 0;
    }
    if (staged) {
#pragma unroll 4
        for (int p = tid; p < P; p += blockDim.x) {
            s_idx[p] = min(max(__ldcg(&a.ws.topk_idx[p]), 0), E - 1);
            s_w[p] = __ldcg(&a.ws.topk_w[p]);
        }
        __syncthreads();
        for (int p = tid; p < P; p += blockDim.x) atomicAdd(&s_cnt[s_idx[p]], 1);
    }
    __syncthreads();
    if (staged && a.cap >= 0) {
        // Capacity-aware token drop ("Capacity-Aware Inference", "Capacity-
        // Aware Token Drop"): an expert routed more than cap pairs keeps the
        // cap with the largest routing weight, ties to the lower token.  The
        // pairs are first grouped by expert (s_seg; the order inside a group
        // is whatever the atomics give, since the ranking breaks ties by the
        // pair index, which orders an expert's pairs by token); a pair of an
        // over-capacity expert is dropped when at least cap pairs of its
        // group beat it.  A dropped pair then belongs to no expert's list
        // (sentinel E) and its mask words read as empty.
        if (warp == 0) {
            int run = 0;
            for (int e0 = 0; e0 < E; e0 += 32) {
                const int e = e0 + lane, c = e < E ? s_cnt[e] : 0;
                int inc = c;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int u = __shfl_up_sync(kFull, inc, o);
                    if (lane >= o) inc += u;
                }
                if (e < E) s_cur[e] = run + inc - c;
                run += __shfl_sync(kFull, inc, 31);
            }
        }
        __syncthreads();
        for (int p = tid; p < P; p += blockDim.x) s_seg[atomicAdd(&s_cur[s_idx[p]], 1)] = p;
        __syncthreads();   // s_cur[e] now ends expert e's group
        uint32_t drop = 0;   // bit i: the pair at group position tid + i * blockDim.x
        for (int i = tid, bit = 0; i < P; i += blockDim.x, ++bit) {
            const int p = s_seg[i], e = s_idx[p];
            if (s_cnt[e] <= a.cap) continue;
            const int g1 = s_cur[e], g0 = g1 - s_cnt[e];
            const float wp = s_w[p];
            int better = 0;
#pragma unroll 8
            for (int j = g0; j < g1; ++j) {
                const int q = s_seg[j];
                const float wq = s_w[q];
                better += (wq > wp || (wq == wp && q < p)) ? 1 : 0;
            }
            if (better >= a.cap) drop |= 1u << bit;
        }
        __syncthreads();
        for (int i = tid, bit = 0; i < P; i += blockDim.x, ++bit)
            if ((drop >> bit) & 1u) {
                const int p = s_seg[i];
                atomicSub(&s_cnt[s_idx[p]], 1);
                s_idx[p] = E;
                for (int c = 0; c < a.mask_words; ++c) a.ws.mask[(size_t)p * a.mask_words + c] = 0u;
            }
        __syncthreads();
    }
    if (warp == 0) {
        // exclusive scans over experts: positions, touched slots, work items, dense tiles
        const int per = (E + 31) / 32;
        const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
        int c_sum = 0, t_sum = 0, i_sum = 0, d_sum = 0;
        for (int e = e0; e < e1; ++e) {
            const int c = s_cnt[e];
            c_sum += c;
            if (c > 0) {
                t_sum += 1;
                i_sum += ((c + a.mt - 1) / a.mt) * a.n_chunks;
                d_sum += (c + kDenseTileM - 1) / kDenseTileM;
            }
        }
        int c_ex = c_sum, t_ex = t_sum, i_ex = i_sum, d_ex = d_sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int c = __shfl_up_sync(kFull, c_ex, o), t = __shfl_up_sync(kFull, t_ex, o);
            int i = __shfl_up_sync(kFull, i_ex, o), dd = __shfl_up_sync(kFull, d_ex, o);
            if (lane >= o) { c_ex += c; t_ex += t; i_ex += i; d_ex += dd; }
        }
        c_ex -= c_sum; t_ex -= t_sum; i_ex -= i_sum; d_ex -= d_sum;
        for (int e = e0; e < e1; ++e) {
            const int c = s_cnt[e];
            plan->offsets[e] = c_ex;
            s_cur[e] = c_ex;
            if (c > 0) {
                plan->touched[t_ex] = e;
                plan->item_prefix[t_ex] = i_ex;
                plan->tile_prefix[t_ex] = d_ex;
                t_ex += 1;
                i_ex += ((c + a.mt - 1) / a.mt) * a.n_chunks;
                d_ex += (c + kDenseTileM - 1) / kDenseTileM;
            }
            c_ex += c;
        }
        if (lane == 31) {
            plan->offsets[E] = c_ex;
            plan->n_touched = t_ex;
            plan->item_prefix[t_ex] = i_ex;
            plan->tile_prefix[t_ex] = d_ex;
            plan->n_routed_items = i_ex;
            plan->n_dense_tiles = d_ex;
            plan->next_item = 0;
        }
        __syncwarp();
        // large batches: the scatter is a kernel of its own (k_plan_scatter),
        // one pair per thread through per-expert cursors, zeroed here
        if (!staged)
            for (int e = lane; e < E; e += 32) a.ws.cursor[e] = 0;
    }
    if (!staged) return;
    __syncthreads();   // s_cur[e]: expert e's first position
    if (P > kSmallPlan) {
        // larger staged plans (the capacity drop's): one pair per thread
        // through the shared-memory cursors; the order inside an expert is
        // then arbitrary, which neither branch's result depends on
        for (int p = tid; p < P; p += blockDim.x) {
            const int e = s_idx[p];
            if (e < E) {   // a dropped pair (expert E) takes no position
                const int pos = atomicAdd(&s_cur[e], 1);
                a.ws.perm[pos] = p;
                a.ws.perm_tok[pos] = p / a.k;
                a.ws.perm_w[pos] = s_w[p];
            }
        }
        return;
    }
    if (warp == 0) {
        // stable scatter, 32 pairs at a time in pair order
        for (int base = 0; base < P; base += 32) {
            const int p = base + lane;
            // a dropped pair (expert E) takes no position
            const int ep = p < P ? (staged ? s_idx[p] : min(max(__ldcg(&a.ws.topk_idx[p]), 0), E - 1)) : E;
            const bool live = ep < E;
            const int e = live ? ep : -1 - lane;
            const unsigned same = __match_any_sync(kFull, e);
            const int rank = __popc(same & ((1u << lane) - 1));
            int pos = 0;
            if (live) pos = s_cur[e] + rank;
            __syncwarp();
            if (live && rank == 0) s_cur[e] += __popc(same);
            if (live) {
                a.ws.perm[pos] = p;
                a.ws.perm_tok[pos] = p / a.k;
                a.ws.perm_w[pos] = staged ? s_w[p] : __ldcg(&a.ws.topk_w[p]);
            }
            __syncwarp();
        }
    }
}

__global__ void __launch_bounds__(256) k_router(RouterArgs a)
{
    extern __shared__ float s_dyn[];   // kRtTok * E floats, reused as 2*E ints
    __shared__ int s_last;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int t0 = blockIdx.y * kRtTok;
    const int nt = min(kRtTok, a.T - t0);

    // let the expert kernel launch now; it waits for this grid to finish
    asm volatile("griddepcontrol.launch_dependents;");
    // every kernel of earlier calls has finished: keep their error code and
    // give this forward a clear error word (read only after this grid ends)
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
        const int e0 = *a.ws.error_word;
        if (e0 != 0) {
            atomicCAS(a.ws.error_sticky, 0, e0);
            *a.ws.error_word = 0;
        }
    }
    const int cta = blockIdx.y * gridDim.x + blockIdx.x;
    unsigned long long *tr = (a.ws.trace_router && cta < a.ws.trace_router_ctas) ? a.ws.trace_router + cta * 8 : nullptr;
    if (tr && threadIdx.x == 0) tr[0] = global_ns();

    // 1. logits of the CTA's `epc` experts for its token tile, the tile's x
    //    rows in shared memory: 2 experts for small batches (the router spread
    //    over E/2 CTAs per tile), more for large ones, whose tiles are many.
    const int quarter = warp & 3;
    uint4 *xs = reinterpret_cast<uint4 *>(s_dyn);                       // [kRtTok][256] 16-byte vectors
    float *qsum = s_dyn + kRtTok * 256 * 4;                              // [8 warps][kRtTok], after x
    const int e_first = blockIdx.x * a.epc;
    if (a.logits_ready) {
        // nothing to compute: the tile's logits are in place
    } else if (a.epc > kRtExp) {
        // large batches (d <= 2048): the tile's rows once, then one expert per
        // warp at a time over the whole of d (lane: 16-byte vectors lane,
        // lane + 32, ...), its router row loaded while the previous expert's
        // dots run; no cross-warp sums
        const int cv = a.d / 8;
        {
            uint4 xv[kRtTok];
#pragma unroll
            for (int j = 0; j < kRtTok; ++j) {
                const int i = threadIdx.x + j * 256;
                if (i < nt * cv) xv[j] = ld_cached(a.x + (size_t)(t0 + i / cv) * a.d + (i % cv) * 8);
            }
#pragma unroll
            for (int j = 0; j < kRtTok; ++j) {
                const int i = threadIdx.x + j * 256;
                if (i < nt * cv) xs[(i / cv) * 256 + i % cv] = xv[j];
            }
        }
        __syncthreads();
        if (a.xtile > 0 && blockIdx.x == 0) {   // the tile's rows of the swizzled token operand
            for (int i = threadIdx.x; i < kRtTok * cv; i += blockDim.x) {
                const int r = i / cv, v = i % cv, t = t0 + r;
                if (t < a.xtile)
                    *reinterpret_cast<uint4 *>(a.ws.x_tiles + ((size_t)(v >> 3) * a.xtile + t) * 64 +
                                               (((v & 7) ^ (t & 7)) << 3)) =
                        r < nt ? xs[r * 256 + v] : make_uint4(0, 0, 0, 0);
            }
        }
        const int e_end = min(e_first + a.epc, a.E);
        uint4 wn[8];
        auto load_row = [&](int e) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int v = lane + 32 * q;
                wn[q] = (e < e_end && v < cv) ? ld_cached(a.wr + (size_t)e * a.d + v * 8) : make_uint4(0, 0, 0, 0);
            }
        };
        load_row(e_first + warp);
#pragma unroll 1
        for (int e = e_first + warp; e < e_end; e += 8) {
            uint4 wv[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) wv[q] = wn[q];
            load_row(e + 8);
            float acc[kRtTok];
#pragma unroll
            for (int r = 0; r < kRtTok; ++r) acc[r] = 0.f;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int v = lane + 32 * q;
                if (v < cv) {
#pragma unroll
                    for (int r = 0; r < kRtTok; ++r)
                        if (r < nt) acc[r] = dot8(wv[q], xs[r * 256 + v], acc[r]);
                }
            }
#pragma unroll
            for (int r = 0; r < kRtTok; ++r) acc[r] = warp_sum(acc[r]);
            if (lane < nt) {
                float v = acc[0];
#pragma unroll
                for (int r = 1; r < kRtTok; ++r) v = lane == r ? acc[r] : v;
                a.ws.logits[(size_t)(t0 + lane) * a.E + e] = v;
            }
        }
    } else {
        // small batches: expert 2 blockIdx.x + w/4 per warp, a quarter of each
        // 2048-wide chunk of d per warp, the four quarter sums meeting in
        // shared memory
        const int e = e_first + (warp >> 2);
        float acc[kRtTok];
#pragma unroll
        for (int r = 0; r < kRtTok; ++r) acc[r] = 0.f;
        for (int c0 = 0; c0 < a.d; c0 += 2048) {
            const int cv = min(2048, a.d - c0) / 8;
            uint4 wv[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int v = quarter * 64 + lane + 32 * q;
                wv[q] = (e < a.E && v < cv) ? ld_cached(a.wr + (size_t)e * a.d + c0 + v * 8) : make_uint4(0, 0, 0, 0);
            }
            // the tile's rows of this chunk: every load issued before the first
            // store (nt * cv <= 8 * 256, at most one 16-byte vector per row and thread)
            uint4 xv[kRtTok];
#pragma unroll
            for (int j = 0; j < kRtTok; ++j) {
                const int i = threadIdx.x + j * 256;
                if (i < nt * cv) xv[j] = ld_cached(a.x + (size_t)(t0 + i / cv) * a.d + c0 + (i % cv) * 8);
            }
            __syncthreads();   // the previous chunk's x is no longer read
#pragma unroll
            for (int j = 0; j < kRtTok; ++j) {
                const int i = threadIdx.x + j * 256;
                if (i < nt * cv) xs[(i / cv) * 256 + i % cv] = xv[j];
            }
            __syncthreads();
            if (a.xtile > 0 && blockIdx.x == 0) {   // the tile's rows of the swizzled token operand
                for (int i = threadIdx.x; i < kRtTok * cv; i += blockDim.x) {
                    const int r = i / cv, v = i % cv, t = t0 + r;
                    if (t < a.xtile) {
                        const int cc = c0 / 8 + v;   // 16-byte block of the row
                        *reinterpret_cast<uint4 *>(a.ws.x_tiles + ((size_t)(cc >> 3) * a.xtile + t) * 64 +
                                                   (((cc & 7) ^ (t & 7)) << 3)) =
                            r < nt ? xs[r * 256 + v] : make_uint4(0, 0, 0, 0);
                    }
                }
            }
            if (e < a.E) {
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int v = quarter * 64 + lane + 32 * q;
                    if (v < cv) {
#pragma unroll
                        for (int r = 0; r < kRtTok; ++r)
                            if (r < nt) acc[r] = dot8(wv[q], xs[r * 256 + v], acc[r]);
                    }
                }
            }
        }
#pragma unroll
        for (int r = 0; r < kRtTok; ++r) acc[r] = warp_sum(acc[r]);
        if (lane == 0)
            for (int r = 0; r < kRtTok; ++r) qsum[warp * kRtTok + r] = acc[r];
        __syncthreads();
        if (threadIdx.x < kRtExp * kRtTok) {
            const int ee = threadIdx.x / kRtTok, r = threadIdx.x % kRtTok;
            const int eg = e_first + ee;
            if (eg < a.E && r < nt) {
                const float *q4 = qsum + (ee * 4) * kRtTok + r;
                a.ws.logits[(size_t)(t0 + r) * a.E + eg] = q4[0] + q4[kRtTok] + q4[2 * kRtTok] + q4[3 * kRtTok];
            }
        }
    }
    if (a.xtile > 0 && blockIdx.x == 0) {   // inputs past d: zero
        const int npad = (a.dp - a.d) / 8;
        for (int i = threadIdx.x; i < kRtTok * npad; i += blockDim.x) {
            const int r = i / npad, t = t0 + r, cc = a.d / 8 + i % npad;
            if (t < a.xtile)
                *reinterpret_cast<uint4 *>(a.ws.x_tiles + ((size_t)(cc >> 3) * a.xtile + t) * 64 +
                                           (((cc & 7) ^ (t & 7)) << 3)) = make_uint4(0, 0, 0, 0);
        }
    }

    // 2. last CTA of this token tile: softmax + top-k
    if (tr && threadIdx.x == 0) tr[1] = global_ns();
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const int tk = atomicAdd(&a.ws.tile_ticket[blockIdx.y], 1);
        s_last = (tk == (int)gridDim.x - 1);
        if (s_last) a.ws.tile_ticket[blockIdx.y] = 0;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (tr && threadIdx.x == 0) tr[2] = global_ns();
    if (warp < nt) {
        const int t = t0 + warp;
        float *row = s_dyn + warp * a.E;
        float m = -INFINITY;
        for (int j = lane; j < a.E; j += 32) {
            const float v = __ldcg(&a.ws.logits[(size_t)t * a.E + j]);
            row[j] = v;
            m = fmaxf(m, v);
        }
        m = warp_max(m);
        float s = 0.f;
        for (int j = lane; j < a.E; j += 32) s += expf(row[j] - m);
        s = warp_sum(s);
        __syncwarp();
        if (a.E <= kRankTopk) {
            // rank of each logit = number of logits ranked before it (larger, or
            // equal with a lower index); the ones with rank < k are the top-k,
            // written straight to their rank -- no serial selection rounds.
            // Valid defaults first: only non-finite logits could leave a rank
            // unwritten.
            for (int r = lane; r < a.k; r += 32) {
                a.ws.topk_idx[(size_t)t * a.k + r] = 0;
                a.ws.topk_w[(size_t)t * a.k + r] = 0.f;
            }
            __syncwarp();
            for (int j = lane; j < a.E; j += 32) {
                const float v = row[j];
                int rank = 0;
                for (int i = 0; i < a.E; ++i) rank += better(row[i], i, v, j) ? 1 : 0;
                if (rank < a.k) {
                    a.ws.topk_idx[(size_t)t * a.k + rank] = j;
                    a.ws.topk_w[(size_t)t * a.k + rank] = expf(v - m) / s;
                    atomicAdd(&a.ws.ecount[j], 1);
                }
            }
        } else {
            unsigned taken = 0;   // bit q: expert lane + 32q already selected
            for (int r = 0; r < a.k; ++r) {
                float bv = -INFINITY;
                int bi = 0x7fffffff;
                for (int q = 0, j = lane; j < a.E; ++q, j += 32) {
                    if (taken & (1u << q)) continue;
                    const float v = row[j];
                    if (bi == 0x7fffffff || better(v, j, bv, bi)) { bv = v; bi = j; }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const float ov = __shfl_xor_sync(kFull, bv, o);
                    const int oi = __shfl_xor_sync(kFull, bi, o);
                    if (oi != 0x7fffffff && (bi == 0x7fffffff || better(ov, oi, bv, bi))) { bv = ov; bi = oi; }
                }
                if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
                if (lane == 0) {
                    a.ws.topk_idx[(size_t)t * a.k + r] = bi;
                    a.ws.topk_w[(size_t)t * a.k + r] = expf(bv - m) / s;
                    atomicAdd(&a.ws.ecount[min(max(bi, 0), a.E - 1)], 1);
                }
            }
        }
    }

    // 3. last token tile: the routing plan (with a single tile, this CTA)
    if (tr && threadIdx.x == 0) tr[3] = global_ns();
    __syncthreads();
    if (gridDim.y > 1) {
        if (threadIdx.x == 0) {
            __threadfence();
            const int tk = atomicAdd(a.ws.done_ticket, 1);
            s_last = (tk == (int)gridDim.y - 1);
            if (s_last) *a.ws.done_ticket = 0;
        }
        __syncthreads();
        if (!s_last) return;
        __threadfence();
    }
    int *s_int = reinterpret_cast<int *>(s_dyn);
    const int P = a.T * a.k;
    const bool staged = plan_staged(P, a.cap);
    if (tr && threadIdx.x == 0) tr[4] = global_ns();
    build_plan(a, s_int, s_int + a.E, staged ? s_int + 2 * a.E : nullptr,
               staged ? reinterpret_cast<float *>(s_int + 2 * a.E + P) : nullptr,
               staged && a.cap >= 0 ? s_int + 2 * a.E + 2 * P : nullptr);
    __syncthreads();
    if (tr && threadIdx.x == 0) tr[5] = global_ns();
}

// The permutation of a larger batch's pairs (more than kSmallPlan, no
// capacity): pair p goes
// to its expert's first position plus a slot taken from the expert's cursor.
// The order of an expert's pairs is then arbitrary, which changes neither
// branch's result (rows are independent; the combine is a sum).
__global__ void __launch_bounds__(256) k_plan_scatter(Workspace ws, int P, int k, int E)
{
    const Plan *plan = ws.plan;
    for (int p = blockIdx.x * blockDim.x + threadIdx.x; p < P; p += gridDim.x * blockDim.x) {
        const int e = min(max(__ldcg(&ws.topk_idx[p]), 0), E - 1);
        const int pos = min(__ldcg(&plan->offsets[e]) + atomicAdd(&ws.cursor[e], 1), P - 1);
        ws.perm[pos] = p;
        ws.perm_tok[pos] = p / k;
        ws.perm_w[pos] = __ldcg(&ws.topk_w[p]);
    }
}

cudaError_t launch_router(const Dims &dm, const DeviceWeights &w, const Workspace &ws,
                          const uint16_t *x, int T, int tile_tokens, cudaStream_t st, int cap, bool logits_ready)
{
    if (cap >= 0 && (long long)T * dm.k > kStagePairs) return cudaErrorNotSupported;
    RouterArgs a;
    a.x = x;
    a.wr = w.wr;
    a.T = T;
    a.d = dm.d;
    a.E = dm.E;
    a.k = dm.k;
    a.mt = tile_tokens;
    a.n_chunks = dm.n_blk;
    a.dp = dm.dp;
    a.xtile = (T <= tile_tokens && tile_tokens <= 16) ? tile_tokens : 0;
    a.cap = cap;
    a.mask_words = dm.f / kChunk;
    a.ws = ws;
    // experts per CTA: 2 unless that makes more than about two CTAs per SM
    // (large batches); then more, so a CTA stages its tile's rows once for
    // several experts (single-chunk rows only, d <= 2048)
    const long long tiles = (T + kRtTok - 1) / kRtTok;
    int epc = kRtExp;
    if (dm.d <= 2048) {
        const long long want = 2 * 148;
        const long long pairs_per_tile = (dm.E + kRtExp - 1) / kRtExp;
        long long per = (pairs_per_tile * tiles + want - 1) / want;   // expert pairs per CTA
        if (per > pairs_per_tile) per = pairs_per_tile;
        if (per > 1) epc = (int)per * kRtExp;
    }
    a.logits_ready = logits_ready ? 1 : 0;
    if (logits_ready) epc = (dm.E + 1) & ~1;   // one CTA per token tile: softmax, top-k, plan
    a.epc = epc;
    dim3 grid((dm.E + epc - 1) / epc, (unsigned)tiles);
    const size_t P = (size_t)T * dm.k;
    size_t smem = sizeof(float) * (size_t)kRtTok * dm.E;   // softmax rows
    if (smem < 16 * (size_t)kRtTok * 256 + 4 * 8 * kRtTok) smem = 16 * (size_t)kRtTok * 256 + 4 * 8 * kRtTok;   // x chunk, quarter sums
    size_t plan_smem = sizeof(int) * 2 * (size_t)dm.E + (plan_staged((long long)P, cap) ? (cap >= 0 ? 12 : 8) * P : 0);
    if (plan_smem > smem) smem = plan_smem;
    // at most max(32 KB, 2*1024*4 + 12*4096 = 56 KB): above the default 48 KB
    // window only with a capacity
    static int smem_set[kMaxDevices] = {};
    if (smem > 48 * 1024) {
        const cudaError_t e = ensure_dynamic_smem(k_router, (int)smem, smem_set);
        if (e != cudaSuccess) return e;
    }
    k_router<<<grid, 256, smem, st>>>(a);
    if (!plan_staged((long long)T * dm.k, cap)) {
        const int P = T * dm.k;
        int blocks = (P + 255) / 256;
        if (blocks > 148 * 8) blocks = 148 * 8;
        k_plan_scatter<<<blocks, 256, 0, st>>>(ws, P, dm.k, dm.E);
    }
    return cudaGetLastError();
}

}  // namespace moe
