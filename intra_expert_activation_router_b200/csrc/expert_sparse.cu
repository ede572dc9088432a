// expert_sparse.cu -- the sparse branch: gate projection on the tensor cores,
// threshold mask, compaction, and the gathered up/down projection of the
// active neurons, in one persistent warp-specialised kernel.
//
// "Uncovering Intra-expert Activation Sparsity for Efficient Mixture-of-Expert
// Model Execution" (technical summary, Methodology item 3):
//   - gate projection, dense ("Gate projection" bullet): g = x Wg[e] for every
//     neuron of the selected expert -- here a tcgen05 MMA per 128-neuron block:
//     D[128 neurons x 16 columns] (TMEM) = Wg block . X tile^T, the block's
//     gate tiles streamed through a ring of 32 KB stages (bulk copies), the
//     token operand in the MMA's K-major swizzled layout;
//   - activation mask in one O(n) pass, no sort ("Activation masking"):
//     active iff |silu(g)| >= tau -- a warp ballot over 32 neurons per token;
//   - fused up-down projection over the active neurons only ("Fused up-down
//     projection"): the active rows of Wu and Wd are gathered and packed
//     densely in shared memory, h = silu(g) * (x Wu[:,j]) and y += w h Wd[j][:]
//     (Hindi summary, "The skip": inactive neurons' weights are never loaded);
//   - shared experts: the same code with the mask off and weight 1 (their
//     execution is unchanged and always dense).
//
// Work items are (expert, tile of up to NT of its tokens, block of 128
// neurons).  With T <= NT ("resident" mode) the whole batch is the gate MMA's
// token operand: the router writes it in the MMA's layout (or, when the batch
// is routed inside this kernel, a TMA tensor map reads it straight from x),
// and each ring stage carries its two 64-input blocks (2 or 4 KB, re-read
// from L2 per item) next to the 32 KB of gate tiles, which leaves the shared memory of a
// resident token tile to the gather buffers.  Items are claimed from a
// counter in the plan, the experts with most tokens first.  A CTA claims its next item only
// once its previous one is masked and at most kClaimBacklog of its gathered
// records are still to be projected: an item's up/down cost (its active
// records) varies several-fold and is known only after its mask, so claims
// paced by the gate stream alone leave some CTAs with three heavy items and
// others idle.  Otherwise each CTA takes a contiguous range of items and
// loads each tile's token rows.  Agents, one CTA per SM:
//   gate lane (warp 8)     publishes item ids; the item's gate tiles, 32 KB
//                          stages into the ring (with the token operand's
//                          blocks in resident mode)
//   MMA lane (warp 9)      per stage 8 MMAs (M 128, N 16, K 16) into one of
//                          four TMEM accumulators; owns the TMEM allocation
//   x warp (warp 10)       tile mode: token rows into the MMA's K-major
//                          128-byte-swizzled layout (cp.async); idle in
//                          resident mode
//   gather warp (warp 11)  once an item's mask is final, the union-active
//                          [up | down] records into a ring of buffers, one
//                          bulk copy per record
//   up warps (0-3)         M(i): the accumulator (one neuron per thread),
//                          silu, threshold, ballot per token, the union per
//                          pass of MT tokens; then per gathered batch the up
//                          dots (each thread holds slices of d of the pass's
//                          tokens, one transposed warp reduction per 4 rows)
//                          and h = silu(g) u where the bit is set
//   down warps (4-7)       per batch, h x the gathered down rows into
//                          per-thread registers kept across consecutive blocks
//                          of the same tokens, then fp32 vector atomics into
//                          y_acc; a small kernel after this one converts y_acc
//                          to bf16 into `out` and re-zeroes it.
// The agents meet on mbarriers (copies, MMA completion, buffer and h hand-off)
// and on monotonic progress counters in shared memory; every wait is bounded.
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"
#include "tma.cuh"

namespace moe {

constexpr int kUpThreads = 128;     // warps 0-3: mask and up projection
constexpr int kDownThreads = 128;   // warps 4-7: down projection and flush
constexpr int kWarpTma = 8, kWarpMma = 9, kWarpX = 10, kWarpGather = 11;
constexpr int kSparseThreads = 384;
constexpr int kGateTile = 16384;     // bytes of one gate tile: 128 neurons x 64 inputs
constexpr int kStageBytes = 2 * kGateTile;
constexpr int kMaxNT = 16;           // tokens per gate tile
constexpr int kMaxSub = 4;           // passes of MT tokens per tile
constexpr int kRows = 4;             // up rows per warp reduction
constexpr int kMaxGB = 8;            // records per gather buffer
constexpr int kAcc = 4;              // TMEM gate accumulators (the MMA runs up to kAcc items ahead)
constexpr int kTmemCols = 16 * kAcc;
constexpr int kSmemLimit = 227 * 1024;
constexpr int kMaxNU = 6;            // gather buffers
constexpr int kIdRing = 16;          // published work-item ids
constexpr int kShareMinRecords = 32;   // gate split: shortest union list whose records the parts share
constexpr int kRecSplitMax = 4;        // record split of dense shared items: most parts per item
constexpr int kClaimBacklog = 24;    // resident mode: records still to project when the next item is claimed
constexpr int kMaxFusedPairs = 128;  // fused routing: (token, expert) pairs kept in shared memory
constexpr int kMaxFusedLogits = 8192;   // fused routing: T * E logits staged in the gate ring
constexpr int kMaxFusedExperts = 256;   // fused routing: rank counting costs E per logit
// mbarriers besides the two rings': gdone, tfree (kAcc each), xfull, xfree,
// mdrain, hsfull, hsfree (2 each)
constexpr int kNumFixedBars = 2 * kAcc + 7;

struct SparseLayout {   // byte offsets from the 1024-aligned base of dynamic shared memory
    int xt_off, xt_kb;                      // token tile (tile mode); bytes per 64-input block (nt * 128)
    int stage_pitch, xs_bytes;              // ring stage: 32 KB of gate tiles, then (resident mode) the
                                            // stage's two 64-input blocks of the token operand
    int ring_off, n_stages;
    int ud_off, ud_buf_bytes, gb, gpitch;   // n_ud buffers of gb [up | down] records (+16-byte skew)
    int n_ud;
    int meta_off, part_off, h_off, last_off, ctr_off, plan_off, perm_off, bar_off;
    int total;                              // dynamic bytes to request (includes alignment slack)
};

struct ItemMeta {
    const uint16_t *wud;          // the expert's [f][2d] up/down records
    long long key;                // (expert slot or shared index, token tile)
    int m, blk, masked, nsub;
    int sidx;                     // shared expert of the item, -1 for a routed expert
    int part;                     // gate split: 0 owner (masks, projects), > 0 publishes partial sums only
    int tok[kMaxNT];
    int pair[kMaxNT];
    float w[kMaxNT];
    unsigned word[kMaxNT][4];     // mask words: token, 32-neuron quarter of the block
    int n_uni[kMaxSub];
    uint8_t uni[kMaxSub][kBlk];   // per pass: union-active neurons of the block, ascending
    uint16_t a[kMaxNT][kBlk];     // silu(g) as bf16 (RNE): fp32's range, relative error <= 2^-9
};

struct SparseArgs {
    CUtensorMap xmap;     // fused mode: x [T][d] as the MMA's token operand (box 64 x nt, 128-byte swizzle)
    const uint16_t *x;
    uint16_t *out;
    DeviceWeights w;
    Workspace ws;
    int T, d, f, k, S;
    int dp, n_kb, n_blk, n_chunks;
    int nt;               // tokens per gate tile
    int resident;         // T <= nt: the whole batch is the MMA's token operand (x_tiles),
                          // and work items are claimed dynamically, heaviest expert first
    float tau;
    float tau_shared;     // shared experts' threshold (masked forwards); <= 0: every shared neuron
    int use_mask;
    int score_shared;     // score mode over the shared experts' neurons instead of the routed pairs'
    int n_tok_tiles;      // ceil(T / nt), for the shared experts
    int n_shared_items;   // S * n_tok_tiles * n_blk
    int max_touched;      // plan cache capacity
    float *score_out;     // score mode: write |silu(g)| [pair][f] (or [token][S][f]), no up/down
    int inject;           // test-only fault: 1 = publish no work item (consumers' waits run out)
    int n_parts;          // gate split: parts per routed item (1: none); part 0, claimed last, owns the item
    int n_parts_s;        // the same for the shared experts' items
    int share_records;    // gate split: the parts also share the item's records (part p projects the
                          // p-th of n_parts ranges of the owner's union list); launches the SH kernel
    int rec_split;        // instead of a gate split: each of a dense shared item's n_parts_s parts streams
                          // the whole gate and projects the p-th range of its records (no hand-off)
    int fused;            // route the batch here (resident mode): logits, top-k and plan per CTA
    const uint16_t *wr;   // fused: router weights [E][d]
    int E;
    int max_pairs;        // fused: T * k (permutation arrays kept in shared memory)
    // rank budget, second pass: the routed pairs' silu(g) [pair][f] from the
    // first pass (score mode, signed) and each pair's cut (v, J) -- neuron j
    // is kept iff |silu(g_j)| > v, or == v and j <= J; routed items then
    // stream no gate (the shared experts' items still do)
    const float *a_in;
    const float *rank_v;
    const int *rank_j;
    int score_signed;     // score mode: write silu(g) itself instead of |silu(g)|
    int tail;             // combine here: y_acc -> bf16 `out` after a grid-wide arrival count
    long long n_out4;     // float4 groups of y_acc converted (0 in score mode)
    SparseLayout L;
};

struct ItemPos {
    int slot;   // routed expert slot, or -1 - s for shared expert s
    int tile, blk;
};

struct PlanCache {      // the routing plan's per-slot arrays, copied to shared memory
    const int *prefix, *expert, *off, *cnt;
    const int *order;   // resident mode: slots by decreasing token count
    int n_touched;
    // the permutation of (token, rank) pairs by expert: the workspace's, or in
    // fused mode this CTA's own copy in shared memory
    const int *perm, *perm_tok;
    const float *perm_w;
};

// DEC: the decode instantiation, always resident (see k_expert_sparse)
template <bool DEC>
__device__ __forceinline__ ItemPos locate_item(const SparseArgs &a, const PlanCache &pc, int item)
{
    ItemPos p;
    if (item < a.n_shared_items) {
        const int per_s = a.n_tok_tiles * a.n_blk;
        p.slot = -1 - item / per_s;
        const int r0 = item % per_s;
        p.tile = r0 / a.n_blk;
        p.blk = r0 % a.n_blk;
    } else if (DEC || a.resident) {   // one tile per expert, slots heaviest first
        const int ir = item - a.n_shared_items;
        p.slot = pc.order[min(ir / a.n_blk, pc.n_touched - 1)];
        p.tile = 0;
        p.blk = ir % a.n_blk;
    } else {
        const int ir = item - a.n_shared_items;
        int lo = 0, hi = pc.n_touched - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (pc.prefix[mid] <= ir) lo = mid; else hi = mid - 1;
        }
        const int local = ir - pc.prefix[lo];
        p.slot = lo;
        p.tile = local / a.n_blk;
        p.blk = local % a.n_blk;
    }
    return p;
}

__device__ __forceinline__ long long item_key(const ItemPos &p)
{
    return ((long long)(p.slot < 0 ? p.slot : p.slot + 1) << 32) | (unsigned)p.tile;
}

// Gate split: claim id -> (item, part).  The shared experts' items come
// first, n_parts_s claims each, then the routed items, n_parts each.  An
// item's parts are claimed in the order P - 1, ..., 1, 0, so the owner (part
// 0), which waits for the others' partial sums, is always claimed after them:
// every such wait points to an earlier claim, which its CTA publishes before
// it reaches any later wait.
// PM, the kernel's part mapping: 2 per-class part counts (the
// record-sharing instantiation), 1 every item n_parts parts, 0 no split (the
// kernels for more than kSplitCols tokens: every item one part, compile-time).
template <int PM>
__device__ __forceinline__ int split_item(const SparseArgs &a, int id)
{
    if constexpr (PM == 2) {
        const int ns = a.n_shared_items * a.n_parts_s;
        return id < ns ? id / a.n_parts_s : a.n_shared_items + (id - ns) / a.n_parts;
    } else if constexpr (PM == 1) {
        return id / a.n_parts;
    } else {
        return id;
    }
}
template <int PM>
__device__ __forceinline__ int split_part(const SparseArgs &a, int id)
{
    if constexpr (PM == 2) {
        const int ns = a.n_shared_items * a.n_parts_s;
        return id < ns ? a.n_parts_s - 1 - id % a.n_parts_s : a.n_parts - 1 - (id - ns) % a.n_parts;
    } else if constexpr (PM == 1) {
        return a.n_parts - 1 - id % a.n_parts;
    } else {
        return 0;
    }
}
template <int PM>
__device__ __forceinline__ int item_parts(const SparseArgs &a, int item)
{
    if constexpr (PM == 2)
        return item < a.n_shared_items ? a.n_parts_s : a.n_parts;
    else if constexpr (PM == 1)
        return a.n_parts;
    else
        return 1;
}

// Stages [lo, hi) of the item's spi gate stages that a part streams.
__device__ __forceinline__ void part_stages(int spi, int n_parts, int part, int &lo, int &hi)
{
    lo = spi * part / n_parts;
    hi = spi * (part + 1) / n_parts;
}

// Tokens of the item's tile: count, and where token r comes from.
__device__ __forceinline__ int tile_tokens(const SparseArgs &a, const PlanCache &pc, const ItemPos &p, int &base)
{
    if (p.slot < 0) {
        base = p.tile * a.nt;   // token ids base .. base + m - 1
        return max(1, min(a.nt, a.T - base));
    }
    base = pc.off[p.slot] + p.tile * a.nt;   // positions in perm
    return max(1, min(a.nt, pc.cnt[p.slot] - p.tile * a.nt));
}

__device__ __forceinline__ int tile_token(const SparseArgs &a, const PlanCache &pc, const ItemPos &p, int base,
                                          int r)
{
    const int t = p.slot < 0 ? base + r : pc.perm_tok[base + r];
    return min(max(t, 0), a.T - 1);
}

// The pass's token rows from global memory (L2-resident), this thread's
// slices of d, widened to fp32 and packed in pairs: xf[p][r][i] holds
// x_r[8 v + 2i] and x_r[8 v + 2i + 1] with v = t128 + 128 p (t128: the
// thread's index among the four up warps).
template <int MT, int NP>
__device__ __forceinline__ void load_x(const uint16_t *x, const int *tok, int m, int d, int t128,
                                       uint64_t (&xf)[NP][MT][4])
{
    const int d8 = d >> 3;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        const int v = t128 + 128 * p;
#pragma unroll
        for (int r = 0; r < MT; ++r) {
            const uint4 xv = (r < m && v < d8) ? ld_cached(x + (size_t)tok[r] * d + 8 * v) : make_uint4(0, 0, 0, 0);
            xf[p][r][0] = bf16x2_f2(xv.x);
            xf[p][r][1] = bf16x2_f2(xv.y);
            xf[p][r][2] = bf16x2_f2(xv.z);
            xf[p][r][3] = bf16x2_f2(xv.w);
        }
    }
}

// Partial up projections of R gathered rows over this warp's slices of d:
// acc[q][r] = sum_{k in slices} w_q[k] x_r[k], rows q < nrows at lo + q*stride,
// even and odd k in the two lanes of packed fp32 FMAs.  All row loads are
// issued before the math.  After one transposed warp reduction the warp-wide
// sum for (q, r) sits in one lane, which stores it to
// part_w[(row_off + q) * MT + r].
template <int R, int MT, int NP>
__device__ __forceinline__ void group_rows(const uint8_t *lo, int stride, int nrows, const uint64_t (&xf)[NP][MT][4],
                                           int d8, int t128, int lane, float *part_w, int row_off)
{
    constexpr int NV = R * MT;
    constexpr int SH = 5 - Log2<NV>::value;
    uint64_t acc2[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) acc2[i] = 0ull;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        const int v = t128 + 128 * p;
        if (v < d8) {
            uint4 wv[R];
#pragma unroll
            for (int q = 0; q < R; ++q)
                wv[q] = q < nrows ? *reinterpret_cast<const uint4 *>(lo + q * stride + 16 * v) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int q = 0; q < R; ++q) {
                const uint64_t w2[4] = {bf16x2_f2(wv[q].x), bf16x2_f2(wv[q].y), bf16x2_f2(wv[q].z),
                                        bf16x2_f2(wv[q].w)};
#pragma unroll
                for (int r = 0; r < MT; ++r) {
                    uint64_t a2 = acc2[q * MT + r];
#pragma unroll
                    for (int i = 0; i < 4; ++i) a2 = ffma2(w2[i], xf[p][r][i], a2);
                    acc2[q * MT + r] = a2;
                }
            }
        }
    }
    float acc[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        float e0, e1;
        f2_unpack(acc2[i], e0, e1);
        acc[i] = e0 + e1;
    }
    const float val = transpose_reduce<NV>(acc, lane);
    const int vi = lane >> SH, q = vi / MT, r = vi % MT;
    if ((lane & ((1 << SH) - 1)) == 0 && q < nrows) part_w[(row_off + q) * MT + r] = val;
}

__device__ __forceinline__ int ld_acquire_gpu(const int *p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ bool route_better(float v1, int i1, float v0, int i0)
{
    return v1 > v0 || (v1 == v0 && i1 < i0);
}

// Routing inside the expert kernel, for batches it takes as one token tile
// (the decode path).  It is the router of the technical summary ("Uncovering
// Intra-expert Activation Sparsity ...", Methodology item 3: the router logic
// is kept unchanged): logits = x Wr^T with fp32 accumulation, softmax over all
// E experts, the top_k experts by probability (ties to the lower index),
// weight = probability.  Computing it here removes the router launch and the
// grid-wide hand-off of its plan from the front of the gate stream:
//   1. CTA b computes the logits of experts b, b + G, ... for all T tokens and
//      publishes them with a release-ordered count;
//   2. once all E experts are counted (bounded wait), every CTA reads the
//      T x E logits and selects each token's top_k (one warp per token, k
//      rounds of a warp arg-max);
//   3. every CTA builds the plan -- per-expert counts, the ascending list of
//      touched experts, their offsets and the stable permutation of the pairs
//      (expert, then token) -- in its own shared memory; CTA 0 also writes it
//      to the workspace, where the statistics and debug calls read it.
// `scratch` (the gate ring, idle until the plan exists) holds the
// temporaries.  Called by every thread of the CTA.  TR: the traced build
// (phase stamps into the workspace's trace buffer).
template <bool TR>
__device__ __noinline__ void route_in_kernel(const SparseArgs &a, uint8_t *scratch, int *s_prefix, int *s_expert,
                                             int *s_off, int *s_cnt, int *s_perm, int *s_perm_tok, float *s_perm_w,
                                             volatile int *s_ntouched, uint64_t *xbar)
{
    // written as short loops: this runs once per forward, so its code is
    // fetched cold -- few instructions matter more than unrolled ones
    constexpr int NW = kSparseThreads / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = a.T, E = a.E, k = a.k, d = a.d, d8 = d >> 3, P = T * k;
    uint4 *xs = reinterpret_cast<uint4 *>(scratch);                  // [T][d8] the batch's rows
    float *red = reinterpret_cast<float *>(xs + (size_t)T * d8);     // [NW][kMaxNT]
    float *lg = red + NW * kMaxNT;                                    // [T][E]
    int *tk_idx = reinterpret_cast<int *>(lg + (size_t)T * E);        // [P]
    float *tk_w = reinterpret_cast<float *>(tk_idx + P);              // [P]
    int *ecnt = reinterpret_cast<int *>(tk_w + P);                    // [E] pairs per expert
    int *eoff = ecnt + E;                                             // [E] first position per expert
    Plan *plan = a.ws.plan;
    unsigned long long *tr = (TR && a.ws.trace_expert && (int)blockIdx.x < a.ws.trace_expert_ctas)
                                 ? a.ws.trace_expert + blockIdx.x * 64 : nullptr;
    if (tr && tid == 0) tr[44] = global_ns();

    // 1. this CTA's experts' logits (fp32 accumulation of bf16 products); the
    //    batch's rows arrive by one bulk copy (x is [T][d], contiguous)
    int mine = 0;
    const uint4 z = make_uint4(0, 0, 0, 0);
    uint4 w0 = z, w1 = z;
    if ((int)blockIdx.x < E) {
        if (tid == 0) {
            mbar_arrive_expect_tx(xbar, (uint32_t)(T * d * 2));
            bulk_g2s(xs, a.x, (uint32_t)(T * d * 2), xbar);
        }
        // the first expert's router row is in flight while x arrives
        const uint16_t *wrow = a.wr + (size_t)blockIdx.x * d;
        if (tid < d8) w0 = ld_cached(wrow + 8 * tid);
        if (tid + kSparseThreads < d8) w1 = ld_cached(wrow + 8 * (tid + kSparseThreads));
        mbar_wait(xbar, 0, a.ws.error_word, 55);
    }
    __syncthreads();
#pragma unroll 1
    for (int e = blockIdx.x; e < E; e += gridDim.x, ++mine) {
        if (e != (int)blockIdx.x) {
            const uint16_t *wrow = a.wr + (size_t)e * d;
            w0 = tid < d8 ? ld_cached(wrow + 8 * tid) : z;
            w1 = tid + kSparseThreads < d8 ? ld_cached(wrow + 8 * (tid + kSparseThreads)) : z;
        }
#pragma unroll 1
        for (int t0 = 0; t0 < T; t0 += 4) {   // four tokens per transposed warp reduction
            float acc[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                acc[u] = 0.f;
                if (t0 + u < T) {
                    if (tid < d8) acc[u] = dot8(w0, xs[(t0 + u) * d8 + tid], acc[u]);
                    if (tid + kSparseThreads < d8) acc[u] = dot8(w1, xs[(t0 + u) * d8 + tid + kSparseThreads], acc[u]);
                }
            }
            const float v = transpose_reduce<4>(acc, lane);   // lanes 8u .. 8u + 7: token t0 + u
            if ((lane & 7) == 0 && t0 + (lane >> 3) < T) red[warp * kMaxNT + t0 + (lane >> 3)] = v;
        }
        __syncthreads();
        if (tid < T) {
            float sum = 0.f;
#pragma unroll 1
            for (int w = 0; w < NW; ++w) sum += red[w * kMaxNT + tid];
            a.ws.logits[(size_t)tid * E + e] = sum;
            __threadfence();
        }
        __syncthreads();
    }
    if (tr && tid == 0) tr[45] = global_ns();
    if (tid == 0 && mine > 0) {
        __threadfence();
        atomicAdd(a.ws.route_count, mine);
    }
    if (tr && tid == 0) tr[58] = global_ns();
    // 2. every expert's logits, then each token's top_k
    if (tid == 0) {
        for (uint32_t spin = 0; ld_acquire_gpu(a.ws.route_count) < E; ++spin) {
            if (spin > kSpinLimit) {
                atomicCAS(a.ws.error_word, 0, 55);
                break;
            }
            __nanosleep(32);
        }
    }
    __syncthreads();
    if (tr && tid == 0) tr[59] = global_ns();
#pragma unroll 4
    for (int i = tid; i < T * E; i += kSparseThreads) lg[i] = __ldcg(&a.ws.logits[i]);
#pragma unroll 1
    for (int e = tid; e < E; e += kSparseThreads) ecnt[e] = 0;
#pragma unroll 1
    for (int p = tid; p < P; p += kSparseThreads) {   // valid defaults: only non-finite logits could
        tk_idx[p] = 0;                                 // leave a rank unwritten
        tk_w[p] = 0.f;
    }
    __syncthreads();
    if (tr && tid == 0) tr[46] = global_ns();
#pragma unroll 1
    for (int t = warp; t < T; t += NW) {   // each token's softmax max and sum (one warp per token)
        const float *row = lg + (size_t)t * E;
        float m = -INFINITY;
#pragma unroll 1
        for (int j = lane; j < E; j += 32) m = fmaxf(m, row[j]);
        m = warp_max(m);
        float sum = 0.f;
#pragma unroll 1
        for (int j = lane; j < E; j += 32) sum += expf(row[j] - m);
        sum = warp_sum(sum);
        if (lane == 0) {
            red[2 * t] = m;
            red[2 * t + 1] = sum;
        }
    }
    __syncthreads();
    // the rank of each logit within its token's row: the logits before it
    // (larger, or equal with a lower index); ranks below k are the top_k, in
    // rank order.  One (token, expert) pair per thread at a time.
#pragma unroll 1
    for (int i = tid; i < T * E; i += kSparseThreads) {
        const int t = i / E, j = i - t * E;
        const float *row = lg + (size_t)t * E;
        const float v = row[j];
        int rank = 0;
#pragma unroll 4
        for (int q = 0; q < E; ++q) rank += route_better(row[q], q, v, j) ? 1 : 0;
        if (rank < k) {
            tk_idx[t * k + rank] = j;
            tk_w[t * k + rank] = expf(v - red[2 * t]) / red[2 * t + 1];
        }
    }
    __syncthreads();
    if (tr && tid == 0) tr[60] = global_ns();
    // 3. the plan: counts, offsets and ascending touched list, stable permutation
#pragma unroll 1
    for (int p = tid; p < P; p += kSparseThreads) atomicAdd(&ecnt[min(max(tk_idx[p], 0), E - 1)], 1);
    __syncthreads();
    if (warp == 0) {
        int run_c = 0, run_t = 0;
#pragma unroll 1
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            const int c = e < E ? ecnt[e] : 0, on = c > 0 ? 1 : 0;
            int ic = c, it = on;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int uc = __shfl_up_sync(kFull, ic, o), ut = __shfl_up_sync(kFull, it, o);
                if (lane >= o) { ic += uc; it += ut; }
            }
            const int off = run_c + ic - c, slot = run_t + it - on;
            if (e < E) eoff[e] = off;
            if (on) {
                s_expert[slot] = e;
                s_off[slot] = off;
                s_cnt[slot] = c;
                s_prefix[slot] = slot * a.n_blk;
            }
            run_c += __shfl_sync(kFull, ic, 31);
            run_t += __shfl_sync(kFull, it, 31);
        }
        if (lane == 0) {
            *s_ntouched = run_t;
            s_prefix[run_t] = run_t * a.n_blk;
        }
    }
    __syncthreads();
#pragma unroll 1
    for (int p = tid; p < P; p += kSparseThreads) {   // pair p after the earlier pairs of its expert
        const int e = min(max(tk_idx[p], 0), E - 1);
        int r = 0;
#pragma unroll 4
        for (int q = 0; q < p; ++q) r += min(max(tk_idx[q], 0), E - 1) == e ? 1 : 0;
        const int pos = eoff[e] + r;
        s_perm[pos] = p;
        s_perm_tok[pos] = p / k;
        s_perm_w[pos] = tk_w[p];
    }
    __syncthreads();
    if (tr && tid == 0) tr[47] = global_ns();
    if (blockIdx.x == 0) {   // the workspace copy for statistics and debug calls
        const int n_t = *s_ntouched;
#pragma unroll 1
        for (int p = tid; p < P; p += kSparseThreads) {
            a.ws.topk_idx[p] = tk_idx[p];
            a.ws.topk_w[p] = tk_w[p];
            a.ws.perm[p] = s_perm[p];
            a.ws.perm_tok[p] = s_perm_tok[p];
            a.ws.perm_w[p] = s_perm_w[p];
        }
#pragma unroll 1
        for (int e = tid; e < E; e += kSparseThreads) plan->offsets[e] = eoff[e];
#pragma unroll 1
        for (int i = tid; i <= n_t; i += kSparseThreads) {
            if (i < n_t) plan->touched[i] = s_expert[i];
            plan->item_prefix[i] = s_prefix[i];
        }
        if (tid == 0) {
            plan->offsets[E] = P;
            plan->n_touched = n_t;
            plan->n_routed_items = n_t * a.n_blk;
        }
    }
    // the gate ring and gather buffers are written by the copy engine from here on
    fence_proxy_async_smem();
    __syncthreads();
}

// The combine, at the end of the kernel: every CTA has flushed its down sums
// into y_acc (fp32 vector atomics, performed in L2) when the arrival count
// reaches the grid; each CTA then converts its slice of y_acc to bf16 (round
// to nearest even) into `out` and re-zeroes it.  The last CTA out resets the
// forward's counters and moves the forward's error code into the sticky
// word.  All CTAs of the grid are resident at once (one per SM, at most one
// per SM), so the count completes; the wait is bounded all the same (code 57,
// and that CTA's slice is left unconverted).
__device__ __noinline__ void combine_tail(const SparseArgs &a, int tid, int *s_flag)
{
    int *tail = a.ws.tail;
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        atomicAdd(&tail[0], 1);
        int ok = 1;
        for (uint32_t spin = 0; ld_acquire_gpu(&tail[0]) < (int)gridDim.x; ++spin) {
            if (spin > kSpinLimit) {
                atomicCAS(a.ws.error_word, 0, 57);
                ok = 0;
                break;
            }
            __nanosleep(64);
        }
        *s_flag = ok;
    }
    __syncthreads();
    if (*s_flag && a.ws.ypart) {
        const int warps = kSparseThreads / 32;
        det_combine(a.ws.ypart, (a.k + a.S) * a.n_blk, a.d, a.out, a.n_out4, (long long)blockIdx.x * warps + (tid >> 5),
                    (long long)gridDim.x * warps, tid & 31);
    } else if (*s_flag) {
        const float4 *src = reinterpret_cast<const float4 *>(a.ws.y_acc);
        float4 *zero = reinterpret_cast<float4 *>(a.ws.y_acc);
        uint2 *dst = reinterpret_cast<uint2 *>(a.out);
#pragma unroll 1
        for (long long i = (long long)blockIdx.x * kSparseThreads + tid; i < a.n_out4;
             i += (long long)gridDim.x * kSparseThreads) {
            const float4 v = __ldcg(src + i);
            uint2 p;
            p.x = (uint32_t)f2bf_bits(v.x) | ((uint32_t)f2bf_bits(v.y) << 16);
            p.y = (uint32_t)f2bf_bits(v.z) | ((uint32_t)f2bf_bits(v.w) << 16);
            dst[i] = p;
            __stcg(zero + i, make_float4(0.f, 0.f, 0.f, 0.f));
        }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        *s_flag = atomicAdd(&tail[1], 1) == (int)gridDim.x - 1;
        __threadfence();
    }
    __syncthreads();
    if (*s_flag) {   // last CTA out: every CTA is past every use of the counters
#pragma unroll 1
        for (int i = tid; a.ws.gcnt && i < a.ws.gcnt_n; i += kSparseThreads) a.ws.gcnt[i] = 0;
        if (tid == 0) {
            *a.ws.route_count = 0;
            a.ws.plan->next_item = 0;
            const int e0 = *reinterpret_cast<volatile int *>(a.ws.error_word);
            if (e0 != 0) {
                atomicCAS(a.ws.error_sticky, 0, e0);
                *a.ws.error_word = 0;
            }
            tail[0] = 0;
            tail[1] = 0;
        }
    }
}

// TR: the traced instantiation, launched only while moe_set_trace holds a
// buffer; the stamps' clock reads and branches cost 4-7 % of a decode step,
// so the untraced kernels have none of them.  DEC: the decode instantiation,
// for batches resident as one token tile, outside the rank budget's passes,
// the calibration's score mode and fault injection: the token-tile mode, the
// rank pass, the score mode and the injection compiled out, and the routing
// (inside the kernel, FU, or by the router kernel) fixed at compile time
// (8-9 % of a decode step).  SH (decode only): the
// parts of a split item also share its records, per-class part counts, the
// record split of dense shared items; a separate instantiation again, since
// code the other kernels never run still slowed them by about a microsecond.
// The traced kernel is the general one (not DEC, not SH).
template <int MT, int NP, bool TR, bool SH, bool DEC, bool FU>
__global__ void __launch_bounds__(kSparseThreads, 1) k_expert_sparse(const __grid_constant__ SparseArgs a)
{
    extern __shared__ uint8_t dsm_raw[];
    // the 128-byte swizzle of the MMA operands needs 1024-byte aligned tiles
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
    const SparseLayout &L = a.L;
    uint8_t *xt = smem + L.xt_off;
    uint8_t *ring = smem + L.ring_off;
    uint8_t *ud = smem + L.ud_off;
    ItemMeta *meta = reinterpret_cast<ItemMeta *>(smem + L.meta_off);   // [2]
    float *part = reinterpret_cast<float *>(smem + L.part_off);        // [2][4 up warps][kMaxGB][MT]
    float *hs = reinterpret_cast<float *>(smem + L.h_off);             // [2][kMaxGB][MT]
    // progress shared between the agents; monotonic, so a reader can never
    // mistake an old value for a new one:
    //   mask_done  items whose mask and union lists are final    (consumers)
    //   pub_items  work-item ids published in s_items           (gate lane)
    //   items_end  number of items of this CTA, once known      (consumers)
    volatile int *mask_done = reinterpret_cast<volatile int *>(smem + L.ctr_off);
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(smem + L.ctr_off + 16);
    volatile int *pub_items = reinterpret_cast<volatile int *>(smem + L.ctr_off + 32);
    volatile int *items_end = reinterpret_cast<volatile int *>(smem + L.ctr_off + 48);
    // items whose down projection and flush are done (down warps)
    volatile int *down_done = reinterpret_cast<volatile int *>(smem + L.ctr_off + 52);
    // records of the masked items (up warps) and records projected (down warps)
    volatile int *rec_masked = reinterpret_cast<volatile int *>(smem + L.ctr_off + 36);
    volatile int *rec_done = reinterpret_cast<volatile int *>(smem + L.ctr_off + 40);
    volatile int *s_items = reinterpret_cast<volatile int *>(smem + L.ctr_off + 64);   // [kIdRing]
    int *s_tail_flag = reinterpret_cast<int *>(smem + L.ctr_off + 20);
    int *s_prefix = reinterpret_cast<int *>(smem + L.plan_off);
    int *s_expert = s_prefix + a.max_touched + 1;
    int *s_off = s_expert + a.max_touched;
    int *s_cnt = s_off + a.max_touched;
    int *s_order = s_cnt + a.max_touched;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    const int NS = L.n_stages;
    uint64_t *full_g = bars, *empty_g = bars + NS;         // gate ring
    uint64_t *gdone = bars + 2 * NS, *tfree = gdone + kAcc;   // TMEM accumulators
    uint64_t *xfull = tfree + kAcc, *xfree = xfull + 1;       // token tile
    uint64_t *mdrain = xfree + 1;
    const int NU = L.n_ud;
    uint64_t *full_u = mdrain + 1, *empty_u = full_u + NU;   // gather buffers
    uint64_t *hsfull = empty_u + NU, *hsfree = hsfull + 2;   // h of a batch, up warps -> down warps

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    Plan *plan = a.ws.plan;
    int *err = a.ws.error_word;
    const int d = a.d;
    constexpr int PM = SH ? 2 : (MT <= kSplitCols ? 1 : 0);   // the part mapping (split_item)
    const bool score_mode = !DEC && a.score_out != nullptr;   // compile-time false in the decode kernel
    const bool fused = DEC ? FU : a.fused != 0;               // compile-time in the decode kernels
    const bool resident = DEC || a.resident;
    const float *const a_in = DEC ? nullptr : a.a_in;   // rank pass, second pass
    const int inject = DEC ? 0 : a.inject;
    unsigned long long *tr = (TR && a.ws.trace_expert && (int)blockIdx.x < a.ws.trace_expert_ctas)
                                 ? a.ws.trace_expert + blockIdx.x * 64 : nullptr;
    if (tr && tid == 0) tr[0] = global_ns();

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full_g[s], 1);
            mbar_init(&empty_g[s], 1);
        }
        for (int b = 0; b < kAcc; ++b) {
            mbar_init(&gdone[b], 1);
            mbar_init(&tfree[b], 4);
        }
        for (int b = 0; b < NU; ++b) {
            mbar_init(&full_u[b], 1);   // the gather lane's expect_tx
            mbar_init(&empty_u[b], 1);
        }
        mbar_init(xfull, 1);
        mbar_init(xfree, 1);
        mbar_init(mdrain, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&hsfull[b], 1);
            mbar_init(&hsfree[b], 1);
        }
        *down_done = 0;
        *mask_done = 0;
        *rec_masked = 0;
        *rec_done = 0;
        *pub_items = 0;
        *items_end = 0x7fffffff;
        fence_mbar_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    // everything above overlaps the router's tail (programmatic dependent
    // launch); the routing plan is read only after the router grid is done
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // fused mode: this CTA's copy of the permutation of pairs
    int *s_perm = reinterpret_cast<int *>(smem + L.perm_off);
    int *s_perm_tok = s_perm + a.max_pairs;
    float *s_perm_w = reinterpret_cast<float *>(s_perm_tok + a.max_pairs);
    volatile int *s_ntouched = reinterpret_cast<volatile int *>(smem + L.ctr_off + 56);
    int n_touched, n_routed_items;
    if (fused) {
        route_in_kernel<TR>(a, ring, s_prefix, s_expert, s_off, s_cnt, s_perm, s_perm_tok, s_perm_w, s_ntouched,
                        xfull);   // the token-tile barrier, unused in resident mode
        n_touched = *s_ntouched;
        n_routed_items = n_touched * a.n_blk;
    } else {
        n_touched = plan->n_touched;
        n_routed_items = plan->n_routed_items;
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
    }
    if (resident) {
        // slots by decreasing token count (ties by slot): claimed in this order,
        // the most expensive items go first and the tail is made of cheap ones
        for (int i = tid; i < n_touched; i += blockDim.x) {
            const int c = s_cnt[i];
            int r = 0;
            for (int j = 0; j < n_touched; ++j) {
                const int cj = s_cnt[j];
                r += (cj > c) || (cj == c && j < i);
            }
            s_order[r] = i;
        }
        __syncthreads();
    }
    if (tr && tid == 0) tr[1] = global_ns();
    const PlanCache pc{s_prefix, s_expert, s_off, s_cnt, s_order, n_touched,
                       fused ? s_perm : a.ws.perm, fused ? s_perm_tok : a.ws.perm_tok,
                       fused ? s_perm_w : a.ws.perm_w};

    const int n_items = PM == 2   ? a.n_shared_items * a.n_parts_s + (a.score_shared ? 0 : n_routed_items) * a.n_parts
                        : PM == 1 ? (a.n_shared_items + (a.score_shared ? 0 : n_routed_items)) * a.n_parts
                                  : a.n_shared_items + (a.score_shared ? 0 : n_routed_items);
    // static ranges (token-tile mode): contiguous items per CTA
    const int G = gridDim.x, b = blockIdx.x;
    const int per = n_items / G, rem = n_items % G;
    const int first = b * per + min(b, rem);
    const int n_my = per + (b < rem ? 1 : 0);
    const size_t gate_per_expert = (size_t)a.n_blk * a.n_kb * (kGateTile / 2);   // elements
    const int spi = a.n_kb / 2;   // ring stages per item
    auto gate_src = [&](const ItemPos &p) -> const uint16_t * {
        const uint16_t *base = p.slot < 0 ? a.w.wsg_t + (size_t)(-1 - p.slot) * gate_per_expert
                                          : a.w.wg_t + (size_t)pc.expert[p.slot] * gate_per_expert;
        return base + (size_t)p.blk * a.n_kb * (kGateTile / 2);
    };
    // the id of this CTA's i-th work item (-1: no more), as published by the gate lane
    auto get_item = [&](int i) -> int {
        for (uint32_t spin = 0; *pub_items <= i; ++spin) {
            if (spin > (kSpinLimit >> 4) || (spin > 1024 && *reinterpret_cast<volatile int *>(err) != 0)) {
                atomicCAS(err, 0, 50);
                return -1;
            }
            __nanosleep(64);
        }
        __threadfence_block();
        return s_items[i % kIdRing];
    };

    // The gather: once an item's mask is final, its union-active records into
    // the gather buffers, batch by batch, one bulk copy per record (measured
    // a little faster than 16-byte cp.async copies spread over the warps).
    auto gather_loop = [&]() {
            uint32_t ub = 0, idle = 0;
            int ubi = 0;        // ub % NU and (ub / NU) & 1, kept without a division (NU is not a constant)
            uint32_t uph = 0;
            for (int ui = 0;;) {
                int go = 0;
                if (lane == 0)
                    go = *mask_done > ui ? 1
                                         : (*items_end <= ui || *reinterpret_cast<volatile int *>(err) != 0 ? -1 : 0);
                go = __shfl_sync(kFull, go, 0);
                if (go < 0) break;
                if (go == 0) {
                    if (++idle > kSpinLimit) {
                        if (lane == 0) atomicCAS(err, 0, 35);
                        break;
                    }
                    __nanosleep(128);
                    continue;
                }
                idle = 0;
                __threadfence_block();
                const ItemMeta &M = meta[ui & 1];
                unsigned long long *tg = (tr && ui < 2 && lane == 0) ? tr + 32 + 4 * ui : nullptr;
                if (tg) tg[0] = global_ns();
                int nbatch = 0;
                const int nsub = min(max(M.nsub, 0), kMaxSub);
                const size_t j0 = (size_t)M.blk * kBlk;
                for (int s = 0; s < nsub; ++s) {
                    const int n = min(max(M.n_uni[s], 0), kBlk);
                    for (int b0 = 0; b0 < n; b0 += L.gb, ++ub, ubi = ubi + 1 < NU ? ubi + 1 : 0, uph ^= ubi == 0) {
                        const int nb = min(L.gb, n - b0);
                        const int bi = ubi;
                        mbar_wait(&empty_u[bi], uph ^ 1, err, 36);
                        if (tg && nbatch < 3) tg[1 + nbatch] = global_ns();
                        ++nbatch;
                        uint8_t *dst = ud + (size_t)bi * L.ud_buf_bytes;
                        // one bulk copy of 4d bytes per record (both ends 16-byte aligned)
                        if (lane == 0) {
                            mbar_arrive_expect_tx(&full_u[bi], (uint32_t)(nb * 4 * d));
                            for (int qq = 0; qq < nb; ++qq) {
                                const size_t j = min(j0 + M.uni[s][b0 + qq], (size_t)a.f - 1);
                                bulk_g2s(dst + (size_t)qq * L.gpitch, M.wud + j * 2 * d, (uint32_t)(4 * d), &full_u[bi]);
                            }
                        }
                        __syncwarp();
                    }
                }
                ++ui;
            }
            // the last batch issued into each buffer has landed before the CTA may exit
            if (lane == 0)
                for (uint32_t b = ub > (uint32_t)NU ? ub - NU : 0; b < ub; ++b)
                    mbar_drain(&full_u[b % NU], (b / NU) & 1);
            __syncwarp();
    };

    if (warp == kWarpTma) {
        // ------------------------------------------------------------ gate lane
        // publishes the work-item ids (claimed from the plan's counter in
        // resident mode, else the CTA's static range), then streams each
        // item's gate tiles into the ring
        if (lane == 0 && inject != 1) {
            const uint64_t pol = policy_evict_first();
            uint32_t g = 0;
            int gs = 0;         // g % NS and (g / NS) & 1, kept without a division
            uint32_t gph = 0;
            unsigned long long t_claim = 0, t_ring = 0, t_last = 0;   // trace only
            // resident mode: CTA b's first item is item b (all CTAs start at once,
            // so no counter round trip); later ones come from the counter, past
            // the grid's first items
            int next = resident ? (int)blockIdx.x : 0;
            for (int i = 0;; ++i) {
                int id;
                if (resident) {
                    if (i > 0 && next < n_items) {
                        // item i - 1 masked and the up/down backlog short: claim the
                        // next item (its gate streams while the backlog drains)
                        const unsigned long long tc0 = tr ? global_ns() : 0;
                        bool ok = true;
                        for (uint32_t spin = 0;; ++spin) {
                            if (*mask_done >= i) {
                                __threadfence_block();
                                if (score_mode || *rec_masked - *rec_done <= kClaimBacklog) break;
                            }
                            if (spin > kSpinLimit || (spin > 1024 && *reinterpret_cast<volatile int *>(err) != 0)) {
                                atomicCAS(err, 0, 54);
                                ok = false;
                                break;
                            }
                            __nanosleep(128);
                        }
                        next = ok ? atomicAdd(&plan->next_item, 1) + (int)gridDim.x : n_items;
                        if (tr) t_claim += global_ns() - tc0;
                    }
                    id = next < n_items ? next : -1;
                } else {
                    id = i < n_my ? first + i : -1;
                }
                // ring slot i % kIdRing is free once the consumers have masked item i - kIdRing
                for (uint32_t spin = 0; *mask_done < i - kIdRing + 1; ++spin) {
                    if (spin > (kSpinLimit >> 4) || (spin > 1024 && *reinterpret_cast<volatile int *>(err) != 0)) {
                        atomicCAS(err, 0, 51);
                        id = -1;
                        break;
                    }
                    __nanosleep(128);
                }
                s_items[i % kIdRing] = id;
                __threadfence_block();
                *pub_items = i + 1;
                if (id < 0) break;
                const ItemPos ip = locate_item<DEC>(a, pc, split_item<PM>(a, id));
                const uint16_t *src = gate_src(ip);
                int s_lo, s_hi;
                if (SH && a.rec_split) {   // every record-split part streams the whole gate
                    s_lo = 0;
                    s_hi = spi;
                } else {
                    part_stages(spi, item_parts<PM>(a, split_item<PM>(a, id)), split_part<PM>(a, id), s_lo, s_hi);
                }
                if (a_in && ip.slot >= 0) s_hi = s_lo;   // rank pass: this gate is computed already
                bool ok = true;
                for (int s = s_lo; s < s_hi; ++s, ++g, gs = gs + 1 < NS ? gs + 1 : 0, gph ^= gs == 0) {
                    const int slot = gs;
                    const unsigned long long tr0 = tr ? global_ns() : 0;
                    if (!mbar_wait(&empty_g[slot], gph ^ 1, err, 30)) { ok = false; break; }
                    if (tr) {
                        t_last = global_ns();
                        t_ring += t_last - tr0;
                        if (g < 4) tr[40 + g] = t_last;
                    }
                    uint8_t *stage = ring + (size_t)slot * L.stage_pitch;
                    mbar_arrive_expect_tx(&full_g[slot], kStageBytes + L.xs_bytes);
                    if (fused) {   // the token operand's blocks 2s, 2s+1 straight from x (L2-resident)
                        tma_load_2d(stage + kStageBytes, &a.xmap, 128 * s, 0, &full_g[slot]);
                        tma_load_2d(stage + kStageBytes + L.xt_kb, &a.xmap, 128 * s + 64, 0, &full_g[slot]);
                    } else if (L.xs_bytes) {   // the same, pre-swizzled by the router
                        bulk_g2s(stage + kStageBytes, a.ws.x_tiles + (size_t)s * (L.xs_bytes / 2), L.xs_bytes,
                                 &full_g[slot]);
                    }
                    bulk_g2s_hint(stage, src + (size_t)s * (kStageBytes / 2), kStageBytes,
                                  &full_g[slot], pol);
                }
                if (!ok) {   // publish the end so that every agent stops
                    s_items[(i + 1) % kIdRing] = -1;
                    __threadfence_block();
                    *pub_items = i + 2;
                    break;
                }
            }
            // every copy issued has landed before the CTA may exit
            for (int s = 0; s < NS && (uint32_t)s < g; ++s) mbar_drain(&full_g[s], (((g - s + NS - 1) / NS) - 1) & 1);
            if (tr) {
                tr[32] = t_claim;
                tr[33] = t_ring;
                tr[34] = g;
                tr[35] = t_last;
            }
        }
        __syncwarp();
    } else if (warp == kWarpMma) {
        // ------------------------------------------------------------- MMA lane
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(128, 16);
            uint32_t g = 0;
            int gs = 0;         // g % NS and (g / NS) & 1, kept without a division
            uint32_t gph = 0;
            int q = -1;
            long long prev_key = 0;
            bool ok = true;
            for (int i = 0; ok; ++i) {
                const int id = get_item(i);
                if (id < 0) break;
                const ItemPos p = locate_item<DEC>(a, pc, split_item<PM>(a, id));
                const long long key = item_key(p);
                int s_lo, s_hi;
                if (SH && a.rec_split) {   // every record-split part streams the whole gate
                    s_lo = 0;
                    s_hi = spi;
                } else {
                    part_stages(spi, item_parts<PM>(a, split_item<PM>(a, id)), split_part<PM>(a, id), s_lo, s_hi);
                }
                const bool skip = a_in && p.slot >= 0;   // rank pass: no MMA for a routed item
                if (skip) s_hi = s_lo;
                if (!resident && (i == 0 || key != prev_key)) {
                    ++q;
                    ok = mbar_wait(xfull, q & 1, err, 31);
                }
                const int bsel = i % kAcc;
                ok = ok && mbar_wait(&tfree[bsel], ((i / kAcc) & 1) ^ 1, err, 32);
                tc_fence_after();
                const uint32_t dt = tmem + 16 * bsel;
                for (int s = s_lo; s < s_hi && ok; ++s, ++g, gs = gs + 1 < NS ? gs + 1 : 0, gph ^= gs == 0) {
                    const int slot = gs;
                    ok = mbar_wait(&full_g[slot], gph, err, 33);
                    tc_fence_after();
                    if (tr && i == 0 && s == 0) tr[56] = global_ns();
                    const uint8_t *A = ring + (size_t)slot * L.stage_pitch;
                    const uint8_t *B = L.xs_bytes ? A + kStageBytes : xt + (size_t)(2 * s) * L.xt_kb;
#pragma unroll
                    for (int kb = 0; kb < 2; ++kb)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_bf16(dt, smem_desc_k_sw128(A + kb * kGateTile + 32 * kk),
                                      smem_desc_k_sw128(B + kb * L.xt_kb + 32 * kk), idesc,
                                      ((s - s_lo) | kb | kk) != 0 ? 1u : 0u);
                    umma_commit(&empty_g[slot]);   // the stage is free once these MMAs have read it
                }
                if (skip)
                    mbar_arrive(&gdone[bsel]);
                else
                    umma_commit(&gdone[bsel]);
                if (tr && i == 0) tr[57] = global_ns();
                if (!resident) {   // static ranges: the next id is first + i + 1
                    const bool last_of_tile =
                        i + 1 >= n_my || item_key(locate_item<DEC>(a, pc, first + i + 1)) != key;
                    if (last_of_tile) umma_commit(xfree);
                }
                prev_key = key;
            }
            umma_commit(mdrain);   // all MMAs complete before the accumulator is freed
            mbar_drain(mdrain, 0);
        }
        __syncwarp();
    } else if (warp == kWarpX) {
        // --------------------------------------------------------------- x warp
        // token rows into the MMA's K-major 128-byte-swizzled layout; inputs
        // past d are the zero padding of the gate tiles
        const int nck = a.dp >> 3;   // 16-byte chunks per padded row
        auto load_rows = [&](int m, auto token_of) {
            for (int r = 0; r < m; ++r) {
                const uint16_t *xrow = a.x + (size_t)token_of(r) * d;
                for (int c = lane; c < nck; c += 32) {
                    const bool in = 8 * c < d;
                    cp_async16(xt + (size_t)(c >> 3) * L.xt_kb + r * 128 + (((c & 7) ^ (r & 7)) << 4),
                               in ? (const void *)(xrow + 8 * c) : (const void *)a.x, in ? 16u : 0u);
                }
            }
            cp_async_wait_all();
            fence_proxy_async_smem();
            __syncwarp();
        };
        if (resident) {
            // the token operand streams with the gate stages: nothing to load here
        } else {
            int q = -1;
            long long prev_key = 0;
            for (int i = 0; i < n_my; ++i) {
                const ItemPos p = locate_item<DEC>(a, pc, first + i);
                const long long key = item_key(p);
                if (i > 0 && key == prev_key) continue;
                prev_key = key;
                ++q;
                if (q > 0 && !mbar_wait(xfree, (q - 1) & 1, err, 34)) break;
                int base;
                const int m = tile_tokens(a, pc, p, base);
                load_rows(m, [&](int r) { return tile_token(a, pc, p, base, r); });
                if (lane == 0) {
                    if (tr && q < 4) tr[48 + q] = global_ns();
                    mbar_arrive(xfull);
                }
            }
        }
        cp_async_wait_all();
        __syncwarp();
    } else if (warp == kWarpGather) {
        // ---------------------------------------------------------- gather warp
        if (!score_mode) gather_loop();
        __syncwarp();
    } else if (warp < 4) {
        // ------------------------------------------------ up warps: mask and up
        // M(i): metadata, the gate accumulator (one neuron per thread), silu,
        // threshold, ballot per token, the union per pass of MT tokens; then,
        // batch by batch, the gathered up rows against the pass's tokens (each
        // thread holds its slices of d in registers), one transposed warp
        // reduction per 4 rows, the four warps' partials summed by warp 0 into
        // h = silu(g) u where the bit is set, handed to the down warps
        const int ct = tid;   // 0..127
        const int d8 = d >> 3;
        uint32_t ub = 0;
        int ubi = 0;        // ub % NU and (ub / NU) & 1, kept without a division
        uint32_t uph = 0;
        int n_rec = 0, ii = 0;
        unsigned long long t_wait = 0, t_work = 0;   // trace only
        auto do_mask = [&](int i, int id) {
            ItemMeta &M = meta[i & 1];
            const int item = split_item<PM>(a, id), part = split_part<PM>(a, id);
            const ItemPos p = locate_item<DEC>(a, pc, item);
            int base;
            const int m = tile_tokens(a, pc, p, base);
            if (ct < m) {
                M.tok[ct] = tile_token(a, pc, p, base, ct);
                if (p.slot < 0) {
                    M.pair[ct] = -1;
                    M.w[ct] = 1.f;
                } else {
                    M.pair[ct] = min(max(pc.perm[base + ct], 0), a.T * a.k - 1);
                    M.w[ct] = pc.perm_w[base + ct];
                }
            }
            if (ct == 0) {
                M.key = item_key(p);
                M.m = m;
                M.blk = p.blk;
                M.masked = part > 0 && !SH ? 0 : p.slot < 0 ? (a.use_mask && a.tau_shared > 0.f ? 1 : 0) : a.use_mask;
                M.sidx = p.slot < 0 ? -1 - p.slot : -1;
                M.part = part;
                // a non-owner part has up/down work only when the records are shared
                M.nsub = part > 0 && !SH ? 0 : (m + MT - 1) / MT;
                M.wud = p.slot < 0 ? a.w.wsud + (size_t)(-1 - p.slot) * 2 * a.f * d
                                   : a.w.wud + (size_t)pc.expert[p.slot] * 2 * a.f * d;
            }
            consumer_sync(kUpThreads);
            unsigned long long *ti = (tr && i < 3) ? tr + 2 + 10 * i : nullptr;   // per-item stamps
            if (ti && ct == 0) ti[0] = global_ns();
            // gate split: the item's partial sums, [part - 1][neuron][token]
            const int np = item_parts<PM>(a, item);
            float *gp = np > 1 && !(SH && a.rec_split) ? a.ws.gpart + (size_t)min(item, a.ws.gcnt_n - 1) * (kMaxParts - 1) * kBlk *
                                                          kSplitCols
                                      : nullptr;
            if (gp && part == 0) {   // the owner waits until the other parts have published theirs
                if (ct == 0) {
                    const int *cnt = a.ws.gcnt + min(item, a.ws.gcnt_n - 1);
                    for (uint32_t spin = 0; ld_acquire_gpu(cnt) < np - 1; ++spin) {
                        if (spin > kSpinLimit || (spin > 1024 && *reinterpret_cast<volatile int *>(err) != 0)) {
                            atomicCAS(err, 0, 56);
                            break;
                        }
                        __nanosleep(32);
                    }
                }
                consumer_sync(kUpThreads);
            }
            if (warp < 4) {
                const int bsel = i % kAcc;
                mbar_wait(&gdone[bsel], (i / kAcc) & 1, err, 40);
                tc_fence_after();
                if (ti && ct == 0) ti[1] = global_ns();
                const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16) + 16 * bsel;
                const int jl = warp * 32 + lane;
                const int j = M.blk * kBlk + jl;
                const bool jv = j < a.f;
                const bool masked = M.masked != 0;
                const float th = M.sidx >= 0 ? a.tau_shared : a.tau;
                const bool from_a = a_in && M.sidx < 0;   // rank pass: silu(g) and the cut from global
                // a rolled loop over the tile's tokens: short code, one TMEM
                // column each (the token's own column in resident mode)
#pragma unroll 1
                for (int t = 0; t < m; ++t) {
                    float av;
                    bool keep;
                    if (from_a) {
                        const int pr = M.pair[t];
                        av = jv ? __ldcg(&a_in[(size_t)pr * a.f + j]) : 0.f;
                        const float sv = fabsf(av), cv = __ldcg(&a.rank_v[pr]);
                        keep = sv > cv || (sv == cv && j <= __ldcg(&a.rank_j[pr]));
                    } else {
                        const int col = resident ? M.tok[t] : t;
                        float g = tmem_ld1(taddr + col);
                        if (gp) {
                            const int c = min(col, kSplitCols - 1);
                            if (part > 0) {   // publish this part's sum; no mask
                                gp[((part - 1) * kBlk + jl) * kSplitCols + c] = g;
                                continue;
                            }
                            for (int r = 1; r < np; ++r)
                                g += __ldcg(&gp[((r - 1) * kBlk + jl) * kSplitCols + c]);
                        }
                        av = silu_f(g);
                        keep = fabsf(av) >= th;
                    }
                    const bool on = jv && (!masked || keep);
                    const unsigned word = __ballot_sync(kFull, on);
                    M.a[t][jl] = f2bf_bits(av);
                    if (lane == 0) M.word[t][warp] = word;
                    if (score_mode && jv) {
                        const size_t row = M.sidx >= 0 ? (size_t)M.tok[t] * a.S + M.sidx : (size_t)M.pair[t];
                        a.score_out[row * a.f + j] = a.score_signed ? av : fabsf(av);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tfree[bsel]);   // the MMA may overwrite this accumulator
                if (ti && ct == 0) ti[2] = ti[3] = global_ns();
            }
            if (gp && part > 0) __threadfence();   // this thread's partial sums before the count
            consumer_sync(kUpThreads);
            if (gp && part > 0 && ct == 0) atomicAdd(a.ws.gcnt + min(item, a.ws.gcnt_n - 1), 1);
            // records shared: the owner adds n_parts more to the count once its
            // union list is published (below); another part waits for that and
            // takes its range of the list.  Every part of an item is claimed in
            // the kernel's first round (parts x items <= grid), so the owner is
            // running; its own wait is only for the parts' sums, published above.
            // (only batches of at most kSplitCols tokens split; the wider
            // instantiations carry none of this code)
            SplitShare *gsh = nullptr;
            if constexpr (SH && MT <= kSplitCols)
                if (gp) gsh = a.ws.gshare + min(item, a.ws.gcnt_n - 1);
            if (gsh && part > 0) {
                if (ct == 0) {
                    const int *cnt = a.ws.gcnt + min(item, a.ws.gcnt_n - 1);
                    for (uint32_t spin = 0; ld_acquire_gpu(cnt) < 2 * np - 1; ++spin) {
                        if (spin > kSpinLimit || (spin > 1024 && *reinterpret_cast<volatile int *>(err) != 0)) {
                            atomicCAS(err, 0, 58);
                            break;
                        }
                        __nanosleep(32);
                    }
                }
                consumer_sync(kUpThreads);
                const int n = min(max(__ldcg(&gsh->n), 0), kBlk);
                const int lo = part * n / np, hi = (part + 1) * n / np;
                if (ct < hi - lo) M.uni[0][ct] = __ldcg(&gsh->uni[lo + ct]);
                for (int t = 0; t < min(m, kSplitCols); ++t) M.a[t][ct] = __ldcg(&gsh->a[t][ct]);
                if (ct < min(m, kSplitCols) * 4) M.word[ct >> 2][ct & 3] = __ldcg(&gsh->word[ct >> 2][ct & 3]);
                if (ct == 0) M.n_uni[0] = hi - lo;
            }
            if (ti && ct == 0) ti[4] = global_ns();
            if (warp < M.nsub && !(gsh && part > 0)) {
                // union of the pass's tokens, compacted in ascending neuron order
                const int s = warp, t0 = s * MT, t1 = min(m, t0 + MT);
                int n = 0;
#pragma unroll
                for (int qw = 0; qw < 4; ++qw) {
                    unsigned uw = 0;
                    for (int t = t0; t < t1; ++t) uw |= M.word[t][qw];
                    const bool on = (uw >> lane) & 1u;
                    const unsigned bal = __ballot_sync(kFull, on);
                    if (on) M.uni[s][n + __popc(bal & ((1u << lane) - 1u))] = (uint8_t)(qw * 32 + lane);
                    n += __popc(bal);
                }
                if constexpr (SH) {
                    if (a.rec_split && np > 1) {   // this part's range of the list, moved to its front
                        const int lo = part * n / np, hi = (part + 1) * n / np;
                        __syncwarp();
                        uint8_t v[kBlk / 32];
#pragma unroll
                        for (int c = 0; c < kBlk / 32; ++c)
                            v[c] = lane + 32 * c < hi - lo ? M.uni[s][lo + lane + 32 * c] : 0;
                        __syncwarp();
#pragma unroll
                        for (int c = 0; c < kBlk / 32; ++c)
                            if (lane + 32 * c < hi - lo) M.uni[s][lane + 32 * c] = v[c];
                        n = hi - lo;
                    }
                }
                if (lane == 0) M.n_uni[s] = n;
            }
            consumer_sync(kUpThreads);
            if (gsh && part == 0) {
                // publish the union list and keep the first range, when the list
                // is long enough for the other parts' extra hand-off and gather
                // round trip to pay; else publish an empty list
                const int n = min(max(M.n_uni[0], 0), kBlk);
                const bool sh = n >= kShareMinRecords;
                if (sh) {
                    if (ct < n) gsh->uni[ct] = M.uni[0][ct];
                    for (int t = 0; t < min(m, kSplitCols); ++t) gsh->a[t][ct] = M.a[t][ct];
                    if (ct < min(m, kSplitCols) * 4) gsh->word[ct >> 2][ct & 3] = M.word[ct >> 2][ct & 3];
                    __threadfence();
                    consumer_sync(kUpThreads);
                }
                if (ct == 0) {
                    gsh->n = sh ? n : 0;
                    __threadfence();
                    atomicAdd(a.ws.gcnt + min(item, a.ws.gcnt_n - 1), np);
                    if (sh) M.n_uni[0] = n / np;
                }
                if (sh) consumer_sync(kUpThreads);
            }
            if (ct == 0) {
                if (!score_mode) {
                    int total = 0;
                    for (int s = 0; s < min(M.nsub, kMaxSub); ++s) total += min(max(M.n_uni[s], 0), kBlk);
                    *rec_masked = *rec_masked + total;
                }
                __threadfence_block();
                *mask_done = i + 1;
                if (ti) ti[5] = global_ns();
            }
            // the pairs' mask words for statistics and the debug lists: written
            // after the publication, off the gather's critical path
            if (M.masked && M.sidx < 0 && (!SH || M.part == 0) && ct < m * 4) {   // routed pairs only, by the owner
                const int t = ct >> 2, qw = ct & 3, chunk = M.blk * 4 + qw;
                if (chunk < a.n_chunks) a.ws.mask[(size_t)M.pair[t] * a.n_chunks + chunk] = M.word[t][qw];
            }
        };
        unsigned long long t_item = 0, t_mask = 0;   // trace only
        for (;; ++ii) {
            const unsigned long long ti0 = tr ? global_ns() : 0;
            const int id = get_item(ii);
            if (id < 0) {
                if (ct == 0) *items_end = ii;   // every item of this CTA has been masked
                break;
            }
            // this metadata slot held item ii - 2: the down warps must be done with it
            for (uint32_t spin = 0; !score_mode && ii >= 2 && *down_done < ii - 1; ++spin) {
                if (spin > kSpinLimit || (spin > 1024 && *reinterpret_cast<volatile int *>(err) != 0)) {
                    atomicCAS(err, 0, 53);
                    break;
                }
                __nanosleep(64);
            }
            const unsigned long long ti1 = tr ? global_ns() : 0;
            do_mask(ii, id);
            if (tr) {
                t_item += ti1 - ti0;
                t_mask += global_ns() - ti1;
            }
            if (score_mode) continue;
            const ItemMeta &M = meta[ii & 1];
            const int m = M.m, nsub = min(M.nsub, kMaxSub);
            unsigned long long *tu = (tr && ii < 3) ? tr + 2 + 10 * ii : nullptr;
            for (int s = 0; s < nsub; ++s) {
                const int r0 = s * MT, ms = min(MT, m - r0);
                uint64_t xf[NP][MT][4];
                load_x<MT, NP>(a.x, M.tok + r0, ms, d, ct, xf);   // the pass's token rows (L2-resident)
                const int n_uni = min(max(M.n_uni[s], 0), kBlk);
                n_rec += n_uni;
                for (int b0 = 0; b0 < n_uni; b0 += L.gb, ++ub, ubi = ubi + 1 < NU ? ubi + 1 : 0, uph ^= ubi == 0) {
                    const int nb = min(L.gb, n_uni - b0);
                    const int bi = ubi, hb = (int)(ub & 1);
                    const unsigned long long tw0 = tr ? global_ns() : 0;
                    mbar_wait(&full_u[bi], uph, err, 41);
                    const unsigned long long tw1 = tr ? global_ns() : 0;
                    t_wait += tw1 - tw0;
                    if (tu && ct == 0 && s == 0 && b0 == 0) tu[6] = global_ns();
                    const uint8_t *buf = ud + (size_t)bi * L.ud_buf_bytes;
                    float *pw = part + (size_t)((hb * 4 + warp) * kMaxGB) * MT;
                    // batches of at most two records (d_model >= 4096): rows per reduction
                    // matched to the batch, no empty rows reduced
                    if (NP >= 4 && L.gb <= 2)
                        group_rows<2, MT, NP>(buf, L.gpitch, nb, xf, d8, ct, lane, pw, 0);
                    else
                        for (int g0 = 0; g0 < nb; g0 += kRows)
                            group_rows<kRows, MT, NP>(buf + (size_t)g0 * L.gpitch, L.gpitch, min(kRows, nb - g0), xf,
                                                      d8, ct, lane, pw, g0);
                    consumer_sync(kUpThreads);   // the four warps' partials are in
                    if (warp == 0) {
                        mbar_wait(&hsfree[hb], ((ub >> 1) & 1) ^ 1, err, 44);   // the down warps read this slot out
                        for (int i = lane; i < nb * MT; i += 32) {
                            const int q = i / MT, r = i % MT;
                            float u = 0.f;
#pragma unroll
                            for (int w4 = 0; w4 < 4; ++w4) u += part[((hb * 4 + w4) * kMaxGB + q) * MT + r];
                            const int jl = M.uni[s][b0 + q];
                            const bool bit = (r < ms) && ((M.word[r0 + r][jl >> 5] >> (jl & 31)) & 1u);
                            hs[(hb * kMaxGB + q) * MT + r] = bit ? bf16_f(M.a[r0 + r][jl]) * u : 0.f;
                        }
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&hsfull[hb]);
                    }
                    if (tr) t_work += global_ns() - tw1;
                }
            }
            if (tu && ct == 0) tu[8] = global_ns();
        }
        if (tr && ct == 0) {
            tr[36] = t_mask;
            tr[37] = t_item;
            tr[52] = t_wait;
            tr[53] = t_work;
            tr[61] = (unsigned long long)n_rec;
            tr[63] = (unsigned long long)ii;
        }
    } else if (warp < 8) {
        // ------------------------------------------ down warps: down and flush
        // batch by batch, h x the gathered down rows into per-thread registers
        // (each thread owns NP x 8 outputs for the pass's tokens), kept across
        // consecutive blocks of the same tokens; then into y_acc by fp32
        // vector atomics
        const int ct = tid - kUpThreads;   // 0..127
        const int d8 = d >> 3;
        uint64_t acc_y[NP][4][MT];   // output pairs (8 v + 2i, 8 v + 2i + 1) of each token, packed
#pragma unroll
        for (int p = 0; p < NP; ++p)
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int r = 0; r < MT; ++r) acc_y[p][i][r] = 0ull;
        uint32_t ub = 0;
        int ubi = 0;        // ub % NU, kept without a division
        unsigned long long t_wait = 0, t_work = 0;   // trace only
        for (int ii = 0; !score_mode; ++ii) {
            bool have = false;
            for (uint32_t spin = 0; spin < kSpinLimit; ++spin) {
                if (*mask_done > ii) { have = true; break; }
                if (*items_end <= ii || *reinterpret_cast<volatile int *>(err) != 0) break;
                __nanosleep(64);
            }
            if (!have) break;
            __threadfence_block();
            const ItemMeta &M = meta[ii & 1];
            const int m = M.m, nsub = min(M.nsub, kMaxSub);
            unsigned long long *tu = (tr && ii < 3) ? tr + 2 + 10 * ii : nullptr;
            for (int s = 0; s < nsub; ++s) {
                const int r0 = s * MT, ms = min(MT, m - r0);
                const int n_uni = min(max(M.n_uni[s], 0), kBlk);
                for (int b0 = 0; b0 < n_uni; b0 += L.gb, ++ub, ubi = ubi + 1 < NU ? ubi + 1 : 0) {
                    const int nb = min(L.gb, n_uni - b0);
                    const int bi = ubi, hb = (int)(ub & 1);
                    const unsigned long long tw0 = tr ? global_ns() : 0;
                    mbar_wait(&hsfull[hb], (ub >> 1) & 1, err, 45);
                    const unsigned long long tw1 = tr ? global_ns() : 0;
                    t_wait += tw1 - tw0;
                    if (tu && ct == 0 && s == 0 && b0 == 0) tu[7] = global_ns();
                    const uint8_t *buf = ud + (size_t)bi * L.ud_buf_bytes;
                    const float *hq = hs + (size_t)(hb * kMaxGB) * MT;
#pragma unroll
                    for (int p = 0; p < NP; ++p) {
                        const int v = ct + 128 * p;
                        if (v < d8) {
#pragma unroll
                            for (int q = 0; q < kRows; ++q) {   // nb <= gb <= kRows records
                                if (q >= nb) break;
                                const uint4 wv =
                                    *reinterpret_cast<const uint4 *>(buf + (size_t)q * L.gpitch + 2 * d + 16 * v);
                                const uint64_t w2[4] = {bf16x2_f2(wv.x), bf16x2_f2(wv.y), bf16x2_f2(wv.z),
                                                        bf16x2_f2(wv.w)};
#pragma unroll
                                for (int r = 0; r < MT; ++r) {
                                    const float hv = hq[q * MT + r];
                                    const uint64_t h2 = f2_pack(hv, hv);
#pragma unroll
                                    for (int i = 0; i < 4; ++i) acc_y[p][i][r] = ffma2(w2[i], h2, acc_y[p][i][r]);
                                }
                            }
                        }
                    }
                    group_sync(2, kDownThreads);
                    if (ct == 0) {
                        mbar_arrive(&hsfree[hb]);   // h slot and gather buffer are free again
                        mbar_arrive(&empty_u[bi]);
                        *rec_done = *rec_done + nb;
                    }
                    if (tr) t_work += global_ns() - tw1;
                }
                // keep accumulating while the next item is the next block of the
                // same tokens (looked up only now: in resident mode the next item
                // is claimed once this one's backlog has drained)
                bool cont = false;
                if (nsub == 1 && !a.ws.ypart) {   // (deterministic mode: one row per block)
                    const int nid = get_item(ii + 1);
                    // (a non-owner part has no up/down work: stop accumulating there)
                    cont = nid >= 0 && split_part<PM>(a, nid) == 0 &&
                           item_key(locate_item<DEC>(a, pc, split_item<PM>(a, nid))) == M.key;
                }
                if (!cont) {
#pragma unroll
                    for (int p = 0; p < NP; ++p) {
                        const int v = ct + 128 * p;
#pragma unroll
                        for (int r = 0; r < MT; ++r) {
                            if (v < d8 && r < ms) {
                                const float wt = M.w[r0 + r];
                                float y[8];
#pragma unroll
                                for (int i = 0; i < 4; ++i) f2_unpack(acc_y[p][i][r], y[2 * i], y[2 * i + 1]);
                                const float4 y0 = make_float4(wt * y[0], wt * y[1], wt * y[2], wt * y[3]);
                                const float4 y1 = make_float4(wt * y[4], wt * y[5], wt * y[6], wt * y[7]);
                                if (a.ws.ypart) {
                                    // deterministic mode: this (routing slot, block)'s own row
                                    // [token][k + S][n_blk][d], summed in order by the combine
                                    const int t = M.tok[r0 + r], kS = a.k + a.S;
                                    const int slot = M.sidx >= 0 ? a.k + M.sidx : M.pair[r0 + r] % a.k;
                                    float4 *dst = reinterpret_cast<float4 *>(
                                        a.ws.ypart + (((size_t)t * kS + slot) * a.n_blk + M.blk) * d + v * 8);
                                    __stcg(dst, y0);
                                    __stcg(dst + 1, y1);
                                } else {
                                    float4 *dst = reinterpret_cast<float4 *>(a.ws.y_acc + (size_t)M.tok[r0 + r] * d + v * 8);
                                    atomicAdd(dst, y0);
                                    atomicAdd(dst + 1, y1);
                                }
                            }
#pragma unroll
                            for (int i = 0; i < 4; ++i) acc_y[p][i][r] = 0ull;
                        }
                    }
                }
            }
            group_sync(2, kDownThreads);
            if (ct == 0) {
                __threadfence_block();
                *down_done = ii + 1;   // this item's metadata slot may be reused
                if (tu) tu[9] = global_ns();
            }
        }
        if (tr && ct == 0) {
            tr[54] = t_wait;
            tr[55] = t_work;
        }
    }
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if (tr && tid == 0) tr[62] = global_ns();
    if (a.tail) combine_tail(a, tid, s_tail_flag);
}

// Routing inside the expert kernel needs: the batch as one token tile
// (resident mode), the permutation (T * k pairs) in shared memory, the T x E
// logits in the idle gate ring, and x at least one 64-input box wide.
bool fused_possible(const Dims &dm, int T)
{
    const SparseTiling t = sparse_tiling(T, dm.d, dm.S);
    return T <= t.nt && T * dm.k <= kMaxFusedPairs && T * dm.E <= kMaxFusedLogits && dm.E <= kMaxFusedExperts &&
           dm.d >= 64;
}

SparseTiling sparse_tiling(int T, int d, int n_shared)
{
    SparseTiling t;
    const int np = (d / 8 + 127) / 128;   // 16-byte slices of d per up/down thread
    // passes of two tokens up to 8 tokens when no shared expert holds all of
    // them (a routed item there mostly has one or two; measured 1-2 us
    // faster), else of four (a shared item's every pass reads all its records)
    t.mt = T <= 1 ? 1 : (T <= 2 || (n_shared == 0 && T <= 8)) ? 2 : 4;
    while (t.mt > 1 && t.mt * np > 8) t.mt >>= 1;
    const int dp = (d + 127) & ~127;
    // 16-token tiles when they fit in 64 KB and the batch needs them: a batch
    // of up to 16 tokens is resident as one tile; from 17 to 32 tokens an
    // expert rarely gets more than 8 and the smaller tile leaves room for
    // gather buffers
    const bool fits16 = 16 * 2 * dp <= 64 * 1024 && 16 <= kMaxSub * t.mt;
    t.nt = (fits16 && T > 8 && (T <= 16 || T > 32)) ? 16 : 8;
    return t;
}

static bool make_layout(int d, int dp, SparseTiling til, bool resident, int max_touched, int perm_pairs,
                        SparseLayout &L)
{
    auto up = [](int v) { return (v + 127) & ~127; };
    const int rec = 4 * d;
    L.xt_kb = til.nt * 128;
    // resident mode streams the token operand with the gate stages; tile mode
    // keeps the tile's rows in shared memory
    const int xt_bytes = resident ? 0 : (dp / 64) * L.xt_kb;   // a multiple of 1024
    L.xs_bytes = resident ? 2 * L.xt_kb : 0;
    L.stage_pitch = kStageBytes + L.xs_bytes;                  // a multiple of 1024
    L.gpitch = rec + 16;
    const int meta_bytes = up(2 * (int)sizeof(ItemMeta));
    const int part_bytes = up(2 * 4 * kMaxGB * til.mt * 4);
    const int h_bytes = up(2 * kMaxGB * til.mt * 4);
    const int plan_bytes = up(4 * (5 * max_touched + 1));
    const int perm_bytes = up(12 * perm_pairs);   // fused mode: perm, perm_tok, perm_w
    const int fixed = xt_bytes + meta_bytes + part_bytes + h_bytes + 128 + 128 + plan_bytes + perm_bytes +
                      up((2 * 8 + 2 * kMaxNU + kNumFixedBars) * 8) + 1024 /* base alignment */;
    // gather buffers of up to four records (rows per up reduction), at least
    // two of them; three gate stages when that leaves two buffers, else two
    int gb = 32768 / rec;
    gb = gb < 1 ? 1 : gb > kRows ? kRows : gb;
    int ns = 3;
    if ((kSmemLimit - fixed - ns * L.stage_pitch) / up(gb * L.gpitch) < 2) ns = 2;
    const int room = kSmemLimit - fixed - ns * L.stage_pitch;
    if (room < 2 * up(L.gpitch)) return false;
    while (gb > 1 && room / up(gb * L.gpitch) < 2) --gb;
    L.gb = gb;
    L.ud_buf_bytes = up(gb * L.gpitch);
    int nu = room / L.ud_buf_bytes;
    L.n_ud = nu > kMaxNU ? kMaxNU : nu;
    L.n_stages = ns;
    int off = 0;
    L.xt_off = off; off += xt_bytes;
    L.ring_off = off; off += ns * L.stage_pitch;
    L.ud_off = off; off += L.n_ud * L.ud_buf_bytes;
    L.meta_off = off; off += meta_bytes;
    L.part_off = off; off += part_bytes;
    L.h_off = off; off += h_bytes;
    L.last_off = off; off += 128;
    L.ctr_off = off; off += 128;
    L.plan_off = off; off += plan_bytes;
    L.perm_off = off; off += perm_bytes;
    L.bar_off = off; off += up((2 * ns + 2 * L.n_ud + kNumFixedBars) * 8);
    L.total = off + 1024;   // slack for aligning the base to 1024 bytes
    return L.n_ud >= 2 && L.total <= kSmemLimit;
}

// out = bf16(y_acc) (round to nearest even), then y_acc = 0; launched after
// the expert kernel as its programmatic dependent.  It also ends the forward
// for the next one: the work-item and route counters go back to zero (CUDA
// graph replays included), and the forward's error code is moved into the
// sticky word and its own word cleared, so a later forward is not cut short.
// With n4 = 0 it only does that.
__global__ void __launch_bounds__(256) k_y_out(float *__restrict__ y_acc, uint16_t *__restrict__ out, size_t n4,
                                               int *route_count, int *next_item, int *error_word, int *error_sticky,
                                               int *gcnt, int gcnt_n, float *ypart, int rows, int d)
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; gcnt && i < gcnt_n; i += gridDim.x * blockDim.x) gcnt[i] = 0;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        *route_count = 0;
        *next_item = 0;
        const int e0 = *error_word;
        if (e0 != 0) {
            atomicCAS(error_sticky, 0, e0);
            *error_word = 0;
        }
    }
    if (ypart)   // deterministic mode: the rows of every token, summed in order
        det_combine(ypart, rows, d, out, (long long)n4, ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5,
                    ((long long)gridDim.x * blockDim.x) >> 5, threadIdx.x & 31);
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; !ypart && i < n4;
         i += (size_t)gridDim.x * blockDim.x) {
        const float4 v = __ldcg(reinterpret_cast<const float4 *>(y_acc) + i);
        uint2 p;
        p.x = (uint32_t)f2bf_bits(v.x) | ((uint32_t)f2bf_bits(v.y) << 16);
        p.y = (uint32_t)f2bf_bits(v.z) | ((uint32_t)f2bf_bits(v.w) << 16);
        reinterpret_cast<uint2 *>(out)[i] = p;
        __stcg(reinterpret_cast<float4 *>(y_acc) + i, make_float4(0.f, 0.f, 0.f, 0.f));
    }
}

static cudaError_t launch_y_out(float *y_acc, uint16_t *out, size_t n4, int n_sm, const Workspace &ws, int rows,
                                int d, cudaStream_t st)
{
    // deterministic mode: 8 threads per four outputs
    const size_t threads = ws.ypart ? n4 * 8 : n4;
    size_t blocks = (threads + 255) / 256;
    if (blocks > (size_t)n_sm * (ws.ypart ? 8 : 4)) blocks = (size_t)n_sm * (ws.ypart ? 8 : 4);
    if (blocks < 1) blocks = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, k_y_out, y_acc, out, n4, ws.route_count, &ws.plan->next_item,
                                       ws.error_word, ws.error_sticky, ws.gcnt, ws.gcnt_n, ws.ypart, rows, d);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int MT, int NP, bool TR, bool SH, bool DEC, bool FU>
static cudaError_t launch_mt_tr(const SparseArgs &a, int grid, cudaStream_t st)
{
    auto kern = k_expert_sparse<MT, NP, TR, SH, DEC, FU>;
    static int smem_set[kMaxDevices] = {};
    cudaError_t e = ensure_dynamic_smem(kern, a.L.total, smem_set);
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

template <int MT, int NP>
static cudaError_t launch_mt(const SparseArgs &a, int grid, cudaStream_t st)
{
    if (a.ws.trace_expert) return launch_mt_tr<MT, NP, true, false, false, false>(a, grid, st);
    if (a.resident && !a.a_in && !a.inject && !a.score_out) {
        if (a.fused)
            return a.share_records ? launch_mt_tr<MT, NP, false, true, true, true>(a, grid, st)
                                   : launch_mt_tr<MT, NP, false, false, true, true>(a, grid, st);
        return a.share_records ? launch_mt_tr<MT, NP, false, true, true, false>(a, grid, st)
                               : launch_mt_tr<MT, NP, false, false, true, false>(a, grid, st);
    }
    return launch_mt_tr<MT, NP, false, false, false, false>(a, grid, st);
}

cudaError_t launch_expert_sparse(const Dims &dm, const DeviceWeights &w, const Workspace &ws,
                                 const uint16_t *x, int T, float tau, bool use_mask,
                                 uint16_t *out, SparseTiling til, int grid_cap, cudaStream_t st,
                                 float *score_out, int inject, bool fused, float tau_shared, bool score_shared,
                                 const RankPass *rank, bool combine_here)
{
    if (rank && !rank->second) score_out = rank->a;   // first pass: signed silu(g) of the routed pairs
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
    a.dp = dm.dp;
    a.n_kb = dm.n_kb;
    a.n_blk = dm.n_blk;
    a.n_chunks = dm.f / kChunk;
    a.nt = til.nt;
    a.resident = T <= til.nt ? 1 : 0;
    a.tau = tau;
    a.tau_shared = tau_shared;
    a.score_shared = (score_out && score_shared) ? 1 : 0;
    a.use_mask = use_mask ? 1 : 0;
    a.score_out = score_out;
    a.inject = inject;
    a.score_signed = (rank && !rank->second) ? 1 : 0;
    a.a_in = (rank && rank->second) ? rank->a : nullptr;
    a.rank_v = a.a_in ? rank->v : nullptr;
    a.rank_j = a.a_in ? rank->j : nullptr;
    // the rank passes use the router's plan (the second pass must see the first one's pairs)
    a.fused = (fused && !score_out && !rank && fused_possible(dm, T)) ? 1 : 0;
    a.wr = w.wr;
    a.E = dm.E;
    a.max_pairs = a.fused ? T * dm.k : 0;
    if (a.fused && !encode(&a.xmap, x, dm.d, T, 2ull * dm.d, til.nt, true)) return cudaErrorInvalidValue;
    a.n_tok_tiles = (T + til.nt - 1) / til.nt;
    a.n_shared_items = (score_out && !a.score_shared) ? 0 : dm.S * a.n_tok_tiles * dm.n_blk;
    const int pairs = T * dm.k;
    a.max_touched = pairs < dm.E ? pairs : dm.E;
    if (!make_layout(dm.d, dm.dp, til, a.resident != 0, a.max_touched, a.max_pairs, a.L)) return cudaErrorInvalidValue;
    const int np = (dm.d / 8 + 127) / 128;
    // gate split: one- and two-token batches whose items are fewer than the SMs
    // stream each item's gate on 2 or 4 CTAs (MOE_SPLIT=0 turns it off)
    a.n_parts = a.n_parts_s = 1;
    // the shared experts' items are the heavy ones when no threshold applies
    // to them (every neuron of a block active: 128 records each)
    // (only the decode kernel has the per-class part counts and the sharing)
    const bool dense_shared = a.n_shared_items > 0 && (!use_mask || tau_shared <= 0.f) && !ws.trace_expert && !inject;
    const long long routed_max = (long long)a.max_touched * dm.n_blk;
    {
        const char *sp = std::getenv("MOE_SPLIT");
        const long long base_max = a.n_shared_items + routed_max;
        if (a.resident && !score_out && !a.a_in && T <= kSplitCols && ws.gpart && ws.gcnt && base_max <= ws.gcnt_n &&
            !(sp && std::strcmp(sp, "0") == 0)) {
            for (int r = kMaxParts; r >= 2; r >>= 1)
                if (base_max * r <= grid_cap && dm.n_kb / 2 >= r) {
                    a.n_parts = a.n_parts_s = r;
                    break;
                }
            // then more parts for heavy shared items where the grid has room
            // (the record-sharing kernel, below, is the one that maps per-class
            // part counts)
            if (dense_shared && til.mt >= T && !ws.ypart && ws.gshare)
                for (int r = kMaxParts; r > a.n_parts_s; r >>= 1)
                    if (a.n_shared_items * r + routed_max * a.n_parts <= grid_cap && dm.n_kb / 2 >= r) {
                        a.n_parts_s = r;
                        break;
                    }
        }
    }
    // the parts also share the item's records where every item is one pass
    // (nsub = 1), the combine takes any number of writers per row, and some
    // items have long union lists (the dense shared experts')
    a.share_records = ((a.n_parts > 1 || a.n_parts_s > 1) && til.mt >= T && !ws.ypart && ws.gshare && dense_shared)
                          ? 1
                          : 0;
    // no gate split: a dense shared item (128 records per pass, the slowest
    // item of the batch) is split by records instead, each part streaming
    // the whole gate (its extra gate traffic buys a shorter critical path)
    // (4 parts where every claim still has an SM of its own, else 2: beyond
    // the grid the extra gate streams compete with the other items)
    a.rec_split = 0;
    if (a.n_parts == 1 && a.n_parts_s == 1 && dense_shared && a.resident && !score_out && !a.a_in && !ws.ypart) {
        a.rec_split = 1;
        a.n_parts_s = (long long)a.n_shared_items * kRecSplitMax + routed_max <= grid_cap ? kRecSplitMax : 2;
        a.share_records = 1;
    }
    const long long bound = (long long)a.n_shared_items * a.n_parts_s +
                            (long long)(a.max_touched + pairs / til.nt) * dm.n_blk * a.n_parts;
    int grid = bound < grid_cap ? (int)bound : grid_cap;
    // the combine at the end of this kernel (one launch per forward), else a
    // separate conversion kernel
    a.tail = combine_here ? 1 : 0;
    a.n_out4 = score_out ? 0 : (long long)T * dm.d / 4;
    if (grid < 1) grid = 1;
    cudaError_t e;
    switch (np * 8 + til.mt) {
    case 8 + 1: e = launch_mt<1, 1>(a, grid, st); break;
    case 8 + 2: e = launch_mt<2, 1>(a, grid, st); break;
    case 8 + 4: e = launch_mt<4, 1>(a, grid, st); break;
    case 16 + 1: e = launch_mt<1, 2>(a, grid, st); break;
    case 16 + 2: e = launch_mt<2, 2>(a, grid, st); break;
    case 16 + 4: e = launch_mt<4, 2>(a, grid, st); break;
    case 32 + 1: e = launch_mt<1, 4>(a, grid, st); break;
    case 32 + 2: e = launch_mt<2, 4>(a, grid, st); break;
    default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    if (a.tail) return cudaSuccess;
    // score mode writes no output: only the counters are reset
    return launch_y_out(ws.y_acc, out, score_out ? 0 : (size_t)T * dm.d / 4, grid_cap, ws, (dm.k + dm.S) * dm.n_blk,
                        dm.d, st);
}

}  // namespace moe
