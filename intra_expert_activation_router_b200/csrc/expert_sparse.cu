// expert_sparse.cu -- fused gate projection, threshold mask, compaction and
// gathered up/down projection for the routed experts (and the dense shared
// experts), on CUDA cores.
//
// "Uncovering Intra-expert Activation Sparsity for Efficient Mixture-of-Expert
// Model Execution" (technical summary, Methodology item 3):
//   - gate projection, dense ("Gate projection" bullet): g = x Wg[e] for every
//     neuron of the selected expert;
//   - activation mask in one O(n) pass, no sort ("Activation masking"):
//     active iff |silu(g)| >= tau -- here a warp ballot over 32 neurons;
//   - fused up-down projection over the active neurons only ("Fused up-down
//     projection"; Hindi summary "The skip": inactive neurons' weights are
//     never loaded): the active rows of Wu and Wd are gathered, h =
//     silu(g) * (x Wu[:,j]) and y += w * h Wd[j][:].
//   - shared experts: the same kernel with the mask off and weight 1 (the
//     shared expert's execution is unchanged and always dense).
//
// Work decomposition.  A work item is (expert, chunk of 32 neurons, tile of
// up to MT of that expert's tokens).  Items of one expert are adjacent, and
// the token tiles of one chunk are adjacent, so the gate rows a tile re-reads
// are still in L2.  The CTA:
//   1. streams the chunk's 32 gate rows (32 x d bf16, contiguous in the
//      neuron-major repack) once and dots them with its tokens; 8 warps x 4
//      rows, fp32 accumulation, one transposed warp reduction;
//   2. evaluates silu and the threshold per (token, neuron), ballots a 32-bit
//      mask word per token (written out as the pair's mask) and compacts the
//      union of its tokens' words into an ascending index list in shared
//      memory;
//   3. gathers the union rows of Wu (one warp per row, 4 rows per warp) and
//      computes h for each token with that token's own mask bit;
//   4. gathers the same rows of Wd (each thread owns 8 output dims, so every
//      row is read with fully coalesced 16-byte loads) and accumulates
//      sum_j h_j Wd[j][:] in registers;
//   5. adds w * partial into the fp32 accumulator y_acc[token] with vector
//      atomics (red.global.add.v4.f32 at L2) and takes a per-token ticket;
//      the last of the (k + S) * (f/32) contributions of a token converts its
//      row to bf16, writes `out`, and re-zeroes the row and the ticket.
#include "common.cuh"
#include "internal.h"

namespace moe {

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
    int n_shared_items;   // S * n_chunks * n_tok_tiles
    int target;           // contributions per token: (k + S) * n_chunks
    float *score_out;     // score mode: write |silu(g)| [pair][f] and stop after the mask
};

template <int MT>
struct SparseSmem {
    float a[kChunk][MT];     // gate pre-activation, then silu(g)
    float h[kChunk][MT];     // h of the union rows (0 where a token's bit is off)
    unsigned word[MT];       // mask word per token
    int tok[MT];
    int pair[MT];
    float w[MT];
    int last[MT];
    int uni[kChunk];         // union-active neuron offsets in the chunk, ascending
    int m;                   // tokens in this item
    int chunk;
    int masked;
    const uint16_t *wg, *wu, *wd;   // expert bases
};

// acc[q*MT + r] += sum_i rows[q][i] * x[tok[r]][i] for the warp's 4 rows.
template <int MT>
__device__ __forceinline__ void dot_rows4(const uint16_t *const (&rows)[4], const bool (&valid)[4],
                                          const uint16_t *x, const int *tok, int m, int d,
                                          int lane, float (&acc)[4 * MT])
{
#pragma unroll
    for (int i = 0; i < 4 * MT; ++i) acc[i] = 0.f;
#pragma unroll 2
    for (int i = lane * 8; i < d; i += 256) {
        uint4 wv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            wv[q] = valid[q] ? ld_stream(rows[q] + i) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int r = 0; r < MT; ++r) {
            if (r < m) {
                const uint4 xv = ld_cached(x + (size_t)tok[r] * d + i);
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[q * MT + r] = dot8(wv[q], xv, acc[q * MT + r]);
            }
        }
    }
}

template <int MT>
__global__ void __launch_bounds__(256, 2) k_expert_sparse(SparseArgs a)
{
    __shared__ SparseSmem<MT> sm;
    constexpr int NV = 4 * MT;                 // values per warp reduction
    constexpr int SH = 5 - Log2<NV>::value;    // lane >> SH = value index
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const Plan *plan = a.ws.plan;
    const int n_items = a.n_shared_items + plan->n_routed_items;
    const size_t fd = (size_t)a.f * a.d;

    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        __syncthreads();   // smem of the previous item is free
        if (tid == 0) {
            int m, tile_base, chunk;
            if (item < a.n_shared_items) {
                const int per = a.n_chunks * a.n_tok_tiles;
                const int s = item / per, rem = item % per;
                chunk = rem / a.n_tok_tiles;
                const int tile = rem % a.n_tok_tiles;
                tile_base = tile * MT;
                m = min(MT, a.T - tile_base);
                sm.wg = a.w.wsg_n + s * fd;
                sm.wu = a.w.wsu_n + s * fd;
                sm.wd = a.w.wsd + s * fd;
                sm.masked = 0;
                for (int r = 0; r < m; ++r) {
                    sm.tok[r] = tile_base + r;
                    sm.pair[r] = -1;
                    sm.w[r] = 1.f;
                }
            } else {
                const int ir = item - a.n_shared_items;
                int lo = 0, hi = plan->n_touched - 1;   // last slot with item_prefix <= ir
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (plan->item_prefix[mid] <= ir) lo = mid; else hi = mid - 1;
                }
                const int e = plan->touched[lo];
                const int off = plan->offsets[e], cnt = plan->offsets[e + 1] - off;
                const int tiles = (cnt + MT - 1) / MT;
                const int local = ir - plan->item_prefix[lo];
                chunk = local / tiles;
                tile_base = (local % tiles) * MT;
                m = min(MT, cnt - tile_base);
                sm.wg = a.w.wg_n + e * fd;
                sm.wu = a.w.wu_n + e * fd;
                sm.wd = a.w.wd + e * fd;
                sm.masked = a.use_mask;
                for (int r = 0; r < m; ++r) {
                    const int p = a.ws.perm[off + tile_base + r];
                    sm.pair[r] = p;
                    sm.tok[r] = p / a.k;
                    sm.w[r] = a.ws.topk_w[p];
                }
            }
            sm.m = m;
            sm.chunk = chunk;
        }
        __syncthreads();
        const int m = sm.m, chunk = sm.chunk, masked = sm.masked;
        const int j0 = chunk * kChunk;

        // 1. gate rows of the chunk
        {
            const uint16_t *rows[4];
            bool valid[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                rows[q] = sm.wg + (size_t)(j0 + warp * 4 + q) * a.d;
                valid[q] = true;
            }
            float acc[NV];
            dot_rows4<MT>(rows, valid, a.x, sm.tok, m, a.d, lane, acc);
            const float g = transpose_reduce<NV>(acc, lane);
            const int vi = lane >> SH, q = vi / MT, r = vi % MT;
            if ((lane & ((1 << SH) - 1)) == 0) sm.a[warp * 4 + q][r] = g;
        }
        __syncthreads();

        // 2. silu, threshold, ballot, union compaction
        for (int r = warp; r < MT; r += 8) {
            const float av = silu_f(sm.a[lane][r]);
            const bool on = (r < m) && (!masked || fabsf(av) >= a.tau);
            const unsigned word = __ballot_sync(kFull, on);
            sm.a[lane][r] = av;
            if (lane == 0) {
                sm.word[r] = word;
                if (masked && r < m)
                    a.ws.mask[(size_t)sm.pair[r] * a.n_chunks + chunk] = word;
            }
            if (a.score_out && r < m && sm.pair[r] >= 0)
                a.score_out[(size_t)sm.pair[r] * a.f + j0 + lane] = fabsf(av);
        }
        __syncthreads();
        if (a.score_out) continue;   // score mode: no up/down, no accumulation
        unsigned uw = 0;
        for (int r = 0; r < m; ++r) uw |= sm.word[r];
        const int n_uni = __popc(uw);
        if (warp == 0 && ((uw >> lane) & 1u)) sm.uni[__popc(uw & ((1u << lane) - 1u))] = lane;
        __syncthreads();

        // 3. gathered up rows -> h
        if (warp < n_uni) {
            const uint16_t *rows[4];
            bool valid[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int pos = warp + 8 * q;
                valid[q] = pos < n_uni;
                rows[q] = sm.wu + (size_t)(j0 + (valid[q] ? sm.uni[pos] : 0)) * a.d;
            }
            float acc[NV];
            dot_rows4<MT>(rows, valid, a.x, sm.tok, m, a.d, lane, acc);
            const float u = transpose_reduce<NV>(acc, lane);
            const int vi = lane >> SH, q = vi / MT, r = vi % MT;
            const int pos = warp + 8 * q;
            if ((lane & ((1 << SH) - 1)) == 0 && pos < n_uni) {
                const int jl = sm.uni[pos];
                const bool bit = (r < m) && ((sm.word[r] >> jl) & 1u);
                sm.h[pos][r] = bit ? sm.a[jl][r] * u : 0.f;
            }
        }
        __syncthreads();

        // 4 + 5. gathered down rows, weighted accumulation (tokens in groups of
        // RG so the accumulators stay in registers)
        if (n_uni > 0) {
            constexpr int RG = MT < 4 ? MT : 4;
            for (int b = tid * 8; b < a.d; b += 256 * 8) {
                for (int r0 = 0; r0 < m; r0 += RG) {
                    float acc[8][RG];
#pragma unroll
                    for (int q = 0; q < 8; ++q)
#pragma unroll
                        for (int r = 0; r < RG; ++r) acc[q][r] = 0.f;
#pragma unroll 4
                    for (int pos = 0; pos < n_uni; ++pos) {
                        float wf[8];
                        unpack8(ld_stream(sm.wd + (size_t)(j0 + sm.uni[pos]) * a.d + b), wf);
#pragma unroll
                        for (int r = 0; r < RG; ++r) {
                            const float hv = sm.h[pos][r0 + r];
#pragma unroll
                            for (int q = 0; q < 8; ++q) acc[q][r] = fmaf(hv, wf[q], acc[q][r]);
                        }
                    }
#pragma unroll
                    for (int r = 0; r < RG; ++r) {
                        const int rr = r0 + r;
                        if (rr < m && sm.word[rr] != 0u) {
                            const float wt = sm.w[rr];
                            float4 *dst = reinterpret_cast<float4 *>(a.ws.y_acc + (size_t)sm.tok[rr] * a.d + b);
                            atomicAdd(dst, make_float4(wt * acc[0][r], wt * acc[1][r], wt * acc[2][r], wt * acc[3][r]));
                            atomicAdd(dst + 1, make_float4(wt * acc[4][r], wt * acc[5][r], wt * acc[6][r], wt * acc[7][r]));
                        }
                    }
                }
            }
        }

        // per-token tickets; the last contributor finishes the token
        __threadfence();
        __syncthreads();
        if (tid < m) {
            const int old = atomicAdd(&a.ws.tok_cnt[sm.tok[tid]], 1);
            sm.last[tid] = (old == a.target - 1);
        }
        __syncthreads();
        for (int r = 0; r < m; ++r) {
            if (!sm.last[r]) continue;
            __threadfence();
            const int t = sm.tok[r];
            float *yrow = a.ws.y_acc + (size_t)t * a.d;
            uint16_t *orow = a.out + (size_t)t * a.d;
            for (int i = tid * 4; i < a.d; i += 256 * 4) {
                const float4 v = __ldcg(reinterpret_cast<const float4 *>(yrow + i));
                uint2 packed;
                packed.x = (uint32_t)f2bf_bits(v.x) | ((uint32_t)f2bf_bits(v.y) << 16);
                packed.y = (uint32_t)f2bf_bits(v.z) | ((uint32_t)f2bf_bits(v.w) << 16);
                *reinterpret_cast<uint2 *>(orow + i) = packed;
                __stcg(reinterpret_cast<float4 *>(yrow + i), make_float4(0.f, 0.f, 0.f, 0.f));
            }
            if (tid == 0) a.ws.tok_cnt[t] = 0;
        }
    }
}

int sparse_tile_tokens(int T)
{
    return T <= 1 ? 1 : T <= 2 ? 2 : T <= 4 ? 4 : 8;
}

template <int MT>
static cudaError_t launch_mt(const SparseArgs &a, int bound, int grid_cap, cudaStream_t st)
{
    int grid = bound < grid_cap ? bound : grid_cap;
    if (grid < 1) grid = 1;
    k_expert_sparse<MT><<<grid, 256, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_expert_sparse(const Dims &dm, const DeviceWeights &w, const Workspace &ws,
                                 const uint16_t *x, int T, float tau, bool use_mask,
                                 uint16_t *out, int mt, int grid_cap, cudaStream_t st,
                                 float *score_out)
{
    SparseArgs a;
    a.score_out = score_out;
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
    a.n_chunks = dm.f / kChunk;
    a.n_tok_tiles = (T + mt - 1) / mt;
    a.n_shared_items = score_out ? 0 : dm.S * a.n_chunks * a.n_tok_tiles;
    a.target = (dm.k + dm.S) * a.n_chunks;
    const int pairs = T * dm.k;
    const int touched_max = pairs < dm.E ? pairs : dm.E;
    const int bound = a.n_shared_items + (touched_max + pairs / mt) * a.n_chunks;
    switch (mt) {
    case 1: return launch_mt<1>(a, bound, grid_cap, st);
    case 2: return launch_mt<2>(a, bound, grid_cap, st);
    case 4: return launch_mt<4>(a, bound, grid_cap, st);
    default: return launch_mt<8>(a, bound, grid_cap, st);
    }
}

}  // namespace moe

namespace moe {

template <int MT>
static int occupancy()
{
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_expert_sparse<MT>, 256, 0) != cudaSuccess) {
        cudaGetLastError();
        n = 1;
    }
    return n > 0 ? n : 1;
}

int sparse_blocks_per_sm(int mt)
{
    switch (mt) {
    case 1: return occupancy<1>();
    case 2: return occupancy<2>();
    case 4: return occupancy<4>();
    default: return occupancy<8>();
    }
}

}  // namespace moe
