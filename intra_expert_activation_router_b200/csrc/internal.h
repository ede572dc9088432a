// internal.h -- data shared by the host library and the kernel launchers.
//
// Everything lives in device memory owned by the handle.  Layouts:
//   repacked weights:
//     wg_t   [E][fp/128][dp/64][128][64]  the gate weights as tensor-core tiles:
//                        one 16 KB tile per (128 neurons, 64 inputs), row j of a
//                        tile = neuron, 128 bytes of inputs with the 16-byte
//                        blocks permuted b -> b ^ (j & 7) (the 128-byte swizzle
//                        of the MMA's K-major shared-memory layout); dp, fp =
//                        d and f rounded up to multiples of 128, padding zero.
//                        A 128-neuron block is contiguous over all its inputs.
//     wud    [E][f][2d]  row j = [up column j | down row j]: one neuron's up and
//                        down weights in a single contiguous 4d-byte record
//     wsg_t, wsud        the same for the shared experts
//     wr     [E][d]
//     wdt    [E][d][f]   dense branch only: down weights transposed (K-major)
//   per-call workspace, sized for max_tokens:
//     logits [T][E] fp32, topk_idx/topk_w [T][k], perm [T*k] (pair ids
//     t*k+rank sorted by expert, stable), mask [T*k][f/32] uint32 (bit j of
//     pair p = neuron j active), y_acc [T][d] fp32 (kept all-zero between
//     calls), tok_cnt [T] (kept zero between calls), plan (below).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

constexpr int kMaxExperts = 1024;
constexpr int kChunk = 32;           // neurons per mask word
constexpr int kBlk = 128;            // neurons per sparse work item (the gate MMA's M)
constexpr int kDenseTileM = 128;     // tokens per dense GEMM tile
constexpr int kSplitCols = 2;        // gate split: batches of at most this many tokens
constexpr int kMaxParts = 4;         // gate split: parts per item

// Gate split, records shared: the owner part's union list and mask of an
// item (kBlk = 128 neurons, at most kSplitCols tokens), published for the
// other parts, which project their own share of the records.
struct SplitShare {
    int n;                                 // union-active neurons of the block
    int pad[3];
    uint8_t uni[128];                      // their positions in the block, ascending
    uint32_t word[kSplitCols][4];          // per token: its active neurons, 32 per word
    uint16_t a[kSplitCols][128];           // per token: silu(g) as bf16
};

// Routing plan written by the router's last CTA.
struct Plan {
    int n_touched;                    // distinct experts selected
    int n_routed_items;               // sparse work items over routed experts
    int n_dense_tiles;                // 128-token tiles over touched experts
    int next_item;                    // sparse work-item counter (dynamic scheduling), reset here
    int touched[kMaxExperts];         // slot -> expert id (ascending)
    int offsets[kMaxExperts + 1];     // expert -> first position in perm
    int item_prefix[kMaxExperts + 1]; // slot -> first sparse work item
    int tile_prefix[kMaxExperts + 1]; // slot -> first dense tile
};

struct Dims {
    int E, k, d, f, S;
    int max_tokens;
    int dp, fp;        // d and f rounded up to multiples of 128 (gate tile padding)
    int n_kb, n_blk;   // dp / 64 input blocks, fp / 128 neuron blocks
};

struct DeviceWeights {
    const uint16_t *wr;
    const uint16_t *wg_t, *wud;
    const uint16_t *wsg_t, *wsud;
    const uint16_t *wdt, *wsdt;   // dense branch only: down weights transposed, [E][d][f] / [S][d][f]
};

// Tensor maps of one dense GEMM launch (kernel parameters).
struct DenseMaps {
    CUtensorMap a;    // GEMM1: x_perm rows; GEMM2: H rows (128-byte swizzle, box 64 x 128)
    CUtensorMap b0;   // GEMM1: unused (gate tiles are plain bulk copies); GEMM2: WdT rows (box 64 x 256)
    CUtensorMap b1;   // GEMM1: up halves of the [up | down] records; GEMM2: unused
};

struct DenseState {
    bool ok;                           // shape supported and maps encoded
    DenseMaps g1r, g1s, g2r, g2s;      // GEMM1/GEMM2, routed/shared
    const uint16_t *gate_r, *gate_s;   // gate tiles, routed / shared experts
    CUtensorMap router_b;              // the router rows Wr [E][d] (box 64 x 256) for the logits GEMM
};

// Element offset of gate weight (neuron j, input k) inside one expert's tiles.
__host__ __device__ __forceinline__ size_t gate_tile_off(int j, int k, int n_kb)
{
    const size_t tile = (size_t)(j >> 7) * n_kb + (k >> 6);
    return tile * 8192 + (size_t)(j & 127) * 64 + ((((k & 63) >> 3) ^ (j & 7)) << 3) + (k & 7);
}

// Token tiling of the sparse branch for a batch of T tokens:
//   nt  tokens per gate tile (8 or 16 of the gate MMA's 16 columns carry tokens)
//   mt  tokens per up/down pass (held in registers; nt / mt <= 4)
struct SparseTiling {
    int nt, mt;
};
SparseTiling sparse_tiling(int T, int d, int n_shared);

struct Workspace {
    float *logits;
    int *topk_idx;
    float *topk_w;
    int *perm;
    int *perm_tok;      // [T*k] token of perm[i]
    float *perm_w;      // [T*k] routing weight of perm[i]
    uint32_t *mask;
    float *y_acc;
    // deterministic combine (moe_set_deterministic), null when off: one fp32
    // row of d per (token, routing slot or shared expert, neuron block) --
    // [T][k + S][n_blk][d] on the sparse path, [T][k + S][d] on the dense one
    // -- each written once with plain stores, summed in a fixed order by the
    // conversion and re-zeroed there (all-zero between calls)
    float *ypart;
    int *tok_cnt;
    int *tile_ticket;   // one per router token tile, kept zero between calls
    int *done_ticket;   // one, kept zero between calls
    // device errors (a bounded wait that ran out, ...): kernels of a forward
    // record their first code in error_word, which the router -- the first
    // kernel of every forward, running after all earlier kernels -- folds
    // into error_sticky and clears, so one forward's error never cuts short a
    // later forward; error_sticky keeps the first code until moe_query_stats
    // reads and clears it
    int *error_word;
    int *error_sticky;
    // the fused decode path's count of experts whose logits are written; like
    // the plan's work-item counter it is zero when a forward starts (the
    // conversion kernel that ends every forward resets both)
    int *route_count;
    // the sparse kernel's combine: [0] CTAs whose down flushes have landed,
    // [1] CTAs done converting; the last CTA out resets both (and the
    // counters above), so they are zero when a forward starts
    int *tail;
    int *cursor;        // [kMaxExperts] per-expert slots of the large-batch scatter
    int *ecount;        // [kMaxExperts] pairs per expert, counted by the router's token tiles
                        // (zeroed again by the plan builder, so zero between calls)
    // gate split over several CTAs (batches of one or two tokens): partial gate
    // sums of an item's non-owner parts [item][part - 1][128 neurons][2 tokens]
    // and per item the count of parts published (zeroed by the conversion
    // kernel that ends every forward); null when the layer's shape does not
    // allow the split
    float *gpart;
    int *gcnt;
    int gcnt_n;
    SplitShare *gshare;   // [item]: the owner's union list, when the parts share the records
    Plan *plan;
    // dense path
    uint16_t *x_perm;   // [T*k + T][d] bf16: tokens in perm order, then x for the shared experts
    // batches of T <= nt <= 16 tokens: x as the gate MMA's token operand,
    // [dp/64][nt][64] bf16 with the 16-byte blocks of row t permuted
    // b -> b ^ (t & 7) (128-byte swizzle), rows t >= T and inputs past d zero;
    // written by the router, streamed by the sparse kernel with the gate tiles
    uint16_t *x_tiles;
    uint16_t *h_perm;   // [T*k + S*T][f] bf16: masked SwiGLU activations, routed then shared
    // host-pointer entry
    uint16_t *x_stage, *out_stage;
    // optional phase timestamps (moe_set_trace); nullptr when off
    unsigned long long *trace_router;   // [router CTAs][8]
    unsigned long long *trace_expert;   // [expert CTAs][64]
    int trace_router_ctas, trace_expert_ctas;
};

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per kernel and device
// rather than on every launch: `done` is a per-kernel array of the largest
// size set so far on each device (the caller keeps one array per kernel).
constexpr int kMaxDevices = 64;
template <typename Kern>
inline cudaError_t ensure_dynamic_smem(Kern kern, int bytes, int (&done)[kMaxDevices])
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (__atomic_load_n(&done[dev], __ATOMIC_ACQUIRE) >= bytes) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) __atomic_store_n(&done[dev], bytes, __ATOMIC_RELEASE);
    return e;
}

__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Launchers (return cudaGetLastError()).
// Routing plan with sparse work items of (expert, tile of `tile_tokens`
// tokens, 128-neuron block).
// cap >= 0: capacity-aware token drop, each expert keeps at most cap pairs
// (batches of up to 4096 pairs; cudaErrorNotSupported above).
cudaError_t launch_router(const Dims &dm, const DeviceWeights &w, const Workspace &ws,
                          const uint16_t *x, int T, int tile_tokens, cudaStream_t st, int cap = -1,
                          bool logits_ready = false);
// inject: test-only fault (MOE_INJECT_WITHHOLD_ITEMS: the gate lane publishes
// no work item, so the consumers' bounded waits run out), 0 otherwise.
// fused: the kernel routes the batch itself (no router launch before it);
// only when fused_possible() holds.  *fused_used reports whether it did.
// The rank budget's two sparse passes: the first (score mode, signed) writes
// silu(g) of every routed pair into `a`; the second reads it back with each
// pair's cut instead of recomputing the routed gates.
struct RankPass {
    float *a;          // [pairs][f] silu(g)
    const float *v;    // [pairs] cut value (second pass)
    const int *j;      // [pairs] last tied index kept (second pass)
    bool second;
};
cudaError_t launch_expert_sparse(const Dims &dm, const DeviceWeights &w, const Workspace &ws,
                                 const uint16_t *x, int T, float tau, bool use_mask,
                                 uint16_t *out, SparseTiling til, int grid_cap, cudaStream_t st,
                                 float *score_out = nullptr, int inject = 0, bool fused = false,
                                 float tau_shared = 0.f, bool score_shared = false, const RankPass *rank = nullptr,
                                 bool combine_here = false);
// Per pair of a [pairs][f] silu(g) buffer, the cut (v, J) keeping its r
// highest |silu(g)| (ties to the lower index, NaN never): neuron j is kept iff
// |silu(g_j)| > v, or == v and j <= J.
cudaError_t launch_rank_select(const float *a, int pairs, int f, int r, float *v_out, int *j_out, cudaStream_t st);
// Whether a sparse forward of T tokens can route inside the expert kernel.
bool fused_possible(const Dims &dm, int T);
// dst[b][c][col_off + r] = src[b][r][c] with row stride ld (elements).
cudaError_t launch_repack_transpose(const uint16_t *src, uint16_t *dst, int batches, int rows, int cols,
                                    int ld, int col_off, cudaStream_t st);
// Gate weights src[b][d][f] (x @ W layout) -> tiles (gate_tile_off); dst zeroed first.
cudaError_t launch_repack_gate_tiles(const uint16_t *src, uint16_t *dst, int batches, const Dims &dm,
                                     cudaStream_t st);
// dst[b][r][col_off + c] = src[b][r][c] with row stride ld (elements).
cudaError_t launch_repack_rows(const uint16_t *src, uint16_t *dst, int batches, int rows, int cols, int ld,
                               int col_off, cudaStream_t st);
cudaError_t launch_mask_compact(const Workspace &ws, int n_pairs, int f, uint16_t *idx_out,
                                int *cnt_out, cudaStream_t st);
cudaError_t launch_stats(const Dims &dm, const Workspace &ws, int T, unsigned long long *out3,
                         cudaStream_t st);

// Read `bytes` (a multiple of 16) of a device buffer once, discarding the values.
cudaError_t launch_read_all(const void *buf, size_t bytes, unsigned *sink, int n_sm, cudaStream_t st);
cudaError_t launch_radix_hist(const uint32_t *v, size_t n, uint32_t prefix, uint32_t prefix_mask,
                              int shift, unsigned *hist, int n_sm, cudaStream_t st);

// Tensor map of a 2D bf16 matrix (`rows` rows of `cols` elements, `ld_bytes`
// apart), boxes of 64 columns x box_rows rows, optionally with the 128-byte
// swizzle; reads outside the matrix return zero.  False if the driver
// rejects it.
bool encode(CUtensorMap *map, const void *base, uint64_t cols, uint64_t rows, uint64_t ld_bytes, uint32_t box_rows,
            bool swizzle);

bool dense_supported(const Dims &dm);
bool dense_setup(const Dims &dm, const DeviceWeights &w, const Workspace &ws, DenseState *st);
// tau_shared: the shared experts' threshold on a masked forward (<= 0: dense).
cudaError_t launch_dense(const Dims &dm, const Workspace &ws, const DenseState &st, const uint16_t *x, int T,
                         float tau, bool use_mask, uint16_t *out, cudaStream_t s, float tau_shared, int n_sm);
// The router's logits (ws.logits [T][E], fp32) as a tcgen05 GEMM of x [T][d]
// and Wr [E][d] on the dense branch's kernel, for large batches; the router
// kernel then runs with logits_ready.
cudaError_t launch_logits_tc(const Dims &dm, const Workspace &ws, const DenseState &st, const uint16_t *x, int T,
                             int n_sm, cudaStream_t s);

}  // namespace moe
