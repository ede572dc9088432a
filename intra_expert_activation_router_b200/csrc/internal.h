// internal.h -- data shared by the host library and the kernel launchers.
//
// Everything lives in device memory owned by the handle.  Layouts:
//   repacked weights (neuron-major, so every neuron's data is contiguous):
//     wg_n   [E][f][d]   row j = gate column j; inside every 128-byte group of a
//                        row the eight 16-byte blocks are permuted b -> b ^ (j & 7)
//                        (the 128-byte swizzle), so that eight consecutive rows
//                        copied contiguously into shared memory are bank-conflict
//                        free for tensor-core fragment loads; a tail of fewer than
//                        eight blocks (d % 64 != 0) is stored unpermuted
//     wud    [E][f][2d]  row j = [up column j | down row j]: one neuron's up and
//                        down weights in a single contiguous 4d-byte record
//     wsg_n, wsud        the same for the shared experts
//     wr     [E][d]
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
constexpr int kChunk = 32;           // neurons per sparse work item (one mask word)
constexpr int kDenseTileM = 128;     // tokens per dense GEMM tile

// Routing plan written by the router's last CTA.
struct Plan {
    int n_touched;                    // distinct experts selected
    int n_routed_items;               // sparse work items over routed experts
    int n_dense_tiles;                // 128-token tiles over touched experts
    int pad_;
    int touched[kMaxExperts];         // slot -> expert id (ascending)
    int offsets[kMaxExperts + 1];     // expert -> first position in perm
    int item_prefix[kMaxExperts + 1]; // slot -> first sparse work item
    int tile_prefix[kMaxExperts + 1]; // slot -> first dense tile
};

struct Dims {
    int E, k, d, f, S;
    int max_tokens;
};

struct DeviceWeights {
    const uint16_t *wr;
    const uint16_t *wg_n, *wud;
    const uint16_t *wsg_n, *wsud;
    const uint16_t *wdt, *wsdt;   // dense branch only: down weights transposed, [E][d][f] / [S][d][f]
};

// Tensor maps of one dense GEMM launch (kernel parameters).
struct DenseMaps {
    CUtensorMap a;    // GEMM1: x_perm rows; GEMM2: H rows (128-byte swizzle, box 64 x 128)
    CUtensorMap b0;   // GEMM1: gate rows (stored pre-swizzled, copied unswizzled); GEMM2: WdT rows (box 64 x 256)
    CUtensorMap b1;   // GEMM1: up halves of the [up | down] records; GEMM2: unused
};

struct DenseState {
    bool ok;                           // shape supported and maps encoded
    DenseMaps g1r, g1s, g2r, g2s;      // GEMM1/GEMM2, routed/shared
};

// Position of element k inside a swizzled gate row j (see wg_n above).
__host__ __device__ __forceinline__ int gate_pos(int j, int k, int d)
{
    const int b = k >> 3, full = (d >> 6) << 3;
    const int sb = b < full ? (b ^ (j & 7)) : b;
    return (sb << 3) | (k & 7);
}

struct Workspace {
    float *logits;
    int *topk_idx;
    float *topk_w;
    int *perm;
    int *perm_tok;      // [T*k] token of perm[i]
    float *perm_w;      // [T*k] routing weight of perm[i]
    uint32_t *mask;
    float *y_acc;
    int *tok_cnt;
    int *tile_ticket;   // one per router token tile, kept zero between calls
    int *done_ticket;   // one, kept zero between calls
    int *error_word;    // nonzero once a kernel reports an error
    Plan *plan;
    // dense path
    uint16_t *x_perm;   // [T*k + T][d] bf16: tokens in perm order, then x for the shared experts
    uint16_t *h_perm;   // [T*k + S*T][f] bf16: masked SwiGLU activations, routed then shared
    // host-pointer entry
    uint16_t *x_stage, *out_stage;
    // optional phase timestamps (moe_set_trace); nullptr when off
    unsigned long long *trace_router;   // [router CTAs][8]
    unsigned long long *trace_expert;   // [expert CTAs][16]
    int trace_router_ctas, trace_expert_ctas;
};

__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Launchers (return cudaGetLastError()).
cudaError_t launch_router(const Dims &dm, const DeviceWeights &w, const Workspace &ws,
                          const uint16_t *x, int T, int mt, cudaStream_t st);
cudaError_t launch_expert_sparse(const Dims &dm, const DeviceWeights &w, const Workspace &ws,
                                 const uint16_t *x, int T, float tau, bool use_mask,
                                 uint16_t *out, int mt, int grid_cap, cudaStream_t st,
                                 float *score_out = nullptr);
// dst[b][c][col_off + pos(c, r)] = src[b][r][c] with row stride ld (elements);
// pos = gate_pos when swizzle, else r.
cudaError_t launch_repack_transpose(const uint16_t *src, uint16_t *dst, int batches, int rows, int cols,
                                    int ld, int col_off, bool swizzle, cudaStream_t st);
// dst[b][r][col_off + c] = src[b][r][c] with row stride ld (elements).
cudaError_t launch_repack_rows(const uint16_t *src, uint16_t *dst, int batches, int rows, int cols, int ld,
                               int col_off, cudaStream_t st);
cudaError_t launch_mask_compact(const Workspace &ws, int n_pairs, int f, uint16_t *idx_out,
                                int *cnt_out, cudaStream_t st);
cudaError_t launch_stats(const Dims &dm, const Workspace &ws, int T, unsigned long long *out3,
                         cudaStream_t st);

cudaError_t launch_radix_hist(const uint32_t *v, size_t n, uint32_t prefix, uint32_t prefix_mask,
                              int shift, unsigned *hist, int n_sm, cudaStream_t st);

bool dense_supported(const Dims &dm);
bool dense_setup(const Dims &dm, const DeviceWeights &w, const Workspace &ws, DenseState *st);
cudaError_t launch_dense(const Dims &dm, const Workspace &ws, const DenseState &st, const uint16_t *x, int T,
                         float tau, bool use_mask, uint16_t *out, cudaStream_t s);

int sparse_tile_tokens(int T, int d);   // tokens per sparse work item for a batch of T

}  // namespace moe
