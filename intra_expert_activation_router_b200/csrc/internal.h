// internal.h -- data shared by the host library and the kernel launchers.
//
// Everything lives in device memory owned by the handle.  Layouts:
//   repacked weights (neuron-major, so every neuron's row is contiguous):
//     wg_n, wu_n   [E][f][d]      row j of expert e = the gate / up column j
//     wd           [E][f][d]      row j = the down-projection row of neuron j
//     wsg_n, wsu_n, wsd [S][f][d] the same for the shared experts
//     wr           [E][d]
//   per-call workspace, sized for max_tokens:
//     logits [T][E] fp32, topk_idx/topk_w [T][k], perm [T*k] (pair ids
//     t*k+rank sorted by expert, stable), mask [T*k][f/32] uint32 (bit j of
//     pair p = neuron j active), y_acc [T][d] fp32 (kept all-zero between
//     calls), tok_cnt [T] (kept zero between calls), plan (below).
#pragma once

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
    const uint16_t *wg_n, *wu_n, *wd;
    const uint16_t *wsg_n, *wsu_n, *wsd;
};

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
    uint16_t *x_perm;   // [T*k][d] bf16, tokens gathered in perm order
    uint16_t *h_perm;   // [T*k][f] bf16, masked SwiGLU activations
    // host-pointer entry
    uint16_t *x_stage, *out_stage;
};

// Launchers (return cudaGetLastError()).
cudaError_t launch_router(const Dims &dm, const DeviceWeights &w, const Workspace &ws,
                          const uint16_t *x, int T, int mt, cudaStream_t st);
cudaError_t launch_expert_sparse(const Dims &dm, const DeviceWeights &w, const Workspace &ws,
                                 const uint16_t *x, int T, float tau, bool use_mask,
                                 uint16_t *out, int mt, int grid_cap, cudaStream_t st,
                                 float *score_out = nullptr);
cudaError_t launch_repack_transpose(const uint16_t *src, uint16_t *dst, int batches, int rows,
                                    int cols, cudaStream_t st);
cudaError_t launch_mask_compact(const Workspace &ws, int n_pairs, int f, uint16_t *idx_out,
                                int *cnt_out, cudaStream_t st);
cudaError_t launch_stats(const Dims &dm, const Workspace &ws, int T, unsigned long long *out3,
                         cudaStream_t st);

cudaError_t launch_radix_hist(const uint32_t *v, size_t n, uint32_t prefix, uint32_t prefix_mask,
                              int shift, unsigned *hist, int n_sm, cudaStream_t st);

int sparse_tile_tokens(int T, int d);   // tokens per sparse work item for a batch of T

}  // namespace moe
