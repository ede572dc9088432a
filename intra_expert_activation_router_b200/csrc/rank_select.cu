// rank_select.cu -- the per-pair rank budget's cut.
//
// The alternative to one threshold: each routed (token, expert) pair keeps
// its r highest-scoring neurons and the lowest-scoring ones are zeroed
// ("Uncovering Intra-expert Activation Sparsity for Efficient Mixture-of-
// Expert Model Execution", technical summary, Methodology item 1).  Scores
// are s_j = |silu(g_j)| in fp32; equal scores go to the lower neuron index; a
// NaN score is never kept.  The cut of a pair is (v, J): neuron j is kept iff
// s_j > v, or s_j == v and j <= J.  It is found without a sort, by an exact
// radix selection over the scores' bit patterns (non-negative floats order
// like their bits), 8 bits per pass, most significant first, then one pass
// for the index of the last tie kept: five O(f) passes per pair.
#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kSelThreads = 256;
constexpr uint32_t kInfBits = 0x7f800000u;   // |x| bits above this are NaN

// block-wide exclusive prefix sum of one value per thread (256 threads)
__device__ __forceinline__ uint32_t block_exclusive_sum(uint32_t v, uint32_t *s_warp, uint32_t &total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
    }
    if (lane == 31) s_warp[warp] = inc;
    __syncthreads();
    uint32_t before = 0;
    total = 0;
#pragma unroll
    for (int w = 0; w < kSelThreads / 32; ++w) {
        const uint32_t t = s_warp[w];
        if (w < warp) before += t;
        total += t;
    }
    __syncthreads();   // s_warp may be reused by the next call
    return before + inc - v;
}

// One CTA per pair.  a: [pairs][f] silu(g) (signed; only |a| is ranked).
__global__ void __launch_bounds__(kSelThreads) k_rank_select(const float *__restrict__ a, int f, int r,
                                                             float *__restrict__ v_out, int *__restrict__ j_out)
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    __shared__ uint32_t hist[256];
    __shared__ uint32_t s_warp[kSelThreads / 32];
    __shared__ uint32_t s_bin, s_above;
    __shared__ int s_j;
    const int tid = threadIdx.x;
    const size_t p = blockIdx.x;
    const uint32_t *row = reinterpret_cast<const uint32_t *>(a) + p * (size_t)f;

    uint32_t nv = 0;
    for (int j = tid; j < f; j += kSelThreads) nv += (__ldcg(row + j) & 0x7fffffffu) <= kInfBits;
    uint32_t n_valid;
    block_exclusive_sum(nv, s_warp, n_valid);
    if (r <= 0 || (uint32_t)r >= n_valid) {   // keep none / every non-NaN score
        if (tid == 0) {
            v_out[p] = r <= 0 ? __uint_as_float(kInfBits) : -1.0f;
            j_out[p] = r <= 0 ? -1 : f;
        }
        return;
    }
    // the r-th largest key: `want` keys of the current prefix rank above it
    uint32_t want = (uint32_t)r - 1, prefix = 0, pmask = 0;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
        hist[tid] = 0;
        __syncthreads();
        for (int j = tid; j < f; j += kSelThreads) {
            const uint32_t key = __ldcg(row + j) & 0x7fffffffu;
            if (key <= kInfBits && (key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        // thread t holds bin 255 - t: its exclusive prefix counts the keys in higher bins
        const uint32_t c = hist[255 - tid];
        uint32_t tot;
        const uint32_t above = block_exclusive_sum(c, s_warp, tot);
        if (c > 0 && above <= want && want < above + c) {
            s_bin = 255u - (uint32_t)tid;
            s_above = above;
        }
        __syncthreads();
        want -= s_above;
        prefix |= s_bin << shift;
        pmask |= 255u << shift;
        __syncthreads();   // s_bin / s_above are rewritten by the next pass
    }
    // keys equal to the cut: the first want + 1 of them in index order are kept
    const int ch = (f + kSelThreads - 1) / kSelThreads;
    const int j0 = tid * ch, j1 = min(f, j0 + ch);
    if (tid == 0) s_j = -1;   // published by the scan's barriers
    uint32_t ties = 0;
    for (int j = j0; j < j1; ++j) ties += (__ldcg(row + j) & 0x7fffffffu) == prefix;
    uint32_t tot;
    const uint32_t before = block_exclusive_sum(ties, s_warp, tot);
    if (ties > 0 && before <= want && want < before + ties) {
        uint32_t left = want - before;
        for (int j = j0; j < j1; ++j)
            if ((__ldcg(row + j) & 0x7fffffffu) == prefix) {
                if (left == 0) {
                    s_j = j;
                    break;
                }
                --left;
            }
    }
    __syncthreads();
    if (tid == 0) {
        v_out[p] = __uint_as_float(prefix);
        j_out[p] = s_j;
    }
}

cudaError_t launch_rank_select(const float *a, int pairs, int f, int r, float *v_out, int *j_out, cudaStream_t st)
{
    if (pairs < 1) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)pairs);
    cfg.blockDim = dim3(kSelThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, k_rank_select, a, f, r, v_out, j_out);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace moe
