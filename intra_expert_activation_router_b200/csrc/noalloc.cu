// noalloc.cu -- the router's softmax top-k for callers that cannot allocate
// device memory.
//
// Some callers must not call cudaMalloc: inference servers that reserve all
// device memory up front in their own arena, custom operators running inside
// another framework that owns the caching allocator, and latency-critical
// paths where an allocation's implicit synchronisation is not acceptable.
// This entry point needs no handle and no workspace: its scratch (router
// logits and the per-token-tile tickets) lives in one file-scope device array
// that every GPU loading the library keeps until the process exits.  The
// caller passes only inputs and outputs.  There is no counterpart of this
// entry point in the paper; it is a packaging of the router step.
#include <cstdint>
#include <mutex>

#include "../../include/moe_sparse.h"
#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kNaTok = 8;   // tokens per CTA
constexpr int kNaExp = 8;   // experts per CTA, one warp each

// Fixed scratch: [T*E] fp32 logits, then ceil(T/8) int tickets.
__device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

__device__ __forceinline__ bool na_better(float v1, int i1, float v0, int i0)
{
    return v1 > v0 || (v1 == v0 && i1 < i0);
}

__global__ void __launch_bounds__(256) k_router_noalloc(const uint16_t *__restrict__ x, const uint16_t *__restrict__ wr,
                                                        int T, int d, int E, int k, float *logits, int *tickets,
                                                        int *idx_out, float *w_out)
{
    __shared__ int s_last;
    __shared__ float s_row[kNaTok][1024];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int t0 = blockIdx.y * kNaTok, nt = min(kNaTok, T - t0);
    const int e = blockIdx.x * kNaExp + warp;
    // logits of this CTA's experts for its tokens, fp32 accumulation
    if (e < E) {
        float acc[kNaTok];
#pragma unroll
        for (int r = 0; r < kNaTok; ++r) acc[r] = 0.f;
        for (int i = lane * 8; i < d; i += 256) {
            const uint4 wv = ld_cached(wr + (size_t)e * d + i);
#pragma unroll
            for (int r = 0; r < kNaTok; ++r)
                if (r < nt) acc[r] = dot8(wv, ld_cached(x + (size_t)(t0 + r) * d + i), acc[r]);
        }
#pragma unroll
        for (int r = 0; r < kNaTok; ++r) acc[r] = warp_sum(acc[r]);
        if (lane == 0)
            for (int r = 0; r < nt; ++r) logits[(size_t)(t0 + r) * E + e] = acc[r];
    }
    // the last CTA of the token tile selects the top-k of each token
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const int tk = atomicAdd(&tickets[blockIdx.y], 1);
        s_last = (tk == (int)gridDim.x - 1);
        if (s_last) tickets[blockIdx.y] = 0;
    }
    __syncthreads();
    if (!s_last || warp >= nt) return;
    __threadfence();
    const int t = t0 + warp;
    float *row = s_row[warp];
    float m = -INFINITY;
    for (int j = lane; j < E; j += 32) {
        row[j] = __ldcg(&logits[(size_t)t * E + j]);
        m = fmaxf(m, row[j]);
    }
    m = warp_max(m);
    float s = 0.f;
    for (int j = lane; j < E; j += 32) s += expf(row[j] - m);
    s = warp_sum(s);
    unsigned taken = 0;   // bit q: expert lane + 32q already selected
    for (int r = 0; r < k; ++r) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int q = 0, j = lane; j < E; ++q, j += 32) {
            if (taken & (1u << q)) continue;
            if (bi == 0x7fffffff || na_better(row[j], j, bv, bi)) { bv = row[j]; bi = j; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(kFull, bv, o);
            const int oi = __shfl_xor_sync(kFull, bi, o);
            if (oi != 0x7fffffff && (bi == 0x7fffffff || na_better(ov, oi, bv, bi))) { bv = ov; bi = oi; }
        }
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (lane == 0) {
            idx_out[(size_t)t * k + r] = bi;
            w_out[(size_t)t * k + r] = expf(bv - m) / s;
        }
    }
}

}  // namespace moe

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_na_mu;
void *g_na_ptr[kMaxDevices];   // device address of g_noalloc_scratch, per device

// The array's name is a host-side stand-in in host code; its device address
// is looked up once per device, with that device current.
int scratch_address(void **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ECUDA;
    std::lock_guard<std::mutex> lk(g_na_mu);
    if (!g_na_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, moe::g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return MOE_ECUDA;
        }
        g_na_ptr[dev] = p;
    }
    *out = g_na_ptr[dev];
    return MOE_OK;
}

}  // namespace

extern "C" int moe_router_topk_noalloc(const void *x, int T, const void *w_router, int E, int d_model,
                                       int top_k, int *idx_out, float *w_out, void *stream)
{
    if (!x || !w_router || !idx_out || !w_out) return MOE_EINVAL;
    if (E < 1 || E > 1024 || top_k < 1 || top_k > E || d_model < 8 || d_model % 8 != 0 || T < 1)
        return MOE_EINVAL;
    if (((uintptr_t)x & 15u) || ((uintptr_t)w_router & 15u)) return MOE_EALIGN;
    const size_t tiles = ((size_t)T + moe::kNaTok - 1) / moe::kNaTok;
    const size_t logit_bytes = (((size_t)T * E * sizeof(float)) + 255) & ~size_t(255);
    if (tiles > 65535 || logit_bytes + tiles * sizeof(int) > (size_t)MOE_NOALLOC_SCRATCH_BYTES) return MOE_ENOTSUP;
    void *base = nullptr;
    const int rc = scratch_address(&base);
    if (rc) return rc;
    float *logits = (float *)base;
    int *tickets = (int *)((char *)base + logit_bytes);
    cudaStream_t st = (cudaStream_t)stream;
    // the tickets must start at zero (a call that failed midway may have left some set)
    if (cudaMemsetAsync(tickets, 0, tiles * sizeof(int), st) != cudaSuccess) return MOE_ECUDA;
    dim3 grid((E + moe::kNaExp - 1) / moe::kNaExp, (unsigned)tiles);
    moe::k_router_noalloc<<<grid, 256, 0, st>>>((const uint16_t *)x, (const uint16_t *)w_router, T, d_model, E,
                                                 top_k, logits, tickets, idx_out, w_out);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ECUDA;
}
