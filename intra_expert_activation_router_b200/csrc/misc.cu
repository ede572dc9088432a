// misc.cu -- weight repacking, active-list compaction and last-call statistics.
#include "common.cuh"
#include "internal.h"

namespace moe {

// dst[b][c][col_off + r] = src[b][r][c], 32x32 tiles through shared memory.
__global__ void k_transpose(const uint16_t *__restrict__ src, uint16_t *__restrict__ dst, int rows, int cols,
                            int ld, int col_off)
{
    __shared__ uint16_t tile[32][33];
    const size_t sbase = (size_t)blockIdx.z * rows * cols;
    const size_t dbase = (size_t)blockIdx.z * cols * ld;
    const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int r = r0 + i, c = c0 + threadIdx.x;
        if (r < rows && c < cols) tile[i][threadIdx.x] = src[sbase + (size_t)r * cols + c];
    }
    __syncthreads();
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int c = c0 + i, r = r0 + threadIdx.x;
        if (r < rows && c < cols) dst[dbase + (size_t)c * ld + col_off + r] = tile[threadIdx.x][i];
    }
}

cudaError_t launch_repack_transpose(const uint16_t *src, uint16_t *dst, int batches, int rows, int cols,
                                    int ld, int col_off, cudaStream_t st)
{
    dim3 grid((cols + 31) / 32, (rows + 31) / 32, batches);
    k_transpose<<<grid, dim3(32, 8), 0, st>>>(src, dst, rows, cols, ld, col_off);
    return cudaGetLastError();
}

// Gate weights src[b][k][j] (input k, neuron j) -> the tensor-core tile layout
// (gate_tile_off), 32x32 tiles through shared memory.
__global__ void k_gate_tiles(const uint16_t *__restrict__ src, uint16_t *__restrict__ dst, int d, int f,
                             int n_kb, size_t per_expert)
{
    __shared__ uint16_t tile[32][33];
    const size_t sbase = (size_t)blockIdx.z * d * f;
    uint16_t *dexp = dst + (size_t)blockIdx.z * per_expert;
    const int j0 = blockIdx.x * 32, k0 = blockIdx.y * 32;
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int k = k0 + i, j = j0 + threadIdx.x;
        if (k < d && j < f) tile[i][threadIdx.x] = src[sbase + (size_t)k * f + j];
    }
    __syncthreads();
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int j = j0 + i, k = k0 + threadIdx.x;
        if (k < d && j < f) dexp[gate_tile_off(j, k, n_kb)] = tile[threadIdx.x][i];
    }
}

cudaError_t launch_repack_gate_tiles(const uint16_t *src, uint16_t *dst, int batches, const Dims &dm,
                                     cudaStream_t st)
{
    const size_t per_expert = (size_t)dm.fp * dm.dp;
    cudaError_t e = cudaMemsetAsync(dst, 0, 2 * per_expert * batches, st);
    if (e != cudaSuccess) return e;
    dim3 grid((dm.f + 31) / 32, (dm.d + 31) / 32, batches);
    k_gate_tiles<<<grid, dim3(32, 8), 0, st>>>(src, dst, dm.d, dm.f, dm.n_kb, per_expert);
    return cudaGetLastError();
}

__global__ void k_copy_rows(const uint16_t *__restrict__ src, uint16_t *__restrict__ dst, size_t n_rows, int cols,
                            int ld, int col_off)
{
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_rows * cols;
         i += (size_t)gridDim.x * blockDim.x) {
        const size_t r = i / cols;
        const int c = (int)(i % cols);
        dst[r * ld + col_off + c] = src[i];
    }
}

cudaError_t launch_repack_rows(const uint16_t *src, uint16_t *dst, int batches, int rows, int cols, int ld,
                               int col_off, cudaStream_t st)
{
    const size_t n_rows = (size_t)batches * rows;
    size_t blocks = (n_rows * cols + 255) / 256;
    if (blocks > 65535 * 8) blocks = 65535 * 8;
    k_copy_rows<<<(unsigned)blocks, 256, 0, st>>>(src, dst, n_rows, cols, ld, col_off);
    return cudaGetLastError();
}

// Mask words -> ascending active-neuron lists, one warp per (token, rank) pair:
// a warp-wide exclusive scan of the words' popcounts places each word's bits.
__global__ void k_mask_compact(const uint32_t *__restrict__ mask, int n_pairs, int words,
                               uint16_t *__restrict__ idx_out, int *__restrict__ cnt_out)
{
    const int lane = threadIdx.x & 31;
    const int p = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (p >= n_pairs) return;
    const uint32_t *row = mask + (size_t)p * words;
    uint16_t *out = idx_out + (size_t)p * words * 32;
    int base = 0;
    for (int w0 = 0; w0 < words; w0 += 32) {
        const uint32_t wv = (w0 + lane < words) ? row[w0 + lane] : 0u;
        const int c = __popc(wv);
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += v;
        }
        int pos = base + incl - c;
        for (uint32_t b = wv; b; b &= b - 1) out[pos++] = (uint16_t)((w0 + lane) * 32 + __ffs(b) - 1);
        base += __shfl_sync(kFull, incl, 31);
    }
    if (lane == 0) cnt_out[p] = base;
}

cudaError_t launch_mask_compact(const Workspace &ws, int n_pairs, int f, uint16_t *idx_out,
                                int *cnt_out, cudaStream_t st)
{
    const int per_block = 8;
    k_mask_compact<<<(n_pairs + per_block - 1) / per_block, 32 * per_block, 0, st>>>(
        ws.mask, n_pairs, f / 32, idx_out, cnt_out);
    return cudaGetLastError();
}

// out[0] += active neurons over all pairs, out[1] += union-active neurons over
// touched experts, out[2] = touched experts.  One CTA per expert slot.
__global__ void k_stats(Plan *plan, const int *perm, const uint32_t *mask, int words,
                        unsigned long long *out)
{
    const int slot = blockIdx.x;
    if (slot >= plan->n_touched) return;
    const int e = plan->touched[slot];
    const int b = plan->offsets[e], n = plan->offsets[e + 1] - b;
    unsigned long long act = 0, uni = 0;
    for (int w = threadIdx.x; w < words; w += blockDim.x) {
        uint32_t u = 0;
        for (int i = 0; i < n; ++i) {
            const uint32_t v = mask[(size_t)perm[b + i] * words + w];
            act += __popc(v);
            u |= v;
        }
        uni += __popc(u);
    }
    atomicAdd(&out[0], act);
    atomicAdd(&out[1], uni);
    if (slot == 0 && threadIdx.x == 0) out[2] = plan->n_touched;
}

cudaError_t launch_stats(const Dims &dm, const Workspace &ws, int T, unsigned long long *out3,
                         cudaStream_t st)
{
    (void)T;
    cudaError_t e = cudaMemsetAsync(out3, 0, 3 * sizeof(unsigned long long), st);
    if (e != cudaSuccess) return e;
    k_stats<<<dm.E, 128, 0, st>>>(ws.plan, ws.perm, ws.mask, dm.f / 32, out3);
    return cudaGetLastError();
}

// One pass of an exact radix select over non-negative float bit patterns
// (their uint32 order is their numeric order): histogram of the 8-bit digit
// at `shift` among the values whose higher digits equal `prefix`.
__global__ void k_radix_hist(const uint32_t *__restrict__ v, size_t n, uint32_t prefix,
                             uint32_t prefix_mask, int shift, unsigned *__restrict__ hist)
{
    __shared__ unsigned sh[256];
    for (int i = threadIdx.x; i < 256; i += blockDim.x) sh[i] = 0;
    __syncthreads();
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const uint32_t u = v[i];
        if ((u & prefix_mask) == prefix) atomicAdd(&sh[(u >> shift) & 255u], 1u);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 256; i += blockDim.x)
        if (sh[i]) atomicAdd(&hist[i], sh[i]);
}

cudaError_t launch_radix_hist(const uint32_t *v, size_t n, uint32_t prefix, uint32_t prefix_mask,
                              int shift, unsigned *hist, int n_sm, cudaStream_t st)
{
    cudaError_t e = cudaMemsetAsync(hist, 0, 256 * sizeof(unsigned), st);
    if (e != cudaSuccess) return e;
    size_t blocks = (n + 255) / 256;
    if (blocks > (size_t)n_sm * 8) blocks = (size_t)n_sm * 8;
    if (blocks < 1) blocks = 1;
    k_radix_hist<<<(unsigned)blocks, 256, 0, st>>>(v, n, prefix, prefix_mask, shift, hist);
    return cudaGetLastError();
}

// Read a buffer once (the L2 flush of the switch-point tuner: after a memset
// of twice the L2, reading it back leaves L2 full of clean lines, so the
// timed forward neither hits in L2 nor pays for write-backs).  `sink` is
// written only if the buffer held the impossible sum below.
__global__ void k_read_all(const uint4 *__restrict__ p, size_t n16, unsigned *sink)
{
    unsigned acc = 0;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += (size_t)gridDim.x * blockDim.x) {
        const uint4 v = __ldcg(p + i);
        acc ^= v.x ^ v.y ^ v.z ^ v.w;
    }
    if (acc == 0x9e3779b9u) *sink = acc;
}

cudaError_t launch_read_all(const void *buf, size_t bytes, unsigned *sink, int n_sm, cudaStream_t st)
{
    k_read_all<<<(unsigned)(n_sm * 4), 256, 0, st>>>(reinterpret_cast<const uint4 *>(buf), bytes / 16, sink);
    return cudaGetLastError();
}

}  // namespace moe
