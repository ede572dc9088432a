// dense_tc.cu -- the dense branch: the same masked layer through tcgen05
// grouped GEMMs, for batches large enough that the union of active neurons
// is dense ("Uncovering Intra-expert Activation Sparsity for Efficient
// Mixture-of-Expert Model Execution", technical summary, Methodology item 3,
// "Dynamic switching": sparse execution for small batches, dense for large).
//
//   gather   token rows in expert order (x_perm), and a copy of x for the
//            shared experts, so every A tile is one TMA box
//   GEMM1    per expert and 128-row tile of its tokens, per 128 neurons:
//            D[128 x 256] = X_tile . [Wg rows | Wu rows]^T in TMEM (one
//            M=128, N=256 MMA per 16 of K); epilogue h = silu(g) u, zeroed
//            where |silu(g)| < tau on the masked path -> bf16 H
//   GEMM2    per expert and tile, per 256 output dims:
//            D[128 x 256] = H_tile . WdT rows^T; epilogue y_acc[token] +=
//            w * D with fp32 vector atomics
//   convert  out = bf16(y_acc), y_acc re-zeroed
// Shared experts run as extra GEMM1/GEMM2 grids over all T tokens with their
// own threshold (none by default) and weight 1.  The GEMM kernel is
// persistent (one CTA per SM walking its tiles): warp 0 issues the TMA loads
// into a 4-stage ring, warp 1 issues the MMAs from one thread into two TMEM
// accumulators in turn, and eight epilogue warps read one accumulator back
// while the MMAs fill the other.  Operands are K-major with the 128-byte
// swizzle; the gate weights are stored in HBM as exactly these tiles
// (gate_tile_off), so each is one plain 16 KB bulk copy.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace moe {

constexpr int kBM = 128;            // token rows per tile
constexpr int kBK = 64;             // K per stage (128 bytes of bf16)
constexpr int kDStages = 4;
constexpr int kDenseThreads = 320;   // warp 0 TMA, warp 1 MMA, warps 2-9 epilogue
constexpr int kEpiWarps = 8;         // two per TMEM lane quarter, each half of the columns
constexpr int kAccCols = 256;        // one accumulator: 128 lanes x 256 fp32 columns
constexpr int kATileBytes = kBM * kBK * 2;    // 16 KB
constexpr int kBTileBytes = 256 * kBK * 2;    // 32 KB
constexpr int kStageBytes = kATileBytes + kBTileBytes;
// Down epilogue staging: per epilogue warp 32 rows x 16 columns of fp32,
// rows padded to 20 floats (16-byte aligned, conflict-free quarter warps)
constexpr int kStgPitch = 20;
constexpr int kStgBytes = kEpiWarps * 32 * kStgPitch * 4;   // 20 KB
constexpr int kDenseSmem = kDStages * kStageBytes + 256 /* barriers */ + kStgBytes + 1024 /* alignment */;

enum DenseMode { kGateUp = 0, kDown = 1, kLogits = 2 };

struct DenseArgs {
    int mode;
    int shared;        // 0: routed tiles from the plan; 1: shared expert `sidx` over all T tokens
    int sidx;
    int T, K, kb;      // tokens, contraction length, K blocks
    int wrows;         // weight rows per expert (f for GEMM1, d for GEMM2)
    int a_base;        // first A row of the launch (shared rows after the routed ones)
    const uint16_t *gate;   // GEMM1: gate tiles of the routed (or shared) experts
    int n_kb, n_blk;        // GEMM1: gate tiles per 128-neuron block, blocks per expert
    int h_base, h_ld;  // GEMM1: first H row, H row length (f)
    float tau;
    int use_mask;
    const Plan *plan;
    const int *perm, *perm_tok;
    const float *perm_w;
    uint16_t *h;       // GEMM1 output
    float *y_acc;      // GEMM2 output
    float *ypart;      // GEMM2 output, deterministic mode: [T][k + S][d] rows
    int k, kS;         // top-k, k + S
    int d;
    int *err;
};

// Token rows in expert order, plus the shared experts' copy of x.
__global__ void k_dense_gather(const uint16_t *__restrict__ x, const int *__restrict__ perm_tok, int P, int T,
                               int d8, int shared_base, uint16_t *__restrict__ x_perm)
{
    const size_t n = (size_t)(P + (shared_base >= 0 ? T : 0)) * d8;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const size_t row = i / d8;
        const int v = (int)(i % d8);
        const int src = row < (size_t)P ? perm_tok[row] : (int)(row - P);
        const size_t dst = row < (size_t)P ? row : (size_t)shared_base + (row - P);
        reinterpret_cast<uint4 *>(x_perm)[dst * d8 + v] = ld_cached(x + ((size_t)src * d8 + v) * 8);
    }
}

// out = bf16(y_acc) (round to nearest even), then y_acc = 0.  The last kernel
// of a dense forward: it also moves the forward's error code into the sticky
// word and clears its own word (as the sparse path's conversion kernel does).
__global__ void k_dense_convert(float *__restrict__ y_acc, uint16_t *__restrict__ out, size_t n4, int *error_word,
                                int *error_sticky, float *ypart, int rows, int d)
{
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        const int e0 = *error_word;
        if (e0 != 0) {
            atomicCAS(error_sticky, 0, e0);
            *error_word = 0;
        }
    }
    if (ypart)   // deterministic mode: each token's k + S rows, summed in order
        det_combine(ypart, rows, d, out, (long long)n4, ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5,
                    ((long long)gridDim.x * blockDim.x) >> 5, threadIdx.x & 31);
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; !ypart && i < n4;
         i += (size_t)gridDim.x * blockDim.x) {
        const float4 v = reinterpret_cast<const float4 *>(y_acc)[i];
        uint2 p;
        p.x = (uint32_t)f2bf_bits(v.x) | ((uint32_t)f2bf_bits(v.y) << 16);
        p.y = (uint32_t)f2bf_bits(v.z) | ((uint32_t)f2bf_bits(v.w) << 16);
        reinterpret_cast<uint2 *>(out)[i] = p;
        reinterpret_cast<float4 *>(y_acc)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

}  // namespace moe

namespace moe {

// One output tile of a launch: A rows [row0, row0 + valid), weight rows
// wrow0 + n0 .. of expert (or shared expert) ex.  Tiles are numbered with
// the output block fastest, so that the tiles in flight at once cover a few
// token tiles completely: a token tile's activations are read by its output
// blocks from L2, an expert's weights by its token tiles at about the same
// time.
struct DenseTile {
    int row0, valid, wrow0, ex, n0, bx;
};

__device__ __forceinline__ int dense_out_blocks(const DenseArgs &a)
{
    return a.mode == kGateUp ? a.wrows / 128 : (a.wrows + 255) / 256;
}

__device__ __forceinline__ int dense_n_tiles(const DenseArgs &a)
{
    const int m_tiles = (a.shared || a.mode == kLogits) ? (a.T + kBM - 1) / kBM : a.plan->n_dense_tiles;
    return m_tiles * dense_out_blocks(a);
}

__device__ __forceinline__ DenseTile dense_tile(const DenseArgs &a, int t)
{
    const int n_out = dense_out_blocks(a);
    DenseTile d;
    d.bx = t % n_out;
    const int by = t / n_out;
    if (a.mode == kLogits) {   // the batch's own rows against all experts' router rows
        d.row0 = kBM * by;
        d.valid = min(kBM, a.T - d.row0);
        d.wrow0 = 0;
        d.ex = 0;
    } else if (!a.shared) {
        const Plan *plan = a.plan;
        int lo = 0, hi = plan->n_touched - 1;   // last slot with tile_prefix <= by
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (plan->tile_prefix[mid] <= by) lo = mid; else hi = mid - 1;
        }
        const int e = plan->touched[lo];
        const int local = by - plan->tile_prefix[lo];
        const int off = plan->offsets[e], cnt = plan->offsets[e + 1] - off;
        d.row0 = off + kBM * local;
        d.valid = min(kBM, cnt - kBM * local);
        d.wrow0 = e * a.wrows;
        d.ex = e;
    } else {
        d.row0 = kBM * by;
        d.valid = min(kBM, a.T - d.row0);
        d.wrow0 = a.sidx * a.wrows;
        d.ex = a.sidx;
    }
    d.n0 = d.bx * (a.mode == kGateUp ? 128 : 256);
    return d;
}

// Persistent: one CTA per SM walks the launch's tiles t = blockIdx.x,
// blockIdx.x + gridDim.x, ...  Warp 0 streams every tile's K blocks into a
// 4-stage ring without pausing between tiles, warp 1 issues the MMAs into one
// of two 256-column TMEM accumulators, and warps 2-9 (two per TMEM lane
// quarter, each half of the columns) run the epilogue of tile i while the
// MMAs of tile i + 1 proceed.
__global__ void __launch_bounds__(kDenseThreads, 1) k_dense_gemm(const __grid_constant__ DenseMaps maps, DenseArgs a)
{
    extern __shared__ uint8_t dsmem_raw[];
    // the 128-byte swizzle needs 1024-byte aligned tiles
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kDStages * kStageBytes);
    uint64_t *empty = full + kDStages;
    uint64_t *accf = empty + kDStages;   // [2] accumulator ready (MMA commit)
    uint64_t *acce = accf + 2;           // [2] accumulator read out (the epilogue warps)
    uint64_t *mdrain = acce + 2;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(mdrain + 1);
    float *stg_all = reinterpret_cast<float *>(smem + kDStages * kStageBytes + 256);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < kDStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accf[b], 1);
            mbar_init(&acce[b], kEpiWarps);
        }
        mbar_init(mdrain, 1);
        fence_mbar_init();
        tma_prefetch_desc(&maps.a);
        if (a.mode == kGateUp) tma_prefetch_desc(&maps.b1);
        else tma_prefetch_desc(&maps.b0);
    }
    if (warp == 1) {
        tmem_alloc(s_tmem, 2 * kAccCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const int n_tiles = dense_n_tiles(a);

    if (warp == 0) {
        if (lane == 0) {
            // ---- TMA producer
            const uint32_t bytes = kATileBytes + (a.mode == kGateUp ? 2 * (kBTileBytes / 2) : kBTileBytes);
            uint32_t st = 0;   // stages issued
            bool ok = true;
            for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
                const DenseTile dt = dense_tile(a, t);
                for (int kb = 0; kb < a.kb; ++kb, ++st) {
                    const int s = (int)(st % kDStages);
                    if (!mbar_wait(&empty[s], ((st / kDStages) & 1) ^ 1, a.err, 31)) {
                        ok = false;
                        break;
                    }
                    uint8_t *A = smem + s * kStageBytes, *B = A + kATileBytes;
                    mbar_arrive_expect_tx(&full[s], bytes);
                    tma_load_2d(A, &maps.a, kb * kBK, a.a_base + dt.row0, &full[s]);
                    if (a.mode == kGateUp) {
                        const uint16_t *gt =
                            a.gate + (((size_t)dt.ex * a.n_blk + dt.bx) * a.n_kb + kb) * (kBM * kBK);
                        bulk_g2s(B, gt, kBTileBytes / 2, &full[s]);
                        tma_load_2d(B + kBTileBytes / 2, &maps.b1, kb * kBK, dt.wrow0 + dt.n0, &full[s]);
                    } else {
                        tma_load_2d(B, &maps.b0, kb * kBK, dt.wrow0 + dt.n0, &full[s]);
                    }
                }
            }
            // every copy issued has landed before the CTA may exit
            for (int s = 0; s < kDStages && (uint32_t)s < st; ++s)
                mbar_drain(&full[s], (((st - s + kDStages - 1) / kDStages) - 1) & 1);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- MMA issuer: M = 128, N = 256, K = 16 per instruction
            const uint32_t idesc = idesc_bf16_f32(kBM, 256);
            uint32_t st = 0;
            int lt = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++lt) {
                const int acc = lt & 1;
                ok = mbar_wait(&acce[acc], ((lt >> 1) & 1) ^ 1, a.err, 34);   // the epilogue read it out
                tc_fence_after();
                const uint32_t dt = tmem + acc * kAccCols;
                for (int kb = 0; kb < a.kb && ok; ++kb, ++st) {
                    const int s = (int)(st % kDStages);
                    ok = mbar_wait(&full[s], (st / kDStages) & 1, a.err, 32);
                    tc_fence_after();
                    const uint8_t *A = smem + s * kStageBytes, *B = A + kATileBytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        umma_bf16(dt, smem_desc_k_sw128(A + 32 * kk), smem_desc_k_sw128(B + 32 * kk), idesc,
                                  (kb | kk) != 0 ? 1u : 0u);
                    umma_commit(&empty[s]);   // the stage is free once these MMAs have read it
                }
                if (ok) umma_commit(&accf[acc]);
            }
            umma_commit(mdrain);   // all MMAs complete before the accumulators are freed
            mbar_drain(mdrain, 0);
        }
        __syncwarp();
    } else {
        // ---- epilogue: thread = accumulator row (TMEM lane 32 * (warp % 4) + lane);
        // warps 2-5 take the first half of the tile's columns, warps 6-9 the second
        const int q = warp & 3, half = (warp - 2) >> 2;
        const int row = q * 32 + lane;
        int lt = 0;
        for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++lt) {
            const int acc = lt & 1;
            const bool ok = mbar_wait(&accf[acc], (lt >> 1) & 1, a.err, 33);
            tc_fence_after();
            if (!ok) break;
            const DenseTile dt = dense_tile(a, t);
            const uint32_t tl = tmem + acc * kAccCols + ((uint32_t)(q * 32) << 16);
            if (a.mode == kGateUp) {
                uint16_t *hrow = a.h + (size_t)(a.h_base + dt.row0 + row) * a.h_ld + dt.n0;
                for (int c = 64 * half; c < 64 * half + 64; c += 16) {
                    float g[16], u[16];
                    tmem_ld16(tl + c, g);
                    tmem_ld16(tl + 128 + c, u);
                    uint32_t pk[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        float hv[2];
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const float av = silu_f(g[2 * i + j]);
                            const bool on = !a.use_mask || fabsf(av) >= a.tau;
                            hv[j] = on ? av * u[2 * i + j] : 0.f;
                        }
                        pk[i] = (uint32_t)f2bf_bits(hv[0]) | ((uint32_t)f2bf_bits(hv[1]) << 16);
                    }
                    if (row < dt.valid) {
                        reinterpret_cast<uint4 *>(hrow + c)[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        reinterpret_cast<uint4 *>(hrow + c)[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                    }
                }
            } else if (a.mode == kLogits) {
                // logits[token][expert] (fp32) for the experts inside the matrix
                float *lrow = a.y_acc + (size_t)(dt.row0 + row) * a.d;
                for (int c = 128 * half; c < 128 * half + 128; c += 16) {
                    float y[16];
                    tmem_ld16(tl + c, y);
                    if (row < dt.valid)
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (dt.n0 + c + i < a.wrows) lrow[dt.n0 + c + i] = y[i];
                }
            } else {
                int tok = 0;
                float w = 1.f;
                if (row < dt.valid) {
                    tok = a.shared ? dt.row0 + row : a.perm_tok[dt.row0 + row];
                    w = a.shared ? 1.f : a.perm_w[dt.row0 + row];
                }
                float *yrow = a.y_acc + (size_t)tok * a.d + dt.n0;
                if (a.ypart) {   // deterministic mode: the pair's own row, each element written once
                    const int slot = a.shared ? a.k + a.sidx
                                              : (row < dt.valid ? a.perm[dt.row0 + row] % a.k : 0);
                    yrow = a.ypart + ((size_t)tok * a.kS + slot) * a.d + dt.n0;
                    for (int c = 128 * half; c < 128 * half + 128; c += 16) {
                        float y[16];
                        tmem_ld16(tl + c, y);
                        if (row < dt.valid)
#pragma unroll
                            for (int i = 0; i < 16; i += 4)
                                __stcg(reinterpret_cast<float4 *>(yrow + c + i),
                                       make_float4(w * y[i], w * y[i + 1], w * y[i + 2], w * y[i + 3]));
                    }
                } else {
                    // the warp's 32 rows, 16 columns at a time, through shared memory,
                    // so that each vector reduction covers 64 contiguous bytes of 8
                    // rows (whole 32-byte sectors) instead of 16 bytes of 32 rows
                    float *stg = stg_all + (warp - 2) * 32 * kStgPitch;
                    const int rr = lane >> 2, c4 = (lane & 3) * 4;
                    int tok_r[4];
                    bool ok_r[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        tok_r[j] = __shfl_sync(0xffffffffu, tok, 8 * j + rr);
                        ok_r[j] = 32 * q + 8 * j + rr < dt.valid;
                    }
                    for (int c = 128 * half; c < 128 * half + 128; c += 16) {
                        float y[16];
                        tmem_ld16(tl + c, y);
#pragma unroll
                        for (int i = 0; i < 16; i += 4)
                            *reinterpret_cast<float4 *>(stg + lane * kStgPitch + i) =
                                make_float4(w * y[i], w * y[i + 1], w * y[i + 2], w * y[i + 3]);
                        __syncwarp();
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const float4 v = *reinterpret_cast<const float4 *>(stg + (8 * j + rr) * kStgPitch + c4);
                            if (ok_r[j])
                                atomicAdd(reinterpret_cast<float4 *>(a.y_acc + (size_t)tok_r[j] * a.d + dt.n0 + c + c4),
                                          v);
                        }
                        __syncwarp();
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acce[acc]);   // the MMA may overwrite this accumulator
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 2 * kAccCols);
    }
}

}  // namespace moe

namespace moe {

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            cudaGetLastError();
    }
    return fn;
}

}  // namespace

// A 2D bf16 matrix of `rows` rows of `cols` elements, `ld_bytes` apart; boxes of
// 64 columns x box_rows rows; elements outside the matrix read as zero.
bool encode(CUtensorMap *map, const void *base, uint64_t cols, uint64_t rows, uint64_t ld_bytes, uint32_t box_rows,
            bool swizzle)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {ld_bytes};
    cuuint32_t box[2] = {(cuuint32_t)kBK, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool dense_supported(const Dims &dm)
{
    return dm.d % 256 == 0 && dm.f % 128 == 0 && encode_fn() != nullptr;
}

bool dense_setup(const Dims &dm, const DeviceWeights &w, const Workspace &ws, DenseState *st)
{
    st->ok = false;
    if (!dense_supported(dm)) return true;   // not an error: the dense path is just unavailable
    const uint64_t d = dm.d, f = dm.f, E = dm.E, S = dm.S;
    const uint64_t Pm = (uint64_t)dm.max_tokens * dm.k, Tm = dm.max_tokens;
    bool ok = true;
    // GEMM1 routed / shared
    ok = ok && encode(&st->g1r.a, ws.x_perm, d, Pm + Tm, 2 * d, kBM, true);
    ok = ok && encode(&st->g1r.b1, w.wud, d, E * f, 4 * d, 128, true);
    st->g1r.b0 = st->g1r.b1;   // unused: gate tiles are bulk copies
    st->gate_r = w.wg_t;
    st->gate_s = w.wsg_t;
    ok = ok && encode(&st->g2r.a, ws.h_perm, f, Pm + S * Tm, 2 * f, kBM, true);
    ok = ok && encode(&st->g2r.b0, w.wdt, f, E * d, 2 * f, 256, true);
    st->g2r.b1 = st->g2r.b0;
    if (S > 0) {
        st->g1s.a = st->g1r.a;
        ok = ok && encode(&st->g1s.b1, w.wsud, d, S * f, 4 * d, 128, true);
        st->g1s.b0 = st->g1s.b1;
        st->g2s.a = st->g2r.a;
        ok = ok && encode(&st->g2s.b0, w.wsdt, f, S * d, 2 * f, 256, true);
        st->g2s.b1 = st->g2s.b0;
    }
    ok = ok && encode(&st->router_b, w.wr, d, E, 2 * d, 256, true);
    st->ok = ok;
    return ok;
}

cudaError_t launch_logits_tc(const Dims &dm, const Workspace &ws, const DenseState &st, const uint16_t *x, int T,
                             int n_sm, cudaStream_t s)
{
    if (!st.ok) return cudaErrorNotSupported;
    static int smem_set[kMaxDevices] = {};
    cudaError_t e = ensure_dynamic_smem(k_dense_gemm, kDenseSmem, smem_set);
    if (e != cudaSuccess) return e;
    DenseMaps maps;
    if (!encode(&maps.a, x, dm.d, T, 2ull * dm.d, kBM, true)) return cudaErrorInvalidValue;
    maps.b0 = st.router_b;
    maps.b1 = st.router_b;
    DenseArgs a = {};
    a.mode = kLogits;
    a.T = T;
    a.K = dm.d;
    a.kb = dm.d / kBK;
    a.wrows = dm.E;
    a.y_acc = ws.logits;
    a.d = dm.E;   // the logits' row length
    a.err = ws.error_word;
    const long long tiles = (long long)((T + kBM - 1) / kBM) * ((dm.E + 255) / 256);
    k_dense_gemm<<<(unsigned)(tiles < n_sm ? tiles : n_sm), kDenseThreads, kDenseSmem, s>>>(maps, a);
    return cudaGetLastError();
}

cudaError_t launch_dense(const Dims &dm, const Workspace &ws, const DenseState &st, const uint16_t *x, int T,
                         float tau, bool use_mask, uint16_t *out, cudaStream_t s, float tau_shared, int n_sm)
{
    // persistent grids: at most one CTA per SM, never more than the launch's tiles
    auto grid = [n_sm](long long tiles) { return (unsigned)(tiles < n_sm ? (tiles > 0 ? tiles : 1) : n_sm); };
    if (!st.ok) return cudaErrorNotSupported;
    static int smem_set[kMaxDevices] = {};
    cudaError_t e = ensure_dynamic_smem(k_dense_gemm, kDenseSmem, smem_set);
    if (e != cudaSuccess) return e;
    const int P = T * dm.k, Pm = dm.max_tokens * dm.k, Tm = dm.max_tokens;
    const int d8 = dm.d / 8;
    // gather
    {
        const size_t n = (size_t)(P + (dm.S > 0 ? T : 0)) * d8;
        size_t blocks = (n + 255) / 256;
        if (blocks > 148 * 16) blocks = 148 * 16;
        k_dense_gather<<<(unsigned)blocks, 256, 0, s>>>(x, ws.perm_tok, P, T, d8, dm.S > 0 ? Pm : -1, ws.x_perm);
    }
    const int mbound = (P < dm.E ? P : dm.E) + P / kBM;
    const int mshared = (T + kBM - 1) / kBM;
    DenseArgs a = {};
    a.T = T;
    a.tau = tau;
    a.use_mask = use_mask ? 1 : 0;
    a.plan = ws.plan;
    a.perm = ws.perm;
    a.perm_tok = ws.perm_tok;
    a.perm_w = ws.perm_w;
    a.h = ws.h_perm;
    a.h_ld = dm.f;
    a.y_acc = ws.y_acc;
    a.ypart = ws.ypart;
    a.k = dm.k;
    a.kS = dm.k + dm.S;
    a.d = dm.d;
    a.err = ws.error_word;
    // GEMM1: gate | up with the mask epilogue
    a.mode = kGateUp;
    a.gate = st.gate_r;
    a.n_kb = dm.n_kb;
    a.n_blk = dm.n_blk;
    a.K = dm.d;
    a.kb = dm.d / kBK;
    a.wrows = dm.f;
    a.shared = 0;
    a.a_base = 0;
    a.h_base = 0;
    k_dense_gemm<<<grid((long long)(dm.f / 128) * mbound), kDenseThreads, kDenseSmem, s>>>(st.g1r, a);
    if (dm.S > 0) {
        a.shared = 1;
        a.a_base = Pm;
        a.use_mask = (use_mask && tau_shared > 0.f) ? 1 : 0;   // the shared experts' own threshold
        a.tau = tau_shared;
        a.gate = st.gate_s;
        for (int z = 0; z < dm.S; ++z) {
            DenseArgs az = a;
            az.sidx = z;
            az.h_base = Pm + z * Tm;   // shared expert z's H rows
            k_dense_gemm<<<grid((long long)(dm.f / 128) * mshared), kDenseThreads, kDenseSmem, s>>>(st.g1s, az);
        }
    }
    // GEMM2: down with the routing-weight epilogue
    a.mode = kDown;
    a.tau = tau;
    a.K = dm.f;
    a.kb = dm.f / kBK;
    a.wrows = dm.d;
    a.shared = 0;
    a.a_base = 0;
    a.use_mask = use_mask ? 1 : 0;
    k_dense_gemm<<<grid((long long)(dm.d / 256) * mbound), kDenseThreads, kDenseSmem, s>>>(st.g2r, a);
    for (int z = 0; z < dm.S; ++z) {
        DenseArgs az = a;
        az.shared = 1;
        az.sidx = z;
        az.a_base = Pm + z * Tm;
        k_dense_gemm<<<grid((long long)(dm.d / 256) * mshared), kDenseThreads, kDenseSmem, s>>>(st.g2s, az);
    }
    // convert
    {
        const size_t n4 = (size_t)T * dm.d / 4;
        size_t blocks = ((ws.ypart ? 8 : 1) * n4 + 255) / 256;   // deterministic: 8 threads per four outputs
        if (blocks > 148 * 16) blocks = 148 * 16;
        k_dense_convert<<<(unsigned)blocks, 256, 0, s>>>(ws.y_acc, out, n4, ws.error_word, ws.error_sticky, ws.ypart,
                                                         dm.k + dm.S, dm.d);
    }
    return cudaGetLastError();
}

}  // namespace moe
