// common.cuh -- small device helpers shared by the kernels.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace moe {

constexpr unsigned kFull = 0xffffffffu;

// 16-byte streaming load of weights: read once, do not keep in L1.
__device__ __forceinline__ uint4 ld_stream(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// 16-byte read-only load that may be cached (activations reused by many warps).
__device__ __forceinline__ uint4 ld_cached(const void *p)
{
    return __ldg(reinterpret_cast<const uint4 *>(p));
}

// bf16 pair (low half = element 0) -> two floats.  Exact widening.
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// One bf16 (its 16 bits) -> float.  Exact widening.
__device__ __forceinline__ float bf16_f(uint16_t v) { return __uint_as_float((uint32_t)v << 16); }

__device__ __forceinline__ void unpack8(const uint4 &v, float (&f)[8])
{
    f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
    f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
    f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
    f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

// Two fp32 lanes in one 64-bit register (element 0 in the low half), for the
// packed fp32 FMA of sm_100 (fma.rn.f32x2: each lane an ordinary fma.rn).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void f2_unpack(uint64_t v, float &lo, float &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

// bf16 pair (low half = element 0) -> the two floats, packed.  Exact widening.
__device__ __forceinline__ uint64_t bf16x2_f2(uint32_t v) { return f2_pack(bf16_lo(v), bf16_hi(v)); }

__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ float dot8(const uint4 &a, const uint4 &b, float acc)
{
    acc = fmaf(bf16_lo(a.x), bf16_lo(b.x), acc);
    acc = fmaf(bf16_hi(a.x), bf16_hi(b.x), acc);
    acc = fmaf(bf16_lo(a.y), bf16_lo(b.y), acc);
    acc = fmaf(bf16_hi(a.y), bf16_hi(b.y), acc);
    acc = fmaf(bf16_lo(a.z), bf16_lo(b.z), acc);
    acc = fmaf(bf16_hi(a.z), bf16_hi(b.z), acc);
    acc = fmaf(bf16_lo(a.w), bf16_lo(b.w), acc);
    acc = fmaf(bf16_hi(a.w), bf16_hi(b.w), acc);
    return acc;
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
    return v;
}

// Reduce N per-lane partial sums across the warp with N-1 + (5-log2 N)
// shuffles instead of 5N: each step hands half of the remaining values to
// the partner lane.  On return, lane l holds the full sum of value index
// (l >> (5 - log2 N)).  N must be a power of two <= 32.  The recursion keeps
// every array index a compile-time constant, so v stays in registers.
template <int M, int N, int O>
struct TransposeReduce {
    static __device__ __forceinline__ void run(float (&v)[M], int lane)
    {
        if constexpr (O == 0) {
            return;
        } else if constexpr (N > 1) {
            const bool upper = (lane & O) != 0;
#pragma unroll
            for (int i = 0; i < N / 2; ++i) {
                const float send = upper ? v[i] : v[i + N / 2];
                const float keep = upper ? v[i + N / 2] : v[i];
                v[i] = keep + __shfl_xor_sync(kFull, send, O);
            }
            TransposeReduce<M, N / 2, O / 2>::run(v, lane);
        } else {
            v[0] += __shfl_xor_sync(kFull, v[0], O);
            TransposeReduce<M, 1, O / 2>::run(v, lane);
        }
    }
};

template <int N>
__device__ __forceinline__ float transpose_reduce(float (&v)[N], int lane)
{
    static_assert(N >= 1 && N <= 32 && (N & (N - 1)) == 0, "N must be a power of two <= 32");
    TransposeReduce<N, N, 16>::run(v, lane);
    return v[0];
}

template <int N>
struct Log2 { static constexpr int value = 1 + Log2<N / 2>::value; };
template <>
struct Log2<1> { static constexpr int value = 0; };

__device__ __forceinline__ float silu_f(float g)
{
    return g / (1.0f + expf(-g));
}

__device__ __forceinline__ uint16_t f2bf_bits(float v)
{
    __nv_bfloat16 b = __float2bfloat16_rn(v);
    return *reinterpret_cast<uint16_t *>(&b);
}

// Deterministic combine: partials [T][rows][d] fp32, one row per
// (routing slot, neuron block) of a token, each written by exactly one
// producer with plain stores; out[t] = bf16(sum of the token's rows), the sum
// taken in one fixed order whatever the schedule was (8 lanes per four
// outputs: lane l adds rows l, l + 8, ... in turn, then a fixed butterfly
// over the 8 lanes), and every row read is re-zeroed, so rows of pairs that
// produced nothing (a dropped pair) read as zero next time.  warp0 / n_warps:
// this warp's index and the warp count of the calling grid; every lane of a
// warp runs the same iterations (the shuffles need all 32).
__device__ __forceinline__ void det_combine(float *__restrict__ part, int rows, int d, uint16_t *__restrict__ out,
                                            long long n_out4, long long warp0, long long n_warps, int lane)
{
    const int d4 = d >> 2, l8 = lane & 7;
    float4 *src = reinterpret_cast<float4 *>(part);
#pragma unroll 1
    for (long long g0 = warp0 * 4; g0 < n_out4; g0 += n_warps * 4) {
        const long long g = g0 + (lane >> 3);
        const bool valid = g < n_out4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (valid) {
            const long long t = g / d4, c4 = g % d4;
            float4 *base = src + (size_t)t * rows * d4 + c4;
            // eight rows per lane in flight at once: all loads, then the zero
            // stores (issued after the loads, so no load waits behind a store
            // it might alias), then the adds in row order
#pragma unroll 1
            for (int j0 = l8; j0 < rows; j0 += 64) {
                float4 v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    v[u] = j0 + 8 * u < rows ? __ldcg(base + (size_t)(j0 + 8 * u) * d4) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    if (j0 + 8 * u < rows) __stcg(base + (size_t)(j0 + 8 * u) * d4, make_float4(0.f, 0.f, 0.f, 0.f));
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    if (j0 + 8 * u < rows) {
                        acc.x += v[u].x;
                        acc.y += v[u].y;
                        acc.z += v[u].z;
                        acc.w += v[u].w;
                    }
            }
        }
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) {
            acc.x += __shfl_xor_sync(0xffffffffu, acc.x, o);
            acc.y += __shfl_xor_sync(0xffffffffu, acc.y, o);
            acc.z += __shfl_xor_sync(0xffffffffu, acc.z, o);
            acc.w += __shfl_xor_sync(0xffffffffu, acc.w, o);
        }
        if (valid && l8 == 0) {
            uint2 p;
            p.x = (uint32_t)f2bf_bits(acc.x) | ((uint32_t)f2bf_bits(acc.y) << 16);
            p.y = (uint32_t)f2bf_bits(acc.z) | ((uint32_t)f2bf_bits(acc.w) << 16);
            reinterpret_cast<uint2 *>(out)[g] = p;
        }
    }
}

}  // namespace moe
