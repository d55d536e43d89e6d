// kvq_warp.cuh -- warp-level helpers shared by the decode kernels: the full
// lane mask, the bounded-wait limit, a base-2 exponential and the fp32
// Walsh-Hadamard transform of a head_dim vector spread over a warp.
#pragma once

#include "kvq_internal.cuh"

namespace kvq {

constexpr unsigned kFull = 0xffffffffu;
constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // 1 s per bounded wait

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Walsh-Hadamard transform of a warp-wide vector (element lane*E + e), fp32,
// Sylvester order: butterfly stages h = 1, 2, 4, ..., D/2 in that order.
template <int D>
__device__ __forceinline__ void fwht_warp(float (&x)[D / 32], int lane)
{
    constexpr int E = D / 32;
#pragma unroll
    for (int h = 1; h < E; h <<= 1)
#pragma unroll
        for (int e = 0; e < E; e++)
            if (!(e & h)) {
                const float a = x[e], b = x[e + h];
                x[e] = a + b;
                x[e + h] = a - b;
            }
#pragma unroll
    for (int m = 1; m < 32; m <<= 1)
#pragma unroll
        for (int e = 0; e < E; e++) {
            const float o = __shfl_xor_sync(kFull, x[e], m);
            x[e] = (lane & m) ? (o - x[e]) : (x[e] + o);
        }
}

// Two vectors transformed together (independent shuffle chains interleave).
template <int D>
__device__ __forceinline__ void fwht_warp2(float (&x)[D / 32], float (&y)[D / 32], int lane)
{
    constexpr int E = D / 32;
#pragma unroll
    for (int h = 1; h < E; h <<= 1)
#pragma unroll
        for (int e = 0; e < E; e++)
            if (!(e & h)) {
                const float a = x[e], b = x[e + h], c = y[e], d = y[e + h];
                x[e] = a + b;
                x[e + h] = a - b;
                y[e] = c + d;
                y[e + h] = c - d;
            }
#pragma unroll
    for (int m = 1; m < 32; m <<= 1)
#pragma unroll
        for (int e = 0; e < E; e++) {
            const float o = __shfl_xor_sync(kFull, x[e], m), q = __shfl_xor_sync(kFull, y[e], m);
            x[e] = (lane & m) ? (o - x[e]) : (x[e] + o);
            y[e] = (lane & m) ? (q - y[e]) : (y[e] + q);
        }
}

}  // namespace kvq
