// kvq_warp.cuh -- warp-level helpers shared by the decode kernels: the full
// lane mask, the bounded-wait limit, a base-2 exponential, the fp32
// Walsh-Hadamard transform of a head_dim vector spread over a warp and the
// bit-reversal permutation of such a vector.
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

// OSCAR's bit-reversal permutation P_br of a warp-wide vector (element
// lane*E + e): element j becomes element br(j) of the input, br reversing the
// log2(D) bits of the index.  br is its own inverse, so the same call undoes
// it.  A lane gathers its E elements with E shuffles each (one per possible
// source register) and keeps the right one.
template <int D> __device__ __forceinline__ int bitrev_index(int j)
{
    constexpr int BITS = D == 128 ? 7 : D == 64 ? 6 : D == 32 ? 5 : 0;
    static_assert(BITS > 0, "head_dim 32, 64 or 128");
    return (int)(__brev((unsigned)j) >> (32 - BITS));
}

template <int D>
__device__ __forceinline__ void warp_bitrev(float (&x)[D / 32], int lane)
{
    constexpr int E = D / 32;
    float y[E];
#pragma unroll
    for (int e = 0; e < E; e++) {
        const int i = bitrev_index<D>(lane * E + e);  // the source element
        const int src = i / E, se = i % E;
        float v = 0.f;
#pragma unroll
        for (int r = 0; r < E; r++) {
            const float t = __shfl_sync(kFull, x[r], src);
            v = r == se ? t : v;
        }
        y[e] = v;
    }
#pragma unroll
    for (int e = 0; e < E; e++) x[e] = y[e];
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

// A head_dim-128 fp16 row at `src` as rotated fp32, lane holding elements
// 4 lane .. 4 lane + 3: signs flipped on the fp16 bits (exact), the
// butterflies of fwht_warp, then each value times rot_scale (rounded once);
// the raw values when the cache does not rotate.
__device__ __forceinline__ void rotated_row_lane4(const AppendParams &p, const __half *src, int lane, float (&x)[4])
{
    uint2 raw = *reinterpret_cast<const uint2 *>(src + 4 * lane);
    if (p.rotate) {
        raw.x ^= p.sign_xor[2 * lane];
        raw.y ^= p.sign_xor[2 * lane + 1];
    }
    const float2 a = __half22float2(bits_h2(raw.x)), b = __half22float2(bits_h2(raw.y));
    x[0] = a.x;
    x[1] = a.y;
    x[2] = b.x;
    x[3] = b.y;
    if (p.rotate) {
        fwht_warp<128>(x, lane);
#pragma unroll
        for (int e = 0; e < 4; e++) x[e] = __fmul_rn(x[e], p.rot_scale);
    }
}

}  // namespace kvq
