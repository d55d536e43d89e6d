// kvq_cert.cuh -- device helpers shared by the certified-mode kernels
// (kvq_certified.cu: bounds, fixed-fraction selection, promotion;
// kvq_ladder.cu: the adaptive ladder): dependent launch, the rotated query,
// dequantisation of one lane's channels, the online-softmax update, raw fp16
// row loads, a CTA-wide bitonic sort of 64-bit keys and CTA-wide scans.
#pragma once

#include <math.h>

#include "kvq_internal.cuh"
#include "kvq_warp.cuh"

namespace kvq {
namespace cert {

constexpr int kSelThreads = 512;   // selection / ladder CTAs
constexpr int kBlkRec = 12;        // block record: P[8], eps, eta, nu, pad
constexpr int kPromWarps = 8;
constexpr int kPromThreads = kPromWarps * 32;
constexpr int kTokBatch = 8;       // tokens whose exact rows a warp has in flight

// Programmatic dependent launch: wait for the stream's previous grid to
// complete (its writes visible) before any memory access, then allow the next
// grid to be set up; only launch latency is hidden, no work overlaps.
__device__ __forceinline__ void pdl_enter()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename Kern>
cudaError_t launch_pdl(Kern kernel, dim3 grid, int threads, size_t smem, cudaStream_t s, const CertParams &p)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, p);
}

__device__ __forceinline__ int clamp_ctx(int T, int max_pages)
{
    return T < 0 ? 0 : (T > max_pages * kPageTokens ? max_pages * kPageTokens : T);
}

// The rotated query row of head (b, head) in lane order: element lane*E + e.
template <int D>
__device__ __forceinline__ void rotated_query(const CertParams &p, int b, int head, int lane, float (&x)[D / 32])
{
    constexpr int E = D / 32;
    const __half *qh = p.q + ((long long)b * p.L.hq + head) * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; e++) x[e] = __half2float(qh[e]);
    if (p.rotate) {
#pragma unroll
        for (int e = 0; e < E; e++) x[e] *= p.signs[lane * E + e];
        fwht_warp<D>(x, lane);
#pragma unroll
        for (int e = 0; e < E; e++) x[e] *= p.rot_scale;
        if (p.rotate == 2) warp_bitrev<D>(x, lane);  // ["OSCAR", 2.2(a)] P_br after H
    }
}

// Dequantised values of channels lane*E .. lane*E+E-1 of token `tok` in a
// chunk (the same arithmetic as the stored codec: code*scale + zero, one
// rounding; int8: code*scale).  The lane's codes are E*bits consecutive bits
// of the token's stream (4, 8, 16 or 32 bits, aligned to their size, inside
// one 16-byte chunk): one load, then shifts.
template <int E>
__device__ __forceinline__ void dequant_lane(const unsigned char *chunk, int codes_off, int meta_off, int row_meta,
                                             int fmt, int tok, int lane, float (&x)[E])
{
    const unsigned char *codes = chunk + codes_off;
    const uint16_t *meta = reinterpret_cast<const uint16_t *>(chunk + meta_off + tok * row_meta);
    const int bits = fmt_bits(fmt);
    const int bit0 = lane * E * bits, byte0 = bit0 >> 3;
    const unsigned char *src = codes + ((byte0 >> 4) * 16 + tok) * 16 + (byte0 & 15);
    const int nbits = E * bits;
    uint32_t w;
    if (nbits == 32) w = *reinterpret_cast<const uint32_t *>(src);
    else if (nbits == 16) w = *reinterpret_cast<const uint16_t *>(src);
    else w = *src >> (bit0 & 7);
    const uint32_t mask = (1u << bits) - 1u;
    if (fmt == KVQ_INT8_SYM) {
        const float s = __half2float(__ushort_as_half(meta[0]));
#pragma unroll
        for (int e = 0; e < E; e++) x[e] = __fmul_rn((float)(int)(int8_t)((w >> (8 * e)) & 0xFFu), s);
    } else {
        const int ng = row_meta / 4;  // asymmetric formats: scales then zeros
        const int gi = fmt == KVQ_INT4_ASYM ? (lane * E) / 32 : 0;
        const float s = __half2float(__ushort_as_half(meta[gi])), z = __half2float(__ushort_as_half(meta[ng + gi]));
#pragma unroll
        for (int e = 0; e < E; e++) x[e] = __fmaf_rn((float)((w >> (bits * e)) & mask), s, z);
    }
}

template <int E>
__device__ __forceinline__ void online_update(float &m, float &l, float (&a)[E], float s, const float (&v)[E])
{
    const float mn = fmaxf(m, s);
    const float al = (m == -INFINITY) ? 0.f : ex2(m - mn);
    const float pe = ex2(s - mn);
    l = fmaf(l, al, pe);
#pragma unroll
    for (int e = 0; e < E; e++) a[e] = fmaf(a[e], al, pe * v[e]);
    m = mn;
}

// A lane's E fp16 values of a row, kept raw (the loads stay in flight in
// half the registers) and widened when used.
template <int E> struct RawRow;
template <> struct RawRow<4> {
    uint2 u;
    __device__ void load(const __half *src) { u = *reinterpret_cast<const uint2 *>(src); }
    __device__ void widen(float (&x)[4]) const
    {
        const float2 a = __half22float2(bits_h2(u.x)), c = __half22float2(bits_h2(u.y));
        x[0] = a.x;
        x[1] = a.y;
        x[2] = c.x;
        x[3] = c.y;
    }
};
template <> struct RawRow<2> {
    uint32_t u;
    __device__ void load(const __half *src) { u = *reinterpret_cast<const uint32_t *>(src); }
    __device__ void widen(float (&x)[2]) const
    {
        const float2 a = __half22float2(bits_h2(u));
        x[0] = a.x;
        x[1] = a.y;
    }
};

// Transpose-reduce: each lane holds 32 partial sums v[0..31] (index i); after
// five halving exchanges lane j holds the warp-wide total of index j.  At the
// step with offset o a lane keeps the half whose index bit log2(o) equals its
// own lane bit and adds the partner's copy of that half: 31 shuffles for 32
// totals (instead of 32 five-step butterflies).
__device__ __forceinline__ float transpose_reduce32(float (&v)[32], int lane)
{
#pragma unroll
    for (int k = 0; k < 16; k++) {
        const bool up = lane & 16;
        const float send = up ? v[k] : v[k + 16], keep = up ? v[k + 16] : v[k];
        v[k] = keep + __shfl_xor_sync(kFull, send, 16);
    }
#pragma unroll
    for (int k = 0; k < 8; k++) {
        const bool up = lane & 8;
        const float send = up ? v[k] : v[k + 8], keep = up ? v[k + 8] : v[k];
        v[k] = keep + __shfl_xor_sync(kFull, send, 8);
    }
#pragma unroll
    for (int k = 0; k < 4; k++) {
        const bool up = lane & 4;
        const float send = up ? v[k] : v[k + 4], keep = up ? v[k + 4] : v[k];
        v[k] = keep + __shfl_xor_sync(kFull, send, 4);
    }
#pragma unroll
    for (int k = 0; k < 2; k++) {
        const bool up = lane & 2;
        const float send = up ? v[k] : v[k + 2], keep = up ? v[k + 2] : v[k];
        v[k] = keep + __shfl_xor_sync(kFull, send, 2);
    }
    const bool up = lane & 1;
    const float send = up ? v[0] : v[1], keep = up ? v[1] : v[0];
    return keep + __shfl_xor_sync(kFull, send, 1);
}

// Sort keys[0..np2) (np2 a power of two) in descending order with NT
// threads; keys past the live entries must be 0.  Up to 2*NT keys stay in
// registers (two per thread, warp shuffles for the stages whose partner is
// under 32 keys away, shared memory for the wider ones); more are sorted in
// shared memory.  Call with every thread of the CTA; ends synchronised.
template <int NT>
__device__ __forceinline__ void sort_keys_desc(unsigned long long *keys, int np2, int tid)
{
    __syncthreads();
    if (np2 <= 2 * NT) {
        unsigned long long v[2];
#pragma unroll
        for (int c = 0; c < 2; c++) v[c] = tid + c * NT < np2 ? keys[tid + c * NT] : 0ull;
        for (int k = 2; k <= np2; k <<= 1)
            for (int jj = k >> 1; jj > 0; jj >>= 1) {
                unsigned long long o[2];
                if (jj >= 32) {
                    __syncthreads();  // the last stage's reads are done
#pragma unroll
                    for (int c = 0; c < 2; c++)
                        if (tid + c * NT < np2) keys[tid + c * NT] = v[c];
                    __syncthreads();
#pragma unroll
                    for (int c = 0; c < 2; c++) o[c] = tid + c * NT < np2 ? keys[(tid + c * NT) ^ jj] : 0ull;
                } else {
#pragma unroll
                    for (int c = 0; c < 2; c++) o[c] = __shfl_xor_sync(kFull, v[c], jj);
                }
#pragma unroll
                for (int c = 0; c < 2; c++) {
                    const int i = tid + c * NT;
                    const bool lower = (i & jj) == 0, desc = (i & k) == 0;
                    const unsigned long long hi = v[c] > o[c] ? v[c] : o[c], lo = v[c] > o[c] ? o[c] : v[c];
                    v[c] = (lower == desc) ? hi : lo;
                }
            }
        __syncthreads();
#pragma unroll
        for (int c = 0; c < 2; c++)
            if (tid + c * NT < np2) keys[tid + c * NT] = v[c];
    } else {
        for (int k = 2; k <= np2; k <<= 1)
            for (int jj = k >> 1; jj > 0; jj >>= 1) {
                for (int i = tid; i < np2; i += NT) {
                    const int ixj = i ^ jj;
                    if (ixj > i) {
                        const unsigned long long a = keys[i], c = keys[ixj];
                        const bool desc = (i & k) == 0;
                        if (desc ? (a < c) : (a > c)) {
                            keys[i] = c;
                            keys[ixj] = a;
                        }
                    }
                }
                __syncthreads();
            }
    }
    __syncthreads();
}

// Key of a sort entry: the non-negative float's bits, then the complement of
// the index (equal scores order the lower index first); index of a key.
__device__ __forceinline__ unsigned long long sort_key(float score, int idx)
{
    if (!(score >= 0.f)) score = 0.f;
    return ((unsigned long long)__float_as_uint(score) << 32) | (unsigned long long)(0xFFFFFFFFu - (unsigned)idx);
}
__device__ __forceinline__ int key_index(unsigned long long key)
{
    return (int)(0xFFFFFFFFu - (unsigned)(key & 0xFFFFFFFFull));
}

struct SumOp {
    __device__ static float id() { return 0.f; }
    __device__ static float op(float a, float b) { return a + b; }
};
struct MaxOp {
    __device__ static float id() { return -INFINITY; }
    __device__ static float op(float a, float b) { return fmaxf(a, b); }
};

// CTA-wide exclusive scan of the first `n_used` of N values per thread in
// thread order (REV: reverse thread order, i.e. over the threads after this
// one), and their totals; entries from n_used on are left as they are.
// sm: NT/32 * N floats.  Every thread of the CTA calls it with the same
// n_used; ends synchronised.
template <int NT, int N, bool REV, typename Op>
__device__ __forceinline__ void block_scan(float (&v)[N], float (&total)[N], float *sm, int tid, int n_used = N)
{
    constexpr int NW = NT / 32;
    static_assert(NW <= 32, "one warp scans the warp totals");
    const int lane = tid & 31, warp = tid >> 5;
    __syncthreads();  // sm may still be read by a previous call
#pragma unroll
    for (int n = 0; n < N; n++) {
        if (n >= n_used) break;
        float inc = v[n];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float t = REV ? __shfl_down_sync(kFull, inc, o) : __shfl_up_sync(kFull, inc, o);
            if (REV ? lane + o < 32 : lane >= o) inc = Op::op(inc, t);
        }
        // exclusive within the warp: the inclusive value of the neighbour
        const float nb = REV ? __shfl_down_sync(kFull, inc, 1) : __shfl_up_sync(kFull, inc, 1);
        v[n] = (REV ? lane == 31 : lane == 0) ? Op::id() : nb;
        if (lane == (REV ? 0 : 31)) sm[warp * N + n] = inc;
    }
    __syncthreads();
    // every warp scans the warp totals (lane w holds warp w's) with shuffles
#pragma unroll
    for (int n = 0; n < N; n++) {
        if (n >= n_used) break;
        const float x = lane < NW ? sm[lane * N + n] : Op::id();
        float inc = x;
#pragma unroll
        for (int o = 1; o < NW; o <<= 1) {
            const float t = REV ? __shfl_down_sync(kFull, inc, o) : __shfl_up_sync(kFull, inc, o);
            if (REV ? lane + o < NW : lane >= o) inc = Op::op(inc, t);
        }
        const bool has = REV ? warp + 1 < NW : warp >= 1;  // warps before this one (after, REV)
        const float nbr = __shfl_sync(kFull, inc, REV ? (has ? warp + 1 : 0) : (has ? warp - 1 : 0));
        const float b = has ? nbr : Op::id();
        total[n] = __shfl_sync(kFull, inc, REV ? 0 : NW - 1);
        v[n] = Op::op(b, v[n]);
    }
    __syncthreads();
}

}  // namespace cert
}  // namespace kvq
