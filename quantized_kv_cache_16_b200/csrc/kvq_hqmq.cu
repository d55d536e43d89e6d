// kvq_hqmq.cu -- the HQMQ codec ["Hurwitz Quaternion Multiplicative
// Quantization for KV Cache Compression", 1-3] on the paged pool:
// quantise-on-append of K/V rows into 20-bit quaternion codes with Med3x
// fp16 outliers, and split-K decode attention over those codes.
//
// Append.  A warp holds one rotated row of 128 elements, lane b owning the
// quaternion block b (elements 4b..4b+3), so the row statistics (radii, the
// lower median by a bitonic sort across lanes, the two largest outliers by
// warp max-reductions) are shuffles and the code of block b is lane b's.
// The codeword search dominates: for each of the 1024 secondary quaternions
// q_s, w = u conj(q_s) and the best of the 24 Hurwitz units is closed-form
// (largest |w_i| or half the sum of |w_i|), 16 multiplies, 12 adds and a
// handful of max/compare operations per candidate; conj(q_s) comes from
// shared memory as one broadcast 16-byte load.  Every operation that decides
// a code is an explicitly rounded fp32 operation in the order kvq.h states,
// so codes match a plain fp32 statement bit for bit.  When there are few rows
// (a decode step appends one token), the 1024 candidates of a row are split
// over the CTA's 8 warps and the per-block winners combined (highest score,
// lowest candidate on ties, which is the sequential rule).
//
// Decode.  CTAs take contiguous page ranges of one (sequence, kv head) and
// hold that head's two codebooks in shared memory (32 KB); each warp streams
// whole 16-token pages into a shared-memory ring by bulk copy.  Lanes rebuild
// K and V blocks as (radius code x step) x q_p q_s (or the fp16 outlier)
// straight into fp16 tensor-core fragments (K, V, the query and the weights
// as hi + lo fp16 pairs, ~22 bits each): scores as K Q^T and the output as V^T P^T
// (m16n8k16, M = tokens or dims, N = 8 heads), with the block-to-
// fragment assignment chosen (a permutation of the contraction index and of
// the output rows) so that every lane rebuilds whole blocks and the score
// fragments become P^T by two 8x8 transposes.  Split partials merge in the
// last CTA of each (sequence, kv head), which also applies the inverse
// rotation.  Rebuilding blocks (lookups and a 16-term quaternion product)
// dominates: the path is bound by instruction issue, not by HBM.
#include <math.h>

#include "kvq_internal.cuh"
#include "kvq_warp.cuh"

namespace kvq {
namespace {

constexpr int kHqWarps = 8;
constexpr int kHqThreads = kHqWarps * 32;
constexpr int kHqD = 128;          // head_dim of HQMQ caches
constexpr int kHqRowCode = 80;     // 32 blocks x 20 bits
constexpr int kHqTok = 8;          // tokens a decode warp has in flight
constexpr unsigned kHqFieldMask = 0xFFFFFu;

// ------------------------------------------------------------------ append --

// w = u c for unit direction u and codeword conj(q_s) = c, exactly as kvq.h
// states: each component is its first product, rounded, then the other three
// products added in order by fused multiply-adds (a subtracted product as
// one with its first factor negated).
__device__ __forceinline__ void hamilton_rn(const float (&u)[4], float4 c, float (&w)[4])
{
    w[0] = __fmaf_rn(-u[3], c.w, __fmaf_rn(-u[2], c.z, __fmaf_rn(-u[1], c.y, __fmul_rn(u[0], c.x))));
    w[1] = __fmaf_rn(-u[3], c.z, __fmaf_rn(u[2], c.w, __fmaf_rn(u[1], c.x, __fmul_rn(u[0], c.y))));
    w[2] = __fmaf_rn(u[3], c.y, __fmaf_rn(u[2], c.x, __fmaf_rn(-u[1], c.w, __fmul_rn(u[0], c.z))));
    w[3] = __fmaf_rn(u[3], c.x, __fmaf_rn(-u[2], c.y, __fmaf_rn(u[1], c.z, __fmul_rn(u[0], c.w))));
}

__device__ __forceinline__ int unit_of(const float (&u)[4], float4 c)
{
    float w[4];
    hamilton_rn(u, c, w);
    float aw[4];
#pragma unroll
    for (int i = 0; i < 4; i++) aw[i] = fabsf(w[i]);
    int ia = 0;
    float ma = aw[0];
#pragma unroll
    for (int i = 1; i < 4; i++)
        if (aw[i] > ma) {
            ma = aw[i];
            ia = i;
        }
    const float mh = __fmul_rn(__fadd_rn(__fadd_rn(__fadd_rn(aw[0], aw[1]), aw[2]), aw[3]), 0.5f);
    if (mh > ma) return 8 + (w[0] < 0.f) + 2 * (w[1] < 0.f) + 4 * (w[2] < 0.f) + 8 * (w[3] < 0.f);
    return 2 * ia + (w[ia] < 0.f);
}

// ascending bitonic sort of one float per lane across the warp
__device__ __forceinline__ float warp_sort_asc(float v, int lane)
{
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            const float o = __shfl_xor_sync(kFull, v, j);
            const bool up = (lane & k) == 0 || k == 32;
            const bool low = (lane & j) == 0;
            v = (low == up) ? fminf(v, o) : fmaxf(v, o);
        }
    return v;
}

// One row's statistics and codes, every lane of the warp (lane = block).
struct HqRow {
    float x[4];      // rotated values of the lane's block
    float u[4];      // unit direction (r > 0)
    float r;         // radius
    unsigned rc;     // radius code
    uint32_t mask;   // outlier blocks
    __half step;
};

__device__ __forceinline__ void hq_prepare(const AppendParams &p, const __half *src, int lane, HqRow &R)
{
    float x[4];
    rotated_row_lane4(p, src, lane, x);  // butterfly stages h = 1, 2, ..., 64, each add rounded
#pragma unroll
    for (int e = 0; e < 4; e++) R.x[e] = x[e];
    const float r = __fsqrt_rn(__fadd_rn(__fadd_rn(__fadd_rn(__fmul_rn(x[0], x[0]), __fmul_rn(x[1], x[1])),
                                                   __fmul_rn(x[2], x[2])),
                                         __fmul_rn(x[3], x[3])));
    R.r = r;
    // Med3x: tau = 3 x the lower median radius (the 16th smallest of 32)
    const float med = __shfl_sync(kFull, warp_sort_asc(r, lane), 15);
    const float tau = __fmul_rn(3.0f, med);
    // outliers: the largest radius above tau, then the next (lowest block on ties);
    // radii above tau are positive, so their bit patterns order like the values
    const bool over = r > tau;
    const unsigned rb = __float_as_uint(r);
    const unsigned m1 = __reduce_max_sync(kFull, over ? rb : 0u);
    const unsigned b1 = __ballot_sync(kFull, over && rb == m1);
    const int pick1 = b1 ? __ffs(b1) - 1 : -1;
    const bool over2 = over && lane != pick1;
    const unsigned m2 = __reduce_max_sync(kFull, over2 ? rb : 0u);
    const unsigned b2 = __ballot_sync(kFull, over2 && rb == m2);
    const int pick2 = b2 ? __ffs(b2) - 1 : -1;
    R.mask = (pick1 >= 0 ? 1u << pick1 : 0u) | (pick2 >= 0 ? 1u << pick2 : 0u);
    // radius step and code
    R.step = __float2half_ru(__fdiv_rn(tau, 31.0f));
    const float sf = __half2float(R.step);
    unsigned rc = 0;
    if (sf > 0.0f) {
        const float v = rintf(__fdiv_rn(r, sf));
        rc = v > 31.0f ? 31u : (unsigned)v;
    }
    R.rc = min(rc, 31u);  // (a NaN radius must not spill into the next field)
#pragma unroll
    for (int e = 0; e < 4; e++) R.u[e] = r > 0.0f ? __fdiv_rn(x[e], r) : 0.0f;
}

// Best candidate of s in [s0, s1) (s0, s1 even): strictly higher score
// wins, so the first of equal scores stays.  Two candidates per step with
// packed f32x2 products and fused multiply-adds (four products and twelve
// multiply-adds per pair instead of 28 scalar operations per candidate).
// Table entries 2j, 2j + 1 hold candidates 2j and 2j + 1 interleaved:
// (c0(2j), c0(2j+1), c1(2j), c1(2j+1)), (c2(2j), c2(2j+1), c3(2j), c3(2j+1)).
__device__ __forceinline__ float pair_score(float2 w0, float2 w1, float2 w2, float2 w3, bool hi)
{
    const float a0 = fabsf(hi ? w0.y : w0.x), a1 = fabsf(hi ? w1.y : w1.x), a2 = fabsf(hi ? w2.y : w2.x),
                a3 = fabsf(hi ? w3.y : w3.x);
    const float ma = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
    const float mh = __fmul_rn(__fadd_rn(__fadd_rn(__fadd_rn(a0, a1), a2), a3), 0.5f);
    return mh > ma ? mh : ma;
}

// Packed f32x2 multiply and fused multiply-add (each lane rounds as the
// scalar operation does).
__device__ __forceinline__ unsigned long long pk(float2 v)
{
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(v.x), "f"(v.y));
    return r;
}
__device__ __forceinline__ float2 upk(unsigned long long r)
{
    float2 v;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
    return v;
}
__device__ __forceinline__ unsigned long long mul2(unsigned long long a, unsigned long long b)
{
    unsigned long long d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b, unsigned long long c)
{
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ void hq_search(const float (&u)[4], const float4 *cb2, int s0, int s1, float &best, int &bs)
{
    const unsigned long long U0 = pk(make_float2(u[0], u[0])), U1 = pk(make_float2(u[1], u[1])),
                             U2 = pk(make_float2(u[2], u[2])), U3 = pk(make_float2(u[3], u[3]));
    const unsigned long long N1 = pk(make_float2(-u[1], -u[1])), N2 = pk(make_float2(-u[2], -u[2])),
                             N3 = pk(make_float2(-u[3], -u[3]));
    best = -INFINITY;
    bs = s0;
#pragma unroll 2
    for (int s = s0; s < s1; s += 2) {
        const float4 a = cb2[s], b = cb2[s + 1];  // (pair s/2 occupies entries s and s + 1)
        const unsigned long long C0 = pk(make_float2(a.x, a.y)), C1 = pk(make_float2(a.z, a.w)),
                                 C2 = pk(make_float2(b.x, b.y)), C3 = pk(make_float2(b.z, b.w));
        const float2 w0 = upk(fma2(N3, C3, fma2(N2, C2, fma2(N1, C1, mul2(U0, C0)))));
        const float2 w1 = upk(fma2(N3, C2, fma2(U2, C3, fma2(U1, C0, mul2(U0, C1)))));
        const float2 w2 = upk(fma2(U3, C1, fma2(U2, C0, fma2(N1, C3, mul2(U0, C2)))));
        const float2 w3 = upk(fma2(U3, C0, fma2(N2, C1, fma2(U1, C2, mul2(U0, C3)))));
        const float sa = pair_score(w0, w1, w2, w3, false), sb = pair_score(w0, w1, w2, w3, true);
        if (sa > best) {
            best = sa;
            bs = s;
        }
        if (sb > best) {
            best = sb;
            bs = s + 1;
        }
    }
}

// Candidate s of the interleaved table as conj(q_s).
__device__ __forceinline__ float4 cand(const float4 *cb2, int s)
{
    const float4 a = cb2[s & ~1], b = cb2[s | 1];
    return (s & 1) ? make_float4(a.y, a.w, b.y, b.w) : make_float4(a.x, a.z, b.x, b.z);
}

// Pack and store a coded row: fields as one little-endian 20-bit stream
// (lane k < 20 writes 32-bit word k), then the meta row.
__device__ __forceinline__ void hq_store(unsigned char *codes, unsigned char *meta, uint32_t field, const HqRow &R,
                                         int lane)
{
    const int blo = (32 * lane) / 20, sh = 32 * lane - 20 * blo;
    const uint32_t f0 = __shfl_sync(kFull, field, min(blo, 31));
    const uint32_t f1 = __shfl_sync(kFull, field, min(blo + 1, 31));
    const uint32_t f2 = __shfl_sync(kFull, field, min(blo + 2, 31));
    const unsigned long long v = (unsigned long long)f0 | ((unsigned long long)(blo + 1 <= 31 ? f1 : 0u) << 20) |
                                 ((unsigned long long)(blo + 2 <= 31 ? f2 : 0u) << 40);
    if (lane < kHqRowCode / 4) reinterpret_cast<uint32_t *>(codes)[lane] = (uint32_t)(v >> sh);
    const int nout = __popc(R.mask);
    if (lane == 0) reinterpret_cast<uint32_t *>(meta)[0] = (uint32_t)__half_as_ushort(R.step);
    if (lane == 1) reinterpret_cast<uint32_t *>(meta)[1] = R.mask;
    if ((R.mask >> lane) & 1u) {
        const int slot = __popc(R.mask & ((1u << lane) - 1u));
        const __half2 h01 = __floats2half2_rn(R.x[0], R.x[1]), h23 = __floats2half2_rn(R.x[2], R.x[3]);
        reinterpret_cast<uint2 *>(meta + 8)[slot] = make_uint2(h2_bits(h01), h2_bits(h23));
    }
    if (lane >= 2 && lane < 2 + kHqmqOut && lane - 2 >= nout)
        reinterpret_cast<uint2 *>(meta + 8)[lane - 2] = make_uint2(0u, 0u);
}

// Grid (CTAs per (kv head, tensor), 2 Hkv): the CTA loads conj(S) of its
// (kv head, tensor) once, then codes rows of tokens n = its own, stride all
// of its column.  WPR warps share a row (1: a warp a row; 8: the CTA a row).
template <int WPR>
__global__ void __launch_bounds__(kHqThreads) hqmq_append_kernel(const __grid_constant__ AppendParams p)
{
    constexpr int RPC = kHqWarps / WPR;  // rows per CTA pass
    constexpr int SPAN = kHqmqNS / WPR;  // candidates per warp
    __shared__ float4 cb2[kHqmqNS];  // conj(S), candidates interleaved in pairs (see hq_search)
    __shared__ float wsc[WPR > 1 ? 2 : 1][kHqWarps][32];
    __shared__ int wsi[WPR > 1 ? 2 : 1][kHqWarps][32];
    const int pair = blockIdx.y, kvh = pair >> 1, tensor = pair & 1;
    const Layout &L = p.L;
    {
        const float4 *S = reinterpret_cast<const float4 *>(p.pool + L.hq_tab) + (long long)pair * kHqmqNS;
        for (int j = threadIdx.x; j < kHqmqNS / 2; j += kHqThreads) {
            const float4 a = S[2 * j], b = S[2 * j + 1];  // conj: exact sign flips
            cb2[2 * j] = make_float4(a.x, b.x, -a.y, -b.y);
            cb2[2 * j + 1] = make_float4(-a.z, -b.z, -a.w, -b.w);
        }
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rgrp = warp / WPR, slice = warp % WPR;
    const int stride = gridDim.x * RPC;
    int par = 0;
    for (int base = blockIdx.x * RPC; base < p.n_tok; base += stride, par ^= 1) {
        const int n = base + rgrp;
        bool active = n < p.n_tok;
        int slot = active ? p.slots[n] : -1;
        if (slot < 0) active = false;
        if (active && slot >= L.num_pages * kPageTokens) {
            if (lane == 0 && slice == 0) set_status(p.pool, KVQ_ERR_OUT_OF_RANGE);
            active = false;
        }
        float best = -INFINITY;
        int bs = 0;
        HqRow R{};
        if (active) {  // warp-uniform
            const __half *src = (tensor ? p.v : p.k) + ((long long)n * L.hkv + kvh) * kHqD;
            hq_prepare(p, src, lane, R);
            hq_search(R.u, cb2, slice * SPAN, slice * SPAN + SPAN, best, bs);
        }
        if constexpr (WPR > 1) {
            wsc[par][warp][lane] = best;
            wsi[par][warp][lane] = bs;
            __syncthreads();  // (two buffers: the next pass writes the other one)
            if (slice == 0) {
#pragma unroll
                for (int w = 1; w < WPR; w++) {
                    const float o = wsc[par][rgrp * WPR + w][lane];
                    if (o > best) {
                        best = o;
                        bs = wsi[par][rgrp * WPR + w][lane];
                    }
                }
            }
        }
        if (active && slice == 0) {
            const bool outl = (R.mask >> lane) & 1u;
            uint32_t field = 0;
            if (!outl) {
                const uint32_t idx = R.r > 0.0f ? (uint32_t)(24 * bs + unit_of(R.u, cand(cb2, bs))) : 0u;
                field = idx | (R.rc << 15);
            }
            const int page = slot / kPageTokens, tok = slot % kPageTokens;
            unsigned char *chunk =
                p.pool + kHeaderBytes + (long long)page * L.page_bytes + (long long)kvh * L.chunk_bytes;
            unsigned char *codes = chunk + (tensor ? L.v_codes : L.k_codes) + tok * kHqRowCode;
            unsigned char *meta = chunk + (tensor ? L.v_meta : L.k_meta) + tok * kHqmqRowMeta;
            hq_store(codes, meta, field, R, lane);
        }
    }
}

// ------------------------------------------------------------------ decode --

// A (page, kv head) chunk of an HQMQ pool: K codes, K meta, V codes, V meta
// of 16 tokens; the decode copies it whole into shared memory.
constexpr int kHqChunk = 2 * kPageTokens * (kHqRowCode + kHqmqRowMeta);  // 3328 bytes
constexpr int kHqStages = 2;                                                // per warp
constexpr int kHqTabBytes = 2 * kHqmqNS * 16;
constexpr int kHqOffStage = kHqTabBytes;
constexpr int kHqOffBar = kHqOffStage + kHqWarps * kHqStages * kHqChunk;
constexpr int kHqSmem = kHqOffBar + kHqWarps * kHqStages * 8;
static_assert(kHqChunk % 16 == 0 && kHqOffStage % 16 == 0 && kHqOffBar % 8 == 0, "bulk copy alignment");
constexpr int kHqMaxSplits = 64;  // the merge holds one weight per split in registers (two per lane)

// The 20-bit field of block `blk` in a token's code row (shared memory).
__device__ __forceinline__ uint32_t hq_field(const unsigned char *row, int blk)
{
    const uint32_t *w = reinterpret_cast<const uint32_t *>(row);
    const int bit = 20 * blk, w0 = bit >> 5, sh = bit & 31;
    const uint32_t lo = w[w0];
    const uint32_t hi = sh > 12 ? w[w0 + 1] : 0u;  // word 20 is never needed
    return __funnelshift_r(lo, hi, sh) & kHqFieldMask;
}

// Block `blk` of a row: (radius code x step) x q_p q_s with q_s from the
// codebook and q_p from the unit table (both in shared memory), or the fp16
// outlier values.  meta = the row's meta (shared memory): step | 0, outlier
// mask, two outlier slots.  The unit table holds 8 copies of the 24 units,
// copy r of unit p at p * 8 + r: a lane reads copy `cpy` = lane % 8, so the
// eight lanes of each 16-byte load phase hit eight different bank groups.
__device__ __forceinline__ void hq_block(uint32_t f, const unsigned char *meta, const float4 *S, const float4 *units,
                                         int blk, int cpy, float (&c)[4])
{
    const uint2 mm = *reinterpret_cast<const uint2 *>(meta);
    const uint32_t idx = f & 0x7FFFu, sq = idx / 24u, pp = idx - 24u * sq;
    const float4 q = S[min(sq, (uint32_t)kHqmqNS - 1u)];
    const float rad = (float)(f >> 15) * __half2float(__ushort_as_half((unsigned short)(mm.x & 0xFFFFu)));
    const float4 qp = units[min(pp, 23u) * 8 + cpy];
    const float a[4] = {qp.x * rad, qp.y * rad, qp.z * rad, qp.w * rad};
    c[0] = a[0] * q.x - a[1] * q.y - a[2] * q.z - a[3] * q.w;
    c[1] = a[0] * q.y + a[1] * q.x + a[2] * q.w - a[3] * q.z;
    c[2] = a[0] * q.z - a[1] * q.w + a[2] * q.x + a[3] * q.y;
    c[3] = a[0] * q.w + a[1] * q.z - a[2] * q.y + a[3] * q.x;
    if (mm.y != 0u) {  // the row has outliers (uniform across the warp): select, no divergent branch
        const int slot = min(__popc(mm.y & ((1u << blk) - 1u)), kHqmqOut - 1);
        const uint2 raw = reinterpret_cast<const uint2 *>(meta + 8)[slot];
        const float2 lo = __half22float2(bits_h2(raw.x)), hi = __half22float2(bits_h2(raw.y));
        const bool mine = (mm.y >> blk) & 1u;
        c[0] = mine ? lo.x : c[0];
        c[1] = mine ? lo.y : c[1];
        c[2] = mine ? hi.x : c[2];
        c[3] = mine ? hi.y : c[3];
    }
}

// A float pair as two fp16 pairs, hi = fp16(x) and lo = fp16(x - hi): the
// tensor-core products keep ~22 bits of each operand.
__device__ __forceinline__ void split_h2(float x0, float x1, uint32_t &hi, uint32_t &lo)
{
    const __half2 h = __floats2half2_rn(x0, x1);
    const float2 b = __half22float2(h);
    hi = h2_bits(h);
    lo = h2_bits(__floats2half2_rn(x0 - b.x, x1 - b.y));
}

// Grid (splits, Hkv, B); split `blockIdx.x` attends pages [x * pps, +pps) of
// its sequence, warp w pages [x * pps + w * ppw, +ppw) (pps = 8 ppw), each
// page copied whole into the warp's two-stage ring by one bulk copy.
// Partials [g][d + 4] (sums, max, sum of weights) go to p.part; the last CTA
// merges them.
template <int G>
__global__ void __launch_bounds__(kHqThreads, 2) hqmq_decode_kernel(const __grid_constant__ DecodeParams p)
{
    const Layout &L = p.L;
    const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = L.g;
    extern __shared__ __align__(128) unsigned char smem[];
    float4 *tab = reinterpret_cast<float4 *>(smem);  // K then V codebook; the warps' sums after the loop
    __shared__ __align__(16) float sq[G * kHqD];
    __shared__ __align__(16) float4 units[24 * 8];
    __shared__ float wm[kHqWarps][G], wl[kHqWarps][G];
    __shared__ int sflag;

    const int p_begin = split * p.pages_per_split + warp * p.pages_per_warp;
    const int32_t *bt = p.block_table + (long long)b * p.max_pages;
    const unsigned char *kv_base = p.pool + kHeaderBytes + (long long)kvh * L.chunk_bytes;
    const uint32_t stage0 = smem_u32(smem + kHqOffStage) + warp * kHqStages * kHqChunk;
    const unsigned char *stage0_ptr = smem + kHqOffStage + warp * kHqStages * kHqChunk;
    const uint32_t bar0 = smem_u32(smem + kHqOffBar) + warp * kHqStages * 8;

    // Launched as a programmatic dependent of the stream's previous kernel:
    // until griddepcontrol.wait returns, only what no kernel writes is read
    // for use (the codebooks, fixed when the cache was created, and the unit
    // table); the context length and block-table entries are read as hints
    // (L2 only) to prefetch the ring's first pages and the query rows.
    {
        const float4 *S = reinterpret_cast<const float4 *>(p.pool + L.hq_tab) + (long long)kvh * 2 * kHqmqNS;
        for (int i = tid; i < 2 * kHqmqNS; i += kHqThreads) tab[i] = __ldg(S + i);
        // the 24 unit Hurwitz quaternions: p < 8 are +-1, +-i, +-j, +-k; p >= 8
        // are (+-1 +-i +-j +-k)/2 with component c negative iff bit c of p - 8
        if (tid < 24 * 8) {
            const int pu = tid >> 3;
            float u4[4];
#pragma unroll
            for (int c = 0; c < 4; c++)
                u4[c] = pu < 8 ? (pu / 2 == c ? ((pu & 1) ? -1.f : 1.f) : 0.f) : ((((pu - 8) >> c) & 1) ? -0.5f : 0.5f);
            units[tid] = make_float4(u4[0], u4[1], u4[2], u4[3]);
        }
        const int Th = min(max(__ldcg(p.ctx_lens + b), 0), p.max_pages * kPageTokens);
        const int npg_h = min(p_begin + p.pages_per_warp, (Th + kPageTokens - 1) / kPageTokens) - p_begin;
        if (lane < npg_h && lane < kHqStages) {
            const int pg = __ldcg(bt + p_begin + lane);
            if (pg >= 0 && pg < L.num_pages) bulk_prefetch_l2(kv_base + (long long)pg * L.page_bytes, kHqChunk);
        }
        if (warp == 0 && lane == 31) bulk_prefetch_l2(p.q + ((long long)b * L.hq + kvh * g) * kHqD, g * kHqD * 2);
        if (lane == 0) {
            for (int st = 0; st < kHqStages; st++) mbar_init(bar0 + 8 * st, 1);
            fence_mbar_init();
        }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    int T = p.ctx_lens[b];
    if (T < 0 || T > p.max_pages * kPageTokens) {
        if (split == 0 && tid == 0) set_status(p.pool, KVQ_ERR_OUT_OF_RANGE);
        T = T < 0 ? 0 : p.max_pages * kPageTokens;
    }
    const int n_pages = (T + kPageTokens - 1) / kPageTokens;
    const int n_act = max(1, (n_pages + p.pages_per_split - 1) / p.pages_per_split);
    if (split >= n_act) return;

    // this warp's pages and its ring; the first copies go out first
    const int npg = max(0, min(p_begin + p.pages_per_warp, n_pages) - p_begin);
    __syncwarp();
    uint32_t vbits = 0;  // bit st: stage st holds a valid page
    auto issue = [&](int i) {  // every lane calls this
        const int st = i % kHqStages;
        int pg = 0;
        if (lane == 0) {
            pg = bt[p_begin + i];
            if (pg < 0 || pg >= L.num_pages) {
                set_status(p.pool, KVQ_ERR_OUT_OF_RANGE);
                pg = -1;
            }
            if (pg >= 0)
                bulk_load(stage0 + st * kHqChunk, kv_base + (long long)pg * L.page_bytes, kHqChunk, bar0 + 8 * st);
            else
                asm volatile("mbarrier.arrive.relaxed.cta.shared::cta.b64 _, [%0];" ::"r"(bar0 + 8 * st) : "memory");
        }
        pg = __shfl_sync(kFull, pg, 0);
        vbits = (vbits & ~(1u << st)) | ((pg >= 0 ? 1u : 0u) << st);
    };
    for (int i = 0; i < kHqStages && i < npg; i++) issue(i);

    if (warp < g) {  // the rotated query in log2 units
        const __half *qh = p.q + ((long long)b * L.hq + kvh * g + warp) * kHqD + lane * 4;
        const uint2 raw = *reinterpret_cast<const uint2 *>(qh);
        const float2 a = __half22float2(bits_h2(raw.x)), c = __half22float2(bits_h2(raw.y));
        float x[4] = {a.x, a.y, c.x, c.y};
        if (p.rotate) {
#pragma unroll
            for (int e = 0; e < 4; e++) x[e] *= p.signs[lane * 4 + e];
            fwht_warp<kHqD>(x, lane);
#pragma unroll
            for (int e = 0; e < 4; e++) x[e] *= p.rot_scale;
        }
#pragma unroll
        for (int e = 0; e < 4; e++) sq[warp * kHqD + lane * 4 + e] = x[e] * p.qscale;
    }
    __syncthreads();
    const float4 *SK = tab, *SV = tab + kHqmqNS;
    // Fragment roles (mma m16n8k16, fp16 in, fp32 out; r = lane / 4, j = lane % 4):
    //   scores S^T [16 tokens x 8 heads] = K [16 x 128] Q^T: k-slice ks holds
    //     blocks 4 ks .. 4 ks + 3, slice position {2j, 2j+1, 2j+8, 2j+9} = dims
    //     0..3 of block 4 ks + j, so lane rebuilds block 4 ks + j of tokens r
    //     and r + 8 and holds the query's block 4 ks + j of head r;
    //   the scores land as tokens r, r + 8 x heads 2j, 2j + 1;
    //   O^T [128 dims x 8 heads] += V^T [128 x 16 tokens] P^T: m-tiles 2i and
    //     2i + 1 hold, in rows r / r + 8, dims 0 / 1 and 2 / 3 of block 8i + r,
    //     so lane rebuilds block 8i + r of tokens 2j, 2j+1, 2j+8, 2j+9; P^T
    //     comes from the score fragments by two 8x8 transposes (movmatrix).
    const int r = lane >> 2, j = lane & 3, cpy = lane & 7;
    uint32_t qb[8][2], ql[8][2];  // the query's hi and lo fp16 parts
#pragma unroll
    for (int ks = 0; ks < 8; ks++) {
        qb[ks][0] = qb[ks][1] = ql[ks][0] = ql[ks][1] = 0u;
        if (r < g) {  // (sq holds g heads)
            const float4 q4 = *reinterpret_cast<const float4 *>(sq + r * kHqD + 4 * (4 * ks + j));
            split_h2(q4.x, q4.y, qb[ks][0], ql[ks][0]);
            split_h2(q4.z, q4.w, qb[ks][1], ql[ks][1]);
        }
    }
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // heads 2j, 2j + 1
    float acc[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; mt++) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;

    for (int i = 0; i < npg; i++) {
        const int st = i % kHqStages;
        const bool ok = mbar_wait_bounded(bar0 + 8 * st, (i / kHqStages) & 1, kWaitLimitNs);
        if (!__all_sync(kFull, ok)) {
            // record it, then wait (bounded) for the copies still in flight
            if (lane == 0) set_status(p.pool, KVQ_ERR_TIMEOUT);
            for (int k = i; k < npg && k < i + kHqStages; k++)
                (void)mbar_wait_bounded(bar0 + 8 * (k % kHqStages), (k / kHqStages) & 1, kWaitLimitNs);
            break;
        }
        const unsigned char *chunk = stage0_ptr + st * kHqChunk;
        const int t_page = (p_begin + i) * kPageTokens;
        const int nvalid = ((vbits >> st) & 1u) ? min(kPageTokens, T - t_page) : 0;

        // ---- scores of tokens r, r + 8 for heads 2j, 2j + 1 ----
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
        {
            const bool va = r < nvalid, vb = r + 8 < nvalid;
            const unsigned char *ra = chunk + L.k_codes + r * kHqRowCode, *rb = ra + 8 * kHqRowCode;
            const unsigned char *ma = chunk + L.k_meta + r * kHqmqRowMeta, *mb = ma + 8 * kHqmqRowMeta;
#pragma unroll
            for (int ks = 0; ks < 8; ks++) {
                const int blk = 4 * ks + j;
                float ka[4], kb[4];
                hq_block(hq_field(ra, blk), ma, SK, units, blk, cpy, ka);
                hq_block(hq_field(rb, blk), mb, SK, units, blk, cpy, kb);
                if (!va) ka[0] = ka[1] = ka[2] = ka[3] = 0.f;
                if (!vb) kb[0] = kb[1] = kb[2] = kb[3] = 0.f;
                uint32_t ah[4], al[4];
                split_h2(ka[0], ka[1], ah[0], al[0]);
                split_h2(kb[0], kb[1], ah[1], al[1]);
                split_h2(ka[2], ka[3], ah[2], al[2]);
                split_h2(kb[2], kb[3], ah[3], al[3]);
                // (K_hi + K_lo)(q_hi + q_lo) without the lo x lo term
                mma16816(sc, ah, qb[ks][0], qb[ks][1]);
                mma16816(sc, al, qb[ks][0], qb[ks][1]);
                mma16816(sc, ah, ql[ks][0], ql[ks][1]);
            }
            if (!va) sc[0] = sc[1] = -INFINITY;
            if (!vb) sc[2] = sc[3] = -INFINITY;
        }
        // ---- online softmax per head over the page's 16 tokens ----
        float mx0 = fmaxf(sc[0], sc[2]), mx1 = fmaxf(sc[1], sc[3]);
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, o));
            mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, o));
        }
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float al0 = m0 == -INFINITY ? 0.f : ex2(m0 - mn0), al1 = m1 == -INFINITY ? 0.f : ex2(m1 - mn1);
        const float p0 = sc[0] == -INFINITY ? 0.f : ex2(sc[0] - mn0), p1 = sc[1] == -INFINITY ? 0.f : ex2(sc[1] - mn1);
        const float p2 = sc[2] == -INFINITY ? 0.f : ex2(sc[2] - mn0), p3 = sc[3] == -INFINITY ? 0.f : ex2(sc[3] - mn1);
        float ps0 = p0 + p2, ps1 = p1 + p3;
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            ps0 += __shfl_xor_sync(kFull, ps0, o);
            ps1 += __shfl_xor_sync(kFull, ps1, o);
        }
        l0 = fmaf(l0, al0, ps0);
        l1 = fmaf(l1, al1, ps1);
        m0 = mn0;
        m1 = mn1;
#pragma unroll
        for (int mt = 0; mt < 8; mt++) {
            acc[mt][0] *= al0;
            acc[mt][1] *= al1;
            acc[mt][2] *= al0;
            acc[mt][3] *= al1;
        }
        // P^T fragments (hi and lo): tokens 2j, 2j+1 (b0) and 2j+8, 2j+9 (b1) of head r
        uint32_t pb[2][2];
        {
            uint32_t t[2][2];
            split_h2(p0, p1, t[0][0], t[1][0]);
            split_h2(p2, p3, t[0][1], t[1][1]);
#pragma unroll
            for (int hl = 0; hl < 2; hl++)
#pragma unroll
                for (int k = 0; k < 2; k++)
                    asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(pb[hl][k]) : "r"(t[hl][k]));
        }
        // ---- values: block 8i + r of tokens 2j, 2j+1, 2j+8, 2j+9 ----
        {
            const int tk[4] = {2 * j, 2 * j + 1, 2 * j + 8, 2 * j + 9};
#pragma unroll
            for (int ib = 0; ib < 4; ib++) {
                const int blk = 8 * ib + r;
                float v[4][4];
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    hq_block(hq_field(chunk + L.v_codes + tk[u] * kHqRowCode, blk),
                             chunk + L.v_meta + tk[u] * kHqmqRowMeta, SV, units, blk, cpy, v[u]);
                    if (tk[u] >= nvalid) v[u][0] = v[u][1] = v[u][2] = v[u][3] = 0.f;
                }
#pragma unroll
                for (int hf = 0; hf < 2; hf++) {  // tile 2 ib + hf: dims 2 hf (rows r), 2 hf + 1 (rows r + 8)
                    uint32_t ah[4], al[4];
                    split_h2(v[0][2 * hf], v[1][2 * hf], ah[0], al[0]);
                    split_h2(v[0][2 * hf + 1], v[1][2 * hf + 1], ah[1], al[1]);
                    split_h2(v[2][2 * hf], v[3][2 * hf], ah[2], al[2]);
                    split_h2(v[2][2 * hf + 1], v[3][2 * hf + 1], ah[3], al[3]);
                    // (V_hi + V_lo)(P_hi + P_lo) without the lo x lo term
                    mma16816(acc[2 * ib + hf], ah, pb[0][0], pb[0][1]);
                    mma16816(acc[2 * ib + hf], ah, pb[1][0], pb[1][1]);
                    mma16816(acc[2 * ib + hf], al, pb[0][0], pb[0][1]);
                }
            }
        }
        // refill this stage (every lane is done reading it)
        __syncwarp();
        if (i + kHqStages < npg) issue(i + kHqStages);
    }

    // warps -> one partial per head: sums, then (max, sum of weights)
    __syncthreads();  // every warp is done with the codebooks
    float *wacc = reinterpret_cast<float *>(tab);  // [kHqWarps][G][128]
#pragma unroll
    for (int hh = 0; hh < 2; hh++) {
        const int h = 2 * j + hh;
        if (h < g) {
#pragma unroll
            for (int ib = 0; ib < 4; ib++) {
                const int blk = 8 * ib + r;
                *reinterpret_cast<float4 *>(wacc + (warp * G + h) * kHqD + 4 * blk) =
                    make_float4(acc[2 * ib][hh], acc[2 * ib][2 + hh], acc[2 * ib + 1][hh], acc[2 * ib + 1][2 + hh]);
            }
            if (r == 0) {
                wm[warp][h] = hh ? m1 : m0;
                wl[warp][h] = hh ? l1 : l0;
            }
        }
    }
    __syncthreads();
    constexpr int REC = kHqD + 4;
    const long long bk = (long long)b * L.hkv + kvh;
    float *part = p.part + (bk * p.n_splits + split) * (long long)g * REC;
    for (int idx = tid; idx < g * kHqD; idx += kHqThreads) {
        const int h = idx / kHqD, ch = idx - h * kHqD;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kHqWarps; w++) M = fmaxf(M, wm[w][h]);
        float a = 0.f, Ls = 0.f;
        if (M != -INFINITY)
#pragma unroll
            for (int w = 0; w < kHqWarps; w++) {
                const float f = wm[w][h] == -INFINITY ? 0.f : ex2(wm[w][h] - M);
                a = fmaf(f, wacc[(w * G + h) * kHqD + ch], a);
                Ls = fmaf(f, wl[w][h], Ls);
            }
        part[h * REC + ch] = a;
        if (ch == 0) {
            part[h * REC + kHqD] = M;
            part[h * REC + kHqD + 1] = Ls;
        }
    }

    // the last CTA of this (sequence, kv head) merges the splits
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(p.counters + bk, 1u);
        sflag = prev == (unsigned)(n_act - 1);
    }
    __syncthreads();
    if (!sflag) return;
    __threadfence();
    if (tid == 0) p.counters[bk] = 0u;
    const float *pb = p.part + bk * p.n_splits * (long long)g * REC;
    for (int h = warp; h < g; h += kHqWarps) {
        // lane c: the weights of splits c and c + 32, then every split's row
        // loaded before any is summed (one round trip)
        float mc[2], lc[2];
#pragma unroll
        for (int k = 0; k < 2; k++) {
            const int c = lane + 32 * k;
            mc[k] = c < n_act ? __ldcg(pb + (c * g + h) * REC + kHqD) : -INFINITY;
            lc[k] = c < n_act ? __ldcg(pb + (c * g + h) * REC + kHqD + 1) : 0.f;
        }
        float M = fmaxf(mc[0], mc[1]);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, o));
        float f[2], Ls = 0.f;
#pragma unroll
        for (int k = 0; k < 2; k++) {
            f[k] = mc[k] == -INFINITY ? 0.f : ex2(mc[k] - M);
            Ls = fmaf(lc[k], f[k], Ls);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) Ls += __shfl_xor_sync(kFull, Ls, o);
        float o4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
        for (int c = 0; c < n_act; c++) {
            const float fc = __shfl_sync(kFull, c < 32 ? f[0] : f[1], c & 31);
            const float4 r = __ldcg(reinterpret_cast<const float4 *>(pb + (c * g + h) * REC + lane * 4));
            o4[0] = fmaf(fc, r.x, o4[0]);
            o4[1] = fmaf(fc, r.y, o4[1]);
            o4[2] = fmaf(fc, r.z, o4[2]);
            o4[3] = fmaf(fc, r.w, o4[3]);
        }
        if (p.rotate) {  // back to the original domain: diag(s) H c
            fwht_warp<kHqD>(o4, lane);
#pragma unroll
            for (int e = 0; e < 4; e++) o4[e] *= p.rot_scale * p.signs[lane * 4 + e];
        }
        float *out = p.out + ((long long)b * L.hq + kvh * g + h) * kHqD + lane * 4;
        *reinterpret_cast<float4 *>(out) = Ls > 0.f ? make_float4(o4[0] / Ls, o4[1] / Ls, o4[2] / Ls, o4[3] / Ls)
                                                    : make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

template <int G>
cudaError_t launch_hq_decode_g(const DecodeParams &p, dim3 grid, cudaStream_t s)
{
    static DeviceOnce once;
    if (once.needed()) {
        const cudaError_t e =
            cudaFuncSetAttribute(hqmq_decode_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, kHqSmem);
        if (e != cudaSuccess) return e;
        once.mark();
    }
    if (p.n_splits > kHqMaxSplits || p.L.chunk_bytes != kHqChunk) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kHqThreads);
    cfg.dynamicSmemBytes = kHqSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, hqmq_decode_kernel<G>, p);
}

// CTAs per (kv head, tensor) column: what stays resident in one wave (the
// instantiation's own occupancy), no more than the tokens need (8 / WPR rows a pass).
template <int WPR>
cudaError_t launch_hq_append_w(const AppendParams &p, int num_sms, cudaStream_t st)
{
    static int resident = 0;
    if (resident == 0) {
        int n = 0;
        const cudaError_t e =
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, hqmq_append_kernel<WPR>, kHqThreads, 0);
        if (e != cudaSuccess) return e;
        resident = n < 1 ? 1 : n;
    }
    const int pairs = 2 * p.L.hkv;
    const long long wave = (long long)resident * num_sms / pairs;
    const long long need = (p.n_tok + kHqWarps / WPR - 1) / (kHqWarps / WPR);
    const int per = (int)(wave < 1 ? 1 : (wave < need ? wave : need));
    hqmq_append_kernel<WPR><<<dim3(per, pairs), kHqThreads, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_hqmq_append(const AppendParams &p, int num_sms, cudaStream_t st)
{
    if (p.n_tok == 0) return cudaSuccess;
    if ((long long)p.n_tok * p.L.hkv > (1ll << 30)) return cudaErrorInvalidValue;  // 32-bit row indexing
    // few rows (a decode step): the CTA shares each row; many: a warp a row
    const long long rows = 2LL * p.n_tok * p.L.hkv;
    if (rows < 2LL * num_sms * kHqWarps) return launch_hq_append_w<8>(p, num_sms, st);
    return launch_hq_append_w<1>(p, num_sms, st);
}

cudaError_t launch_hqmq_decode(const DecodeParams &p, dim3 grid, cudaStream_t s)
{
    const int g = p.L.g;
    if (g <= 1) return launch_hq_decode_g<1>(p, grid, s);
    if (g <= 2) return launch_hq_decode_g<2>(p, grid, s);
    if (g <= 4) return launch_hq_decode_g<4>(p, grid, s);
    return launch_hq_decode_g<8>(p, grid, s);
}

}  // namespace kvq
