// kvq_decode.cu -- split-K decode attention over the packed paged cache
// ["OSCAR", 2.2b: a fused kernel that unpacks, dequantises and attends over a
// paged low-bit cache and applies the inverse rotation to the output].
//
// Grid (split, kv head, sequence); 8 warps per CTA.  Each warp streams its
// own contiguous run of 16-token pages: one bulk copy per (page, kv head)
// chunk into a shared-memory ring guarded by mbarriers.  Per page (16 tokens),
// with the MMA row dimension over tokens:
//
//   QK  int8 tensor cores (mma.m16n8k32.s8, exact int32): A = the key codes of
//       the 16 tokens as bytes (int4/int2 codes unpack with a mask and shift;
//       int8 codes are used as stored); B = the rotated, pre-scaled query of
//       every head of the GQA group as three signed 7-bit digits
//       q*2^E = d1*2^14 + d2*2^7 + d3 (~21 bits), one column per (head, digit).
//       One MMA per quantisation group; the digits recombine in int32, the
//       group scale applies in fp32, and the group-zero term
//       sum_g zero[t][g] * sum_{i in g} q_i is one fp16 MMA (zeros exact,
//       query sums as hi + lo).  No dequantised key is ever rounded.
//   softmax online in the log2 domain; lane (r, j) owns head j for tokens r
//       and r+8, so the running max, sum and the accumulator columns of a
//       head all live in the same lanes.  The running max is raised only when
//       a page's max exceeds it by more than 8 (exact: any reference works).
//   PV  fp16 tensor cores with M = channels: A = value codes of 16 tokens
//       transposed by ldmatrix.trans (exact fp16 integers); B = p * scale of
//       each token and group as an (fp16 hi, fp16 lo) column pair per head,
//       transposed into B layout with movmatrix; the zero term is the fp16
//       zeros against p (hi, lo) in one more MMA.
//
// The 8 warps' (m, l, acc) merge through shared memory into one partial per
// (sequence, kv head, split, head); the last CTA of each (sequence, kv head)
// merges all splits by the log-sum-exp rule with every thread loading in
// parallel, applies the inverse rotation R^T = diag(s) H c_d, writes fp32.
#include <math.h>

#include "kvq_internal.cuh"
#include "kvq_warp.cuh"

namespace kvq {
namespace {

constexpr int kCombineSplits = 40;  // most splits per (sequence, kv head)

// fp16x2 constants (bit patterns)
constexpr uint32_t kH1024 = 0x64006400u;  // (1024, 1024)

__device__ __forceinline__ uint32_t hsub2u(uint32_t a, uint32_t b)
{
    return h2_bits(__hsub2(bits_h2(a), bits_h2(b)));
}

__device__ __forceinline__ uint32_t hfma2u(uint32_t a, uint32_t b, uint32_t c)
{
    return h2_bits(__hfma2(bits_h2(a), bits_h2(b), bits_h2(c)));
}

// (a & m) | c in one three-input logic instruction.  The masks come in as
// registers (see nib_masks): with both as immediates the compiler splits the
// operation in two.
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t m, uint32_t c)
{
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(m), "r"(c));
    return d;
}

// The constants of nib (4-bit values: two masks) and fld2 (2-bit values:
// four masks), held in registers for the whole loop.
template <int VF> struct NibMasks {
    uint32_t m[VF == KVQ_INT2_ASYM ? 4 : 2];
    uint32_t h1024;
};
template <int VF> __device__ __forceinline__ NibMasks<VF> nib_masks()
{
    NibMasks<VF> k;
    if constexpr (VF == KVQ_INT2_ASYM) {
        asm volatile("mov.b32 %0, 0x00030003;" : "=r"(k.m[0]));
        asm volatile("mov.b32 %0, 0x000C000C;" : "=r"(k.m[1]));
        asm volatile("mov.b32 %0, 0x00300030;" : "=r"(k.m[2]));
        asm volatile("mov.b32 %0, 0x00C000C0;" : "=r"(k.m[3]));
    } else {
        asm volatile("mov.b32 %0, 0x000F000F;" : "=r"(k.m[0]));
        asm volatile("mov.b32 %0, 0x00F000F0;" : "=r"(k.m[1]));
    }
    asm volatile("mov.b32 %0, 0x64006400;" : "=r"(k.h1024));
    return k;
}

// Nibble n (0..3) of each 16-bit half of w as exact fp16 integers:
// (w & mask) | 0x6400 is 1024 + c * 16^(n&1); subtract / rescale exactly.
template <int VF> __device__ __forceinline__ uint32_t nib(uint32_t w, int n, const NibMasks<VF> &k)
{
    const uint32_t x = (n & 2) ? (w >> 8) : w;
    if (n & 1) return hfma2u(and_or(x, k.m[1], k.h1024), 0x2C002C00u /*1/16*/, 0xD400D400u /*-64*/);
    return hsub2u(and_or(x, k.m[0], k.h1024), kH1024);
}

// 2-bit field f (0..7) of each 16-bit half as exact fp16 integers.
template <int VF> __device__ __forceinline__ uint32_t fld2(uint32_t w, int f, const NibMasks<VF> &k)
{
    const uint32_t x = (f >= 4) ? (w >> 8) : w;
    const int q = f & 3;
    const uint32_t v = and_or(x, k.m[q], k.h1024);  // 1024 + c * 4^q
    switch (q) {
    case 0: return hsub2u(v, kH1024);
    case 1: return hfma2u(v, 0x34003400u /*1/4*/, 0xDC00DC00u /*-256*/);
    case 2: return hfma2u(v, 0x2C002C00u /*1/16*/, 0xD400D400u /*-64*/);
    default: return hfma2u(v, 0x24002400u /*1/64*/, 0xCC00CC00u /*-16*/);
    }
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) { return h2_bits(__floats2half2_rn(lo, hi)); }


// x ~= hi + lo as the fp16 pair (hi, lo) = (fp16(x), fp16(x - hi)), for two
// values at once (one packed conversion each way): rx for x, ry for y
__device__ __forceinline__ void hilo_pair(float x, float y, uint32_t &rx, uint32_t &ry)
{
    const float2 hf = __half22float2(__floats2half2_rn(x, y));
    rx = pack_h2(hf.x, x - hf.x);  // hf.x is an fp16 value: packing it is exact
    ry = pack_h2(hf.y, y - hf.y);
}

// NG fp16 values stored consecutively (4-byte aligned for NG >= 2) as fp32
template <int NG>
__device__ __forceinline__ void load_h(const unsigned char *p, float (&s)[NG])
{
    if constexpr (NG == 4) {
        const uint2 u = *reinterpret_cast<const uint2 *>(p);
        const float2 a = __half22float2(bits_h2(u.x)), b = __half22float2(bits_h2(u.y));
        s[0] = a.x;
        s[1] = a.y;
        s[2] = b.x;
        s[3] = b.y;
    } else if constexpr (NG == 2) {
        const float2 a = __half22float2(bits_h2(*reinterpret_cast<const uint32_t *>(p)));
        s[0] = a.x;
        s[1] = a.y;
    } else {
        static_assert(NG == 1, "1, 2 or 4 groups");
        s[0] = __half2float(__ushort_as_half(*reinterpret_cast<const uint16_t *>(p)));
    }
}

__device__ __forceinline__ uint32_t movm_t(uint32_t x)
{
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// D(16x8 s32) += A(16x32 s8, row) * B(32x8 s8, col)
__device__ __forceinline__ void imma16832(int *d, const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D(16x8 s32) = A(16x32 s8, row) * B(32x8 s8, col), no accumulator input
__device__ __forceinline__ void imma16832_z(int *d, const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(0));
}

// D(16x8 f32) = A(16x16 f16, row) * B(16x8 f16, col), no accumulator input
__device__ __forceinline__ void mma16816_z(float *d, const uint32_t *a, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
}


// The signs of a lane's E consecutive elements (lane*E .. lane*E+E-1) as
// bits (1 = negative), from the per-call bit words: a per-lane index into
// the parameter space touches at most four words, not one address per lane.
template <int E>
__device__ __forceinline__ uint32_t lane_sign_bits(const uint32_t (&bits)[kMaxD / 32], int lane)
{
    return (bits[(lane * E) >> 5] >> ((lane * E) & 31)) & ((1u << E) - 1u);
}

// x with its sign flipped where bit e of sg is set (multiplication by +-1,
// exactly)
__device__ __forceinline__ float flip_sign(float x, uint32_t sg, int e)
{
    return __uint_as_float(__float_as_uint(x) ^ (((sg >> e) & 1u) << 31));
}

// ------------------------------------------------------------ fused append ---
// Quantise-on-append of one K or V row by a whole warp: lane l holds elements
// [l*E, l*E+E).  Same fp32 operations in the same order as the append kernel
// (sign, butterflies h = 1, 2, 4, ..., d/2 as (a+b, a-b), times c_d; group
// statistics; fp16 scale/zero; rounding), so the stored bytes are identical.
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ uint32_t round_code(float v, float lo, float hi)
{
    v = fminf(fmaxf(v, lo), hi);
    return __float_as_uint(__fadd_rn(v, kRoundMagic)) & 0xFFu;
}

__device__ __forceinline__ float code_value(uint32_t c, bool is_signed)
{
    return (float)(is_signed ? (int)(int8_t)c : (int)c);
}

template <int LANES> __device__ __forceinline__ float group_min(float v)
{
#pragma unroll
    for (int m = 1; m < LANES; m <<= 1) v = fminf(v, __shfl_xor_sync(kFull, v, m));
    return v;
}
template <int LANES> __device__ __forceinline__ float group_max(float v)
{
#pragma unroll
    for (int m = 1; m < LANES; m <<= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, m));
    return v;
}

// A store of the appended row's bytes to the pool's page and, when stage is
// not null, to the same offset of the page's staged copy.
template <typename T>
__device__ __forceinline__ void put2(unsigned char *pool, unsigned char *stage, int off, T v)
{
    *reinterpret_cast<T *>(pool + off) = v;
    if (stage) *reinterpret_cast<T *>(stage + off) = v;
}

// The new token's row (raw: this lane's E fp16 values, already loaded) coded
// into the pool's page (codes[], scale and zero at meta_row[]) and, when
// codes_s and meta_s are not null, into the page's staged copy at the same
// offsets.  BR: OSCAR's bit reversal after H (rotate 2), through perm, D
// floats of shared memory.
template <int D, int FMT, bool BR>
__device__ __forceinline__ void warp_append_row(uint2 raw, uint32_t sg, int rotate, float rot_scale, float clip,
                                                unsigned char *codes, unsigned char *meta_row, unsigned char *codes_s,
                                                unsigned char *meta_s, int tok, unsigned int *desc, int tensor,
                                                int lane, float *perm)
{
    constexpr int E = D / 32;
    float x[E];
    if constexpr (E == 4) {
        const float2 f0 = __half22float2(bits_h2(raw.x)), f1 = __half22float2(bits_h2(raw.y));
        x[0] = f0.x;
        x[1] = f0.y;
        x[2] = f1.x;
        x[3] = f1.y;
    } else {
        const float2 f0 = __half22float2(bits_h2(raw.x));
        x[0] = f0.x;
        x[1] = f0.y;
    }
    if (rotate) {
#pragma unroll
        for (int e = 0; e < E; e++) x[e] = flip_sign(x[e], sg, e);
#pragma unroll
        for (int h = 1; h < E; h <<= 1)
#pragma unroll
            for (int e = 0; e < E; e++)
                if (!(e & h)) {
                    const float a = x[e], b = x[e + h];
                    x[e] = __fadd_rn(a, b);
                    x[e + h] = __fsub_rn(a, b);
                }
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
            const float sg = (lane & m) ? -1.0f : 1.0f;  // upper partner: a - b
#pragma unroll
            for (int e = 0; e < E; e++) x[e] = __fmaf_rn(sg, x[e], __shfl_xor_sync(kFull, x[e], m));
        }
#pragma unroll
        for (int e = 0; e < E; e++) x[e] = __fmul_rn(x[e], rot_scale);
        if constexpr (BR) {  // ["OSCAR", 2.2(a)] P_br after H: a permutation (exact), through shared memory
            __syncwarp();
#pragma unroll
            for (int e = 0; e < E; e++) perm[lane * E + e] = x[e];
            __syncwarp();
#pragma unroll
            for (int e = 0; e < E; e++) x[e] = perm[bitrev_index<D>(lane * E + e)];
            __syncwarp();
        }
    }
    const bool want_desc = desc != nullptr;
    float emax = 0.f, amax = 0.f;
    if constexpr (FMT == KVQ_INT8_SYM) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < E; e++) a = fmaxf(a, fabsf(x[e]));
        a = group_max<32>(a);
        const __half shh = __float2half_ru(__fdiv_rn(a, 127.0f));
        const float sf = __half2float(shh);
        const float inv = (sf == 0.0f) ? 0.0f : __fdiv_rn(1.0f, sf);
        amax = a;
        uint32_t packed = 0;
#pragma unroll
        for (int e = 0; e < E; e++) {
            const uint32_t c = round_code(__fmul_rn(x[e], inv), -127.0f, 127.0f);
            packed |= c << (8 * e);
            emax = fmaxf(emax, fabsf(__fsub_rn(x[e], __fmul_rn(code_value(c, true), sf))));
        }
        const int byte0 = lane * E;  // stream byte
        const int off = ((byte0 / 16) * 16 + tok) * 16 + byte0 % 16;
        if constexpr (E == 4) put2<uint32_t>(codes, codes_s, off, packed);
        else put2<uint16_t>(codes, codes_s, off, (uint16_t)packed);
        if (lane == 0) put2<uint16_t>(meta_row, meta_s, 0, __half_as_ushort(shh));
    } else {
        constexpr bool I4 = FMT == KVQ_INT4_ASYM;
        constexpr int GL = I4 ? 32 / E : 32;  // lanes per group
        constexpr int NG = I4 ? D / 32 : 1;
        constexpr float QMAX = I4 ? 15.0f : 3.0f;
        float lo = x[0], hi = x[0];
#pragma unroll
        for (int e = 1; e < E; e++) {
            lo = fminf(lo, x[e]);
            hi = fmaxf(hi, x[e]);
        }
        lo = group_min<GL>(lo);
        hi = group_max<GL>(hi);
        if (clip < 1.0f) {
            lo = __fmul_rn(lo, clip);
            hi = __fmul_rn(hi, clip);
        }
        const __half shh = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), QMAX));
        const __half zhh = __float2half_rn(lo);
        const float sf = __half2float(shh), zf = __half2float(zhh);
        const float inv = (sf == 0.0f) ? 0.0f : __fdiv_rn(1.0f, sf);
        uint32_t packed = 0;
#pragma unroll
        for (int e = 0; e < E; e++) {
            const uint32_t c = round_code(__fmul_rn(__fsub_rn(x[e], zf), inv), 0.0f, QMAX);
            packed |= c << ((I4 ? 4 : 2) * e);
            emax = fmaxf(emax, fabsf(__fsub_rn(x[e], __fadd_rn(__fmul_rn(code_value(c, false), sf), zf))));
            amax = fmaxf(amax, fabsf(x[e]));
        }
        if constexpr (I4) {
            const int gi = lane / GL, q = lane % GL;  // q-th run of E codes in group gi
            const int off = (gi * 16 + tok) * 16 + (q * E) / 2;
            if constexpr (E == 4) put2<uint16_t>(codes, codes_s, off, (uint16_t)packed);
            else put2<uint8_t>(codes, codes_s, off, (uint8_t)packed);
            if (q == 0) {
                put2<uint16_t>(meta_row, meta_s, 2 * gi, __half_as_ushort(shh));
                put2<uint16_t>(meta_row, meta_s, 2 * (NG + gi), __half_as_ushort(zhh));
            }
        } else {
            static_assert(I4 || E == 4, "2-bit fused append needs head_dim 128");
            put2<uint8_t>(codes, codes_s, ((lane / 16) * 16 + tok) * 16 + lane % 16, (uint8_t)packed);  // stream byte = lane
            if (lane == 0)
                put2<uint32_t>(meta_row, meta_s, 0, __half_as_ushort(shh) | (uint32_t(__half_as_ushort(zhh)) << 16));
        }
    }
    if (want_desc) {
        emax = group_max<32>(emax);
        amax = group_max<32>(amax);
        if (lane == 0) {
            if (tensor == 0) {
                atomicMax(desc + 0, __float_as_uint(emax));
            } else {
                atomicMax(desc + 1, __float_as_uint(emax));
                atomicMax(desc + 2, __float_as_uint(amax));
            }
        }
    }
}

// ------------------------------------------------------------ key codecs ---
// A operand of the QK IMMA: thread (r, j) holds, for k-step kq (32 virtual
// channels), 4 bytes at virtual k = 4j..4j+3 and 4j+16..4j+19 of tokens r and
// r+8.  chan(kq, k) maps virtual k to the physical channel; the query digits
// follow the same map, so the codes never need reordering.

template <int FMT, int D> struct KCodec;

template <int D> struct KCodec<KVQ_INT4_ASYM, D> {
    static constexpr int NCH = D / 32;  // 16-byte chunks per token row (= groups)
    static constexpr int NG = D / 32;
    static constexpr int KQ = D / 32;   // IMMA k-steps
    static constexpr bool ZERO = true;
    static constexpr int ROW_META = 4 * NG;
    __device__ static int chan(int kq, int k) { return 32 * kq + 8 * ((k & 15) >> 2) + 2 * (k & 3) + (k >> 4); }
    __device__ static int group_of_kq(int kq) { return kq; }
    __device__ static void inv_chan(int ch, int &kq, int &k)
    {
        const int c = ch & 31;
        kq = ch >> 5;
        k = 16 * (c & 1) + 4 * (c >> 3) + ((c >> 1) & 3);
    }
    // w[c] / w8[c]: word j of chunk c for tokens r / r+8
    __device__ static void afrag(const uint32_t (&w)[NCH], const uint32_t (&w8)[NCH], int kq, uint32_t (&a)[4])
    {
        a[0] = w[kq] & 0x0F0F0F0Fu;
        a[1] = w8[kq] & 0x0F0F0F0Fu;
        a[2] = (w[kq] >> 4) & 0x0F0F0F0Fu;
        a[3] = (w8[kq] >> 4) & 0x0F0F0F0Fu;
    }
};

template <int D> struct KCodec<KVQ_INT8_SYM, D> {
    static constexpr int NCH = D / 16;
    static constexpr int NG = 1;
    static constexpr int KQ = D / 32;
    static constexpr bool ZERO = false;
    static constexpr int ROW_META = 2;
    __device__ static int chan(int kq, int k) { return 32 * kq + k; }
    __device__ static int group_of_kq(int) { return 0; }
    __device__ static void inv_chan(int ch, int &kq, int &k)
    {
        kq = ch >> 5;
        k = ch & 31;
    }
    __device__ static void afrag(const uint32_t (&w)[NCH], const uint32_t (&w8)[NCH], int kq, uint32_t (&a)[4])
    {
        a[0] = w[2 * kq];
        a[1] = w8[2 * kq];
        a[2] = w[2 * kq + 1];
        a[3] = w8[2 * kq + 1];
    }
};

template <int D> struct KCodec<KVQ_INT2_ASYM, D> {
    static constexpr int NCH = D / 64;
    static constexpr int NG = 1;
    static constexpr int KQ = D / 32;
    static constexpr bool ZERO = true;
    static constexpr int ROW_META = 4;
    __device__ static int chan(int kq, int k)
    {
        return 64 * (kq >> 1) + 16 * ((k & 15) >> 2) + 4 * (k & 3) + 2 * (kq & 1) + (k >> 4);
    }
    __device__ static int group_of_kq(int) { return 0; }
    __device__ static void inv_chan(int ch, int &kq, int &k)
    {
        const int rem = ch & 63;
        kq = 2 * (ch >> 6) + ((rem >> 1) & 1);
        k = 16 * (rem & 1) + 4 * (rem >> 4) + ((rem >> 2) & 3);
    }
    __device__ static void afrag(const uint32_t (&w)[NCH], const uint32_t (&w8)[NCH], int kq, uint32_t (&a)[4])
    {
        const int c = kq >> 1, s = 2 * (kq & 1);
        a[0] = (w[c] >> (2 * s)) & 0x03030303u;
        a[1] = (w8[c] >> (2 * s)) & 0x03030303u;
        a[2] = (w[c] >> (2 * s + 2)) & 0x03030303u;
        a[3] = (w8[c] >> (2 * s + 2)) & 0x03030303u;
    }
};

// ---------------------------------------------------------- value codecs ---
// A operand of PV (M = channels, K = 16 tokens).  ldmatrix.trans of a chunk
// over 8 tokens hands thread (r, j) the r-th 16-bit piece of tokens 2j and
// 2j+1 packed together (wA; tokens 2j+8, 2j+9 in wB).  chan(mt, row) maps an
// accumulator row back to the physical channel.

template <int FMT, int D> struct VCodec;

template <int D> struct VCodec<KVQ_INT4_ASYM, D> {
    static constexpr int NCH = D / 32;
    static constexpr int NG = D / 32;
    static constexpr int ROW_META = 4 * NG;
    static constexpr int MT_PER_CHUNK = 2;
    __device__ static int chan(int mt, int row) { return 32 * (mt >> 1) + 4 * (row & 7) + 2 * (mt & 1) + (row >> 3); }
    __device__ static int group_of_mt(int mt) { return mt >> 1; }
    __device__ static int group_of_chan(int ch) { return ch / 32; }
    __device__ static void afrag(uint32_t wA, uint32_t wB, int u, uint32_t (&a)[4], const NibMasks<KVQ_INT4_ASYM> &k)
    {
        a[0] = nib(wA, 2 * u, k);
        a[1] = nib(wA, 2 * u + 1, k);
        a[2] = nib(wB, 2 * u, k);
        a[3] = nib(wB, 2 * u + 1, k);
    }
};

template <int D> struct VCodec<KVQ_INT2_ASYM, D> {
    static constexpr int NCH = D / 64;
    static constexpr int NG = 1;
    static constexpr int ROW_META = 4;
    static constexpr int MT_PER_CHUNK = 4;
    __device__ static int chan(int mt, int row) { return 64 * (mt >> 2) + 8 * (row & 7) + 2 * (mt & 3) + (row >> 3); }
    __device__ static int group_of_mt(int) { return 0; }
    __device__ static int group_of_chan(int) { return 0; }
    __device__ static void afrag(uint32_t wA, uint32_t wB, int u, uint32_t (&a)[4], const NibMasks<KVQ_INT2_ASYM> &k)
    {
        a[0] = fld2(wA, 2 * u, k);
        a[1] = fld2(wA, 2 * u + 1, k);
        a[2] = fld2(wB, 2 * u, k);
        a[3] = fld2(wB, 2 * u + 1, k);
    }
};

template <int KF, int VF, int D, bool G8> struct Cfg {
    using K = KCodec<KF, D>;
    using V = VCodec<VF, D>;
    static constexpr int NH = G8 ? 2 : 1;  // heads per lane (j, j+4)
    static constexpr int NT = G8 ? 3 : 2;  // IMMA n-tiles of query digits
    static constexpr int K_CODES = 0;
    static constexpr int K_META = 16 * (D * (KF == KVQ_INT4_ASYM ? 4 : KF == KVQ_INT8_SYM ? 8 : 2) / 8);
    static constexpr int V_CODES = K_META + 16 * K::ROW_META;
    static constexpr int V_META = V_CODES + 16 * (D * (VF == KVQ_INT4_ASYM ? 4 : 2) / 8);
    static constexpr int CHUNK = V_META + 16 * V::ROW_META;
    static constexpr int NST = CHUNK > 3000 ? 3 : 4;
    static constexpr int STAGE = (CHUNK + 127) / 128 * 128;
    static constexpr int MT = D / 16;  // m-tiles of PV
    static constexpr int E = D / 32;   // elements per lane in warp-wide vectors
    // shared memory map
    static constexpr int RING = kDecodeWarps * NST * STAGE;
    static constexpr int OFF_QV = RING;                              // s8 [NT][KQ][8][32]
    static constexpr int OFF_QSUM = OFF_QV + NT * K::KQ * 8 * 32;    // f32 [8][4]
    static constexpr int OFF_QEXP = OFF_QSUM + kMaxGqa * 4 * 4;      // i32 [8]
    static constexpr int OFF_BAR = OFF_QEXP + kMaxGqa * 4;
    static constexpr int END = OFF_BAR + kDecodeWarps * NST * 8;
    static constexpr int OFF_FLAG = (END + 7) / 8 * 8;                   // the last-CTA flag (int)
    static constexpr int OFF_RBAR = OFF_FLAG + 8;                         // mbarrier of the record copy
    // final merge: split weights [kCombineSplits][8], per-head rescale,
    // max and sum [8] each, the normalised rows [8][D]
    static constexpr int OFF_FW = OFF_RBAR + 8;
    static constexpr int OFF_FC = OFF_FW + kCombineSplits * kMaxGqa * 4;
    static constexpr int OFF_FM = OFF_FC + kMaxGqa * 4;
    static constexpr int OFF_FL = OFF_FM + kMaxGqa * 4;
    static constexpr int OFF_FROW = (OFF_FL + kMaxGqa * 4 + 15) / 16 * 16;
    static constexpr int SMEM = OFF_FROW + kMaxGqa * D * 4;
    // split records staged per piece of the final merge (in the ring)
    static constexpr int REC = D + 4;
    // merge scratch (aliases the ring after the page loop): per warp and
    // head a row of D sums at a padded stride (the four heads a warp stores
    // at once then fall on different banks), and the (max, sum) pairs
    static constexpr int MS = D + 8;
    static constexpr int MERGE_ACC = 0;                                       // [W][8][MS] f32
    static constexpr int MERGE_ML = MERGE_ACC + kDecodeWarps * kMaxGqa * MS * 4;  // [W][8] float2
    static_assert(MERGE_ML + kDecodeWarps * kMaxGqa * 8 <= RING, "merge scratch must fit in the ring");
    static_assert(OFF_BAR % 8 == 0, "mbarriers need 8-byte alignment");
};

// Key chunks, not transposed, tokens r (w) and r+8 (w8): ldmatrix.x4 over the
// matrices (c, tok 0-7), (c, tok 8-15), (c+1, tok 0-7), (c+1, tok 8-15).
template <int NCH>
__device__ __forceinline__ void ld_krows(uint32_t base, int lane, uint32_t (&w)[NCH], uint32_t (&w8)[NCH])
{
    const int row = lane & 7, mi = lane >> 3;
    if constexpr (NCH >= 2) {
#pragma unroll
        for (int q = 0; q < NCH / 2; q++) {
            const int c = 2 * q + (mi >> 1), tok = (mi & 1) * 8 + row;
            ldsm_x4(base + (c * 16 + tok) * 16, w[2 * q], w8[2 * q], w[2 * q + 1], w8[2 * q + 1]);
        }
    } else {
        const int tok = (mi & 1) * 8 + row;
        uint32_t d0, d1;
        ldsm_x4(base + tok * 16, w[0], w8[0], d0, d1);
    }
}

// Value chunks transposed: wA[c] = tokens (2j, 2j+1), wB[c] = tokens
// (2j+8, 2j+9), 16-bit piece r of chunk c.
template <int NCH>
__device__ __forceinline__ void ld_vrows_t(uint32_t base, int lane, uint32_t (&wA)[NCH], uint32_t (&wB)[NCH])
{
    const int row = lane & 7, mi = lane >> 3;
    if constexpr (NCH >= 2) {
#pragma unroll
        for (int q = 0; q < NCH / 2; q++) {
            const int c = 2 * q + (mi >> 1), tok = (mi & 1) * 8 + row;
            ldsm_x4_t(base + (c * 16 + tok) * 16, wA[2 * q], wB[2 * q], wA[2 * q + 1], wB[2 * q + 1]);
        }
    } else {
        const int tok = (mi & 1) * 8 + row;
        uint32_t d0, d1;
        ldsm_x4_t(base + tok * 16, wA[0], wB[0], d0, d1);
    }
}


// Which (head, digit) a query-digit column holds; digit -1 = unused column.
template <bool G8>
__device__ __forceinline__ void col_src(int nt, int n, int &head, int &digit)
{
    if (!G8) {
        head = n >> 1;
        digit = nt == 0 ? (n & 1) : ((n & 1) ? -1 : 2);
    } else {
        if (nt < 2) {
            head = 4 * nt + (n >> 1);
            digit = n & 1;
        } else {
            head = (n & 1) ? 4 + (n >> 1) : (n >> 1);
            digit = 2;
        }
    }
}

// Column (n-tile, col) holding digit dg of head h (the inverse of col_src).
template <bool G8>
__device__ __forceinline__ void digit_col(int h, int dg, int &nt, int &col)
{
    if (!G8) {
        nt = dg == 2 ? 1 : 0;
        col = 2 * h + (dg == 1 ? 1 : 0);
    } else {
        const int hh = h & 3, hi = h >> 2;
        if (dg < 2) {
            nt = hi;
            col = 2 * hh + dg;
        } else {
            nt = 2;
            col = 2 * hh + hi;
        }
    }
}

// BR: the cache stores the rotated channels in bit-reversed order (rotate 2);
// a template parameter so that the rotate 0/1 kernels carry none of it.
template <int D, int KF, int VF, bool G8, bool BR>
__global__ void __launch_bounds__(kDecodeThreads, G8 ? 1 : 2) decode_kernel(const __grid_constant__ DecodeParams p)
{
    using C = Cfg<KF, VF, D, G8>;
    using KC = typename C::K;
    using VC = typename C::V;
    constexpr int E = C::E;
    constexpr int NST = C::NST;
    constexpr int NH = C::NH;
    constexpr int NT = C::NT;

    const Layout &L = p.L;
    const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r = lane >> 2, j = lane & 3;
    const int g = L.g;

    // Launched as a programmatic dependent of the stream's previous kernel,
    // this CTA may start while that grid is still finishing.  Until
    // griddepcontrol.wait returns, nothing read can be trusted (the previous
    // kernel may be writing the context lengths, the block table, the query
    // or the pages), so this phase only reads hints and warms L2: the context
    // length and this warp's block-table entries are read (L2 only, never
    // kept in L1), clamped into the pool, and the first pages they name, the
    // query rows and the appended rows are prefetched into L2.
    extern __shared__ __align__(128) unsigned char smem[];
    const uint32_t bar0 = smem_u32(smem + C::OFF_BAR) + warp * NST * 8;
    const int p_begin = split * p.pages_per_split + warp * p.pages_per_warp;
    const int32_t *bt = p.block_table + (long long)b * p.max_pages;
    int Th, id_h = -1;  // hints: the context length, page p_begin + lane
    {
        Th = min(max(__ldcg(p.ctx_lens + b), 0), p.max_pages * kPageTokens);
        const int npg_h = min(p_begin + p.pages_per_warp, (Th + kPageTokens - 1) / kPageTokens) - p_begin;
        if (lane < npg_h && lane < 32) {
            const int pg = __ldcg(bt + p_begin + lane);
            if (pg >= 0 && pg < L.num_pages) {
                id_h = pg;
                // only the ring's first fill: prefetching the whole run at once
                // queued the first pages behind the rest (measured slower)
                if (lane < NST) bulk_prefetch_l2(p.pool + kHeaderBytes + (long long)kvh * L.chunk_bytes + (long long)pg * L.page_bytes,
                                 L.chunk_bytes);
            }
        }
        // the group's query rows (contiguous) and the rows the step appends
        if (warp == 0 && lane == 31) bulk_prefetch_l2(p.q + ((long long)b * L.hq + kvh * g) * D, g * D * 2);
        if (warp == 1 && lane == 31 && p.new_k != nullptr) {
            bulk_prefetch_l2(p.new_k + ((long long)b * L.hkv + kvh) * D, D * 2);
            bulk_prefetch_l2(p.new_v + ((long long)b * L.hkv + kvh) * D, D * 2);
        }
        if (lane == 0) {  // the ring's barriers (this CTA's own shared memory)
            for (int s = 0; s < NST; s++) mbar_init(bar0 + 8 * s, 1);
            fence_mbar_init();
        }
    }
    // wait for the previous grid to complete (its writes visible), then let
    // the next dependent grid be set up early
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (p.rec_ready != nullptr) {
        // a step from host buffers: the previous step's record is consumed
        // (its grid is complete); this step's record comes on the library's
        // copy stream, announced by its flag.  The mark is a plain store:
        // nothing written before it needs ordering (the previous grid only
        // read the record, and its completion is what the mark says)
        if (p.rec_consumed != nullptr && split == 0 && kvh == 0 && b == 0 && tid == 0)
            asm volatile("st.relaxed.sys.global.u32 [%0], %1;" ::"l"(p.rec_consumed), "r"(p.rec_seq - 1u) : "memory");
        bool ok = true;
        if (lane == 0) ok = flag_wait_bounded(p.rec_ready, p.rec_seq, kWaitLimitNs);
        __syncwarp();  // the other lanes' record loads come after lane 0's acquire
        if (!__shfl_sync(kFull, ok, 0) && lane == 0) set_status(p.pool, KVQ_ERR_TIMEOUT);
    }

    // the true values: the context length, this warp's first 32 block-table
    // entries and the query row all go out together, ahead of any copy
    int T = p.ctx_lens[b];
    const int id_raw = (lane < p.pages_per_warp && p_begin + lane < p.max_pages) ? bt[p_begin + lane] : -1;
    uint2 q_raw = make_uint2(0u, 0u);
    if (warp < g) {
        const __half *qh = p.q + ((long long)b * L.hq + kvh * g + warp) * D + lane * E;
        if constexpr (E == 4) q_raw = *reinterpret_cast<const uint2 *>(qh);
        else q_raw.x = *reinterpret_cast<const uint32_t *>(qh);
    }

    // The contents of every page are final now; only the page ids of the
    // hints are guesses.  The first copies go out at once from them, while
    // the loads above are in flight.  A guess that turns out wrong is waited
    // out and its copy made again.
    const uint32_t stage0 = smem_u32(smem) + warp * NST * C::STAGE;
    const unsigned char *stage0_ptr = smem + warp * NST * C::STAGE;
    const unsigned char *kv_base = p.pool + kHeaderBytes + (long long)kvh * L.chunk_bytes;
    int n_spec = 0;
    {
        const unsigned lead = __ballot_sync(kFull, id_h >= 0);
        n_spec = min(NST, __ffs(~lead) - 1 < 0 ? 32 : __ffs(~lead) - 1);
        for (int i = 0; i < n_spec; i++) {
            const int pg = __shfl_sync(kFull, id_h, i);
            bulk_load_or_arrive(lane == 0, false, stage0 + i * C::STAGE, kv_base + (long long)pg * L.page_bytes,
                                C::CHUNK, bar0 + 8 * i);
        }
    }

    if (T < 0 || T > p.max_pages * kPageTokens) {
        if (split == 0 && tid == 0) set_status(p.pool, KVQ_ERR_OUT_OF_RANGE);
        T = T < 0 ? 0 : p.max_pages * kPageTokens;
    }
    const int n_pages = (T + kPageTokens - 1) / kPageTokens;
    const int n_active = max(1, (n_pages + p.pages_per_split - 1) / p.pages_per_split);
    const int q_lo = min(p.win_sink, T), q_hi = max(q_lo, T - p.win_recent);  // tokens attended here

    int8_t *qv = reinterpret_cast<int8_t *>(smem + C::OFF_QV);
    float *qsum = reinterpret_cast<float *>(smem + C::OFF_QSUM);
    int *qexp = reinterpret_cast<int *>(smem + C::OFF_QEXP);
    int *sflag = reinterpret_cast<int *>(smem + C::OFF_FLAG);

    // ---- this warp's pages: the first copies go out before any query work,
    //      so the page data is in flight during it ----
    const int p_end = min(p_begin + p.pages_per_warp, n_pages);
    const int npg = split >= n_active ? 0 : max(0, p_end - p_begin);

    auto fetch_ids = [&](int i0) -> int {
        const int i = i0 + lane;
        int pg = -1;
        if (i < npg) {
            pg = bt[p_begin + i];
            if (pg < 0 || pg >= L.num_pages) {
                set_status(p.pool, KVQ_ERR_OUT_OF_RANGE);
                pg = -1;
            }
        }
        return pg;
    };
    int ids = -1;  // page ids of the issue window [32k, 32k+32)
    if (lane < npg) {
        ids = id_raw;
        if (ids < 0 || ids >= L.num_pages) {
            set_status(p.pool, KVQ_ERR_OUT_OF_RANGE);
            ids = -1;
        }
    }
    const bool appends = p.new_k != nullptr && T > 0 && npg > 0 && n_pages - 1 >= p_begin && n_pages - 1 < p_end;
    // the guesses hold if page i < n_spec is the true page i (the test
    // hook's mode 2 discards them all)
    const bool spec_ok = __all_sync(kFull, lane >= n_spec || (lane < npg && ids == id_h)) && p.expire_first_wait != 2;
    uint32_t phm = 0;  // bit s: the parity stage s's next page completes
    int n_done = n_spec;
    if (!spec_ok && n_spec > 0) {
        // wait (bounded) for the guessed copies, so none lands on a stage that
        // is refilled or of a CTA that has left; their stages move on a phase
        bool landed = true;
        for (int i = 0; i < n_spec; i++) landed &= mbar_wait_bounded(bar0 + 8 * i, 0, kWaitLimitNs);
        if (!__all_sync(kFull, landed) && lane == 0) set_status(p.pool, KVQ_ERR_TIMEOUT);
        phm = (1u << n_spec) - 1u;
        n_done = 0;
    }
    if (split >= n_active) return;
    uint32_t vbits = (1u << n_done) - 1u;  // bit s: stage s holds a valid page
    auto issue = [&](int i) {  // every lane calls this; lane 0 alone copies (predicated, no branch)
        const int pg = __shfl_sync(kFull, ids, i & 31);
        const int st = i % NST;
        vbits = (vbits & ~(1u << st)) | ((pg >= 0 ? 1u : 0u) << st);
        // (a stage was last read by this warp's ldmatrix loads, complete before
        // the __syncwarp that precedes every refill; no generic-proxy write to
        // the ring precedes the copy, so no proxy fence)
        bulk_load_or_arrive(lane == 0 && pg >= 0, lane == 0 && pg < 0, stage0 + st * C::STAGE,
                            kv_base + (long long)max(pg, 0) * L.page_bytes, C::CHUNK, bar0 + 8 * st);
    };
    const int n_first = min(NST, npg);
    for (int i = n_done; i < n_first; i++) issue(i);
    // Fused append: the warp that owns the page of position T-1 (its last
    // page) codes the new token's K and V rows into it once that page's copy
    // has landed, storing the bytes both to the pool and to the staged copy
    // (see the page loop); no other warp waits for it.  The rows and the
    // slot are copied now (cp.async) into the final merge's row buffer,
    // unused until every warp has left its page loop, so their latency
    // hides behind the query work and the first pages.
    const int app_tok = (T - 1) % kPageTokens;
    bool app_pending = appends;  // the rows are yet to be stored
    unsigned char *app_buf = smem + C::OFF_FROW;  // K row, V row, slot; at +1024 the bit-reversal scratch
    static_assert(kMaxGqa * D * 4 >= 1024 + D * 4, "the append's scratch fits in the row buffer");
    if (appends) {
        const long long app_row = ((long long)b * L.hkv + kvh) * D + lane * E;
        const uint32_t dst = smem_u32(app_buf) + lane * E * 2;
        asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(dst), "l"(p.new_k + app_row), "n"(E * 2) : "memory");
        asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(dst + D * 2), "l"(p.new_v + app_row), "n"(E * 2)
                     : "memory");
        if (lane == 0)
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(app_buf) + D * 4), "l"(p.new_slots + b)
                         : "memory");
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
    // codes the rows into the pool's page app_pg and, if stage is not null,
    // into its staged copy
    auto append_rows = [&](int app_pg, unsigned char *stage) {
        app_pending = false;
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncwarp();
        const int app_slot = *reinterpret_cast<const int *>(app_buf + D * 4);
        if (app_pg < 0 || app_pg >= L.num_pages || app_slot != app_pg * kPageTokens + app_tok) {
            if (lane == 0) set_status(p.pool, KVQ_ERR_OUT_OF_RANGE);
            return false;
        }
        uint2 app_k = make_uint2(0u, 0u), app_v = make_uint2(0u, 0u);
        if constexpr (E == 4) {
            app_k = *reinterpret_cast<const uint2 *>(app_buf + lane * 8);
            app_v = *reinterpret_cast<const uint2 *>(app_buf + D * 2 + lane * 8);
        } else {
            app_k.x = *reinterpret_cast<const uint32_t *>(app_buf + lane * 4);
            app_v.x = *reinterpret_cast<const uint32_t *>(app_buf + D * 2 + lane * 4);
        }
        unsigned char *chunk = const_cast<unsigned char *>(kv_base) + (long long)app_pg * L.page_bytes;
        unsigned int *desc = L.desc_off ? reinterpret_cast<unsigned int *>(const_cast<unsigned char *>(p.pool) +
                                                                            L.desc_off + ((long long)app_pg * L.hkv + kvh) * 16)
                                        : nullptr;
        const uint32_t sg = lane_sign_bits<E>(p.sign_bits, lane);
        float *perm = reinterpret_cast<float *>(app_buf + 1024);  // past the rows and the slot
        warp_append_row<D, KF, BR>(app_k, sg, p.rotate, p.rot_scale, p.clip, chunk + L.k_codes,
                               chunk + L.k_meta + app_tok * L.k_row_meta, stage ? stage + C::K_CODES : nullptr,
                               stage ? stage + C::K_META + app_tok * KC::ROW_META : nullptr, app_tok, desc, 0, lane,
                               perm);
        warp_append_row<D, VF, BR>(app_v, sg, p.rotate, p.rot_scale, p.clip, chunk + L.v_codes,
                               chunk + L.v_meta + app_tok * L.v_row_meta, stage ? stage + C::V_CODES : nullptr,
                               stage ? stage + C::V_META + app_tok * VC::ROW_META : nullptr, app_tok, desc, 1, lane,
                               perm);
        return true;
    };

    // ---- query (warp h): rotate, pre-scale, group sums, and the three signed
    //      7-bit digits of q * 2^E written straight into the B layout ----
    if (warp < g) {
        const int h = warp;
        float x[E];
        if constexpr (E == 4) {
            const uint2 u = q_raw;
            const float2 f0 = __half22float2(bits_h2(u.x)), f1 = __half22float2(bits_h2(u.y));
            x[0] = f0.x;
            x[1] = f0.y;
            x[2] = f1.x;
            x[3] = f1.y;
        } else {
            const float2 f0 = __half22float2(bits_h2(q_raw.x));
            x[0] = f0.x;
            x[1] = f0.y;
        }
        float sc = p.qscale;
        if (p.rotate) {
#pragma unroll
            for (int e = 0; e < E; e++) x[e] = flip_sign(x[e], lane_sign_bits<E>(p.sign_bits, lane), e);
            fwht_warp<D>(x, lane);
            sc *= p.rot_scale;
        }
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < E; e++) {
            x[e] *= sc;
            amax = fmaxf(amax, fabsf(x[e]));
        }
        // ["OSCAR", 2.2(a)] P_br after H (rotate 2): the query in the stored
        // channel order, so the digits and group sums below are the plain ones
        if constexpr (BR) warp_bitrev<D>(x, lane);
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, m));
        // amax < 2^ex with ex = biased exponent - 126; E = 20 - ex keeps
        // |q * 2^E| < 2^20, so the leading digit stays within +-64
        const int ex = amax > 0.f ? (int)((__float_as_uint(amax) >> 23) & 0xFF) - 126 : 20;
        const int Eh = max(-126, min(127, 20 - ex));
        if (lane == 0) qexp[h] = Eh;
        const float pw2 = __int_as_float((127 + Eh) << 23);
#pragma unroll
        for (int e = 0; e < E; e++) {
            const int ch = lane * E + e;
            const int Q = __float2int_rn(x[e] * pw2);
            const int d3 = ((Q + 64) & 127) - 64;
            const int R = (Q - d3) >> 7;
            const int d2 = ((R + 64) & 127) - 64;
            const int d1 = (R - d2) >> 7;
            int kq, k;
            KC::inv_chan(ch, kq, k);
            const int dig[3] = {d1, d2, d3};
#pragma unroll
            for (int dg = 0; dg < 3; dg++) {
                int nt, col;
                digit_col<G8>(h, dg, nt, col);
                qv[((nt * KC::KQ + kq) * 8 + col) * 32 + k] = (int8_t)dig[dg];
            }
        }
        if constexpr (KC::ZERO) {
            float sm = 0.f;
#pragma unroll
            for (int e = 0; e < E; e++) sm += x[e];
            constexpr int LANES = (KF == KVQ_INT4_ASYM) ? 32 / E : 32;
#pragma unroll
            for (int m = 1; m < LANES; m <<= 1) sm += __shfl_xor_sync(kFull, sm, m);
            if ((lane % LANES) == 0) qsum[h * 4 + (lane * E) / (KF == KVQ_INT4_ASYM ? 32 : D)] = sm;
        }
    }
    // warps without a head clear the digit columns no head writes
    if (warp >= g) {
        uint32_t *qv32 = reinterpret_cast<uint32_t *>(qv);
        for (int idx = (warp - g) * 32 + lane; idx < NT * KC::KQ * 8 * 8; idx += (kDecodeWarps - g) * 32) {
            const int col = (idx >> 3) & 7, nt = (idx >> 6) / KC::KQ;
            int head, digit;
            col_src<G8>(nt, col, head, digit);
            if (digit < 0 || head >= g) qv32[idx] = 0u;
        }
    }
    __syncthreads();

    // ---- per-lane constants: query digit B fragments, zero-term B fragments ----
    uint32_t qb[NT][KC::KQ][2];
#pragma unroll
    for (int nt = 0; nt < NT; nt++)
#pragma unroll
        for (int kq = 0; kq < KC::KQ; kq++) {
            const int8_t *src = qv + ((nt * KC::KQ + kq) * 8 + r) * 32;
            qb[nt][kq][0] = *reinterpret_cast<const uint32_t *>(src + 4 * j);
            qb[nt][kq][1] = *reinterpret_cast<const uint32_t *>(src + 16 + 4 * j);
        }
    uint32_t zb[NH];
#pragma unroll
    for (int t = 0; t < NH; t++) zb[t] = 0u;
    if constexpr (KC::ZERO) {
#pragma unroll
        for (int t = 0; t < NH; t++) {
            const int head = (r >> 1) + 4 * t;
            if (head < g && 2 * j < KC::NG) {
                float q0 = qsum[head * 4 + 2 * j];
                float q1 = (2 * j + 1 < KC::NG) ? qsum[head * 4 + 2 * j + 1] : 0.f;
                if (r & 1) {  // low part
                    q0 -= __half2float(__float2half_rn(q0));
                    q1 -= __half2float(__float2half_rn(q1));
                }
                zb[t] = pack_h2(q0, q1);
            }
        }
    }
    float qinv[NH];
#pragma unroll
    for (int t = 0; t < NH; t++) qinv[t] = (j + 4 * t < g) ? __int_as_float((127 - qexp[j + 4 * t]) << 23) : 0.f;

    float oacc[NH][C::MT][4];
    float oz[NH][4];
    // m_ref: the exponentials' reference, m_run while it is finite; before
    // any token every score is -inf and ex2(-inf - (-inf)) would be NaN
    float m_run[NH], l_part[NH], m_ref[NH];
#pragma unroll
    for (int t = 0; t < NH; t++) {
        m_ref[t] = 0.f;
#pragma unroll
        for (int mt = 0; mt < C::MT; mt++) oacc[t][mt][0] = oacc[t][mt][1] = oacc[t][mt][2] = oacc[t][mt][3] = 0.f;
        oz[t][0] = oz[t][1] = oz[t][2] = oz[t][3] = 0.f;
        m_run[t] = -INFINITY;
        l_part[t] = 0.f;
    }

    // Pages whose 16 tokens are all attended here and whose copy exists take
    // the plain path; the first/last pages of the context or of a window
    // boundary, and pages the block table got wrong, mask their tokens.
    // Iterations [i_full0, i_full1) are the warp's pages inside [q_lo, q_hi).
    const int i_full0 = (q_lo + kPageTokens - 1) / kPageTokens - p_begin;
    const int i_full1 = q_hi / kPageTokens - p_begin;
    const NibMasks<VF> nmask = nib_masks<VF>();
    int st = 0;  // the ring stage of page i
    int n_loop = npg;
    if (p.expire_first_wait == 1 && npg > 0) {
        // test hook: the first wait counts as expired.  The timeout path
        // runs as it would: record the status, then wait (bounded, the
        // normal limit) for the copies in flight; no page is attended.
        if (lane == 0) set_status(p.pool, KVQ_ERR_TIMEOUT);
        for (int k = 0; k < npg && k < NST; k++) (void)mbar_wait_bounded(bar0 + 8 * k, (phm >> k) & 1u, kWaitLimitNs);
        n_loop = 0;
    }
    for (int i = 0; i < n_loop; i++) {
        const uint32_t bar = bar0 + 8 * st, ph = (phm >> st) & 1u;
        if (!__all_sync(kFull, mbar_try_wait(bar, ph))) {
            // slow path: the page is not in yet; wait, but not forever
            if (!__all_sync(kFull, mbar_wait_bounded(bar, ph, kWaitLimitNs))) {
                // give up on this warp's run: record it, then wait (bounded) for
                // the copies still in flight so none lands after the ring is reused
                if (lane == 0) set_status(p.pool, KVQ_ERR_TIMEOUT);
                for (int k = i; k < npg && k < i + NST; k++)
                    (void)mbar_wait_bounded(bar0 + 8 * (k % NST), (phm >> (k % NST)) & 1u, kWaitLimitNs);
                break;
            }
        }
        const uint32_t sb = stage0 + st * C::STAGE;
        const unsigned char *sp = stage0_ptr + st * C::STAGE;
        if (app_pending && i == npg - 1) {
            // the appended row: into the pool and into the staged copy of its
            // page, which was copied before the row existed
            if (append_rows(__shfl_sync(kFull, ids, i & 31), const_cast<unsigned char *>(sp))) __syncwarp();
        }
        const bool page_ok = (vbits >> st) & 1u;
        const bool ragged = i < i_full0 || i >= i_full1 || !page_ok;  // warp-uniform
        // valid tokens of a ragged page: r in [vlo, vhi) (the tail, windows attended elsewhere)
        int vlo = 0, vhi = kPageTokens;
        if (ragged) {
            const int t0 = (p_begin + i) * kPageTokens;
            vlo = page_ok ? min(max(q_lo - t0, 0), kPageTokens) : kPageTokens;
            vhi = page_ok ? min(max(q_hi - t0, 0), kPageTokens) : 0;
        }
        const bool tv_r = r >= vlo && r < vhi, tv_r8 = r + 8 >= vlo && r + 8 < vhi;

        // ---------------- QK: scores of tokens r, r+8 for the lane's heads ----
        float s_r[NH], s_r8[NH];
        {
            uint32_t kw[KC::NCH], kw8[KC::NCH];
            ld_krows<KC::NCH>(sb + C::K_CODES, lane, kw, kw8);
            const unsigned char *meta_r = sp + C::K_META + r * KC::ROW_META;
            const unsigned char *meta_r8 = sp + C::K_META + (r + 8) * KC::ROW_META;
            float zr[NH], zr8[NH];
#pragma unroll
            for (int t = 0; t < NH; t++) zr[t] = zr8[t] = 0.f;
            if constexpr (KC::ZERO) {
                // zeros of groups (2j, 2j+1) of tokens r and r+8 as the A
                // fragment; lanes j with no such group read an in-row word
                // and drop it (their B rows are zero as well)
                uint32_t a[4] = {0u, 0u, 0u, 0u};
                if constexpr (KC::NG >= 2) {
                    const int jj = (2 * j < KC::NG) ? j : 0;
                    const uint32_t z0 = *reinterpret_cast<const uint32_t *>(meta_r + 2 * KC::NG + 4 * jj);
                    const uint32_t z1 = *reinterpret_cast<const uint32_t *>(meta_r8 + 2 * KC::NG + 4 * jj);
                    a[0] = (2 * j < KC::NG) ? z0 : 0u;
                    a[1] = (2 * j < KC::NG) ? z1 : 0u;
                } else {
                    const uint32_t z0 = *reinterpret_cast<const uint16_t *>(meta_r + 2);
                    const uint32_t z1 = *reinterpret_cast<const uint16_t *>(meta_r8 + 2);
                    a[0] = j == 0 ? z0 : 0u;
                    a[1] = j == 0 ? z1 : 0u;
                }
#pragma unroll
                for (int t = 0; t < NH; t++) {
                    float dz[4];
                    mma16816_z(dz, a, zb[t], 0u);
                    zr[t] = dz[0] + dz[1];
                    zr8[t] = dz[2] + dz[3];
                }
            }
            float acc_r[NH], acc_r8[NH];
            float skr[KC::NG], skr8[KC::NG];  // the rows' group scales
            load_h<KC::NG>(meta_r, skr);
            load_h<KC::NG>(meta_r8, skr8);
#pragma unroll
            for (int gi = 0; gi < KC::NG; gi++) {
                int d[NT][4];
                bool first = true;
#pragma unroll
                for (int kq = 0; kq < KC::KQ; kq++) {
                    if (KC::group_of_kq(kq) != gi) continue;
                    uint32_t a[4];
                    KC::afrag(kw, kw8, kq, a);
#pragma unroll
                    for (int nt = 0; nt < NT; nt++) {
                        if (first) imma16832_z(d[nt], a, qb[nt][kq][0], qb[nt][kq][1]);
                        else imma16832(d[nt], a, qb[nt][kq][0], qb[nt][kq][1]);
                    }
                    first = false;
                }
                const float sk_r = skr[gi], sk_r8 = skr8[gi];
#pragma unroll
                for (int t = 0; t < NH; t++) {
                    // digits of head j + 4t: (d1, d2, d3) for row r (c0/c1) and r+8 (c2/c3)
                    const int n12 = G8 ? t : 0, n3 = G8 ? 2 : 1, c3 = G8 ? t : 0;
                    float v_r, v_r8;
                    if constexpr (KF == KVQ_INT8_SYM) {
                        v_r = fmaf(__int2float_rn(d[n12][0]), 16384.f,
                                   fmaf(__int2float_rn(d[n12][1]), 128.f, __int2float_rn(d[n3][c3])));
                        v_r8 = fmaf(__int2float_rn(d[n12][2]), 16384.f,
                                    fmaf(__int2float_rn(d[n12][3]), 128.f, __int2float_rn(d[n3][2 + c3])));
                    } else {
                        v_r = __int2float_rn(d[n12][0] * 16384 + d[n12][1] * 128 + d[n3][c3]);
                        v_r8 = __int2float_rn(d[n12][2] * 16384 + d[n12][3] * 128 + d[n3][2 + c3]);
                    }
                    if (gi == 0) {
                        acc_r[t] = sk_r * v_r;
                        acc_r8[t] = sk_r8 * v_r8;
                    } else {
                        acc_r[t] = fmaf(sk_r, v_r, acc_r[t]);
                        acc_r8[t] = fmaf(sk_r8, v_r8, acc_r8[t]);
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < NH; t++) {
                s_r[t] = fmaf(acc_r[t], qinv[t], zr[t]);
                s_r8[t] = fmaf(acc_r8[t], qinv[t], zr8[t]);
            }
            if (ragged) {
#pragma unroll
                for (int t = 0; t < NH; t++) {
                    s_r[t] = tv_r ? s_r[t] : -INFINITY;
                    s_r8[t] = tv_r8 ? s_r8[t] : -INFINITY;
                }
            }
        }

        // ---------------- online softmax (log2 domain) ----------------
        float p_r[NH], p_r8[NH];
        {
            float mx[NH];
            bool need = false;
#pragma unroll
            for (int t = 0; t < NH; t++) {
                float m = fmaxf(s_r[t], s_r8[t]);
                m = fmaxf(m, __shfl_xor_sync(kFull, m, 4));
                m = fmaxf(m, __shfl_xor_sync(kFull, m, 8));
                m = fmaxf(m, __shfl_xor_sync(kFull, m, 16));
                mx[t] = m;
                need |= m > m_run[t] + 8.0f;
            }
            if (__any_sync(kFull, need)) {
#pragma unroll
                for (int t = 0; t < NH; t++) {
                    const float m_new = mx[t] > m_run[t] + 8.0f ? mx[t] : m_run[t];
                    const float alpha = (m_new == -INFINITY) ? 1.f : ex2(m_run[t] - m_new);
                    m_run[t] = m_new;
                    m_ref[t] = m_new == -INFINITY ? 0.f : m_new;
                    l_part[t] *= alpha;
#pragma unroll
                    for (int mt = 0; mt < C::MT; mt++) {
                        oacc[t][mt][0] *= alpha;
                        oacc[t][mt][1] *= alpha;
                        oacc[t][mt][2] *= alpha;
                        oacc[t][mt][3] *= alpha;
                    }
                    oz[t][0] *= alpha;
                    oz[t][1] *= alpha;
                    oz[t][2] *= alpha;
                    oz[t][3] *= alpha;
                }
            }
#pragma unroll
            for (int t = 0; t < NH; t++) {
                p_r[t] = ex2(s_r[t] - m_ref[t]);
                p_r8[t] = ex2(s_r8[t] - m_ref[t]);
                l_part[t] += p_r[t] + p_r8[t];
            }
            if (p.page_stats != nullptr) {  // certified mode: this page's (m, l) per head
                float2 *ps = p.page_stats + (((long long)b * L.hkv + kvh) * p.max_pages + p_begin + i) * g;
#pragma unroll
                for (int t = 0; t < NH; t++) {
                    float l = p_r[t] + p_r8[t];
                    l += __shfl_xor_sync(kFull, l, 4);
                    l += __shfl_xor_sync(kFull, l, 8);
                    l += __shfl_xor_sync(kFull, l, 16);
                    if (r == 0 && j + 4 * t < g) ps[j + 4 * t] = make_float2(m_run[t], l);
                }
            }
        }

        // ---------------- PV ----------------
        {
            const unsigned char *vmeta_r = sp + C::V_META + r * VC::ROW_META;
            const unsigned char *vmeta_r8 = sp + C::V_META + (r + 8) * VC::ROW_META;
            float sv_r[VC::NG], sv_r8[VC::NG];
            load_h<VC::NG>(vmeta_r, sv_r);
            load_h<VC::NG>(vmeta_r8, sv_r8);
            // zero term: A = zeros^T (group r, tokens 2j, 2j+1 | 2j+8, 2j+9);
            // rows r >= NG read group r % NG and drop it
            uint32_t az[4] = {0u, 0u, 0u, 0u};
            {
                const unsigned char *zrow = sp + C::V_META + 2 * VC::NG + 2 * (r % VC::NG);
                uint32_t z0 = *reinterpret_cast<const uint16_t *>(zrow + (2 * j) * VC::ROW_META);
                uint32_t z1 = *reinterpret_cast<const uint16_t *>(zrow + (2 * j + 1) * VC::ROW_META);
                uint32_t z2 = *reinterpret_cast<const uint16_t *>(zrow + (2 * j + 8) * VC::ROW_META);
                uint32_t z3 = *reinterpret_cast<const uint16_t *>(zrow + (2 * j + 9) * VC::ROW_META);
                if (ragged) {
                    // masked tokens: weight and zero both 0 (their stage bytes may be stale)
#pragma unroll
                    for (int gi = 0; gi < VC::NG; gi++) {
                        sv_r[gi] = tv_r ? sv_r[gi] : 0.f;
                        sv_r8[gi] = tv_r8 ? sv_r8[gi] : 0.f;
                    }
                    if (2 * j < vlo || 2 * j >= vhi) z0 = 0;
                    if (2 * j + 1 < vlo || 2 * j + 1 >= vhi) z1 = 0;
                    if (2 * j + 8 < vlo || 2 * j + 8 >= vhi) z2 = 0;
                    if (2 * j + 9 < vlo || 2 * j + 9 >= vhi) z3 = 0;
                }
                if (r < VC::NG) {
                    az[0] = z0 | (z1 << 16);
                    az[2] = z2 | (z3 << 16);
                }
            }
            uint32_t vA[VC::NCH], vB[VC::NCH];
            ld_vrows_t<VC::NCH>(sb + C::V_CODES, lane, vA, vB);
#pragma unroll
            for (int t = 0; t < NH; t++) {
                // p as (hi, lo) columns, transposed into B layout
                uint32_t h0, h1;
                hilo_pair(p_r[t], p_r8[t], h0, h1);
                mma16816(oz[t], az, movm_t(h0), movm_t(h1));
                uint32_t wb[VC::NG][2];
#pragma unroll
                for (int gi = 0; gi < VC::NG; gi++) {
                    hilo_pair(p_r[t] * sv_r[gi], p_r8[t] * sv_r8[gi], h0, h1);
                    wb[gi][0] = movm_t(h0);
                    wb[gi][1] = movm_t(h1);
                }
#pragma unroll
                for (int c = 0; c < VC::NCH; c++) {
#pragma unroll
                    for (int u = 0; u < VC::MT_PER_CHUNK; u++) {
                        const int mt = c * VC::MT_PER_CHUNK + u;
                        uint32_t a[4];
                        VC::afrag(vA[c], vB[c], u, a, nmask);
                        const int gi = VC::group_of_mt(mt);
                        mma16816(oacc[t][mt], a, wb[gi][0], wb[gi][1]);
                    }
                }
            }
        }

        // ---------------- refill this stage ----------------
        __syncwarp();
        const int nxt = i + NST;
        if (nxt < npg) {
            if ((nxt & 31) == 0) ids = fetch_ids(nxt);
            issue(nxt);
        }
        phm ^= 1u << st;
        if (++st == NST) st = 0;
    }
    if (app_pending) (void)append_rows(bt[n_pages - 1], nullptr);  // the run ended early: the pool still gets the rows

    // ---- warp state -> shared memory, CTA merge ----
    // The zero term of group gi for head j sits in lane (gi, j): add it to
    // the accumulator rows of that group, and the row pair (c, c + 1) a lane
    // holds becomes two finished sums.
#pragma unroll
    for (int t = 0; t < NH; t++) {
        l_part[t] += __shfl_xor_sync(kFull, l_part[t], 4);
        l_part[t] += __shfl_xor_sync(kFull, l_part[t], 8);
        l_part[t] += __shfl_xor_sync(kFull, l_part[t], 16);
        const float zs = oz[t][0] + oz[t][1];
        float zg[VC::NG];
#pragma unroll
        for (int gi = 0; gi < VC::NG; gi++) zg[gi] = __shfl_sync(kFull, zs, gi * 4 + j);
#pragma unroll
        for (int mt = 0; mt < C::MT; mt++) {
            const float z = zg[VC::group_of_mt(mt)];
            oacc[t][mt][0] = oacc[t][mt][0] + oacc[t][mt][1] + z;
            oacc[t][mt][2] = oacc[t][mt][2] + oacc[t][mt][3] + z;
        }
    }
    __syncthreads();  // every warp is done with the stage ring
    float *macc = reinterpret_cast<float *>(smem + C::MERGE_ACC);  // [warp][head][MS]
    float2 *mml = reinterpret_cast<float2 *>(smem + C::MERGE_ML);  // [warp][head] (max, sum)
#pragma unroll
    for (int t = 0; t < NH; t++) {
        const int head = j + 4 * t;
        if (head < g) {
            float *row = macc + (warp * kMaxGqa + head) * C::MS;
#pragma unroll
            for (int mt = 0; mt < C::MT; mt++)
                *reinterpret_cast<float2 *>(row + VC::chan(mt, r)) = make_float2(oacc[t][mt][0], oacc[t][mt][2]);
            if (r == 0) mml[warp * kMaxGqa + head] = make_float2(m_run[t], l_part[t]);
        }
    }
    __syncthreads();

    // thread: head h, channels (ch, ch + 1); the 8 warps' (max, sum) of the
    // head are broadcast reads, their weights 2^(m_w - M) computed here
    const int n_splits = p.n_splits;
    float *part_base = p.part + (((long long)b * L.hkv + kvh) * n_splits) * g * (D + 4);
    for (int idx = tid; idx < g * (D / 2); idx += kDecodeThreads) {
        const int h = idx / (D / 2), ch = 2 * (idx % (D / 2));
        float2 mlw[kDecodeWarps];
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; w++) {
            mlw[w] = mml[w * kMaxGqa + h];
            M = fmaxf(M, mlw[w].x);
        }
        float2 acc = make_float2(0.f, 0.f);
        float Lsum = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kDecodeWarps; w++) {
                const float f = (mlw[w].x == -INFINITY) ? 0.f : ex2(mlw[w].x - M);
                const float2 a = *reinterpret_cast<const float2 *>(macc + (w * kMaxGqa + h) * C::MS + ch);
                acc.x = fmaf(f, a.x, acc.x);
                acc.y = fmaf(f, a.y, acc.y);
                Lsum = fmaf(f, mlw[w].y, Lsum);
            }
        }
        float *dst = part_base + ((long long)split * g + h) * (D + 4);
        *reinterpret_cast<float2 *>(dst + ch) = acc;
        if (ch == 0) *reinterpret_cast<float2 *>(dst + D) = make_float2(M, Lsum);
    }

    // ---- last CTA of this (sequence, kv head) merges the splits ----
    __syncthreads();
    if (tid == 0) {
        // release: this CTA's record (ordered by the barrier above) is visible
        // before the count; acquire: the last CTA then sees every record
        unsigned prev;
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                     : "=r"(prev)
                     : "l"(p.counters + (b * L.hkv + kvh))
                     : "memory");
        *sflag = (prev == (unsigned)(n_active - 1));
    }
    __syncthreads();
    if (!*sflag) return;

    // The splits' records (contiguous, [split][head][D + 4]) come into the
    // free ring with one bulk copy per piece; warp h turns the piece's
    // (max, sum) pairs of head h into weights 2^(m_s - M) and the running
    // (M, L); every thread then accumulates its (head, channel pair) over
    // the piece from shared memory.
    float *fw = reinterpret_cast<float *>(smem + C::OFF_FW);  // [split in piece][8]
    float *fc = reinterpret_cast<float *>(smem + C::OFF_FC);  // [8] rescale of what came before
    float *fM = reinterpret_cast<float *>(smem + C::OFF_FM);
    float *fL = reinterpret_cast<float *>(smem + C::OFF_FL);
    float *frow = reinterpret_cast<float *>(smem + C::OFF_FROW);  // [8][D]
    const float *recs = reinterpret_cast<const float *>(smem);
    const uint32_t rbar = smem_u32(smem + C::OFF_RBAR);
    constexpr int REC = C::REC;
    const int split_bytes = g * REC * 4;
    const int per_piece = min(n_active, C::RING / split_bytes);
    constexpr int OPT = (kMaxGqa * (D / 2) + kDecodeThreads - 1) / kDecodeThreads;  // pairs a thread owns
    float2 o[OPT];
#pragma unroll
    for (int k = 0; k < OPT; k++) o[k] = make_float2(0.f, 0.f);
    if (tid < kMaxGqa) {
        fM[tid] = -INFINITY;
        fL[tid] = 0.f;
    }
    if (tid == 0) {
        p.counters[b * L.hkv + kvh] = 0u;  // self-resetting for the next call
        mbar_init(rbar, 1);
        fence_mbar_init();
        // the records were written by other CTAs through the generic proxy
        // and are read here by the bulk-copy (async) proxy
        asm volatile("fence.proxy.async.global;" ::: "memory");
    }
    __syncthreads();
    bool rec_ok = true;
    uint32_t rph = 0;
    for (int s0 = 0; s0 < n_active; s0 += per_piece) {
        const int ns = min(per_piece, n_active - s0);
        if (tid == 0)
            bulk_load(smem_u32(smem), part_base + (long long)s0 * g * REC, (uint32_t)(ns * split_bytes), rbar);
        // while the accumulators stream in: warp h reads the piece's (max,
        // sum) pairs of head h straight from the records and turns them into
        // weights 2^(m_s - M) and the running (M, L)
        if (warp < g) {
            const int h = warp;
            const float Mold = fM[h];
            float mloc = -INFINITY, lloc = 0.f, mloc2 = -INFINITY, lloc2 = 0.f;
            if (lane < ns) {
                const float2 ml = __ldcg(reinterpret_cast<const float2 *>(part_base + ((long long)(s0 + lane) * g + h) * REC + D));
                mloc = ml.x;
                lloc = ml.y;
            }
            if (lane + 32 < ns) {
                const float2 ml =
                    __ldcg(reinterpret_cast<const float2 *>(part_base + ((long long)(s0 + lane + 32) * g + h) * REC + D));
                mloc2 = ml.x;
                lloc2 = ml.y;
            }
            float Mp = fmaxf(mloc, mloc2);
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) Mp = fmaxf(Mp, __shfl_xor_sync(kFull, Mp, m));
            const float Mn = fmaxf(Mold, Mp);
            const float f1 = mloc == -INFINITY ? 0.f : ex2(mloc - Mn);
            const float f2 = mloc2 == -INFINITY ? 0.f : ex2(mloc2 - Mn);
            if (lane < ns) fw[lane * kMaxGqa + h] = f1;
            if (lane + 32 < ns) fw[(lane + 32) * kMaxGqa + h] = f2;
            float Lp = f1 * lloc + f2 * lloc2;
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) Lp += __shfl_xor_sync(kFull, Lp, m);
            if (lane == 0) {
                const float c = Mold == -INFINITY ? 0.f : ex2(Mold - Mn);
                fc[h] = c;
                fM[h] = Mn;
                fL[h] = fL[h] * c + Lp;
            }
        }
        rec_ok = __syncthreads_and(mbar_wait_bounded(rbar, rph, kWaitLimitNs));
        if (!rec_ok) {
            // record it; wait (bounded) once more so the copy is not left
            // landing in the shared memory of an exited CTA; no output
            if (tid == 0) {
                set_status(p.pool, KVQ_ERR_TIMEOUT);
                (void)mbar_wait_bounded(rbar, rph, kWaitLimitNs);
            }
            return;
        }
        rph ^= 1u;
#pragma unroll
        for (int k = 0; k < OPT; k++) {
            const int idx = tid + k * kDecodeThreads;
            if (idx < g * (D / 2)) {
                const int h = idx / (D / 2), ch = 2 * (idx % (D / 2));
                const float c = fc[h];
                // two independent chains (even and odd records)
                float2 a = make_float2(o[k].x * c, o[k].y * c), a2 = make_float2(0.f, 0.f);
                int sp = 0;
                for (; sp + 1 < ns; sp += 2) {
                    const float f = fw[sp * kMaxGqa + h], f2 = fw[(sp + 1) * kMaxGqa + h];
                    const float2 v = *reinterpret_cast<const float2 *>(recs + (sp * g + h) * REC + ch);
                    const float2 v2 = *reinterpret_cast<const float2 *>(recs + ((sp + 1) * g + h) * REC + ch);
                    a.x = fmaf(f, v.x, a.x);
                    a.y = fmaf(f, v.y, a.y);
                    a2.x = fmaf(f2, v2.x, a2.x);
                    a2.y = fmaf(f2, v2.y, a2.y);
                }
                if (sp < ns) {
                    const float f = fw[sp * kMaxGqa + h];
                    const float2 v = *reinterpret_cast<const float2 *>(recs + (sp * g + h) * REC + ch);
                    a.x = fmaf(f, v.x, a.x);
                    a.y = fmaf(f, v.y, a.y);
                }
                o[k] = make_float2(a.x + a2.x, a.y + a2.y);
            }
        }
        __syncthreads();  // the next piece overwrites the staged records
    }
#pragma unroll
    for (int k = 0; k < OPT; k++) {
        const int idx = tid + k * kDecodeThreads;
        if (idx < g * (D / 2)) {
            const int h = idx / (D / 2), ch = 2 * (idx % (D / 2));
            const float Ls = fL[h];
            const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
            *reinterpret_cast<float2 *>(frow + h * D + ch) = make_float2(o[k].x * inv, o[k].y * inv);
        }
    }
    __syncthreads();
    // warp h: inverse rotation of head h's normalised row, then the output
    for (int h = warp; h < g; h += kDecodeWarps) {
        float v[E];
        if constexpr (BR) {  // the row is in the stored (bit-reversed) channel order: gather it back
#pragma unroll
            for (int e = 0; e < E; e++) v[e] = frow[h * D + bitrev_index<D>(lane * E + e)];
        } else {
#pragma unroll
            for (int e = 0; e < E; e++) v[e] = frow[h * D + lane * E + e];
        }
        if (lane == 0 && p.head_ml) p.head_ml[((long long)b * L.hkv + kvh) * g + h] = make_float2(fM[h], fL[h]);
        if (p.rotate) {
            fwht_warp<D>(v, lane);
            const uint32_t sg = lane_sign_bits<E>(p.sign_bits, lane);
#pragma unroll
            for (int e = 0; e < E; e++) v[e] = flip_sign(v[e] * p.rot_scale, sg, e);
        }
        float *dst = p.out + ((long long)b * L.hq + kvh * g + h) * D + lane * E;
        if constexpr (E == 4) {
            *reinterpret_cast<float4 *>(dst) = make_float4(v[0], v[1], v[2], v[3]);
        } else {
            *reinterpret_cast<float2 *>(dst) = make_float2(v[0], v[1]);
        }
    }
}

template <int D, int KF, int VF, bool G8, bool BR>
cudaError_t launch_t(const DecodeParams &p, dim3 grid, cudaStream_t s)
{
    using C = Cfg<KF, VF, D, G8>;
    static DeviceOnce once;
    if (once.needed()) {
        cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, KF, VF, G8, BR>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return e;
        once.mark();
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kDecodeThreads);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_kernel<D, KF, VF, G8, BR>, p);
}

template <int D, int KF, int VF>
cudaError_t launch_g(const DecodeParams &p, dim3 grid, cudaStream_t s)
{
    if (p.rotate == 2)
        return p.L.g > 4 ? launch_t<D, KF, VF, true, true>(p, grid, s) : launch_t<D, KF, VF, false, true>(p, grid, s);
    return p.L.g > 4 ? launch_t<D, KF, VF, true, false>(p, grid, s) : launch_t<D, KF, VF, false, false>(p, grid, s);
}

}  // namespace

bool decode_supported(const Layout &L)
{
    if (L.g < 1 || L.g > kMaxGqa) return false;
    if (L.v_fmt != KVQ_INT4_ASYM && L.v_fmt != KVQ_INT2_ASYM) return false;
    if (L.d == 64) return L.k_fmt == KVQ_INT4_ASYM && L.v_fmt == KVQ_INT4_ASYM;
    return L.d == 128;
}

int decode_max_splits(const Layout &) { return kCombineSplits; }

cudaError_t launch_decode(const DecodeParams &p, dim3 grid, cudaStream_t s)
{
    const Layout &L = p.L;
    if (L.d == 64) return launch_g<64, KVQ_INT4_ASYM, KVQ_INT4_ASYM>(p, grid, s);
    if (L.v_fmt == KVQ_INT4_ASYM) {
        switch (L.k_fmt) {
        case KVQ_INT4_ASYM: return launch_g<128, KVQ_INT4_ASYM, KVQ_INT4_ASYM>(p, grid, s);
        case KVQ_INT8_SYM: return launch_g<128, KVQ_INT8_SYM, KVQ_INT4_ASYM>(p, grid, s);
        default: return launch_g<128, KVQ_INT2_ASYM, KVQ_INT4_ASYM>(p, grid, s);
        }
    }
    switch (L.k_fmt) {
    case KVQ_INT4_ASYM: return launch_g<128, KVQ_INT4_ASYM, KVQ_INT2_ASYM>(p, grid, s);
    case KVQ_INT8_SYM: return launch_g<128, KVQ_INT8_SYM, KVQ_INT2_ASYM>(p, grid, s);
    default: return launch_g<128, KVQ_INT2_ASYM, KVQ_INT2_ASYM>(p, grid, s);
    }
}

}  // namespace kvq
