// kvq_append.cu -- quantise-on-append: load an fp16 K or V row, apply the
// random sign and the Walsh-Hadamard butterflies in fp32, compute per-group
// statistics, scale/zero, round to codes and store them packed into the paged
// pool ["When Quantization Is Free", Methodology 2: sign in registers,
// butterfly passes, per-group scaling, rounding, nibble packing; "Runtime-
// Certified Bounded-Error Quantized Attention", Methodology 1: INT8 keys,
// INT4 values, per-block error descriptors; "OSCAR", 2.2: INT2 with clipping].
//
// A row of d elements is spread over d/64 consecutive lanes (one lane for
// d = 64, two for d = 128), 64 elements each, held as 32 fp32 pairs.  The
// butterfly stage h = 1 pairs the two halves of a register pair (scalar
// add/sub); stages h = 2..32 pair register pairs (packed f32x2 add / fma);
// stage h = 64 pairs the row's two lanes (one shuffle per element and a
// packed exact fma(+-1, x, partner)).  The stages run in the order h = 1, 2,
// 4, ... of a plain fp32 statement of the transform, each result rounded to
// nearest, and every codec operation is an explicitly rounded operation, so
// the integer codes match that plain statement bit for bit.  For int4 a lane
// holds two quantisation groups; int2/int8 row statistics reduce over the
// row's lanes.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23: x + magic rounds x to an integer (ties to even)
constexpr unsigned long long kAppendWaitNs = 1000000000ull;  // 1 s per bounded wait

__device__ __forceinline__ float code_value(uint32_t cw) { return __fsub_rn(__uint_as_float(cw), kRoundMagic); }

__device__ __forceinline__ uint32_t pack4bytes(uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3)
{
    const uint32_t t01 = __byte_perm(b0, b1, 0x0040);
    const uint32_t t23 = __byte_perm(b2, b3, 0x0040);
    return __byte_perm(t01, t23, 0x5410);
}

__device__ __forceinline__ float min3(float a, float b, float c)
{
    float r;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ float max3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// A constant pair held in a register pair: the packed instructions take
// their operands from registers, and a pair the compiler may re-materialise
// costs a move at every use.
__device__ __forceinline__ float2 reg_pair(float x, float y)
{
    float2 r;
    asm volatile("mov.b32 %0, %2;\n\tmov.b32 %1, %3;" : "=f"(r.x), "=f"(r.y) : "f"(x), "f"(y));
    return r;
}

// The constant pairs of the packed arithmetic: (-1, -1) and the rounding
// magic, set up once per row.
struct PackC {
    float2 m1, magic;
};
__device__ __forceinline__ PackC pack_consts()
{
    return PackC{reg_pair(-1.0f, -1.0f), reg_pair(kRoundMagic, kRoundMagic)};
}

// a - b, rounded once: fma(b, -1, a)
__device__ __forceinline__ float2 sub2(float2 a, float2 b, const PackC &k) { return __ffma2_rn(b, k.m1, a); }

// codes of a pair: clamp(rint((y - z) * inv), lo, hi) as the low bits of
// (value + magic); the clamp comes before the rounding, which gives the same
// integer
__device__ __forceinline__ void quant_pair(float2 y, float2 z2, float2 inv2, float lo, float hi, uint32_t &c0,
                                           uint32_t &c1, const PackC &k)
{
    float2 t = __fmul2_rn(sub2(y, z2, k), inv2);
    t.x = fminf(fmaxf(t.x, lo), hi);
    t.y = fminf(fmaxf(t.y, lo), hi);
    t = __fadd2_rn(t, k.magic);
    c0 = __float_as_uint(t.x);
    c1 = __float_as_uint(t.y);
}

// The same codes for rows whose largest element already codes at most the
// top code: every step (subtract, multiply by inv > 0 or 0, add the rounding
// magic) is monotone in y, so no element needs the upper clamp.  The lower
// clamp stays: it also keeps the multiply and the add apart (fused into one
// multiply-add they would round once where the codec rounds twice, and a
// product just below a half-way point that rounds up onto it would then
// code differently).
__device__ __forceinline__ void quant_pair_lo(float2 y, float2 z2, float2 inv2, float lo, uint32_t &c0, uint32_t &c1,
                                              const PackC &k)
{
    float2 t = __fmul2_rn(sub2(y, z2, k), inv2);
    t.x = fmaxf(t.x, lo);
    t.y = fmaxf(t.y, lo);
    t = __fadd2_rn(t, k.magic);
    c0 = __float_as_uint(t.x);
    c1 = __float_as_uint(t.y);
}

// The unclamped integer code of one value, by the same operations.
__device__ __forceinline__ int code_of(float y, float z, float inv)
{
    return (int)(__float_as_uint(__fadd_rn(__fmul_rn(__fsub_rn(y, z), inv), kRoundMagic)) - 0x4B400000u);
}

// The value of lane ^ 16, every operand an immediate.
__device__ __forceinline__ float shfl_xor16(float v)
{
    float r;
    asm volatile("shfl.sync.bfly.b32 %0, %1, 16, 0x1f, 0xffffffff;" : "=f"(r) : "f"(v));
    return r;
}

// min / max over the row's lanes (lane and lane ^ 16 for d = 128)
template <int LANES> __device__ __forceinline__ float row_min(float v)
{
    if constexpr (LANES == 2) v = fminf(v, __shfl_xor_sync(kFull, v, 16));
    return v;
}
template <int LANES> __device__ __forceinline__ float row_max(float v)
{
    if constexpr (LANES == 2) v = fmaxf(v, __shfl_xor_sync(kFull, v, 16));
    return v;
}

// min and max of the N pairs y[0 .. N), 3-input min/max in four independent
// chains (short dependency chains; min/max are exact in any order)
template <int N>
__device__ __forceinline__ void pair_minmax(const float2 *y, float &lo, float &hi)
{
    static_assert(N % 4 == 0, "four chains");
    float l[4], h[4];
#pragma unroll
    for (int c = 0; c < 4; c++) {
        l[c] = fminf(y[c].x, y[c].y);
        h[c] = fmaxf(y[c].x, y[c].y);
    }
#pragma unroll
    for (int i = 4; i < N; i += 4)
#pragma unroll
        for (int c = 0; c < 4; c++) {
            l[c] = min3(l[c], y[i + c].x, y[i + c].y);
            h[c] = max3(h[c], y[i + c].x, y[i + c].y);
        }
    lo = fminf(min3(l[0], l[1], l[2]), l[3]);
    hi = fmaxf(max3(h[0], h[1], h[2]), h[3]);
}

// Dequantisation error and magnitude of a pair (descriptors): the stored
// value is code * scale + zero, each step rounded.
__device__ __forceinline__ void pair_err(float2 y, uint32_t c0, uint32_t c1, float2 s2, float2 z2, float &emax,
                                         float &amax, const PackC &k)
{
    float2 yh = make_float2(code_value(c0), code_value(c1));
    yh = __fadd2_rn(__fmul2_rn(yh, s2), z2);
    const float2 e = sub2(y, yh, k);
    emax = max3(emax, fabsf(e.x), fabsf(e.y));
    amax = max3(amax, fabsf(y.x), fabsf(y.y));
}

// Squared reconstruction error of NP pairs quantised with scale sf and zero
// z (the codec's arithmetic), summed in fp32 with the even and the odd
// elements apart, in order, then added.  The reconstruction and the sums use
// the scalar _rn operations, which are never fused into a multiply-add (a
// fused square-and-add rounds once instead of twice and was seen to move a
// near-tie decision).
template <int NP>
__device__ __forceinline__ float run_sq_error(const float2 *y, float2 z2, float sf, float lo, float hi, const PackC &k)
{
    const float inv = (sf == 0.0f) ? 0.0f : __fdiv_rn(1.0f, sf);
    const float2 inv2 = make_float2(inv, inv);
    float ev = 0.0f, od = 0.0f;
#pragma unroll
    for (int i = 0; i < NP; i++) {
        uint32_t c0, c1;
        quant_pair(y[i], z2, inv2, lo, hi, c0, c1, k);
        const float h0 = __fadd_rn(__fmul_rn(code_value(c0), sf), z2.x);
        const float h1 = __fadd_rn(__fmul_rn(code_value(c1), sf), z2.x);
        const float e0 = __fsub_rn(y[i].x, h0), e1 = __fsub_rn(y[i].y, h1);
        ev = __fadd_rn(ev, __fmul_rn(e0, e0));
        od = __fadd_rn(od, __fmul_rn(e1, e1));
    }
    return __fadd_rn(ev, od);
}

// ScaleSearch ["Search Your Block Floating Point Scales!", ScaleSearch] on
// the fp16 scale: the candidates' bit patterns are the default's plus f,
// tried as f = 0, -1, 1, -2, 2, 3, 4, 5, 6 (positive finite ones only); the
// least squared error wins, a later candidate only if strictly better.  A
// group spread over the row's two lanes adds the two lanes' sums (each lane
// holds a run of 64 consecutive elements).  Every lane of the warp runs every
// candidate, so the shuffle never diverges.
template <int NP, int LANES>
__device__ __forceinline__ __half search_scale(const float2 *y, __half sh0, float zf, float lo, float hi, const PackC &kc)
{
    const int b0 = __half_as_ushort(sh0);
    const bool searchable = b0 != 0 && b0 < 0x7C00;
    const float2 z2 = make_float2(zf, zf);
    int best = b0;
    float best_err = 0.0f;
#pragma unroll 1
    for (int k = 0; k < 9; k++) {
        const int f = k == 0 ? 0 : k == 1 ? -1 : k == 2 ? 1 : k == 3 ? -2 : k - 2;
        const int bits = b0 + f;
        const bool valid = searchable && bits > 0 && bits < 0x7C00;
        const float sf = valid ? __half2float(__ushort_as_half((unsigned short)bits)) : 0.0f;
        float err = run_sq_error<NP>(y, z2, sf, lo, hi, kc);
        if constexpr (LANES == 2) err = __fadd_rn(err, __shfl_xor_sync(kFull, err, 16));
        if (valid && (k == 0 || err < best_err)) {
            best = bits;
            best_err = err;
        }
    }
    return __ushort_as_half((unsigned short)best);
}

// (a + b, a - b) of the fp16 halves (a low, b high) of w: the exact fp16
// values added and subtracted in fp32 with one rounding each (b widened,
// then two mixed-precision operations)
__device__ __forceinline__ float2 h1_butterfly(uint32_t w)
{
    float s, d, b;
    asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %3;\n cvt.f32.f16 %2, hi;\n"
        " add.rn.f32.f16 %0, lo, %2;\n sub.rn.f32.f16 %1, lo, %2;\n}"
        : "=f"(s), "=f"(d), "=f"(b)
        : "r"(w));
    return make_float2(s, d);
}

// v with its low n bits in reverse order
__host__ __device__ constexpr int rev_bits(int v, int n) { return n == 0 ? 0 : ((v & 1) << (n - 1)) | rev_bits(v >> 1, n - 1); }

// OSCAR's bit-reversal permutation P_br of a rotated row, after H and c_d
// ("OSCAR", 2.2(a)): element i moves to position br(i), br reversing the
// log2(d) index bits.  d = 128, two lanes a row: half s holds elements
// 64 s + k as pairs y[t] = (k = 2t, 2t + 1); element (s, t, c) lands in half
// c at pair br5(t), component s.  So lane s keeps component s of each pair,
// trades the other with its partner (one shuffle a pair) and the pairs move
// to slot br5(t).  d = 64, one lane a row: a fixed reordering of the lane's
// registers.  A permutation: every value is moved, none is changed.
template <int LANES>
__device__ __forceinline__ void bitrev_row(float2 (&y)[32], int s)
{
    float2 z[32];
    if constexpr (LANES == 2) {
#pragma unroll
        for (int t = 0; t < 32; t++) {
            const float recv = shfl_xor16(s ? y[t].x : y[t].y);
            z[rev_bits(t, 5)] = s ? make_float2(recv, y[t].y) : make_float2(y[t].x, recv);
        }
    } else {
#pragma unroll
        for (int u = 0; u < 32; u++) {
            const int k0 = rev_bits(2 * u, 6), k1 = rev_bits(2 * u + 1, 6);
            z[u] = make_float2((k0 & 1) ? y[k0 >> 1].y : y[k0 >> 1].x, (k1 & 1) ? y[k1 >> 1].y : y[k1 >> 1].x);
        }
    }
#pragma unroll
    for (int t = 0; t < 32; t++) y[t] = z[t];
}

template <int D, int FMT, bool SEARCH>
__device__ __forceinline__ void half_row(const AppendParams &p, const uint32_t *sign_xor, const unsigned char *src,
                                         unsigned char *chunk, int tok, int tensor, int s, bool active,
                                         unsigned int *desc, int x, const float (&csc)[8])
{
    constexpr int LANES = D / 64;
    constexpr unsigned PARTNER = 16;  // the row's other lane (d = 128)
    const Layout &L = p.L;
    const PackC kc = pack_consts();
    // ---- 64 fp16 from the staged row (shared memory), flip signs (exact), widen to 32 pairs ----
    // Slot i takes the row's 16-byte chunk i ^ x (x = this lane's row mod 8
    // when rotating, else 0), so that the lanes of a row group read distinct
    // banks of the densely staged rows.  The butterflies undo the
    // permutation: a Sylvester Hadamard transform of a vector whose index is
    // XORed with x is the transform of the vector with entry k negated when
    // popcount(k & x) is odd.  Each butterfly then forms the same sum (its
    // operands swapped) or the negated difference of the unpermuted order,
    // so every value is exactly plus or minus the unpermuted one, and the
    // final scale by +-c_d (csc, per chunk) restores the signs exactly.
    float2 y[32];
    {
        const uint4 *s4 = reinterpret_cast<const uint4 *>(src + 128 * s);
        uint4 w[8];
#pragma unroll
        for (int i = 0; i < 8; i++) w[i] = s4[i ^ x];
        const uint4 *sx4 = reinterpret_cast<const uint4 *>(sign_xor + 32 * s);
#pragma unroll
        for (int i = 0; i < 8; i++) {
            uint32_t ww[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
            if (p.rotate) {
                const uint4 m = sx4[i ^ x];
                ww[0] ^= m.x;
                ww[1] ^= m.y;
                ww[2] ^= m.z;
                ww[3] ^= m.w;
            }
            if (p.rotate) {
                // butterfly h = 1 straight from the fp16 pair: (a + b, a - b),
                // each rounded once in fp32 from the exact fp16 values
#pragma unroll
                for (int e = 0; e < 4; e++) y[4 * i + e] = h1_butterfly(ww[e]);
            } else {
#pragma unroll
                for (int e = 0; e < 4; e++) y[4 * i + e] = __half22float2(bits_h2(ww[e]));
            }
        }
    }
    // ---- butterflies: h = 2..32 across pairs, h = 64 across lanes ----
    if (p.rotate) {
#pragma unroll
        for (int hh = 1; hh < 32; hh <<= 1)
#pragma unroll
            for (int i = 0; i < 32; i++)
                if (!(i & hh)) {
                    const float2 a = y[i], b = y[i + hh];
                    y[i] = __fadd2_rn(a, b);
                    y[i + hh] = sub2(a, b, kc);
                }
        if constexpr (LANES == 2) {
            // lower lane: a + b; upper lane: a - b with a = the lower lane's value
            const float sg = s ? -1.0f : 1.0f;
            const float2 sg2 = make_float2(sg, sg);
#pragma unroll
            for (int i = 0; i < 32; i++) {
                const float2 o = make_float2(shfl_xor16(y[i].x), shfl_xor16(y[i].y));
                y[i] = __ffma2_rn(sg2, y[i], o);
            }
        }
#pragma unroll
        for (int i = 0; i < 32; i++) y[i] = __fmul2_rn(y[i], reg_pair(csc[i >> 2], csc[i >> 2]));
        if (p.rotate == 2) bitrev_row<LANES>(y, s);
    }

    unsigned char *codes = chunk + (tensor ? L.v_codes : L.k_codes);
    unsigned char *meta = chunk + (tensor ? L.v_meta : L.k_meta) + tok * (tensor ? L.v_row_meta : L.k_row_meta);
    const bool want_desc = desc != nullptr;
    float emax = 0.0f, amax = 0.0f;

    if (FMT == KVQ_INT4_ASYM) {
        // two groups of 32 per lane (16 pairs each), one 16-byte chunk each
        uint32_t sz[2][2];  // [scale|zero][group] fp16 bits
        float zfs[2], infs[2], sfs[2];
        bool fits = true;  // both groups' largest elements code at most 15
#pragma unroll
        for (int gq = 0; gq < 2; gq++) {
            const float2 *yg = y + 16 * gq;
            float lo, hi;
            pair_minmax<16>(yg, lo, hi);
            const float hi_y = hi;
            if (p.clip < 1.0f) {
                lo = __fmul_rn(lo, p.clip);
                hi = __fmul_rn(hi, p.clip);
            }
            __half shh = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 15.0f));
            const __half zhh = __float2half_rn(lo);
            if constexpr (SEARCH) shh = search_scale<16, 1>(yg, shh, __half2float(zhh), 0.0f, 15.0f, kc);
            sfs[gq] = __half2float(shh);
            zfs[gq] = __half2float(zhh);
            infs[gq] = (sfs[gq] == 0.0f) ? 0.0f : __fdiv_rn(1.0f, sfs[gq]);
            fits = fits && code_of(hi_y, zfs[gq], infs[gq]) <= 15;
            sz[0][gq] = __half_as_ushort(shh);
            sz[1][gq] = __half_as_ushort(zhh);
        }
        fits = __all_sync(kFull, fits || !active);
#pragma unroll
        for (int gq = 0; gq < 2; gq++) {
            const float2 *yg = y + 16 * gq;
            const float2 z2 = make_float2(zfs[gq], zfs[gq]), inv2 = make_float2(infs[gq], infs[gq]);
            const float2 s2 = make_float2(sfs[gq], sfs[gq]);
            uint32_t w[4];
            if (fits && !want_desc) {
#pragma unroll
                for (int m = 0; m < 4; m++) {
                    uint32_t bb[4];
#pragma unroll
                    for (int k = 0; k < 4; k++) {
                        uint32_t c0, c1;
                        quant_pair_lo(yg[4 * m + k], z2, inv2, 0.0f, c0, c1, kc);
                        bb[k] = c0 + (c1 << 4);
                    }
                    w[m] = pack4bytes(bb[0], bb[1], bb[2], bb[3]);
                }
            } else {
#pragma unroll
                for (int m = 0; m < 4; m++) {
                    uint32_t bb[4];
#pragma unroll
                    for (int k = 0; k < 4; k++) {
                        uint32_t c0, c1;
                        quant_pair(yg[4 * m + k], z2, inv2, 0.0f, 15.0f, c0, c1, kc);
                        if (want_desc) pair_err(yg[4 * m + k], c0, c1, s2, z2, emax, amax, kc);
                        bb[k] = c0 + (c1 << 4);
                    }
                    w[m] = pack4bytes(bb[0], bb[1], bb[2], bb[3]);
                }
            }
            if (active) *reinterpret_cast<uint4 *>(codes + ((2 * s + gq) * 16 + tok) * 16) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        if (active) {
            constexpr int NG = D / 32;
            *reinterpret_cast<uint32_t *>(meta + 4 * s) = sz[0][0] | (sz[0][1] << 16);
            *reinterpret_cast<uint32_t *>(meta + 2 * NG + 4 * s) = sz[1][0] | (sz[1][1] << 16);
        }
    } else if (FMT == KVQ_INT2_ASYM) {
        // one group over the row; this lane's 64 codes are stream bytes [16s, 16s+16)
        float lo, hi;
        pair_minmax<32>(y, lo, hi);
        lo = row_min<LANES>(lo);
        hi = row_max<LANES>(hi);
        const float hi_y = hi;
        if (p.clip < 1.0f) {
            lo = __fmul_rn(lo, p.clip);
            hi = __fmul_rn(hi, p.clip);
        }
        __half shh = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 3.0f));
        const __half zhh = __float2half_rn(lo);
        if constexpr (SEARCH) shh = search_scale<32, LANES>(y, shh, __half2float(zhh), 0.0f, 3.0f, kc);
        const float sf = __half2float(shh), zf = __half2float(zhh);
        const float inv = (sf == 0.0f) ? 0.0f : __fdiv_rn(1.0f, sf);
        const float2 z2 = make_float2(zf, zf), inv2 = make_float2(inv, inv), s2 = make_float2(sf, sf);
        // the row's largest element codes at most 3 (clipping leaves it there
        // for rows around zero): then no element needs the upper clamp
        const bool fits = __all_sync(kFull, code_of(hi_y, zf, inv) <= 3 || !active);
        uint32_t w[4];
        if (fits && !want_desc) {
#pragma unroll
            for (int m = 0; m < 4; m++) {
                uint32_t bb[4];
#pragma unroll
                for (int k = 0; k < 4; k++) {
                    uint32_t c[4];
                    quant_pair_lo(y[8 * m + 2 * k], z2, inv2, 0.0f, c[0], c[1], kc);
                    quant_pair_lo(y[8 * m + 2 * k + 1], z2, inv2, 0.0f, c[2], c[3], kc);
                    bb[k] = c[0] + (c[1] << 2) + (c[2] << 4) + (c[3] << 6);
                }
                w[m] = pack4bytes(bb[0], bb[1], bb[2], bb[3]);
            }
        } else {
#pragma unroll
            for (int m = 0; m < 4; m++) {
                uint32_t bb[4];
#pragma unroll
                for (int k = 0; k < 4; k++) {
                    uint32_t c[4];
                    quant_pair(y[8 * m + 2 * k], z2, inv2, 0.0f, 3.0f, c[0], c[1], kc);
                    quant_pair(y[8 * m + 2 * k + 1], z2, inv2, 0.0f, 3.0f, c[2], c[3], kc);
                    if (want_desc) {
                        pair_err(y[8 * m + 2 * k], c[0], c[1], s2, z2, emax, amax, kc);
                        pair_err(y[8 * m + 2 * k + 1], c[2], c[3], s2, z2, emax, amax, kc);
                    }
                    bb[k] = c[0] + (c[1] << 2) + (c[2] << 4) + (c[3] << 6);
                }
                w[m] = pack4bytes(bb[0], bb[1], bb[2], bb[3]);
            }
        }
        if (active) {
            *reinterpret_cast<uint4 *>(codes + (s * 16 + tok) * 16) = make_uint4(w[0], w[1], w[2], w[3]);
            if (s == 0)
                *reinterpret_cast<uint32_t *>(meta) = __half_as_ushort(shh) | (uint32_t(__half_as_ushort(zhh)) << 16);
        }
    } else {
        // symmetric int8, one fp16 scale (rounded up) per row; 64 bytes per lane
        float am[4];
#pragma unroll
        for (int c = 0; c < 4; c++) am[c] = fmaxf(fabsf(y[c].x), fabsf(y[c].y));
#pragma unroll
        for (int i = 4; i < 32; i += 4)
#pragma unroll
            for (int c = 0; c < 4; c++) am[c] = max3(am[c], fabsf(y[i + c].x), fabsf(y[i + c].y));
        float a = fmaxf(max3(am[0], am[1], am[2]), am[3]);
        a = row_max<LANES>(a);
        __half shh = __float2half_ru(__fdiv_rn(a, 127.0f));
        if constexpr (SEARCH) shh = search_scale<32, LANES>(y, shh, 0.0f, -127.0f, 127.0f, kc);
        const float sf = __half2float(shh);
        const float inv = (sf == 0.0f) ? 0.0f : __fdiv_rn(1.0f, sf);
        if (want_desc) amax = a;
        const float2 inv2 = make_float2(inv, inv), s2 = make_float2(sf, sf), z2 = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int c = 0; c < 4; c++) {
            uint32_t w[4];
#pragma unroll
            for (int m = 0; m < 4; m++) {
                uint32_t cw[4];
                quant_pair(y[8 * c + 2 * m], z2, inv2, -127.0f, 127.0f, cw[0], cw[1], kc);
                quant_pair(y[8 * c + 2 * m + 1], z2, inv2, -127.0f, 127.0f, cw[2], cw[3], kc);
                if (want_desc) {
                    float unused = 0.0f;
                    pair_err(y[8 * c + 2 * m], cw[0], cw[1], s2, z2, emax, unused, kc);
                    pair_err(y[8 * c + 2 * m + 1], cw[2], cw[3], s2, z2, emax, unused, kc);
                }
                w[m] = pack4bytes(cw[0], cw[1], cw[2], cw[3]);
            }
            if (active) *reinterpret_cast<uint4 *>(codes + ((4 * s + c) * 16 + tok) * 16) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        if (active && s == 0) *reinterpret_cast<uint16_t *>(meta) = __half_as_ushort(shh);
    }
    if (want_desc) {
        emax = row_max<LANES>(emax);
        amax = row_max<LANES>(amax);
        // non-negative floats order like their bit patterns
        if (active && s == 0) {
            if (tensor == 0) {
                atomicMax(desc + 0, __float_as_uint(emax));
            } else {
                atomicMax(desc + 1, __float_as_uint(emax));
                atomicMax(desc + 2, __float_as_uint(amax));
            }
        }
    }
}

// Rows are processed in groups of 32/LANES consecutive rows of one tensor per
// warp (16 rows for d = 128).  Each group (contiguous in the input) is staged
// in shared memory by one bulk copy, double-buffered so the next group
// streams in while this one is computed; lane (row = lane & 15, half =
// lane >> 4) reads its half-row with 16-byte loads in the chunk order
// i ^ (row & 7), which keeps the eight rows of a load phase on distinct banks
// (see half_row).  Persistent grid: each warp takes groups g, g + all
// warps, ...
constexpr int kAppendWarps = 8;

template <int D> struct AppendSmem {
    static constexpr int LANES = D / 64;
    static constexpr int ROWS = 32 / LANES;       // rows per group
    static constexpr int ROW_BYTES = 2 * D;
    static constexpr int STRIDE = ROW_BYTES;
    static constexpr int BUF = ROWS * STRIDE;
    static constexpr int BYTES = kAppendWarps * 2 * BUF + kAppendWarps * 2 * 8;  // buffers + mbarriers
};

template <int D, int KF, int VF, bool SEARCH>
__global__ void __launch_bounds__(kAppendWarps * 32, SEARCH ? 1 : 2) append_kernel(const __grid_constant__ AppendParams p)
{
    using S = AppendSmem<D>;
    constexpr int LANES = S::LANES, ROWS = S::ROWS;
    __shared__ __align__(16) uint32_t sign_xor[kMaxD / 2];
    extern __shared__ __align__(128) unsigned char smem[];
    if (threadIdx.x < D / 2) sign_xor[threadIdx.x] = p.sign_xor[threadIdx.x];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = lane % ROWS, s = lane / ROWS;  // row in the group, half of the row
    unsigned char *buf0 = smem + warp * 2 * S::BUF;
    const uint32_t bar0 = smem_u32(smem + kAppendWarps * 2 * S::BUF) + warp * 16;
    if (lane == 0) {
        mbar_init(bar0, 1);
        mbar_init(bar0 + 8, 1);
        fence_mbar_init();
    }
    __syncthreads();

    const int rows_per_tensor = p.n_tok * p.L.hkv;
    const int groups_per_tensor = (rows_per_tensor + ROWS - 1) / ROWS;
    const int n_groups = 2 * groups_per_tensor;
    const int stride = gridDim.x * kAppendWarps;
    const bool hkv_pow2 = (p.L.hkv & (p.L.hkv - 1)) == 0;
    const int hkv_shift = __ffs(p.L.hkv) - 1;
    const int g0 = blockIdx.x * kAppendWarps + warp;
    // this lane's chunk order and the signed output scales it implies (half_row)
    const int xr = p.rotate ? (r & 7) : 0;
    float csc[8];
#pragma unroll
    for (int c = 0; c < 8; c++) csc[c] = (__popc(c & xr) & 1) ? -p.rot_scale : p.rot_scale;

    // start the copy of group gi (its nrows rows, contiguous) into buffer bsel
    auto issue = [&](int gi, int bsel) {
        const int tensor = gi >= groups_per_tensor;
        const int row0 = (gi - tensor * groups_per_tensor) * ROWS;
        const int nrows = min(ROWS, rows_per_tensor - row0);
        // relaxed arm, no proxy fence: the buffer was last read (generic
        // loads, complete before the __syncwarp ending its group) and the
        // copy's completion is what publishes the data
        if (lane == 0)
            bulk_load(smem_u32(buf0 + bsel * S::BUF), (tensor ? p.v : p.k) + (long long)row0 * D,
                      (uint32_t)(nrows * S::ROW_BYTES), bar0 + 8 * bsel);
    };

    if (g0 < n_groups) issue(g0, 0);
    int it = 0;
    for (int gi = g0; gi < n_groups; gi += stride, it++) {
        const int bsel = it & 1;
        if (gi + stride < n_groups) issue(gi + stride, bsel ^ 1);
        // this group's row: slot, page, chunk (independent of the staged data)
        const int tensor = gi >= groups_per_tensor;
        const int row = (gi - tensor * groups_per_tensor) * ROWS + r;
        bool active = row < rows_per_tensor;
        const int rem = active ? row : 0;
        const int n = hkv_pow2 ? (rem >> hkv_shift) : rem / p.L.hkv, kvh = rem - n * p.L.hkv;
        const int slot = p.slots[n];
        if (slot < 0) active = false;
        if (active && slot >= p.L.num_pages * kPageTokens) {
            if (s == 0) set_status(p.pool, KVQ_ERR_OUT_OF_RANGE);
            active = false;
        }
        const int page = active ? slot / kPageTokens : 0, tok = active ? slot % kPageTokens : 0;
        unsigned char *chunk =
            p.pool + kHeaderBytes + (long long)page * p.L.page_bytes + (long long)kvh * p.L.chunk_bytes;
        unsigned int *desc = p.L.desc_off ? reinterpret_cast<unsigned int *>(p.pool + p.L.desc_off +
                                                                             ((long long)page * p.L.hkv + kvh) * 16)
                                          : nullptr;
        if (!mbar_wait_bounded(bar0 + 8 * bsel, (it >> 1) & 1, kAppendWaitNs)) {
            if (lane == 0) set_status(p.pool, KVQ_ERR_TIMEOUT);
            // the other buffer may still have copies in flight: wait for them (bounded) and stop
            if (gi + stride < n_groups) (void)mbar_wait_bounded(bar0 + 8 * (bsel ^ 1), ((it + 1) >> 1) & 1, kAppendWaitNs);
            break;
        }
        const unsigned char *src = buf0 + bsel * S::BUF + r * S::STRIDE;
        if (tensor == 0) half_row<D, KF, SEARCH>(p, sign_xor, src, chunk, tok, 0, s, active, desc, xr, csc);
        else half_row<D, VF, SEARCH>(p, sign_xor, src, chunk, tok, 1, s, active, desc, xr, csc);
        __syncwarp();  // every lane is done with this buffer before it is refilled
    }
    (void)LANES;
}

// Persistent grid: as many CTAs as stay resident (the instantiation's own
// occupancy), at most one per eight groups of work.
template <int D, int KF, int VF, bool SEARCH>
cudaError_t launch_one_s(const AppendParams &p, long long want, int num_sms, cudaStream_t st)
{
    static DeviceOnce once;
    static int resident = 1;
    if (once.needed()) {
        cudaError_t e = cudaFuncSetAttribute(append_kernel<D, KF, VF, SEARCH>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, AppendSmem<D>::BYTES);
        if (e != cudaSuccess) return e;
        int n = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, append_kernel<D, KF, VF, SEARCH>, kAppendWarps * 32,
                                                          AppendSmem<D>::BYTES);
        if (e != cudaSuccess) return e;
        resident = n < 1 ? 1 : (n > 2 ? 2 : n);
        once.mark();
    }
    const long long cap = (long long)resident * num_sms;
    const int blocks = (int)(want < cap ? want : cap);
    append_kernel<D, KF, VF, SEARCH><<<blocks, kAppendWarps * 32, AppendSmem<D>::BYTES, st>>>(p);
    return cudaGetLastError();
}

// The scale search is its own instantiation so that the kernel without it
// keeps its register budget (two CTAs per SM).
template <int D, int KF, int VF>
cudaError_t launch_one(const AppendParams &p, long long want, int num_sms, cudaStream_t st)
{
    return p.scale_search ? launch_one_s<D, KF, VF, true>(p, want, num_sms, st)
                          : launch_one_s<D, KF, VF, false>(p, want, num_sms, st);
}

template <int D, int KF>
cudaError_t launch_d_k(const AppendParams &p, long long want, int num_sms, cudaStream_t st)
{
    switch (p.L.v_fmt) {
    case KVQ_INT4_ASYM: return launch_one<D, KF, KVQ_INT4_ASYM>(p, want, num_sms, st);
    case KVQ_INT8_SYM: return launch_one<D, KF, KVQ_INT8_SYM>(p, want, num_sms, st);
    default: return launch_one<D, KF, KVQ_INT2_ASYM>(p, want, num_sms, st);
    }
}

template <int D>
cudaError_t launch_d(const AppendParams &p, long long want, int num_sms, cudaStream_t st)
{
    switch (p.L.k_fmt) {
    case KVQ_INT4_ASYM: return launch_d_k<D, KVQ_INT4_ASYM>(p, want, num_sms, st);
    case KVQ_INT8_SYM: return launch_d_k<D, KVQ_INT8_SYM>(p, want, num_sms, st);
    default: return launch_d_k<D, KVQ_INT2_ASYM>(p, want, num_sms, st);
    }
}

}  // namespace

cudaError_t launch_append(const AppendParams &p, int num_sms, cudaStream_t st)
{
    const long long rows_per_tensor = (long long)p.n_tok * p.L.hkv;
    if (rows_per_tensor == 0) return cudaSuccess;
    if (rows_per_tensor > (1ll << 30)) return cudaErrorInvalidValue;  // 32-bit row indexing
    const int rows = p.L.d == 64 ? 32 : 16;
    const long long groups = 2 * ((rows_per_tensor + rows - 1) / rows);
    const long long want = (groups + kAppendWarps - 1) / kAppendWarps;
    return p.L.d == 64 ? launch_d<64>(p, want, num_sms, st) : launch_d<128>(p, want, num_sms, st);
}

}  // namespace kvq
