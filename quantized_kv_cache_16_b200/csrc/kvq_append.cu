// kvq_append.cu -- quantise-on-append: load an fp16 K or V row, apply the
// random sign and the Walsh-Hadamard butterflies in fp32, compute per-group
// statistics, scale/zero, round to codes and store them packed into the paged
// pool ["When Quantization Is Free", Methodology 2: sign in registers,
// butterfly passes, per-group scaling, rounding, nibble packing; "Runtime-
// Certified Bounded-Error Quantized Attention", Methodology 1: INT8 keys,
// INT4 values, per-block error descriptors; "OSCAR", 2.2: INT2 with clipping].
//
// One thread owns one token-head row, so all log2(d) butterfly stages run in
// registers with no exchange between threads.  Every codec operation is an
// explicitly rounded intrinsic: the integer codes must match a plain fp32
// statement of the same steps bit for bit.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23: x + magic rounds x to an integer (ties to even)

template <int D>
__device__ __forceinline__ void fwht(float (&y)[D])
{
    // Sylvester order: half-width h = 1, 2, 4, ..., D/2; (a, b) -> (a + b, a - b).
#pragma unroll
    for (int h = 1; h < D; h <<= 1) {
#pragma unroll
        for (int j = 0; j < D; j++) {
            if (!(j & h)) {
                const float a = y[j], b = y[j + h];
                y[j] = __fadd_rn(a, b);
                y[j + h] = __fsub_rn(a, b);
            }
        }
    }
}

// Load one fp16 row, flip the signs (exact), rotate in fp32.
template <int D>
__device__ __forceinline__ void load_rotated(const AppendParams &p, const __half *src, float (&y)[D])
{
    const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
#pragma unroll
    for (int i = 0; i < D / 8; i++) {
        const uint4 w = __ldg(s4 + i);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; e++) {
            uint32_t x = ww[e];
            if (p.rotate) x ^= p.sign_xor[i * 4 + e];
            const float2 f = __half22float2(bits_h2(x));
            y[8 * i + 2 * e] = f.x;
            y[8 * i + 2 * e + 1] = f.y;
        }
    }
    if (p.rotate) {
        fwht<D>(y);
#pragma unroll
        for (int i = 0; i < D; i++) y[i] = __fmul_rn(y[i], p.rot_scale);
    }
}

// code (as the low bits of x + magic), clamped to [lo, hi] before rounding
__device__ __forceinline__ uint32_t round_code(float v, float lo, float hi)
{
    v = fminf(fmaxf(v, lo), hi);
    return __float_as_uint(__fadd_rn(v, kRoundMagic));
}

__device__ __forceinline__ float code_value(uint32_t cw) { return __fsub_rn(__uint_as_float(cw), kRoundMagic); }

__device__ __forceinline__ uint32_t pack4bytes(uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3)
{
    const uint32_t t01 = __byte_perm(b0, b1, 0x0040);
    const uint32_t t23 = __byte_perm(b2, b3, 0x0040);
    return __byte_perm(t01, t23, 0x5410);
}

struct RowOut {
    unsigned char *codes;  // region start of this (page, kv head, tensor)
    unsigned char *meta;   // this token's meta row
    int tok;
};

// Asymmetric int4, groups of 32: 16 bytes of codes per group = one chunk.
template <int D>
__device__ __forceinline__ void store_int4(const float (&y)[D], float clip, const RowOut &o, float &emax,
                                           float &amax, bool want_desc)
{
    constexpr int NG = D / 32;
    uint16_t sh[NG], zh[NG];
#pragma unroll
    for (int gi = 0; gi < NG; gi++) {
        float lo = y[32 * gi], hi = lo;
#pragma unroll
        for (int i = 1; i < 32; i++) {
            lo = fminf(lo, y[32 * gi + i]);
            hi = fmaxf(hi, y[32 * gi + i]);
        }
        if (clip < 1.0f) {
            lo = __fmul_rn(lo, clip);
            hi = __fmul_rn(hi, clip);
        }
        const __half shh = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 15.0f));
        const __half zhh = __float2half_rn(lo);
        const float sf = __half2float(shh), zf = __half2float(zhh);
        const float inv = (sf == 0.0f) ? 0.0f : __fdiv_rn(1.0f, sf);
        sh[gi] = __half_as_ushort(shh);
        zh[gi] = __half_as_ushort(zhh);
        uint32_t cw[32];
#pragma unroll
        for (int i = 0; i < 32; i++) {
            const float yi = y[32 * gi + i];
            cw[i] = round_code(__fmul_rn(__fsub_rn(yi, zf), inv), 0.0f, 15.0f);
            if (want_desc) {
                const float yhat = __fadd_rn(__fmul_rn(code_value(cw[i]), sf), zf);
                emax = fmaxf(emax, fabsf(__fsub_rn(yi, yhat)));
                amax = fmaxf(amax, fabsf(yi));
            }
        }
        uint32_t w[4];
#pragma unroll
        for (int m = 0; m < 4; m++) {
            uint32_t b[4];
#pragma unroll
            for (int k = 0; k < 4; k++) b[k] = cw[8 * m + 2 * k] + (cw[8 * m + 2 * k + 1] << 4);
            w[m] = pack4bytes(b[0], b[1], b[2], b[3]);
        }
        *reinterpret_cast<uint4 *>(o.codes + (gi * 16 + o.tok) * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (NG == 4) {
        *reinterpret_cast<uint4 *>(o.meta) =
            make_uint4(sh[0] | (uint32_t(sh[1 % NG]) << 16), sh[2 % NG] | (uint32_t(sh[3 % NG]) << 16),
                       zh[0] | (uint32_t(zh[1 % NG]) << 16), zh[2 % NG] | (uint32_t(zh[3 % NG]) << 16));
    } else {
        *reinterpret_cast<uint2 *>(o.meta) =
            make_uint2(sh[0] | (uint32_t(sh[1 % NG]) << 16), zh[0] | (uint32_t(zh[1 % NG]) << 16));
    }
}

// Asymmetric int2, one group over the whole row.
template <int D>
__device__ __forceinline__ void store_int2(const float (&y)[D], float clip, const RowOut &o, float &emax,
                                           float &amax, bool want_desc)
{
    float lo = y[0], hi = lo;
#pragma unroll
    for (int i = 1; i < D; i++) {
        lo = fminf(lo, y[i]);
        hi = fmaxf(hi, y[i]);
    }
    if (clip < 1.0f) {
        lo = __fmul_rn(lo, clip);
        hi = __fmul_rn(hi, clip);
    }
    const __half shh = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 3.0f));
    const __half zhh = __float2half_rn(lo);
    const float sf = __half2float(shh), zf = __half2float(zhh);
    const float inv = (sf == 0.0f) ? 0.0f : __fdiv_rn(1.0f, sf);
    uint32_t w[D / 16];
#pragma unroll
    for (int m = 0; m < D / 16; m++) {
        uint32_t b[4];
#pragma unroll
        for (int k = 0; k < 4; k++) {
            uint32_t cw[4];
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const float yi = y[16 * m + 4 * k + e];
                cw[e] = round_code(__fmul_rn(__fsub_rn(yi, zf), inv), 0.0f, 3.0f);
                if (want_desc) {
                    const float yhat = __fadd_rn(__fmul_rn(code_value(cw[e]), sf), zf);
                    emax = fmaxf(emax, fabsf(__fsub_rn(yi, yhat)));
                    amax = fmaxf(amax, fabsf(yi));
                }
            }
            b[k] = cw[0] + (cw[1] << 2) + (cw[2] << 4) + (cw[3] << 6);
        }
        w[m] = pack4bytes(b[0], b[1], b[2], b[3]);
    }
#pragma unroll
    for (int c = 0; c < D / 64; c++)
        *reinterpret_cast<uint4 *>(o.codes + (c * 16 + o.tok) * 16) =
            make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
    *reinterpret_cast<uint32_t *>(o.meta) = __half_as_ushort(shh) | (uint32_t(__half_as_ushort(zhh)) << 16);
}

// Symmetric int8, one fp16 scale (rounded up) per token-head.
template <int D>
__device__ __forceinline__ void store_int8(const float (&y)[D], const RowOut &o, float &emax, float &amax,
                                           bool want_desc)
{
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < D; i++) a = fmaxf(a, fabsf(y[i]));
    const __half shh = __float2half_ru(__fdiv_rn(a, 127.0f));
    const float sf = __half2float(shh);
    const float inv = (sf == 0.0f) ? 0.0f : __fdiv_rn(1.0f, sf);
    if (want_desc) amax = a;
#pragma unroll
    for (int c = 0; c < D / 16; c++) {
        uint32_t w[4];
#pragma unroll
        for (int m = 0; m < 4; m++) {
            uint32_t cw[4];
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const float yi = y[16 * c + 4 * m + e];
                cw[e] = round_code(__fmul_rn(yi, inv), -127.0f, 127.0f);
                if (want_desc) {
                    const float yhat = __fmul_rn(code_value(cw[e]), sf);
                    emax = fmaxf(emax, fabsf(__fsub_rn(yi, yhat)));
                }
            }
            w[m] = pack4bytes(cw[0], cw[1], cw[2], cw[3]);
        }
        *reinterpret_cast<uint4 *>(o.codes + (c * 16 + o.tok) * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    *reinterpret_cast<uint16_t *>(o.meta) = __half_as_ushort(shh);
}

template <int D, int FMT>
__device__ __forceinline__ void append_row(const AppendParams &p, const __half *src, unsigned char *chunk, int tok,
                                           int tensor, unsigned int *desc)
{
    float y[D];
    load_rotated<D>(p, src, y);
    const Layout &L = p.L;
    RowOut o;
    o.codes = chunk + (tensor ? L.v_codes : L.k_codes);
    o.meta = chunk + (tensor ? L.v_meta : L.k_meta) + tok * (tensor ? L.v_row_meta : L.k_row_meta);
    o.tok = tok;
    const bool want_desc = desc != nullptr;
    float emax = 0.0f, amax = 0.0f;
    if (FMT == KVQ_INT4_ASYM) store_int4<D>(y, p.clip, o, emax, amax, want_desc);
    else if (FMT == KVQ_INT2_ASYM) store_int2<D>(y, p.clip, o, emax, amax, want_desc);
    else store_int8<D>(y, o, emax, amax, want_desc);
    if (want_desc) {
        // non-negative floats order like their bit patterns
        if (tensor == 0) {
            atomicMax(desc + 0, __float_as_uint(emax));
        } else {
            atomicMax(desc + 1, __float_as_uint(emax));
            atomicMax(desc + 2, __float_as_uint(amax));
        }
    }
}

template <int D, int KF, int VF>
__global__ void __launch_bounds__(128) append_kernel(const __grid_constant__ AppendParams p)
{
    const long long rows_per_tensor = (long long)p.n_tok * p.L.hkv;
    const long long r = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= 2 * rows_per_tensor) return;
    const int tensor = r >= rows_per_tensor;
    const long long rem = r - tensor * rows_per_tensor;
    const int n = (int)(rem / p.L.hkv), kvh = (int)(rem % p.L.hkv);
    const int slot = p.slots[n];
    if (slot < 0) return;
    if (slot >= p.L.num_pages * kPageTokens) {
        set_status(p.pool, KVQ_ERR_OUT_OF_RANGE);
        return;
    }
    const int page = slot / kPageTokens, tok = slot % kPageTokens;
    unsigned char *chunk = p.pool + kHeaderBytes + (long long)page * p.L.page_bytes + (long long)kvh * p.L.chunk_bytes;
    unsigned int *desc =
        p.L.desc_off ? reinterpret_cast<unsigned int *>(p.pool + p.L.desc_off + ((long long)page * p.L.hkv + kvh) * 16)
                     : nullptr;
    const __half *src = (tensor ? p.v : p.k) + rem * D;
    if (tensor == 0) append_row<D, KF>(p, src, chunk, tok, 0, desc);
    else append_row<D, VF>(p, src, chunk, tok, 1, desc);
}

template <int D, int KF>
cudaError_t launch_d_k(const AppendParams &p, int vf, dim3 grid, cudaStream_t s)
{
    switch (vf) {
    case KVQ_INT4_ASYM: append_kernel<D, KF, KVQ_INT4_ASYM><<<grid, 128, 0, s>>>(p); break;
    case KVQ_INT8_SYM: append_kernel<D, KF, KVQ_INT8_SYM><<<grid, 128, 0, s>>>(p); break;
    default: append_kernel<D, KF, KVQ_INT2_ASYM><<<grid, 128, 0, s>>>(p); break;
    }
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const AppendParams &p, dim3 grid, cudaStream_t s)
{
    switch (p.L.k_fmt) {
    case KVQ_INT4_ASYM: return launch_d_k<D, KVQ_INT4_ASYM>(p, p.L.v_fmt, grid, s);
    case KVQ_INT8_SYM: return launch_d_k<D, KVQ_INT8_SYM>(p, p.L.v_fmt, grid, s);
    default: return launch_d_k<D, KVQ_INT2_ASYM>(p, p.L.v_fmt, grid, s);
    }
}

}  // namespace

cudaError_t launch_append(const AppendParams &p, int, int, cudaStream_t s)
{
    const long long rows = 2LL * p.n_tok * p.L.hkv;
    if (rows == 0) return cudaSuccess;
    const dim3 grid((unsigned)((rows + 127) / 128));
    return p.L.d == 64 ? launch_d<64>(p, grid, s) : launch_d<128>(p, grid, s);
}

}  // namespace kvq
