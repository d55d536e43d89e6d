// kvq_append.cu -- quantise-on-append: load an fp16 K or V row, apply the
// random sign and the Walsh-Hadamard butterflies in fp32, compute per-group
// statistics, scale/zero, round to codes and store them packed into the paged
// pool ["When Quantization Is Free", Methodology 2: sign in registers,
// butterfly passes, per-group scaling, rounding, nibble packing; "Runtime-
// Certified Bounded-Error Quantized Attention", Methodology 1: INT8 keys,
// INT4 values, per-block error descriptors; "OSCAR", 2.2: INT2 with clipping].
//
// A row of d elements is spread over d/32 consecutive lanes, one 32-element
// slice each.  Butterfly stages h = 1..16 stay inside a slice (registers);
// stages h = 32 and 64 pair slice s with s^1 and s^2 (one shuffle and one
// exact fma(+-1, x, partner) per element), in the same stage order as a plain
// fp32 statement of the transform.  For int4 a slice is one quantisation
// group; int2/int8 row statistics reduce over the row's lanes.  Every codec
// operation is an explicitly rounded intrinsic so the integer codes match
// that plain statement bit for bit.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23: x + magic rounds x to an integer (ties to even)

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

// min/max/sum over the `lanes` consecutive lanes that hold one row
template <int LANES> __device__ __forceinline__ float row_min(float v)
{
#pragma unroll
    for (int m = 1; m < LANES; m <<= 1) v = fminf(v, __shfl_xor_sync(kFull, v, m));
    return v;
}
template <int LANES> __device__ __forceinline__ float row_max(float v)
{
#pragma unroll
    for (int m = 1; m < LANES; m <<= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, m));
    return v;
}

template <int D, int FMT>
__device__ __forceinline__ void slice_row(const AppendParams &p, const uint32_t *sign_xor, const __half *src,
                                          unsigned char *chunk, int tok, int tensor, int s, bool active,
                                          unsigned int *desc)
{
    constexpr int LANES = D / 32;
    const Layout &L = p.L;
    // ---- load 32 fp16, flip signs (exact), widen ----
    float y[32];
    {
        const uint4 *s4 = reinterpret_cast<const uint4 *>(src + 32 * s);
#pragma unroll
        for (int i = 0; i < 4; i++) {
            uint4 w = active ? __ldg(s4 + i) : make_uint4(0, 0, 0, 0);
            uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; e++) {
                uint32_t x = ww[e];
                if (p.rotate) x ^= sign_xor[16 * s + 4 * i + e];
                const float2 f = __half22float2(bits_h2(x));
                y[8 * i + 2 * e] = f.x;
                y[8 * i + 2 * e + 1] = f.y;
            }
        }
    }
    // ---- butterflies: h = 1..16 in the slice, h = 32, 64 across slices ----
    if (p.rotate) {
#pragma unroll
        for (int h = 1; h < 32; h <<= 1)
#pragma unroll
            for (int jj = 0; jj < 32; jj++)
                if (!(jj & h)) {
                    const float a = y[jj], b = y[jj + h];
                    y[jj] = __fadd_rn(a, b);
                    y[jj + h] = __fsub_rn(a, b);
                }
#pragma unroll
        for (int m = 1; m < LANES; m <<= 1) {
            // lower slice: a + b; upper slice: a - b with a = the lower's value
            const float sg = (s & m) ? -1.0f : 1.0f;
#pragma unroll
            for (int jj = 0; jj < 32; jj++) {
                const float o = __shfl_xor_sync(kFull, y[jj], m);
                y[jj] = __fmaf_rn(sg, y[jj], o);
            }
        }
#pragma unroll
        for (int jj = 0; jj < 32; jj++) y[jj] = __fmul_rn(y[jj], p.rot_scale);
    }

    unsigned char *codes = chunk + (tensor ? L.v_codes : L.k_codes);
    unsigned char *meta = chunk + (tensor ? L.v_meta : L.k_meta) + tok * (tensor ? L.v_row_meta : L.k_row_meta);
    const bool want_desc = desc != nullptr;
    float emax = 0.0f, amax = 0.0f;

    if (FMT == KVQ_INT4_ASYM) {
        // one group per slice, 16 bytes = one chunk
        float lo = y[0], hi = y[0];
#pragma unroll
        for (int i = 1; i < 32; i++) {
            lo = fminf(lo, y[i]);
            hi = fmaxf(hi, y[i]);
        }
        if (p.clip < 1.0f) {
            lo = __fmul_rn(lo, p.clip);
            hi = __fmul_rn(hi, p.clip);
        }
        const __half shh = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 15.0f));
        const __half zhh = __float2half_rn(lo);
        const float sf = __half2float(shh), zf = __half2float(zhh);
        const float inv = (sf == 0.0f) ? 0.0f : __fdiv_rn(1.0f, sf);
        uint32_t w[4];
#pragma unroll
        for (int m = 0; m < 4; m++) {
            uint32_t bb[4];
#pragma unroll
            for (int k = 0; k < 4; k++) {
                uint32_t cw[2];
#pragma unroll
                for (int e = 0; e < 2; e++) {
                    const float yi = y[8 * m + 2 * k + e];
                    cw[e] = round_code(__fmul_rn(__fsub_rn(yi, zf), inv), 0.0f, 15.0f);
                    if (want_desc) {
                        const float yhat = __fadd_rn(__fmul_rn(code_value(cw[e]), sf), zf);
                        emax = fmaxf(emax, fabsf(__fsub_rn(yi, yhat)));
                        amax = fmaxf(amax, fabsf(yi));
                    }
                }
                bb[k] = cw[0] + (cw[1] << 4);
            }
            w[m] = pack4bytes(bb[0], bb[1], bb[2], bb[3]);
        }
        if (active) {
            *reinterpret_cast<uint4 *>(codes + (s * 16 + tok) * 16) = make_uint4(w[0], w[1], w[2], w[3]);
            reinterpret_cast<uint16_t *>(meta)[s] = __half_as_ushort(shh);
            reinterpret_cast<uint16_t *>(meta)[LANES + s] = __half_as_ushort(zhh);
        }
    } else if (FMT == KVQ_INT2_ASYM) {
        // one group over the row; this slice's 32 codes are bytes [8s, 8s+8)
        float lo = y[0], hi = y[0];
#pragma unroll
        for (int i = 1; i < 32; i++) {
            lo = fminf(lo, y[i]);
            hi = fmaxf(hi, y[i]);
        }
        lo = row_min<LANES>(lo);
        hi = row_max<LANES>(hi);
        if (p.clip < 1.0f) {
            lo = __fmul_rn(lo, p.clip);
            hi = __fmul_rn(hi, p.clip);
        }
        const __half shh = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 3.0f));
        const __half zhh = __float2half_rn(lo);
        const float sf = __half2float(shh), zf = __half2float(zhh);
        const float inv = (sf == 0.0f) ? 0.0f : __fdiv_rn(1.0f, sf);
        uint32_t w[2];
#pragma unroll
        for (int m = 0; m < 2; m++) {
            uint32_t bb[4];
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
                bb[k] = cw[0] + (cw[1] << 2) + (cw[2] << 4) + (cw[3] << 6);
            }
            w[m] = pack4bytes(bb[0], bb[1], bb[2], bb[3]);
        }
        if (active) {
            const int byte0 = 8 * s;  // stream byte of this slice
            *reinterpret_cast<uint2 *>(codes + ((byte0 / 16) * 16 + tok) * 16 + byte0 % 16) = make_uint2(w[0], w[1]);
            if (s == 0)
                *reinterpret_cast<uint32_t *>(meta) =
                    __half_as_ushort(shh) | (uint32_t(__half_as_ushort(zhh)) << 16);
        }
    } else {
        // symmetric int8, one fp16 scale (rounded up) per row; 32 bytes per slice
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; i++) a = fmaxf(a, fabsf(y[i]));
        a = row_max<LANES>(a);
        const __half shh = __float2half_ru(__fdiv_rn(a, 127.0f));
        const float sf = __half2float(shh);
        const float inv = (sf == 0.0f) ? 0.0f : __fdiv_rn(1.0f, sf);
        if (want_desc) amax = a;
        uint32_t w[8];
#pragma unroll
        for (int m = 0; m < 8; m++) {
            uint32_t cw[4];
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const float yi = y[4 * m + e];
                cw[e] = round_code(__fmul_rn(yi, inv), -127.0f, 127.0f);
                if (want_desc) {
                    const float yhat = __fmul_rn(code_value(cw[e]), sf);
                    emax = fmaxf(emax, fabsf(__fsub_rn(yi, yhat)));
                }
            }
            w[m] = pack4bytes(cw[0], cw[1], cw[2], cw[3]);
        }
        if (active) {
            *reinterpret_cast<uint4 *>(codes + ((2 * s) * 16 + tok) * 16) = make_uint4(w[0], w[1], w[2], w[3]);
            *reinterpret_cast<uint4 *>(codes + ((2 * s + 1) * 16 + tok) * 16) = make_uint4(w[4], w[5], w[6], w[7]);
            if (s == 0) *reinterpret_cast<uint16_t *>(meta) = __half_as_ushort(shh);
        }
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

template <int D, int KF, int VF>
__global__ void __launch_bounds__(256) append_kernel(const __grid_constant__ AppendParams p)
{
    constexpr int LANES = D / 32;
    __shared__ uint32_t sign_xor[kMaxD / 2];
    if (threadIdx.x < D / 2) sign_xor[threadIdx.x] = p.sign_xor[threadIdx.x];
    __syncthreads();

    // K rows take the first k_threads threads, V rows start on the next warp
    // boundary: every warp runs one format path, so the full-warp shuffles
    // below are always executed by all 32 lanes together
    const long long rows_per_tensor = (long long)p.n_tok * p.L.hkv;
    const long long k_threads = (rows_per_tensor * LANES + 31) / 32 * 32;
    const long long gthread = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const int tensor = gthread >= k_threads;
    const long long row = (gthread - tensor * k_threads) / LANES;
    const int s = (int)(gthread % LANES);
    // lanes past the last row still run the butterflies (partners stay inside
    // the row's lane group) but store nothing
    bool active = row < rows_per_tensor;
    const long long rem = active ? row : 0;
    const int n = (int)(rem / p.L.hkv), kvh = (int)(rem % p.L.hkv);
    const int slot = p.slots[n];
    if (slot < 0) active = false;
    if (active && slot >= p.L.num_pages * kPageTokens) {
        if (s == 0) set_status(p.pool, KVQ_ERR_OUT_OF_RANGE);
        active = false;
    }
    const int page = active ? slot / kPageTokens : 0, tok = active ? slot % kPageTokens : 0;
    unsigned char *chunk = p.pool + kHeaderBytes + (long long)page * p.L.page_bytes + (long long)kvh * p.L.chunk_bytes;
    unsigned int *desc =
        p.L.desc_off ? reinterpret_cast<unsigned int *>(p.pool + p.L.desc_off + ((long long)page * p.L.hkv + kvh) * 16)
                     : nullptr;
    const __half *src = (tensor ? p.v : p.k) + rem * D;
    if (tensor == 0) slice_row<D, KF>(p, sign_xor, src, chunk, tok, 0, s, active, desc);
    else slice_row<D, VF>(p, sign_xor, src, chunk, tok, 1, s, active, desc);
}

template <int D, int KF>
cudaError_t launch_d_k(const AppendParams &p, int vf, dim3 grid, cudaStream_t st)
{
    switch (vf) {
    case KVQ_INT4_ASYM: append_kernel<D, KF, KVQ_INT4_ASYM><<<grid, 256, 0, st>>>(p); break;
    case KVQ_INT8_SYM: append_kernel<D, KF, KVQ_INT8_SYM><<<grid, 256, 0, st>>>(p); break;
    default: append_kernel<D, KF, KVQ_INT2_ASYM><<<grid, 256, 0, st>>>(p); break;
    }
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const AppendParams &p, dim3 grid, cudaStream_t st)
{
    switch (p.L.k_fmt) {
    case KVQ_INT4_ASYM: return launch_d_k<D, KVQ_INT4_ASYM>(p, p.L.v_fmt, grid, st);
    case KVQ_INT8_SYM: return launch_d_k<D, KVQ_INT8_SYM>(p, p.L.v_fmt, grid, st);
    default: return launch_d_k<D, KVQ_INT2_ASYM>(p, p.L.v_fmt, grid, st);
    }
}

}  // namespace

cudaError_t launch_append(const AppendParams &p, int, int, cudaStream_t st)
{
    const long long rows_per_tensor = (long long)p.n_tok * p.L.hkv;
    if (rows_per_tensor == 0) return cudaSuccess;
    const long long threads = 2 * ((rows_per_tensor * (p.L.d / 32) + 31) / 32 * 32);
    const dim3 grid((unsigned)((threads + 255) / 256));
    return p.L.d == 64 ? launch_d<64>(p, grid, st) : launch_d<128>(p, grid, st);
}

}  // namespace kvq
