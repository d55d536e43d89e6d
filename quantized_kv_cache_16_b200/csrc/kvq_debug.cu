// kvq_debug.cu -- read stored rows back (codes, scales/zeros, dequantised
// rotated values) and reset page descriptors.  Not on the hot path.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

__global__ void dequant_kernel(const __grid_constant__ DequantParams p)
{
    const Layout &L = p.L;
    const long long rr = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (rr >= 2LL * p.n * L.hkv) return;
    const int tensor = (int)(rr & 1);
    const long long rest = rr >> 1;
    const int kvh = (int)(rest % L.hkv), i = (int)(rest / L.hkv);
    const int slot = p.slots[i];
    if (slot < 0 || slot >= L.num_pages * kPageTokens) {
        set_status(p.pool, KVQ_ERR_OUT_OF_RANGE);
        return;
    }
    const int page = slot / kPageTokens, tok = slot % kPageTokens;
    const unsigned char *chunk = p.pool + kHeaderBytes + (long long)page * L.page_bytes + (long long)kvh * L.chunk_bytes;
    const int fmt = tensor ? L.v_fmt : L.k_fmt;
    const int bits = fmt_bits(fmt);
    const unsigned char *codes = chunk + (tensor ? L.v_codes : L.k_codes);
    const int row_meta = tensor ? L.v_row_meta : L.k_row_meta;
    const unsigned char *meta = chunk + (tensor ? L.v_meta : L.k_meta) + tok * row_meta;
    const int d = L.d;
    const int ng = fmt == KVQ_INT4_ASYM ? d / 32 : 1;
    const int group = fmt == KVQ_INT4_ASYM ? 32 : d;
    float s[4], z[4];
    uint16_t sh[4] = {0, 0, 0, 0}, zh[4] = {0, 0, 0, 0};
    for (int gi = 0; gi < ng; gi++) {
        sh[gi] = reinterpret_cast<const uint16_t *>(meta)[gi];
        zh[gi] = fmt == KVQ_INT8_SYM ? 0 : reinterpret_cast<const uint16_t *>(meta)[ng + gi];
        s[gi] = __half2float(__ushort_as_half(sh[gi]));
        z[gi] = __half2float(__ushort_as_half(zh[gi]));
    }
    const long long row = (long long)i * L.hkv + kvh;
    for (int ch = 0; ch < d; ch++) {
        const int bit = ch * bits;
        const int byte = bit / 8;
        const unsigned char bv = codes[((byte / 16) * 16 + tok) * 16 + byte % 16];
        const int raw = (bv >> (bit % 8)) & ((1 << bits) - 1);
        const int code = fmt == KVQ_INT8_SYM ? (int)(int8_t)raw : raw;
        const int gi = ch / group;
        const float val = fmt == KVQ_INT8_SYM ? __fmul_rn((float)code, s[0]) : __fmaf_rn((float)code, s[gi], z[gi]);
        if (p.codes_out) p.codes_out[(row * 2 + tensor) * d + ch] = (uint8_t)raw;
        float *dst = tensor ? p.v_out : p.k_out;
        if (dst) dst[row * d + ch] = val;
    }
    if (p.meta_out) {
        uint16_t *m = p.meta_out + (row * 2 + tensor) * 8;
        for (int k = 0; k < 4; k++) {
            m[k] = sh[k];
            m[4 + k] = zh[k];
        }
    }
}

__global__ void reset_pages_kernel(unsigned char *pool, Layout L, const int32_t *pages, int n)
{
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= (long long)n * L.hkv) return;
    const int kvh = (int)(t % L.hkv), pg = pages[t / L.hkv];
    if (pg < 0 || pg >= L.num_pages) {
        set_status(pool, KVQ_ERR_OUT_OF_RANGE);
        return;
    }
    *reinterpret_cast<uint4 *>(pool + L.desc_off + ((long long)pg * L.hkv + kvh) * 16) = make_uint4(0, 0, 0, 0);
}

}  // namespace

cudaError_t launch_dequant(const DequantParams &p, cudaStream_t s)
{
    const long long rows = 2LL * p.n * p.L.hkv;
    dequant_kernel<<<(unsigned)((rows + 127) / 128), 128, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_reset_pages(unsigned char *pool, Layout L, const int32_t *pages, int n, cudaStream_t s)
{
    const long long t = (long long)n * L.hkv;
    reset_pages_kernel<<<(unsigned)((t + 127) / 128), 128, 0, s>>>(pool, L, pages, n);
    return cudaGetLastError();
}

}  // namespace kvq
