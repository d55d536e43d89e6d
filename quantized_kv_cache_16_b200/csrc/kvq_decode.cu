// kvq_decode.cu -- split-K decode attention over the packed paged cache
// ["OSCAR", 2.2b: a fused kernel that unpacks, dequantises and attends over a
// paged low-bit cache and applies the inverse rotation to the output].
//
// Grid (split, kv head, sequence); 8 warps per CTA.  Each warp streams its
// own contiguous run of 16-token pages: one bulk copy per (page, kv head)
// chunk into a 4-deep shared-memory ring guarded by mbarriers.  Per page:
//
//   QK  on tensor cores (mma.m16n8k16, fp32 accumulate).  B = the key codes of
//       8 tokens, turned into fp16 integers exactly (magic-number unpack, no
//       rounding); A = the rotated, pre-scaled query of the GQA group split
//       into an fp16 high part (rows 0..g-1) and low part (rows 8..8+g-1), so
//       q ~= hi + lo to ~22 bits.  One accumulator per quantisation group;
//       the per-token group scale is applied in fp32 afterwards and the
//       group-zero term  sum_g zero[t][g] * sum_{i in g} q_i  is one more MMA
//       with the fp16 zeros as B.  So scores = sum_g s_g (q.c_g) + z_g qsum_g,
//       the dequantised dot product, without ever rounding a dequantised key.
//   softmax online in the log2 domain, with the running max raised only when
//       a page's max exceeds it by more than 8 (exact: any reference works).
//   PV  on tensor cores with M = channels: A = value codes of 16 tokens
//       transposed by ldmatrix.trans (exact fp16 integers), B = p * scale of
//       each token and group split into fp16 hi + lo (two MMAs); the zero term
//       is the fp16 zeros against p (hi + lo).
//
// The 8 warps' (m, l, acc) are merged through shared memory into one partial
// per (sequence, kv head, split, head); the last CTA of each (sequence, kv
// head) to finish merges all splits by the log-sum-exp rule, applies the
// inverse rotation R^T = diag(s) H c_d and writes fp32.
#include <math.h>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // 1 s per stage wait

// fp16x2 constants (bit patterns)
constexpr uint32_t kH1024 = 0x64006400u;   // (1024, 1024)
constexpr uint32_t kH1152 = 0x64806480u;   // (1152, 1152)
constexpr uint32_t kMagicB = 0x64646464u;  // bytes 0x64 for PRMT

__device__ __forceinline__ uint32_t hsub2u(uint32_t a, uint32_t b)
{
    return h2_bits(__hsub2(bits_h2(a), bits_h2(b)));
}

__device__ __forceinline__ uint32_t hfma2u(uint32_t a, uint32_t b, uint32_t c)
{
    return h2_bits(__hfma2(bits_h2(a), bits_h2(b), bits_h2(c)));
}

// Nibbles at bits [0,4) and [16,20) of w as exact fp16 integers.
__device__ __forceinline__ uint32_t nib0(uint32_t w) { return hsub2u((w & 0x000F000Fu) | kH1024, kH1024); }
// Nibbles at bits [4,8) and [20,24): (1024 + 16c) / 16 - 64 = c exactly.
__device__ __forceinline__ uint32_t nib1(uint32_t w)
{
    return hfma2u((w & 0x00F000F0u) | kH1024, 0x2C002C00u /*1/16*/, 0xD400D400u /*-64*/);
}
// Nibble n (0..3) of each 16-bit half.
__device__ __forceinline__ uint32_t nib(uint32_t w, int n)
{
    return (n & 1) ? nib1(n & 2 ? w >> 8 : w) : nib0(n & 2 ? w >> 8 : w);
}

// 2-bit field f (0..7) of each 16-bit half as exact fp16 integers.
__device__ __forceinline__ uint32_t fld2(uint32_t w, int f)
{
    const uint32_t x = (f >= 4) ? (w >> 8) : w;
    const int q = f & 3;
    const uint32_t v = (x & (0x00030003u << (2 * q))) | kH1024;  // 1024 + c * 4^q
    switch (q) {
    case 0: return hsub2u(v, kH1024);
    case 1: return hfma2u(v, 0x34003400u /*1/4*/, 0xDC00DC00u /*-256*/);
    case 2: return hfma2u(v, 0x2C002C00u /*1/16*/, 0xD400D400u /*-64*/);
    default: return hfma2u(v, 0x24002400u /*1/64*/, 0xCC00CC00u /*-16*/);
    }
}

// Signed bytes 0,1 (sel 0) or 2,3 (sel 1) of w as exact fp16 integers.
__device__ __forceinline__ uint32_t i8pair(uint32_t w, int sel)
{
    const uint32_t biased = w ^ 0x80808080u;  // c + 128 as unsigned bytes
    const uint32_t x = __byte_perm(biased, kMagicB, sel ? 0x7362 : 0x5140);
    return hsub2u(x, kH1152);
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) { return h2_bits(__floats2half2_rn(lo, hi)); }

// (x0, x1) ~= hi + lo with hi = fp16(x) and lo = fp16(x - hi), packed pairs.
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t &hi, uint32_t &lo)
{
    const __half2 h = __floats2half2_rn(x0, x1);
    hi = h2_bits(h);
    lo = pack_h2(x0 - __low2float(h), x1 - __high2float(h));
}

// ------------------------------------------------------------ key codecs ---
// B operand of QK: thread (r = lane/4, j = lane%4) holds for k-step ks the
// fp16 pairs at virtual k (2j, 2j+1) and (2j+8, 2j+9) of token r.  chan()
// maps a virtual (ks, kk) to the physical channel, which the query fragment
// follows; the unpack never needs to reorder codes.

template <int FMT, int D> struct KCodec;

template <int D> struct KCodec<KVQ_INT4_ASYM, D> {
    static constexpr int NCH = D / 32;  // 16-byte chunks per token row (= groups)
    static constexpr int NG = D / 32;
    static constexpr bool ZERO = true;
    static constexpr int ROW_META = 4 * NG;
    __device__ static int chan(int ks, int kk)
    {
        const int jj = (kk & 7) >> 1, e = kk & 1, hb = kk >> 3;
        return 32 * (ks >> 1) + 8 * jj + 2 * (ks & 1) + hb + 4 * e;
    }
    __device__ static int group_of_chan(int ch) { return ch / 32; }
    __device__ static int group_of_chunk(int c) { return c; }
    static constexpr int KS_PER_CHUNK = 2;
    __device__ static void unpack(uint32_t w, uint32_t (&b)[KS_PER_CHUNK][2])
    {
        b[0][0] = nib(w, 0);
        b[0][1] = nib(w, 1);
        b[1][0] = nib(w, 2);
        b[1][1] = nib(w, 3);
    }
};

template <int D> struct KCodec<KVQ_INT8_SYM, D> {
    static constexpr int NCH = D / 16;
    static constexpr int NG = 1;
    static constexpr bool ZERO = false;
    static constexpr int ROW_META = 2;
    __device__ static int chan(int ks, int kk)
    {
        const int jj = (kk & 7) >> 1, e = kk & 1, hb = kk >> 3;
        return 16 * ks + 4 * jj + 2 * hb + e;
    }
    __device__ static int group_of_chan(int) { return 0; }
    __device__ static int group_of_chunk(int) { return 0; }
    static constexpr int KS_PER_CHUNK = 1;
    __device__ static void unpack(uint32_t w, uint32_t (&b)[KS_PER_CHUNK][2])
    {
        b[0][0] = i8pair(w, 0);
        b[0][1] = i8pair(w, 1);
    }
};

template <int D> struct KCodec<KVQ_INT2_ASYM, D> {
    static constexpr int NCH = D / 64;
    static constexpr int NG = 1;
    static constexpr bool ZERO = true;
    static constexpr int ROW_META = 4;
    __device__ static int chan(int ks, int kk)
    {
        const int jj = (kk & 7) >> 1, e = kk & 1, hb = kk >> 3;
        return 64 * (ks >> 2) + 16 * jj + 2 * (ks & 3) + hb + 8 * e;
    }
    __device__ static int group_of_chan(int) { return 0; }
    __device__ static int group_of_chunk(int) { return 0; }
    static constexpr int KS_PER_CHUNK = 4;
    __device__ static void unpack(uint32_t w, uint32_t (&b)[KS_PER_CHUNK][2])
    {
#pragma unroll
        for (int u = 0; u < 4; u++) {
            b[u][0] = fld2(w, 2 * u);
            b[u][1] = fld2(w, 2 * u + 1);
        }
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
    __device__ static void afrag(uint32_t wA, uint32_t wB, int u, uint32_t (&a)[4])
    {
        a[0] = nib(wA, 2 * u);
        a[1] = nib(wA, 2 * u + 1);
        a[2] = nib(wB, 2 * u);
        a[3] = nib(wB, 2 * u + 1);
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
    __device__ static void afrag(uint32_t wA, uint32_t wB, int u, uint32_t (&a)[4])
    {
        a[0] = fld2(wA, 2 * u);
        a[1] = fld2(wA, 2 * u + 1);
        a[2] = fld2(wB, 2 * u);
        a[3] = fld2(wB, 2 * u + 1);
    }
};

template <int KF, int VF, int D> struct Cfg {
    using K = KCodec<KF, D>;
    using V = VCodec<VF, D>;
    static constexpr int K_CODES = 0;
    static constexpr int K_META = 16 * (D * (KF == KVQ_INT4_ASYM ? 4 : KF == KVQ_INT8_SYM ? 8 : 2) / 8);
    static constexpr int V_CODES = K_META + 16 * K::ROW_META;
    static constexpr int V_META = V_CODES + 16 * (D * (VF == KVQ_INT4_ASYM ? 4 : 2) / 8);
    static constexpr int CHUNK = V_META + 16 * V::ROW_META;
    static constexpr int NST = CHUNK > 3000 ? 3 : 4;
    static constexpr int STAGE = (CHUNK + 127) / 128 * 128;
    static constexpr int KST = D / 16;  // k-steps of QK
    static constexpr int MT = D / 16;   // m-tiles of PV
    static constexpr int E = D / 32;    // elements per lane in warp-wide vectors
    // shared memory map
    static constexpr int OFF_QS = kDecodeWarps * NST * STAGE;
    static constexpr int OFF_QSUM = OFF_QS + kMaxGqa * D * 4;
    static constexpr int OFF_BAR = OFF_QSUM + kMaxGqa * 4 * 4;
    static constexpr int OFF_FLAG = OFF_BAR + kDecodeWarps * NST * 8;
    static constexpr int SMEM = OFF_FLAG + 16;
    // merge scratch (aliases the stage ring after the page loop)
    static constexpr int MERGE_ACC = 0;                                       // [W][8][D]
    static constexpr int MERGE_Z = MERGE_ACC + kDecodeWarps * kMaxGqa * D * 4;  // [W][4][8]
    static constexpr int MERGE_M = MERGE_Z + kDecodeWarps * 4 * kMaxGqa * 4;    // [W][8]
    static constexpr int MERGE_L = MERGE_M + kDecodeWarps * kMaxGqa * 4;        // [W][8]
    static_assert(MERGE_L + kDecodeWarps * kMaxGqa * 4 <= OFF_QS, "merge scratch must fit in the stage ring");
};

// Load NCH 16-byte chunks of rows [8*nt, 8*nt+8) of a chunk-major code region
// (non-transposed): out[c] = bytes [4j, 4j+4) of chunk c of token 8*nt + r.
template <int NCH>
__device__ __forceinline__ void ld_rows(uint32_t base, int nt, int lane, uint32_t (&w)[NCH])
{
    const int row = lane & 7, mi = lane >> 3;
    if constexpr (NCH >= 4) {
#pragma unroll
        for (int q = 0; q < NCH / 4; q++) {
            const uint32_t addr = base + ((4 * q + mi) * 16 + 8 * nt + row) * 16;
            ldsm_x4(addr, w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        }
    } else if constexpr (NCH == 2) {
        const uint32_t addr = base + (((mi & 1)) * 16 + 8 * nt + row) * 16;
        ldsm_x2(addr, w[0], w[1]);
    } else {
        const uint32_t addr = base + (8 * nt + row) * 16;
        uint32_t dummy;
        ldsm_x2(addr, w[0], dummy);
    }
}

// Load NCH chunks of a value region transposed: wA[c] = tokens (2j, 2j+1),
// wB[c] = tokens (2j+8, 2j+9), 16-bit piece r of chunk c.
template <int NCH>
__device__ __forceinline__ void ld_rows_t(uint32_t base, int lane, uint32_t (&wA)[NCH], uint32_t (&wB)[NCH])
{
    const int row = lane & 7, mi = lane >> 3;
    if constexpr (NCH >= 2) {
#pragma unroll
        for (int q = 0; q < NCH / 2; q++) {
            const int c = 2 * q + (mi >> 1), tok = (mi & 1) * 8 + row;
            const uint32_t addr = base + (c * 16 + tok) * 16;
            ldsm_x4_t(addr, wA[2 * q], wB[2 * q], wA[2 * q + 1], wB[2 * q + 1]);
        }
    } else {
        const int tok = (mi & 1) * 8 + row;
        const uint32_t addr = base + tok * 16;
        uint32_t d0, d1;
        ldsm_x4_t(addr, wA[0], wB[0], d0, d1);
    }
}

// Walsh-Hadamard transform of a warp-wide vector (element lane*E + e), fp32.
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

__device__ __forceinline__ float h2f_bits(uint16_t u) { return __half2float(__ushort_as_half(u)); }

template <int D, int KF, int VF>
__global__ void __launch_bounds__(kDecodeThreads, 2) decode_kernel(const __grid_constant__ DecodeParams p)
{
    using C = Cfg<KF, VF, D>;
    using KC = typename C::K;
    using VC = typename C::V;
    constexpr int E = C::E;
    constexpr int NST = C::NST;

    const Layout &L = p.L;
    const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r = lane >> 2, j = lane & 3;
    const int g = L.g;

    int T = p.ctx_lens[b];
    if (T < 0 || T > p.max_pages * kPageTokens) {
        if (split == 0 && tid == 0) set_status(p.pool, KVQ_ERR_OUT_OF_RANGE);
        T = T < 0 ? 0 : p.max_pages * kPageTokens;
    }
    const int n_pages = (T + kPageTokens - 1) / kPageTokens;
    const int n_active = max(1, (n_pages + p.pages_per_split - 1) / p.pages_per_split);
    if (split >= n_active) return;

    extern __shared__ __align__(128) unsigned char smem[];
    float *qs = reinterpret_cast<float *>(smem + C::OFF_QS);
    float *qsum = reinterpret_cast<float *>(smem + C::OFF_QSUM);
    int *sflag = reinterpret_cast<int *>(smem + C::OFF_FLAG);
    const uint32_t bar0 = smem_u32(smem + C::OFF_BAR) + warp * NST * 8;
    const uint32_t stage0 = smem_u32(smem) + warp * NST * C::STAGE;
    const unsigned char *stage0_ptr = smem + warp * NST * C::STAGE;

    // ---- query: rotate, pre-scale, group sums (warp w handles head w) ----
    for (int h = warp; h < g; h += kDecodeWarps) {
        const __half *qh = p.q + ((long long)b * L.hq + kvh * g + h) * D + lane * E;
        float x[E];
        if constexpr (E == 4) {
            const uint2 u = *reinterpret_cast<const uint2 *>(qh);
            const float2 f0 = __half22float2(bits_h2(u.x)), f1 = __half22float2(bits_h2(u.y));
            x[0] = f0.x;
            x[1] = f0.y;
            x[2] = f1.x;
            x[3] = f1.y;
        } else {
            const float2 f0 = __half22float2(bits_h2(*reinterpret_cast<const uint32_t *>(qh)));
            x[0] = f0.x;
            x[1] = f0.y;
        }
        float sc = p.qscale;
        if (p.rotate) {
#pragma unroll
            for (int e = 0; e < E; e++) x[e] *= p.signs[lane * E + e];
            fwht_warp<D>(x, lane);
            sc *= p.rot_scale;
        }
#pragma unroll
        for (int e = 0; e < E; e++) {
            x[e] *= sc;
            qs[h * D + lane * E + e] = x[e];
        }
        if constexpr (KC::ZERO) {
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < E; e++) s += x[e];
            // lanes sharing a group: int4 -> 32/E lanes, int2 -> all 32
            constexpr int LANES = (KF == KVQ_INT4_ASYM) ? 32 / E : 32;
#pragma unroll
            for (int m = 1; m < LANES; m <<= 1) s += __shfl_xor_sync(kFull, s, m);
            if ((lane % LANES) == 0) qsum[h * 4 + (lane * E) / (KF == KVQ_INT4_ASYM ? 32 : D)] = s;
        }
    }
    if (lane == 0) {
        for (int s = 0; s < NST; s++) mbar_init(bar0 + 8 * s, 1);
        fence_mbar_init();
    }
    __syncthreads();

    // ---- this warp's pages ----
    const int p_begin = split * p.pages_per_split + warp * p.pages_per_warp;
    const int p_end = min(p_begin + p.pages_per_warp, n_pages);
    const int npg = max(0, p_end - p_begin);
    const int32_t *bt = p.block_table + (long long)b * p.max_pages;
    const unsigned char *kv_base = p.pool + kHeaderBytes + (long long)kvh * L.chunk_bytes;

    // page ids of pages [i0, i0+32) of this warp, one per lane
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
    int ids = fetch_ids(0);  // page ids of the issue window [32k, 32k+32)
    uint32_t vbits = 0;      // bit s: stage s holds a valid page
    auto issue = [&](int i) {  // every lane calls this
        const int pg = __shfl_sync(kFull, ids, i & 31);
        const int st = i % NST;
        vbits = (vbits & ~(1u << st)) | ((pg >= 0 ? 1u : 0u) << st);
        if (lane == 0) {
            fence_proxy_async();
            if (pg >= 0)
                bulk_load(stage0 + st * C::STAGE, kv_base + (long long)pg * L.page_bytes, C::CHUNK, bar0 + 8 * st);
            else
                asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar0 + 8 * st) : "memory");
        }
    };
    for (int i = 0; i < NST && i < npg; i++) issue(i);

    // ---- query fragments (A operands) ----
    uint32_t aq[C::KST][4];
#pragma unroll
    for (int ks = 0; ks < C::KST; ks++) {
#pragma unroll
        for (int half = 0; half < 2; half++) {
            const int kk = 2 * j + 8 * half;
            uint32_t hi = 0, lo = 0;
            if (r < g) {
                const float x0 = qs[r * D + KC::chan(ks, kk)], x1 = qs[r * D + KC::chan(ks, kk + 1)];
                const __half2 h2 = __floats2half2_rn(x0, x1);
                hi = h2_bits(h2);
                lo = pack_h2(x0 - __low2float(h2), x1 - __high2float(h2));
            }
            aq[ks][2 * half] = hi;
            aq[ks][2 * half + 1] = lo;
        }
    }
    uint32_t aqz[4] = {0, 0, 0, 0};
    if constexpr (KC::ZERO) {
        if (r < g && 2 * j < KC::NG) {
            const float x0 = qsum[r * 4 + 2 * j];
            const float x1 = (2 * j + 1 < KC::NG) ? qsum[r * 4 + 2 * j + 1] : 0.f;
            const __half2 h2 = __floats2half2_rn(x0, x1);
            aqz[0] = h2_bits(h2);
            aqz[1] = pack_h2(x0 - __low2float(h2), x1 - __high2float(h2));
        }
    }

    float oacc[C::MT][4];
#pragma unroll
    for (int mt = 0; mt < C::MT; mt++) oacc[mt][0] = oacc[mt][1] = oacc[mt][2] = oacc[mt][3] = 0.f;
    float oz[4] = {0.f, 0.f, 0.f, 0.f};
    float m_run = -INFINITY, l_part = 0.f;

    for (int i = 0; i < npg; i++) {
        const int st = i % NST;
        const bool ok = mbar_wait_bounded(bar0 + 8 * st, (i / NST) & 1, kWaitLimitNs);
        if (!__all_sync(kFull, ok)) {
            // give up on this warp's run: record it, then wait (bounded) for
            // the copies still in flight so none lands after the ring is reused
            if (lane == 0) set_status(p.pool, KVQ_ERR_TIMEOUT);
            for (int k = i; k < npg && k < i + NST; k++)
                (void)mbar_wait_bounded(bar0 + 8 * (k % NST), (k / NST) & 1, kWaitLimitNs);
            break;
        }
        const int t0 = (p_begin + i) * kPageTokens;
        const int nvalid = min(kPageTokens, T - t0);
        const uint32_t sb = stage0 + st * C::STAGE;
        const unsigned char *sp = stage0_ptr + st * C::STAGE;
        const bool page_ok = (vbits >> st) & 1u;

        // per-thread tokens of the score fragment / PV B operand
        const int tk[4] = {2 * j, 2 * j + 1, 2 * j + 8, 2 * j + 9};

        // ---------------- QK ----------------
        float sk[4][KC::NG];
#pragma unroll
        for (int q = 0; q < 4; q++) {
            const unsigned char *mrow = sp + C::K_META + tk[q] * KC::ROW_META;
#pragma unroll
            for (int gi = 0; gi < KC::NG; gi++) sk[q][gi] = h2f_bits(*reinterpret_cast<const uint16_t *>(mrow + 2 * gi));
        }
        float sc[4];
#pragma unroll
        for (int nt = 0; nt < 2; nt++) {
            uint32_t kw[KC::NCH];
            ld_rows<KC::NCH>(sb + C::K_CODES, nt, lane, kw);
            float dz[4] = {0.f, 0.f, 0.f, 0.f};
            if constexpr (KC::ZERO) {
                const unsigned char *mrow = sp + C::K_META + (8 * nt + r) * KC::ROW_META + 2 * KC::NG;
                uint32_t bz = 0;
                if constexpr (KC::NG >= 2) {
                    if (2 * j < KC::NG) bz = *reinterpret_cast<const uint32_t *>(mrow + 4 * j);
                } else {
                    if (j == 0) bz = *reinterpret_cast<const uint16_t *>(mrow);
                }
                mma16816(dz, aqz, bz, 0u);
            }
            float s0 = dz[0] + dz[2], s1 = dz[1] + dz[3];
#pragma unroll
            for (int gi = 0; gi < KC::NG; gi++) {
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c = 0; c < KC::NCH; c++) {
                    if (KC::group_of_chunk(c) != gi) continue;
                    uint32_t bb[KC::KS_PER_CHUNK][2];
                    KC::unpack(kw[c], bb);
#pragma unroll
                    for (int u = 0; u < KC::KS_PER_CHUNK; u++)
                        mma16816(acc, aq[c * KC::KS_PER_CHUNK + u], bb[u][0], bb[u][1]);
                }
                s0 = fmaf(sk[2 * nt][gi], acc[0] + acc[2], s0);
                s1 = fmaf(sk[2 * nt + 1][gi], acc[1] + acc[3], s1);
            }
            sc[2 * nt] = s0;
            sc[2 * nt + 1] = s1;
        }
        if (nvalid < kPageTokens || !page_ok) {
#pragma unroll
            for (int q = 0; q < 4; q++)
                if (tk[q] >= nvalid || !page_ok) sc[q] = -INFINITY;
        }

        // ---------------- online softmax (log2 domain) ----------------
        float mx = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
        const bool need = mx > m_run + 8.0f;
        if (__any_sync(kFull, need)) {
            const float m_new = need ? mx : m_run;
            const float alpha = (m_new == -INFINITY) ? 1.f : exp2f(m_run - m_new);
            m_run = m_new;
            l_part *= alpha;
            const float a0 = __shfl_sync(kFull, alpha, 8 * j), a1 = __shfl_sync(kFull, alpha, 8 * j + 4);
#pragma unroll
            for (int mt = 0; mt < C::MT; mt++) {
                oacc[mt][0] *= a0;
                oacc[mt][1] *= a1;
                oacc[mt][2] *= a0;
                oacc[mt][3] *= a1;
            }
            oz[0] *= a0;
            oz[1] *= a1;
            oz[2] *= a0;
            oz[3] *= a1;
        }
        float pr[4];
#pragma unroll
        for (int q = 0; q < 4; q++) {
            pr[q] = (m_run == -INFINITY) ? 0.f : exp2f(sc[q] - m_run);
            l_part += pr[q];
        }

        // ---------------- PV ----------------
        float sv[4][VC::NG];
        uint16_t zv[4];
#pragma unroll
        for (int q = 0; q < 4; q++) {
            const unsigned char *mrow = sp + C::V_META + tk[q] * VC::ROW_META;
            const bool valid = page_ok && tk[q] < nvalid;
#pragma unroll
            for (int gi = 0; gi < VC::NG; gi++)
                sv[q][gi] = valid ? h2f_bits(*reinterpret_cast<const uint16_t *>(mrow + 2 * gi)) : 0.f;
            zv[q] = (valid && r < VC::NG) ? *reinterpret_cast<const uint16_t *>(mrow + 2 * VC::NG + 2 * r) : 0;
        }
        // p and p*scale enter the MMAs as fp16 hi + lo pairs (two MMAs each),
        // so the weights carry ~22 bits instead of fp16's 11
        {
            uint32_t ph[2], pl[2];
            split_pair(pr[0], pr[1], ph[0], pl[0]);
            split_pair(pr[2], pr[3], ph[1], pl[1]);
            const uint32_t az[4] = {uint32_t(zv[0]) | (uint32_t(zv[1]) << 16), 0u,
                                    uint32_t(zv[2]) | (uint32_t(zv[3]) << 16), 0u};
            mma16816(oz, az, ph[0], ph[1]);
            mma16816(oz, az, pl[0], pl[1]);
        }
        uint32_t wh[VC::NG][2], wl[VC::NG][2];
#pragma unroll
        for (int gi = 0; gi < VC::NG; gi++) {
            split_pair(pr[0] * sv[0][gi], pr[1] * sv[1][gi], wh[gi][0], wl[gi][0]);
            split_pair(pr[2] * sv[2][gi], pr[3] * sv[3][gi], wh[gi][1], wl[gi][1]);
        }
        uint32_t vA[VC::NCH], vB[VC::NCH];
        ld_rows_t<VC::NCH>(sb + C::V_CODES, lane, vA, vB);
#pragma unroll
        for (int c = 0; c < VC::NCH; c++) {
#pragma unroll
            for (int u = 0; u < VC::MT_PER_CHUNK; u++) {
                const int mt = c * VC::MT_PER_CHUNK + u;
                uint32_t a[4];
                VC::afrag(vA[c], vB[c], u, a);
                const int gi = VC::group_of_mt(mt);
                mma16816(oacc[mt], a, wh[gi][0], wh[gi][1]);
                mma16816(oacc[mt], a, wl[gi][0], wl[gi][1]);
            }
        }

        // ---------------- refill this stage ----------------
        __syncwarp();
        const int nxt = i + NST;
        if (nxt < npg) {
            if ((nxt & 31) == 0) ids = fetch_ids(nxt);
            issue(nxt);
        }
    }

    // ---- warp state -> shared memory, CTA merge ----
    l_part += __shfl_xor_sync(kFull, l_part, 1);
    l_part += __shfl_xor_sync(kFull, l_part, 2);
    __syncthreads();  // every warp is done with the stage ring
    float *macc = reinterpret_cast<float *>(smem + C::MERGE_ACC);
    float *mz = reinterpret_cast<float *>(smem + C::MERGE_Z);
    float *mm = reinterpret_cast<float *>(smem + C::MERGE_M);
    float *ml = reinterpret_cast<float *>(smem + C::MERGE_L);
#pragma unroll
    for (int mt = 0; mt < C::MT; mt++) {
#pragma unroll
        for (int q = 0; q < 4; q++) {
            const int row = r + 8 * (q >> 1), col = 2 * j + (q & 1);
            if (col < g) macc[(warp * kMaxGqa + col) * D + VC::chan(mt, row)] = oacc[mt][q];
        }
    }
#pragma unroll
    for (int q = 0; q < 2; q++) {
        const int col = 2 * j + q;
        if (r < VC::NG && col < g) mz[(warp * 4 + r) * kMaxGqa + col] = oz[q];
    }
    if (j == 0 && r < g) {
        mm[warp * kMaxGqa + r] = m_run;
        ml[warp * kMaxGqa + r] = l_part;
    }
    __syncthreads();

    const int n_splits = p.n_splits;
    float *part_base = p.part + (((long long)b * L.hkv + kvh) * n_splits) * g * (D + 4);
    for (int idx = tid; idx < g * D; idx += kDecodeThreads) {
        const int h = idx / D, ch = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; w++) M = fmaxf(M, mm[w * kMaxGqa + h]);
        float acc = 0.f, Lsum = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kDecodeWarps; w++) {
                const float mw = mm[w * kMaxGqa + h];
                const float f = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
                acc += f * (macc[(w * kMaxGqa + h) * D + ch] + mz[(w * 4 + VC::group_of_chan(ch)) * kMaxGqa + h]);
                Lsum += f * ml[w * kMaxGqa + h];
            }
        }
        float *dst = part_base + ((long long)split * g + h) * (D + 4);
        dst[ch] = acc;
        if (ch == 0) {
            dst[D] = M;
            dst[D + 1] = Lsum;
        }
    }

    // ---- last CTA of this (sequence, kv head) merges the splits ----
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(p.counters + (b * L.hkv + kvh), 1u);
        *sflag = (prev == (unsigned)(n_active - 1));
    }
    __syncthreads();
    if (!*sflag) return;
    __threadfence();
    if (tid == 0) p.counters[b * L.hkv + kvh] = 0u;

    for (int h = warp; h < g; h += kDecodeWarps) {
        float M = -INFINITY;
        for (int s = lane; s < n_active; s += 32) M = fmaxf(M, __ldcg(part_base + ((long long)s * g + h) * (D + 4) + D));
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, m));
        float o[E];
#pragma unroll
        for (int e = 0; e < E; e++) o[e] = 0.f;
        float Lsum = 0.f;
        if (M != -INFINITY) {
            for (int s = 0; s < n_active; s++) {
                const float *src = part_base + ((long long)s * g + h) * (D + 4);
                const float ms = __ldcg(src + D), ls = __ldcg(src + D + 1);
                const float f = (ms == -INFINITY) ? 0.f : exp2f(ms - M);
                Lsum += f * ls;
                if constexpr (E == 4) {
                    const float4 v = __ldcg(reinterpret_cast<const float4 *>(src) + lane);
                    o[0] += f * v.x;
                    o[1] += f * v.y;
                    o[2] += f * v.z;
                    o[3] += f * v.w;
                } else {
                    const float2 v = __ldcg(reinterpret_cast<const float2 *>(src) + lane);
                    o[0] += f * v.x;
                    o[1] += f * v.y;
                }
            }
        }
        const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
#pragma unroll
        for (int e = 0; e < E; e++) o[e] *= inv;
        if (p.rotate) {
            fwht_warp<D>(o, lane);
#pragma unroll
            for (int e = 0; e < E; e++) o[e] *= p.rot_scale * p.signs[lane * E + e];
        }
        float *dst = p.out + ((long long)b * L.hq + kvh * g + h) * D + lane * E;
        if constexpr (E == 4) {
            *reinterpret_cast<float4 *>(dst) = make_float4(o[0], o[1], o[2], o[3]);
        } else {
            *reinterpret_cast<float2 *>(dst) = make_float2(o[0], o[1]);
        }
    }
}

template <int D, int KF, int VF>
cudaError_t launch_t(const DecodeParams &p, dim3 grid, cudaStream_t s)
{
    using C = Cfg<KF, VF, D>;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, KF, VF>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::SMEM);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    decode_kernel<D, KF, VF><<<grid, kDecodeThreads, C::SMEM, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

bool decode_supported(const Layout &L)
{
    if (L.g < 1 || L.g > kMaxGqa) return false;
    if (L.v_fmt != KVQ_INT4_ASYM && L.v_fmt != KVQ_INT2_ASYM) return false;
    if (L.d == 64) return L.k_fmt == KVQ_INT4_ASYM && L.v_fmt == KVQ_INT4_ASYM;
    return L.d == 128;
}

cudaError_t launch_decode(const DecodeParams &p, dim3 grid, cudaStream_t s)
{
    const Layout &L = p.L;
    if (L.d == 64) return launch_t<64, KVQ_INT4_ASYM, KVQ_INT4_ASYM>(p, grid, s);
    if (L.v_fmt == KVQ_INT4_ASYM) {
        switch (L.k_fmt) {
        case KVQ_INT4_ASYM: return launch_t<128, KVQ_INT4_ASYM, KVQ_INT4_ASYM>(p, grid, s);
        case KVQ_INT8_SYM: return launch_t<128, KVQ_INT8_SYM, KVQ_INT4_ASYM>(p, grid, s);
        default: return launch_t<128, KVQ_INT2_ASYM, KVQ_INT4_ASYM>(p, grid, s);
        }
    }
    switch (L.k_fmt) {
    case KVQ_INT4_ASYM: return launch_t<128, KVQ_INT4_ASYM, KVQ_INT2_ASYM>(p, grid, s);
    case KVQ_INT8_SYM: return launch_t<128, KVQ_INT8_SYM, KVQ_INT2_ASYM>(p, grid, s);
    default: return launch_t<128, KVQ_INT2_ASYM, KVQ_INT2_ASYM>(p, grid, s);
    }
}

}  // namespace kvq
