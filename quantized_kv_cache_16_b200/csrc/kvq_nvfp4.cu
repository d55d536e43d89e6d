// kvq_nvfp4.cu -- the NVFP4 codec ["Search Your Block Floating Point
// Scales!", NVFP4 and ScaleSearch] on the paged pool: e2m1 codes with one
// E4M3 scale per block of 16 elements, the default scale round(max|x| / 6)
// or, with scale_search, the best of nine neighbouring scale bit patterns.
//
// Append.  A warp holds one rotated row of 128 elements, lane holding 4
// consecutive ones, so a 16-element block is four lanes: its maximum and its
// squared error are two xor-shuffles.  The scale is the E4M3 conversion
// (nearest, saturating) of max / 6; codes are e2m1 of x / scale by explicit
// round-to-nearest-even thresholds.  Every operation that decides a code is
// an explicitly rounded fp32 operation in the order kvq.h states.
//
// Decode.  e2m1 x E4M3 values are exact in fp16 (at most five significant
// bits, magnitudes 2^-10 .. 2688), so K and V go to the tensor cores as
// single fp16 operands straight from the hardware conversions: each lane
// turns a byte of two codes into an fp16 pair and multiplies it by its
// block's scale.  The query and the softmax weights are hi + lo fp16 pairs.
// Fragments as in the HQMQ decode (scores K Q^T with M = the page's 16
// tokens and N = 8 heads, output V^T P^T with M = dims), but the contraction
// index and the output rows are permuted so that a lane reads one 16-byte
// span of each of its two key rows and one 8-byte span of each of its four
// value rows.
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <math.h>

#include "kvq_internal.cuh"
#include "kvq_warp.cuh"

namespace kvq {
namespace {

constexpr int kNvWarps = 8;
constexpr int kNvThreads = kNvWarps * 32;
constexpr int kNvD = 128;
constexpr int kNvRowCode = kNvD / 2;   // 64 code bytes a row
constexpr int kNvRowMeta = kNvD / 16;  // 8 scale bytes a row

// ------------------------------------------------------------------ append --

// E4M3 byte as fp32 (exact).
__device__ __forceinline__ float e4m3_f(uint8_t b)
{
    const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)b, __NV_E4M3);
    return __half2float(__half(h));
}

// e2m1 code of v: nearest of +-{0, 0.5, 1, 1.5, 2, 3, 4, 6}, ties to the
// even magnitude index, beyond 6 (infinity included) to 6; zero and NaN are
// code 0; bit 3 = sign.
__device__ __forceinline__ uint32_t e2m1_code(float v)
{
    const float a = fabsf(v);
    uint32_t m = a <= 0.25f ? 0u : a < 0.75f ? 1u : a <= 1.25f ? 2u : a < 1.75f ? 3u
               : a <= 2.5f ? 4u : a < 3.5f ? 5u : a <= 5.0f ? 6u : 7u;
    if (a != a) m = 0u;  // NaN
    return m == 0u ? 0u : (m | (signbit(v) ? 8u : 0u));
}

__device__ __forceinline__ float e2m1_val(uint32_t c)
{
    const uint32_t m = c & 7u;  // 0, 0.5, 1, 1.5, then 2, 3, 4, 6
    const float v = m < 4u ? 0.5f * (float)m : (m < 7u ? (float)(m - 2u) : 6.0f);
    return (c & 8u) ? -v : v;
}

// The lane's four codes under scale sf (all zero when sf is 0).
__device__ __forceinline__ void lane_codes(const float (&x)[4], float sf, uint32_t (&c)[4])
{
#pragma unroll
    for (int e = 0; e < 4; e++) c[e] = sf > 0.0f ? e2m1_code(__fdiv_rn(x[e], sf)) : 0u;
}

// Squared error of the lane's four elements, ((e0^2 + e1^2) + e2^2) + e3^2,
// summed over the block's four lanes as (r0 + r1) + (r2 + r3).
__device__ __forceinline__ float block_sq_error(const float (&x)[4], float sf)
{
    uint32_t c[4];
    lane_codes(x, sf, c);
    float acc = 0.0f;
#pragma unroll
    for (int e = 0; e < 4; e++) {
        const float d = __fsub_rn(x[e], __fmul_rn(e2m1_val(c[e]), sf));
        const float d2 = __fmul_rn(d, d);
        acc = e == 0 ? d2 : __fadd_rn(acc, d2);
    }
    acc = __fadd_rn(acc, __shfl_xor_sync(kFull, acc, 1));
    return __fadd_rn(acc, __shfl_xor_sync(kFull, acc, 2));
}

// The default scale byte of the lane's block: E4M3 (nearest, saturating) of
// max |x| / 6 over the block's four lanes.
__device__ __forceinline__ int default_scale(const float (&x)[4])
{
    float am = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
    am = fmaxf(am, __shfl_xor_sync(kFull, am, 1));
    am = fmaxf(am, __shfl_xor_sync(kFull, am, 2));
    return (int)__nv_cvt_float_to_fp8(__fdiv_rn(am, 6.0f), __NV_SATFINITE, __NV_E4M3);
}

// Code the lane's four elements under scale byte sc and store them (two
// code bytes a lane) and the block's scale byte (its first lane).
// (and, when codes_s / meta_s are not null, the same bytes there too)
__device__ __forceinline__ void store_row(const float (&x)[4], int sc, unsigned char *codes, unsigned char *meta,
                                          int lane, unsigned char *codes_s = nullptr, unsigned char *meta_s = nullptr)
{
    uint32_t c[4];
    lane_codes(x, e4m3_f((uint8_t)sc), c);
    const uint16_t w = (uint16_t)(c[0] | (c[1] << 4) | (c[2] << 8) | (c[3] << 12));
    reinterpret_cast<uint16_t *>(codes)[lane] = w;
    if (codes_s) reinterpret_cast<uint16_t *>(codes_s)[lane] = w;
    if ((lane & 3) == 0) {
        meta[lane >> 2] = (unsigned char)sc;
        if (meta_s) meta_s[lane >> 2] = (unsigned char)sc;
    }
}

// Grid: persistent CTAs, a warp codes rows r, r + all warps, ... (K rows
// then V rows, row = token * Hkv + kv head).
template <bool SEARCH>
__global__ void __launch_bounds__(kNvThreads) nvfp4_append_kernel(const __grid_constant__ AppendParams p)
{
    const Layout &L = p.L;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long rows_per_tensor = (long long)p.n_tok * L.hkv;
    const long long n_rows = 2 * rows_per_tensor;
    for (long long row = (long long)blockIdx.x * kNvWarps + warp; row < n_rows;
         row += (long long)gridDim.x * kNvWarps) {
        const int tensor = row >= rows_per_tensor;
        const long long rr = row - tensor * rows_per_tensor;
        const int n = (int)(rr / L.hkv), kvh = (int)(rr - (long long)n * L.hkv);
        const int slot = p.slots[n];
        if (slot < 0) continue;  // warp-uniform
        if (slot >= L.num_pages * kPageTokens) {
            if (lane == 0) set_status(p.pool, KVQ_ERR_OUT_OF_RANGE);
            continue;
        }
        float x[4];
        rotated_row_lane4(p, (tensor ? p.v : p.k) + rr * kNvD, lane, x);
        const int b0 = default_scale(x);  // the block's (lanes 4k .. 4k + 3)
        int best = b0;
        if constexpr (SEARCH) {
            // candidates b0 + f, f = 0, -1, 1, -2, 2, 3, 4, 5, 6: positive finite
            // codes only; a later one replaces only when strictly better
            const bool searchable = b0 != 0 && b0 <= 0x7E;  // uniform over the block's lanes
            float be = 0.0f;
#pragma unroll 1
            for (int k = 0; k < 9; k++) {
                const int f = k == 0 ? 0 : k == 1 ? -1 : k == 2 ? 1 : k == 3 ? -2 : k - 2;
                const int b = b0 + f;
                const bool valid = searchable && b >= 1 && b <= 0x7E;
                const float e = block_sq_error(x, valid ? e4m3_f((uint8_t)b) : 0.0f);  // every lane shuffles
                if (valid && (k == 0 || e < be)) {
                    be = e;
                    best = b;
                }
            }
        }
        const int page = slot / kPageTokens, tok = slot % kPageTokens;
        unsigned char *chunk = p.pool + kHeaderBytes + (long long)page * L.page_bytes + (long long)kvh * L.chunk_bytes;
        store_row(x, best, chunk + (tensor ? L.v_codes : L.k_codes) + tok * kNvRowCode,
                  chunk + (tensor ? L.v_meta : L.k_meta) + tok * kNvRowMeta, lane);
    }
}

template <bool SEARCH>
cudaError_t launch_nv_append(const AppendParams &p, int num_sms, cudaStream_t st)
{
    static int resident = 0;
    if (resident == 0) {
        int n = 0;
        const cudaError_t e =
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, nvfp4_append_kernel<SEARCH>, kNvThreads, 0);
        if (e != cudaSuccess) return e;
        resident = n < 1 ? 1 : n;
    }
    const long long rows = 2LL * p.n_tok * p.L.hkv;
    const long long want = (rows + kNvWarps - 1) / kNvWarps, cap = (long long)resident * num_sms;
    nvfp4_append_kernel<SEARCH><<<(int)(want < cap ? want : cap), kNvThreads, 0, st>>>(p);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ decode --

constexpr int kNvChunk = 2 * kPageTokens * (kNvRowCode + kNvRowMeta);  // 2304 bytes
constexpr int kNvStages = 4;
constexpr int kNvOffBar = kNvWarps * kNvStages * kNvChunk;
constexpr int kNvSmem = kNvOffBar + kNvWarps * kNvStages * 8;
constexpr int kNvMaxSplits = 64;
static_assert(kNvChunk % 16 == 0, "bulk copy size");
static_assert(kNvWarps * 8 * kNvD * 4 <= kNvOffBar, "the warps' sums fit in the ring");

__device__ __forceinline__ void split_h2(float x0, float x1, uint32_t &hi, uint32_t &lo)
{
    const __half2 h = __floats2half2_rn(x0, x1);
    const float2 b = __half22float2(h);
    hi = h2_bits(h);
    lo = h2_bits(__floats2half2_rn(x0 - b.x, x1 - b.y));
}

// Two e2m1 codes (a byte, low nibble first) times the block scale, as an
// fp16 pair (exact).
__device__ __forceinline__ __half2 fp4x2_scaled(uint32_t byte, __half2 s2)
{
    const __half2_raw r = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)(byte & 0xFFu), __NV_E2M1);
    return __hmul2(__half2(r), s2);
}

__device__ __forceinline__ __half2 scale_h2(uint8_t b)
{
    const __half s = __half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)b, __NV_E4M3));
    return __halves2half2(s, s);
}

// Grid (splits, Hkv, B) as the HQMQ decode: split x attends pages
// [x * pps, +pps), warp w pages [x * pps + w * ppw, +ppw), each page (the
// 2304-byte (page, kv head) chunk) copied into the warp's two-stage ring by
// one bulk copy; partials [g][d + 4] go to p.part, the last CTA merges them.
template <int G>
__global__ void __launch_bounds__(kNvThreads, 2) nvfp4_decode_kernel(const __grid_constant__ DecodeParams p)
{
    const Layout &L = p.L;
    const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = L.g;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(16) float sq[G * kNvD];
    __shared__ float wm[kNvWarps][G], wl[kNvWarps][G];
    __shared__ int sflag;

    const int p_begin = split * p.pages_per_split + warp * p.pages_per_warp;
    const int32_t *bt = p.block_table + (long long)b * p.max_pages;
    const unsigned char *kv_base = p.pool + kHeaderBytes + (long long)kvh * L.chunk_bytes;
    const uint32_t stage0 = smem_u32(smem) + warp * kNvStages * kNvChunk;
    const unsigned char *stage0_ptr = smem + warp * kNvStages * kNvChunk;
    const uint32_t bar0 = smem_u32(smem + kNvOffBar) + warp * kNvStages * 8;

    // Launched as a programmatic dependent of the stream's previous kernel:
    // until griddepcontrol.wait returns nothing read is trusted, so this
    // phase reads the context length and this warp's block-table entries as
    // hints only (L2, never L1) and prefetches the pages of the ring's first
    // fill, the query rows and the appended rows into L2.
    {
        const int Th = min(max(__ldcg(p.ctx_lens + b), 0), p.max_pages * kPageTokens);
        const int npg_h = min(p_begin + p.pages_per_warp, (Th + kPageTokens - 1) / kPageTokens) - p_begin;
        if (lane < npg_h && lane < kNvStages) {
            const int pg = __ldcg(bt + p_begin + lane);
            if (pg >= 0 && pg < L.num_pages) bulk_prefetch_l2(kv_base + (long long)pg * L.page_bytes, kNvChunk);
        }
        if (warp == 0 && lane == 31) bulk_prefetch_l2(p.q + ((long long)b * L.hq + kvh * g) * kNvD, g * kNvD * 2);
        if (warp == 1 && lane == 31 && p.new_k != nullptr) {
            bulk_prefetch_l2(p.new_k + ((long long)b * L.hkv + kvh) * kNvD, kNvD * 2);
            bulk_prefetch_l2(p.new_v + ((long long)b * L.hkv + kvh) * kNvD, kNvD * 2);
        }
        if (lane == 0) {
            for (int st = 0; st < kNvStages; st++) mbar_init(bar0 + 8 * st, 1);
            fence_mbar_init();
        }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // the true context length, this warp's first 32 block-table entries and
    // the query row go out together
    int T = p.ctx_lens[b];
    const int id_raw = (lane < p.pages_per_warp && p_begin + lane < p.max_pages) ? bt[p_begin + lane] : -1;
    uint2 q_raw = make_uint2(0u, 0u);
    if (warp < g) q_raw = *reinterpret_cast<const uint2 *>(p.q + ((long long)b * L.hq + kvh * g + warp) * kNvD + lane * 4);
    if (T < 0 || T > p.max_pages * kPageTokens) {
        if (split == 0 && tid == 0) set_status(p.pool, KVQ_ERR_OUT_OF_RANGE);
        T = T < 0 ? 0 : p.max_pages * kPageTokens;
    }
    const int n_pages = (T + kPageTokens - 1) / kPageTokens;
    const int n_act = max(1, (n_pages + p.pages_per_split - 1) / p.pages_per_split);
    if (split >= n_act) return;
    const int npg = max(0, min(p_begin + p.pages_per_warp, n_pages) - p_begin);
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
    int ids = -1;  // page ids of the issue window [32k, 32k + 32)
    if (lane < npg) {
        ids = id_raw;
        if (ids < 0 || ids >= L.num_pages) {
            set_status(p.pool, KVQ_ERR_OUT_OF_RANGE);
            ids = -1;
        }
    }
    uint32_t vbits = 0;  // bit st: stage st holds a valid page
    auto issue = [&](int i) {  // every lane calls this; lane 0 alone copies (predicated)
        const int pg = __shfl_sync(kFull, ids, i & 31);
        const int st = i % kNvStages;
        vbits = (vbits & ~(1u << st)) | ((pg >= 0 ? 1u : 0u) << st);
        bulk_load_or_arrive(lane == 0 && pg >= 0, lane == 0 && pg < 0, stage0 + st * kNvChunk,
                            kv_base + (long long)max(pg, 0) * L.page_bytes, kNvChunk, bar0 + 8 * st);
    };
    for (int i = 0; i < kNvStages && i < npg; i++) issue(i);
    // fused append (decode step): the warp that owns the page of position
    // T - 1 (its last page) codes the new token's K and V rows (default
    // scales) once that page's copy has landed, storing the bytes both to
    // the pool and to the staged copy; no other warp waits for it.  The rows
    // and the slot are copied now (cp.async) into app_buf, so their latency
    // hides behind the query work and the first pages.
    const uint32_t sgb = (p.sign_bits[lane >> 3] >> ((lane & 7) * 4)) & 0xFu;  // signs of elements 4 lane .. + 3
    const int app_tok = (T - 1) % kPageTokens;
    __shared__ __align__(16) unsigned char app_buf[2 * kNvD * 2 + 16];  // K row, V row, slot
    bool app_pending = p.new_k != nullptr && T > 0 && n_pages - 1 >= p_begin && n_pages - 1 < p_begin + npg;
    if (app_pending) {
        const long long row = ((long long)b * L.hkv + kvh) * kNvD + 4 * lane;
        const uint32_t dst = smem_u32(app_buf) + lane * 8;
        asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(p.new_k + row) : "memory");
        asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst + kNvD * 2), "l"(p.new_v + row) : "memory");
        if (lane == 0)
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(app_buf) + kNvD * 4), "l"(p.new_slots + b)
                         : "memory");
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
    // codes the rows into the pool's page pg and, if stage is not null, into its staged copy
    auto append_rows = [&](int pg, unsigned char *stage) -> bool {
        app_pending = false;
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncwarp();
        const int slot = *reinterpret_cast<const int *>(app_buf + kNvD * 4);
        if (pg < 0 || pg >= L.num_pages || slot != pg * kPageTokens + app_tok) {
            if (lane == 0) set_status(p.pool, KVQ_ERR_OUT_OF_RANGE);
            return false;
        }
        unsigned char *chunk = const_cast<unsigned char *>(kv_base) + (long long)pg * L.page_bytes;
#pragma unroll 1
        for (int tensor = 0; tensor < 2; tensor++) {
            const uint2 raw = *reinterpret_cast<const uint2 *>(app_buf + tensor * kNvD * 2 + lane * 8);
            const float2 a = __half22float2(bits_h2(raw.x)), c = __half22float2(bits_h2(raw.y));
            float x[4] = {a.x, a.y, c.x, c.y};
            if (p.rotate) {  // the append's rotation: exact sign flips, butterflies, one rounded scale
#pragma unroll
                for (int e = 0; e < 4; e++) x[e] = __uint_as_float(__float_as_uint(x[e]) ^ (((sgb >> e) & 1u) << 31));
                fwht_warp<kNvD>(x, lane);
#pragma unroll
                for (int e = 0; e < 4; e++) x[e] = __fmul_rn(x[e], p.rot_scale);
            }
            const int co = (tensor ? L.v_codes : L.k_codes) + app_tok * kNvRowCode;
            const int mo = (tensor ? L.v_meta : L.k_meta) + app_tok * kNvRowMeta;
            store_row(x, default_scale(x), chunk + co, chunk + mo, lane, stage ? stage + co : nullptr,
                      stage ? stage + mo : nullptr);
        }
        return true;
    };

    if (warp < g) {  // the rotated query in log2 units
        const float2 a = __half22float2(bits_h2(q_raw.x)), c = __half22float2(bits_h2(q_raw.y));
        float x[4] = {a.x, a.y, c.x, c.y};
        if (p.rotate) {
#pragma unroll
            for (int e = 0; e < 4; e++) x[e] = __uint_as_float(__float_as_uint(x[e]) ^ (((sgb >> e) & 1u) << 31));
            fwht_warp<kNvD>(x, lane);
#pragma unroll
            for (int e = 0; e < 4; e++) x[e] *= p.rot_scale;
        }
#pragma unroll
        for (int e = 0; e < 4; e++) sq[warp * kNvD + lane * 4 + e] = x[e] * p.qscale;
    }
    __syncthreads();
    // Fragments (r = lane / 4, j = lane % 4).  Rows of the score tile and
    // the contraction index of PV are the page's tokens in the order
    // tok(m) = m ^ ((m >> 1) & 1), so the four token rows a value load of a
    // half-warp touches alternate between the two bank halves of a 128-byte
    // line (64-byte rows).  Scores S^T = K Q^T: k-slice ks position {2j,
    // 2j+1, 2j+8, 2j+9} = dims 32j + 4ks .. + 3, so a lane's eight slices are
    // the 16 code bytes [16j, 16j + 16) of tokens tok(r) and tok(r + 8)
    // (one conflict-free 16-byte load each).  Output O^T = V^T P^T: m-tiles
    // 2ib, 2ib + 1 rows r / r + 8 = dims 0 / 1 and 2 / 3 of 16r + 4ib, so a
    // lane's four tile pairs are the 8 code bytes [8r, 8r + 8) of tokens
    // tok(2j), tok(2j+1), tok(2j+8), tok(2j+9).  The score fragments become
    // P^T by two 8x8 transposes.
    const int r = lane >> 2, j = lane & 3;
    auto tok = [](int m) { return m ^ ((m >> 1) & 1); };
    uint32_t qb[8][2], ql[8][2];
#pragma unroll
    for (int ks = 0; ks < 8; ks++) {
        qb[ks][0] = qb[ks][1] = ql[ks][0] = ql[ks][1] = 0u;
        if (r < g) {
            const float4 q4 = *reinterpret_cast<const float4 *>(sq + r * kNvD + 32 * j + 4 * ks);
            split_h2(q4.x, q4.y, qb[ks][0], ql[ks][0]);
            split_h2(q4.z, q4.w, qb[ks][1], ql[ks][1]);
        }
    }
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // heads 2j, 2j + 1
    float acc[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; mt++) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
    const int ta = tok(r), tb = tok(r + 8);
    const int tv[4] = {tok(2 * j), tok(2 * j + 1), tok(2 * j + 8), tok(2 * j + 9)};

    for (int i = 0; i < npg; i++) {
        const int st = i % kNvStages;
        const bool ok = mbar_wait_bounded(bar0 + 8 * st, (i / kNvStages) & 1, kWaitLimitNs);
        if (!__all_sync(kFull, ok)) {
            if (lane == 0) set_status(p.pool, KVQ_ERR_TIMEOUT);
            for (int k = i; k < npg && k < i + kNvStages; k++)
                (void)mbar_wait_bounded(bar0 + 8 * (k % kNvStages), (k / kNvStages) & 1, kWaitLimitNs);
            break;
        }
        const unsigned char *chunk = stage0_ptr + st * kNvChunk;
        if (app_pending && i == npg - 1) {  // the appended row: into the pool and the staged copy of its page
            if (append_rows(__shfl_sync(kFull, ids, i & 31), const_cast<unsigned char *>(chunk))) __syncwarp();
        }
        const int t_page = (p_begin + i) * kPageTokens;
        const int nvalid = ((vbits >> st) & 1u) ? min(kPageTokens, T - t_page) : 0;

        // ---- scores of tokens tok(r), tok(r + 8) for heads 2j, 2j + 1 ----
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
        const bool va = ta < nvalid, vb = tb < nvalid;
        {
            const uint4 ka = *reinterpret_cast<const uint4 *>(chunk + L.k_codes + ta * kNvRowCode + 16 * j);
            const uint4 kb = *reinterpret_cast<const uint4 *>(chunk + L.k_codes + tb * kNvRowCode + 16 * j);
            const uint32_t sa2 = *reinterpret_cast<const uint16_t *>(chunk + L.k_meta + ta * kNvRowMeta + 2 * j);
            const uint32_t sb2 = *reinterpret_cast<const uint16_t *>(chunk + L.k_meta + tb * kNvRowMeta + 2 * j);
            const uint32_t wa[4] = {ka.x, ka.y, ka.z, ka.w}, wb[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
            for (int ks = 0; ks < 8; ks++) {
                const __half2 sa = scale_h2((uint8_t)(sa2 >> (ks < 4 ? 0 : 8)));
                const __half2 sb = scale_h2((uint8_t)(sb2 >> (ks < 4 ? 0 : 8)));
                const uint32_t ca = wa[ks >> 1] >> (16 * (ks & 1)), cb = wb[ks >> 1] >> (16 * (ks & 1));
                uint32_t a[4];
                a[0] = va ? h2_bits(fp4x2_scaled(ca, sa)) : 0u;
                a[1] = vb ? h2_bits(fp4x2_scaled(cb, sb)) : 0u;
                a[2] = va ? h2_bits(fp4x2_scaled(ca >> 8, sa)) : 0u;
                a[3] = vb ? h2_bits(fp4x2_scaled(cb >> 8, sb)) : 0u;
                mma16816(sc, a, qb[ks][0], qb[ks][1]);
                mma16816(sc, a, ql[ks][0], ql[ks][1]);
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
        uint32_t pb[2][2];  // P^T (hi, lo): tokens tok(2j), tok(2j+1) (b0) and tok(2j+8), tok(2j+9) (b1) of head r
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
        // ---- values: dims 16r .. 16r + 15 of the lane's four tokens ----
        {
            uint2 cv[4];
            __half2 s2[4];
#pragma unroll
            for (int u = 0; u < 4; u++) {
                cv[u] = *reinterpret_cast<const uint2 *>(chunk + L.v_codes + tv[u] * kNvRowCode + 8 * r);
                s2[u] = scale_h2(chunk[L.v_meta + tv[u] * kNvRowMeta + r]);
                if (tv[u] >= nvalid) {  // zero codes and scale (a stale scale byte may be NaN)
                    cv[u] = make_uint2(0u, 0u);
                    s2[u] = __float2half2_rn(0.f);
                }
            }
#pragma unroll
            for (int ib = 0; ib < 4; ib++) {
                __half2 v01[4], v23[4];
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    const uint32_t w = ((ib < 2 ? cv[u].x : cv[u].y) >> (16 * (ib & 1))) & 0xFFFFu;
                    v01[u] = fp4x2_scaled(w, s2[u]);
                    v23[u] = fp4x2_scaled(w >> 8, s2[u]);
                }
                uint32_t a[4];
                a[0] = h2_bits(__lows2half2(v01[0], v01[1]));
                a[1] = h2_bits(__highs2half2(v01[0], v01[1]));
                a[2] = h2_bits(__lows2half2(v01[2], v01[3]));
                a[3] = h2_bits(__highs2half2(v01[2], v01[3]));
                mma16816(acc[2 * ib], a, pb[0][0], pb[0][1]);
                mma16816(acc[2 * ib], a, pb[1][0], pb[1][1]);
                a[0] = h2_bits(__lows2half2(v23[0], v23[1]));
                a[1] = h2_bits(__highs2half2(v23[0], v23[1]));
                a[2] = h2_bits(__lows2half2(v23[2], v23[3]));
                a[3] = h2_bits(__highs2half2(v23[2], v23[3]));
                mma16816(acc[2 * ib + 1], a, pb[0][0], pb[0][1]);
                mma16816(acc[2 * ib + 1], a, pb[1][0], pb[1][1]);
            }
        }
        __syncwarp();
        const int nxt = i + kNvStages;
        if (nxt < npg) {
            if ((nxt & 31) == 0) ids = fetch_ids(nxt);
            issue(nxt);
        }
    }
    if (app_pending) (void)append_rows(bt[n_pages - 1], nullptr);  // the run ended early: the pool still gets the rows

    // warps -> one partial per head (the ring holds the warps' sums now)
    __syncthreads();
    float *wacc = reinterpret_cast<float *>(smem);  // [kNvWarps][G][128]
#pragma unroll
    for (int hh = 0; hh < 2; hh++) {
        const int h = 2 * j + hh;
        if (h < g) {
#pragma unroll
            for (int ib = 0; ib < 4; ib++)
                *reinterpret_cast<float4 *>(wacc + (warp * G + h) * kNvD + 16 * r + 4 * ib) =
                    make_float4(acc[2 * ib][hh], acc[2 * ib][2 + hh], acc[2 * ib + 1][hh], acc[2 * ib + 1][2 + hh]);
            if (r == 0) {
                wm[warp][h] = hh ? m1 : m0;
                wl[warp][h] = hh ? l1 : l0;
            }
        }
    }
    __syncthreads();
    constexpr int REC = kNvD + 4;
    const long long bk = (long long)b * L.hkv + kvh;
    float *part = p.part + (bk * p.n_splits + split) * (long long)g * REC;
    for (int idx = tid; idx < g * kNvD; idx += kNvThreads) {
        const int h = idx / kNvD, ch = idx - h * kNvD;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kNvWarps; w++) M = fmaxf(M, wm[w][h]);
        float a = 0.f, Ls = 0.f;
        if (M != -INFINITY)
#pragma unroll
            for (int w = 0; w < kNvWarps; w++) {
                const float f = wm[w][h] == -INFINITY ? 0.f : ex2(wm[w][h] - M);
                a = fmaf(f, wacc[(w * G + h) * kNvD + ch], a);
                Ls = fmaf(f, wl[w][h], Ls);
            }
        part[h * REC + ch] = a;
        if (ch == 0) {
            part[h * REC + kNvD] = M;
            part[h * REC + kNvD + 1] = Ls;
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
    const float *pbase = p.part + bk * p.n_splits * (long long)g * REC;
    for (int h = warp; h < g; h += kNvWarps) {
        float mc[2], lc[2];
#pragma unroll
        for (int k = 0; k < 2; k++) {
            const int c = lane + 32 * k;
            mc[k] = c < n_act ? __ldcg(pbase + (c * g + h) * REC + kNvD) : -INFINITY;
            lc[k] = c < n_act ? __ldcg(pbase + (c * g + h) * REC + kNvD + 1) : 0.f;
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
            const float4 rr = __ldcg(reinterpret_cast<const float4 *>(pbase + (c * g + h) * REC + lane * 4));
            o4[0] = fmaf(fc, rr.x, o4[0]);
            o4[1] = fmaf(fc, rr.y, o4[1]);
            o4[2] = fmaf(fc, rr.z, o4[2]);
            o4[3] = fmaf(fc, rr.w, o4[3]);
        }
        if (p.rotate) {  // back to the original domain: diag(s) H c
            fwht_warp<kNvD>(o4, lane);
#pragma unroll
            for (int e = 0; e < 4; e++) o4[e] = __uint_as_float(__float_as_uint(o4[e] * p.rot_scale) ^ (((sgb >> e) & 1u) << 31));
        }
        float *out = p.out + ((long long)b * L.hq + kvh * g + h) * kNvD + lane * 4;
        *reinterpret_cast<float4 *>(out) = Ls > 0.f ? make_float4(o4[0] / Ls, o4[1] / Ls, o4[2] / Ls, o4[3] / Ls)
                                                    : make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

template <int G>
cudaError_t launch_nv_decode_g(const DecodeParams &p, dim3 grid, cudaStream_t s)
{
    static DeviceOnce once;
    if (once.needed()) {
        const cudaError_t e =
            cudaFuncSetAttribute(nvfp4_decode_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, kNvSmem);
        if (e != cudaSuccess) return e;
        once.mark();
    }
    if (p.n_splits > kNvMaxSplits || p.L.chunk_bytes != kNvChunk) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kNvThreads);
    cfg.dynamicSmemBytes = kNvSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, nvfp4_decode_kernel<G>, p);
}

}  // namespace

cudaError_t launch_nvfp4_append(const AppendParams &p, int num_sms, cudaStream_t st)
{
    if (p.n_tok == 0) return cudaSuccess;
    return p.scale_search ? launch_nv_append<true>(p, num_sms, st) : launch_nv_append<false>(p, num_sms, st);
}

cudaError_t launch_nvfp4_decode(const DecodeParams &p, dim3 grid, cudaStream_t s)
{
    const int g = p.L.g;
    if (g <= 1) return launch_nv_decode_g<1>(p, grid, s);
    if (g <= 2) return launch_nv_decode_g<2>(p, grid, s);
    if (g <= 4) return launch_nv_decode_g<4>(p, grid, s);
    return launch_nv_decode_g<8>(p, grid, s);
}

}  // namespace kvq
