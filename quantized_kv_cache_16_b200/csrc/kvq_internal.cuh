// kvq_internal.cuh -- internal definitions shared by the library's .cu files:
// the pool layout, the cache handle, kernel parameter blocks and the inline
// PTX wrappers (bulk copy + mbarrier, ldmatrix, mma.sync).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

constexpr int kPageTokens = 16;
constexpr int kHeaderBytes = 256;
constexpr int kMaxD = 128;
constexpr int kMaxGqa = 8;

// Status word lives at the start of the pool header.
struct PoolHeader {
    unsigned int status;
    unsigned int pad[63];
};

// HQMQ: 1024 secondary codewords per (kv head, K|V); two fp16 outlier blocks
// per row; 20 bits per 4-element block (5 bits an element); 24 meta bytes.
constexpr int kHqmqNS = 1024;
constexpr int kHqmqOut = 2;
constexpr int kHqmqRowMeta = 8 + 8 * kHqmqOut;

inline __host__ __device__ int fmt_bits(int fmt)
{
    return fmt == KVQ_INT4_ASYM || fmt == KVQ_NVFP4 ? 4 : fmt == KVQ_INT8_SYM ? 8 : fmt == KVQ_HQMQ ? 5 : 2;
}

// Byte layout of the pool (see kvq_pool_bytes in kvq.h).
struct Layout {
    int d, hq, hkv, g;
    int k_fmt, v_fmt;
    int k_row_code, v_row_code;  // code bytes of one token row
    int k_row_meta, v_row_meta;  // meta bytes of one token row
    int k_codes, k_meta, v_codes, v_meta;  // region offsets inside a chunk
    int chunk_bytes;                       // one (page, kv head)
    long long page_bytes;
    int num_pages;
    long long desc_off;  // from the pool start; 0 when descriptors are off
    int bound_block;
    long long hq_tab;    // HQMQ codebooks [Hkv][2][1024] float4 from the pool start; 0 otherwise
};

inline __host__ Layout make_layout(const kvq_config &c)
{
    Layout L{};
    L.d = c.head_dim;
    L.hq = c.num_q_heads;
    L.hkv = c.num_kv_heads;
    L.g = c.num_q_heads / c.num_kv_heads;
    L.k_fmt = c.k_fmt;
    L.v_fmt = c.v_fmt;
    L.k_row_code = L.d * fmt_bits(c.k_fmt) / 8;
    L.v_row_code = L.d * fmt_bits(c.v_fmt) / 8;
    L.k_row_meta = c.k_fmt == KVQ_HQMQ    ? kHqmqRowMeta
                   : c.k_fmt == KVQ_NVFP4 ? L.d / 16
                   : c.k_fmt == KVQ_INT8_SYM ? 2
                                              : 4 * (L.d / c.k_group);
    L.v_row_meta = c.v_fmt == KVQ_HQMQ    ? kHqmqRowMeta
                   : c.v_fmt == KVQ_NVFP4 ? L.d / 16
                   : c.v_fmt == KVQ_INT8_SYM ? 2
                                              : 4 * (L.d / c.v_group);
    L.k_codes = 0;
    L.k_meta = kPageTokens * L.k_row_code;
    L.v_codes = L.k_meta + kPageTokens * L.k_row_meta;
    L.v_meta = L.v_codes + kPageTokens * L.v_row_code;
    L.chunk_bytes = L.v_meta + kPageTokens * L.v_row_meta;
    L.page_bytes = (long long)L.hkv * L.chunk_bytes;
    L.num_pages = c.num_pages;
    L.bound_block = c.bound_block_tokens;
    L.desc_off = c.bound_block_tokens > 0 ? kHeaderBytes + (long long)c.num_pages * L.page_bytes : 0;
    L.hq_tab = 0;
    if (c.k_fmt == KVQ_HQMQ)
        L.hq_tab = kHeaderBytes + (long long)c.num_pages * L.page_bytes +
                   (c.bound_block_tokens > 0 ? (long long)c.num_pages * L.hkv * 16 : 0);
    return L;
}

}  // namespace kvq

struct kvq_cache {
    kvq_config cfg;
    kvq::Layout L;
    unsigned char *pool;
    size_t pool_bytes;
    int device;
    int num_sms;
    float signs[kvq::kMaxD];       // +1 / -1
    uint32_t sign_xor[kvq::kMaxD / 2];  // per half2 word: 0x8000 / 0x80000000 where the sign is -1
    float rot_scale;               // fp32(1/sqrt(d))
    void *last_stream;
    // kvq_decode_step_host: record copies on their own stream, two record
    // buffers used alternately (created on first use)
    cudaStream_t copy_stream = nullptr;
    cudaEvent_t ev_copied[2] = {nullptr, nullptr};   // record b is on the device
    cudaEvent_t ev_consumed[2] = {nullptr, nullptr}; // the kernel that read record b is done
    int io_next = 0;
    size_t io_bytes = 0;        // record size and buffer of the last call:
    const void *io_buf = nullptr;  // when either changes, the copy waits for both halves
    // the integer decode's record handshake (no event between the steps'
    // kernels, so they overlap through the dependent launch): ready[2] in
    // device memory, consumed[2] in mapped page-locked host memory (and its
    // device view), the step number of the last call
    unsigned int *io_flags = nullptr;
    unsigned int *io_marks = nullptr;
    unsigned int *io_marks_dev = nullptr;
    unsigned long long io_seq = 0;
    int expire_first_wait = 0;  // test hook (kvq_debug_expire_first_wait)
};

namespace kvq {

// ---------------------------------------------------------------- kernels ---

struct AppendParams {
    const __half *k;
    const __half *v;
    const int32_t *slots;
    int n_tok;
    unsigned char *pool;
    Layout L;
    float clip;
    float rot_scale;
    int rotate;
    int scale_search;
    uint32_t sign_xor[kMaxD / 2];
};

struct DecodeParams {
    const unsigned char *pool;
    const __half *q;
    const int32_t *block_table;
    const int32_t *ctx_lens;
    int max_pages;
    int batch;
    Layout L;
    float qscale;  // softmax scale * log2(e)
    float rot_scale;
    int rotate;
    float signs[kMaxD];
    uint32_t sign_bits[kMaxD / 32];  // bit i % 32 of word i / 32: sign i is -1
    int pages_per_split;
    int pages_per_warp;
    int n_splits;
    float *part;              // [B][Hkv][n_splits][g][d + 4]
    unsigned int *counters;   // [B][Hkv] finished CTAs, zero between calls
    float *out;
    // fused append of one token per sequence before attending (null = off)
    const __half *new_k;      // [B][Hkv][d]
    const __half *new_v;
    const int32_t *new_slots; // [B]: the slot of position ctx_lens[b] - 1
    float clip;
    // certified mode: per page and head (m, l) = (running max, sum of
    // 2^(s - m) over the page's tokens), log2 units; null = off
    float2 *page_stats;       // [B][Hkv][max_pages][g]
    // sink and recent windows attended elsewhere (0, 0 = none): only tokens
    // [min(sink, T), max(that, T - recent)) are attended here
    int win_sink, win_recent;
    float2 *head_ml;          // [B][Hkv][g]: totals (M, L) of the softmax, certified mode only
    int expire_first_wait;    // test hook: each warp's first page wait counts as expired
    // kvq_decode_step_host: the step's record (context lengths, query, new
    // rows) is on the device once *rec_ready reaches rec_seq (written after
    // its copy on the library's copy stream); CTA (0, 0, 0) marks the previous
    // step's record consumed (*rec_consumed = rec_seq - 1) once the previous
    // grid is complete.  Null otherwise.
    const unsigned int *rec_ready;
    unsigned int *rec_consumed;
    unsigned int rec_seq;
};

struct DequantParams {
    const unsigned char *pool;
    const int32_t *slots;
    int n;
    Layout L;
    float *k_out;
    float *v_out;
    uint8_t *codes_out;
    uint16_t *meta_out;
};

// Certified mode ["Runtime-Certified Bounded-Error Quantized Attention",
// Methodology 1-3]: after the quantised decode (which records page_stats),
// one CTA per (sequence, kv head) turns the page statistics and the block
// descriptors into per-block error bounds and picks the top blocks; then up
// to kCertChunks CTAs per (sequence, kv head) recompute those blocks from the
// exact fp16 rows (tier 2) and correct the output in place.
constexpr int kCertChunks = 16;       // promote CTAs per (sequence, kv head)
constexpr int kCertMaxBlocks = 16384; // bound blocks per sequence the selection can sort

struct CertParams {
    const unsigned char *pool;
    const __half *q;
    const int32_t *block_table;
    const int32_t *ctx_lens;
    int max_pages;
    Layout L;
    float scale;   // softmax scale (natural units)
    float qscale;  // scale * log2(e)
    float rot_scale;
    int rotate;
    float signs[kMaxD];
    float frac;        // promoted fraction of each (sequence, kv head)'s blocks
    int sort_cap;      // power of two >= every sequence's block count
    int kmax_out;      // columns of promoted_out
    int n_chunks;      // promote CTAs per (sequence, kv head)
    const float2 *page_stats;  // [B][Hkv][max_pages][g] from the decode kernel
    const float2 *head_ml;     // [B][Hkv][g]: (M, L) of the quantised pass, log2 units (decode kernel)
    float *blk;                // [B][Hkv][sort_cap][12]: per-block masses and descriptors
    float *spart;              // [B][Hkv][g][n_chunk_cap]: per-chunk sums of P_b e^(Delta_b)
    float *dq;                 // [B][Hkv][g]: scale * ||q_r||_1
    int n_chunk_cap;           // page chunks of the blocks kernel: ceil(max_pages / 256)
    int32_t *prom;             // [B][Hkv][sort_cap]: promoted blocks, highest bound first
    int32_t *prom_count;       // [B][Hkv]
    int32_t *promoted_out;     // optional [B][Hkv][kmax_out], -1 padded
    const __half *k2;          // tier 2: exact rows [num_pages*16][Hkv][d] fp16, device-accessible
    const __half *v2;
    float *cpart;              // [B][Hkv][n_chunks][g][3d + 4]: sums of the mixed (exact values, dequantised
                               // values) and quantised sides, then (m, l) of each side
    unsigned int *ccount;      // [B][Hkv], zero between calls
    float *out;                // [B][Hq][d]

    // adaptive ladder ["Runtime-Certified...", Methodology 3]; frac is then
    // the budget of key-promoted blocks.  prom entries carry flags in bits
    // 24-25 (kPromKey, kPromVal); the fixed-fraction mode promotes both.
    int ladder;
    float tau_cov, key_tol, v_tol, rank_tol, cert_tol;
    int layer_thresh;          // every head falls back when more than this many do on their own
    unsigned char *flags;      // [B][Hkv][sort_cap]: bit 0 key exact, bit 1 value exact
    float2 *bml;               // [B][Hkv][sort_cap][g]: (m, l) of key-promoted blocks' exact scores, log2 units
    float2 *mix;               // [B][Hkv][g]: (R, den) of the mixed output's softmax (promote's merge)
    int32_t *gstat;            // [B][Hkv]: group status bits and K* (bits 16+)
    int32_t *status;           // [B][Hq]: status bits of each head
    float *bound;              // [B][Hq]: certified bound of each head's mixed output
    unsigned int *nfall;       // heads that fell back on their own (one counter)
    int32_t *k_star_out;       // optional [B][Hkv]
    unsigned char *flags_out;  // optional [B][Hkv][nb_out]
    int nb_out;
    float *bound_out;          // optional [B][Hq]
    int32_t *status_out;       // optional [B][Hq]
    int sink, recent;             // window decode: the store's sink rows and recent ring length (k2/v2 = the store)
    int n_dsplit, dsplit_tokens;  // dense fallback: splits per (sequence, kv head) and tokens per split
    int batch, dense_ctas;        // the persistent dense-fallback grid
    float *dpart;              // [B][Hkv][n_dsplit][g][d + 4]
    unsigned int *dcount;      // [B][Hkv], zero between calls
};

constexpr int kPromKey = 1 << 24, kPromVal = 1 << 25, kPromIdx = (1 << 24) - 1;
constexpr int kDenseSplitsMax = 64;

// ladder status bits (kvq.h: KVQ_LADDER_*)
constexpr int kStExpanded = 1, kStCapped = 2, kStValues = 4, kStRankFail = 8, kStBoundFail = 16,
              kStHeadDense = 32, kStLayerDense = 64;

// launchers (return cudaGetLastError() of the launch)
cudaError_t launch_append(const AppendParams &p, int num_sms, cudaStream_t s);
cudaError_t launch_decode(const DecodeParams &p, dim3 grid, cudaStream_t s);
cudaError_t launch_dequant(const DequantParams &p, cudaStream_t s);
cudaError_t launch_reset_pages(unsigned char *pool, Layout L, const int32_t *pages, int n, cudaStream_t s);
cudaError_t launch_cert_blocks(const CertParams &p, int batch, cudaStream_t s);
cudaError_t launch_cert_select(const CertParams &p, int batch, cudaStream_t s);
cudaError_t launch_cert_promote(const CertParams &p, int batch, cudaStream_t s);
cudaError_t launch_ladder_select(const CertParams &p, int batch, cudaStream_t s);
cudaError_t launch_ladder_finish(const CertParams &p, int batch, cudaStream_t s);
cudaError_t launch_windows(const CertParams &p, int batch, cudaStream_t s);
cudaError_t launch_hqmq_append(const AppendParams &p, int num_sms, cudaStream_t s);
cudaError_t launch_hqmq_decode(const DecodeParams &p, dim3 grid, cudaStream_t s);
cudaError_t launch_nvfp4_append(const AppendParams &p, int num_sms, cudaStream_t s);
cudaError_t launch_nvfp4_decode(const DecodeParams &p, dim3 grid, cudaStream_t s);
bool decode_supported(const Layout &L);
int decode_max_splits(const Layout &L);
constexpr int kDecodeWarps = 8;

// Decode workspace head: the finished-CTA counters [B][Hkv], rounded to 256
// bytes.  Zero before the first call; every call leaves them zero.
inline size_t decode_counter_bytes(int batch, int hkv)
{
    return ((size_t)batch * hkv * 4 + 255) / 256 * 256;
}
constexpr int kDecodeThreads = kDecodeWarps * 32;

// One-time setup per device (a kernel's shared-memory attribute is a
// property of the device it was set on): a bit per device, 64 devices.
struct DeviceOnce {
    unsigned long long done = 0;
    static int device()
    {
        int dev = 0;
        return cudaGetDevice(&dev) == cudaSuccess ? dev : 0;
    }
    bool needed() const
    {
        const int dev = device();
        return dev >= 64 || !((done >> dev) & 1ull);
    }
    void mark()
    {
        const int dev = device();
        if (dev < 64) done |= 1ull << dev;
    }
};

// ------------------------------------------------------------- device util ---

__device__ __forceinline__ void set_status(const unsigned char *pool, unsigned int code)
{
    unsigned int *st = reinterpret_cast<unsigned int *>(const_cast<unsigned char *>(pool));
    atomicCAS(st, 0u, code);
}

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, unsigned count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Arm the barrier for `bytes` and start a bulk global->shared copy that
// completes the transaction on it.  src/dst 16-byte aligned, bytes % 16 == 0.
// The arrive is relaxed: the copy's completion publishes the data to the
// waiting consumer, and the issuing thread has nothing of its own to publish,
// so its earlier memory operations (e.g. an atomic in flight) need not finish
// first.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile("mbarrier.arrive.expect_tx.relaxed.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// The warp-uniform form of a ring refill: every lane executes it, only the
// lane whose `copy` is set arms the barrier and starts the bulk copy, and only
// the lane whose `skip` is set arrives on the barrier without a copy (a slot
// with nothing to load).  Predicated instructions, no branch.
__device__ __forceinline__ void bulk_load_or_arrive(bool copy, bool skip, uint32_t dst, const void *src,
                                                    uint32_t bytes, uint32_t bar)
{
    asm volatile(
        "{\n"
        " .reg .pred pc, ps;\n"
        " setp.ne.u32 pc, %4, 0;\n"
        " setp.ne.u32 ps, %5, 0;\n"
        " @pc mbarrier.arrive.expect_tx.relaxed.cta.shared::cta.b64 _, [%3], %2;\n"
        " @pc cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n"
        " @ps mbarrier.arrive.relaxed.cta.shared::cta.b64 _, [%3];\n"
        "}\n" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar), "r"((uint32_t)copy), "r"((uint32_t)skip)
        : "memory");
}

// Hint: bring `bytes` at src into L2 (no data returned, no completion to
// wait for).  src 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t phase)
{
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(phase)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ unsigned long long globaltimer_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Wait for phase `phase` of the barrier, giving up after ~limit_ns.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t phase, unsigned long long limit_ns)
{
    if (mbar_try_wait(bar, phase)) return true;
    unsigned long long t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, phase)) return true;
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
}

// Wait until the 32-bit flag *f (written by a stream memory operation, i.e.
// from outside the SMs) reaches v in modular order, giving up after
// ~limit_ns.  Acquire at system scope: what was written before the flag is
// visible after it.
__device__ __forceinline__ bool flag_wait_bounded(const unsigned int *f, unsigned int v, unsigned long long limit_ns)
{
    unsigned int x;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(x) : "l"(f) : "memory");
    if ((int)(x - v) >= 0) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (true) {
        __nanosleep(32);
        asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(x) : "l"(f) : "memory");
        if ((int)(x - v) >= 0) return true;
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t &r0, uint32_t &r1)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// D(16x8 f32) += A(16x16 f16, row) * B(16x8 f16, col)
__device__ __forceinline__ void mma16816(float *d, const uint32_t *a, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }

__device__ __forceinline__ __half2 bits_h2(uint32_t u) { return *reinterpret_cast<__half2 *>(&u); }

}  // namespace kvq
