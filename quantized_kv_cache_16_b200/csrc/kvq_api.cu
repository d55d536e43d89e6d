// kvq_api.cu -- the C ABI: argument checks on the host, cache handle, kernel
// launches on the caller's stream, workspace sizing and the status word.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <new>

#include <cuda.h>

#include "kvq_internal.cuh"

using namespace kvq;

namespace {

// SplitMix64 (Steele, Lea & Flood 2014): add the golden-ratio increment to the
// state, then two xor-shift-multiply rounds and a final xor-shift.
uint64_t splitmix64_next(uint64_t &state)
{
    uint64_t z = (state += 0x9E3779B97F4A7C15ULL);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// HQMQ secondary codebook of (kv head h, tensor t) ["Hurwitz Quaternion
// Multiplicative Quantization for KV Cache Compression", 1: random unit
// quaternions per head and role, no calibration]: candidates of four
// SplitMix64 draws mapped to [-1, 1) by (out >> 40) / 2^23 - 1, rejected
// unless 1e-4 < |a|^2 <= 1, then normalised, all in fp32 (kvq.h states the
// exact recipe; the host computes it, the pool stores it).
void hqmq_codebook(uint64_t seed, int h, int t, float *S)
{
    uint64_t state = seed ^ ((uint64_t)(2 * h + t + 1) * 0xD1B54A32D192ED03ULL);
    for (int n = 0; n < kHqmqNS;) {
        float a[4];
        for (int i = 0; i < 4; i++) {
            const float m = (float)(splitmix64_next(state) >> 40);  // < 2^24: exact
            a[i] = m * (1.0f / 8388608.0f) - 1.0f;
        }
        // each square and each sum rounded to fp32, in order (the stores
        // through volatile keep a product from fusing into the next add)
        volatile float sq[4];
        for (int i = 0; i < 4; i++) sq[i] = a[i] * a[i];
        volatile float n2 = sq[0];
        for (int i = 1; i < 4; i++) n2 = n2 + sq[i];
        const float q = n2;
        if (!(q > 1e-4f && q <= 1.0f)) continue;
        const float r = sqrtf(q);
        for (int i = 0; i < 4; i++) S[4 * n + i] = a[i] / r;
        n++;
    }
}

kvq_status check_config(const kvq_config *c)
{
    if (!c) return KVQ_ERR_INVALID_ARG;
    if (c->head_dim != 64 && c->head_dim != 128) return KVQ_ERR_UNSUPPORTED;
    if (c->num_kv_heads <= 0 || c->num_q_heads <= 0 || c->num_q_heads % c->num_kv_heads) return KVQ_ERR_INVALID_ARG;
    if (c->num_q_heads / c->num_kv_heads > kMaxGqa) return KVQ_ERR_UNSUPPORTED;
    if (c->page_tokens != kPageTokens) return KVQ_ERR_UNSUPPORTED;
    if (c->num_pages <= 0) return KVQ_ERR_INVALID_ARG;
    const int fmts[2] = {c->k_fmt, c->v_fmt}, groups[2] = {c->k_group, c->v_group};
    for (int t = 0; t < 2; t++) {
        switch (fmts[t]) {
        case KVQ_INT4_ASYM:
            if (groups[t] != 32) return KVQ_ERR_UNSUPPORTED;
            break;
        case KVQ_INT2_ASYM:
            if (groups[t] != c->head_dim) return KVQ_ERR_UNSUPPORTED;
            break;
        case KVQ_INT8_SYM:
            if (t == 1) return KVQ_ERR_UNSUPPORTED;  // values: int4 or int2
            if (groups[t] != c->head_dim) return KVQ_ERR_UNSUPPORTED;
            break;
        case KVQ_HQMQ:
            if (groups[t] != 4 || c->head_dim != 128) return KVQ_ERR_UNSUPPORTED;
            break;
        case KVQ_NVFP4:
            if (groups[t] != 16 || c->head_dim != 128) return KVQ_ERR_UNSUPPORTED;
            break;
        default: return KVQ_ERR_INVALID_ARG;
        }
    }
    const bool hq = c->k_fmt == KVQ_HQMQ;
    if (hq != (c->v_fmt == KVQ_HQMQ)) return KVQ_ERR_UNSUPPORTED;  // HQMQ keys and values, or neither
    if (hq && (c->bound_block_tokens != 0 || c->scale_search != 0)) return KVQ_ERR_UNSUPPORTED;
    const bool nv = c->k_fmt == KVQ_NVFP4;
    if (nv != (c->v_fmt == KVQ_NVFP4)) return KVQ_ERR_UNSUPPORTED;  // NVFP4 keys and values, or neither
    if (nv && c->bound_block_tokens != 0) return KVQ_ERR_UNSUPPORTED;
    if (!(c->clip_ratio > 0.0f && c->clip_ratio <= 1.0f)) return KVQ_ERR_INVALID_ARG;
    if (c->bound_block_tokens < 0 || c->bound_block_tokens % kPageTokens) return KVQ_ERR_INVALID_ARG;
    if (c->rotate < 0 || c->rotate > 2) return KVQ_ERR_INVALID_ARG;
    if (c->rotate == 2 && (hq || nv)) return KVQ_ERR_UNSUPPORTED;  // the bit reversal: integer formats
    if (c->scale_search != 0 && c->scale_search != 1) return KVQ_ERR_INVALID_ARG;
    return KVQ_OK;
}

struct SplitPlan {
    int pages_per_warp, pages_per_split, n_splits;
};

// Split the context so that the grid of (split, kv head, sequence) CTAs
// fills the two CTA slots of every SM in one wave when every sequence is as
// long as the block table allows: as many splits as the slots allow per
// (sequence, kv head) pair (at most the final merge's limit), pages spread
// evenly over them in whole pages per warp.  More pairs than slots take one
// split each.
SplitPlan plan_splits(const kvq_cache *c, int batch, int max_pages)
{
    SplitPlan s{};
    const long long pairs = (long long)batch * c->L.hkv;
    const long long slots = 2LL * c->num_sms;
    long long want = pairs > 0 ? slots / pairs : 1;
    if (want < 1) want = 1;
    if (want > decode_max_splits(c->L)) want = decode_max_splits(c->L);
    const long long per_split = (max_pages + want - 1) / want;
    s.pages_per_warp = (int)((per_split + kDecodeWarps - 1) / kDecodeWarps);
    if (s.pages_per_warp < 1) s.pages_per_warp = 1;
    s.pages_per_split = s.pages_per_warp * kDecodeWarps;
    s.n_splits = (max_pages + s.pages_per_split - 1) / s.pages_per_split;
    if (s.n_splits < 1) s.n_splits = 1;
    return s;
}

size_t counters_bytes(int batch, int hkv) { return decode_counter_bytes(batch, hkv); }

size_t round256(size_t n) { return (n + 255) / 256 * 256; }

// Bound blocks a sequence of max_pages pages can hold, and the power of two
// the selection sorts.
int cert_blocks(const kvq_cache *c, int max_pages)
{
    const long long blk = c->L.bound_block;
    return blk > 0 ? (int)(((long long)max_pages * kPageTokens + blk - 1) / blk) : 0;
}

int pow2_at_least(int n)
{
    int p = 1;
    while (p < n) p <<= 1;
    return p;
}

// ceil(frac * n_blocks) in fp64 with a 1e-9 guard, clamped to [0, n_blocks]
int promote_count(float frac, int n_blocks)
{
    if (!(frac > 0.0f) || n_blocks <= 0) return 0;
    int k = (int)ceil((double)frac * (double)n_blocks - 1e-9);
    return k < 0 ? 0 : (k > n_blocks ? n_blocks : k);
}

// Page chunks of the certified blocks kernel (256 pages each).
size_t cert_chunks(int max_pages) { return ((size_t)max_pages + 255) / 256; }

// Certified-mode workspace, after the decode partials: page statistics,
// per-head totals, promoted-block lists and counts, promote partials and
// the promote counters (zero between calls).
struct CertWs {
    size_t page_stats, head_ml, blk, spart, dq, prom, prom_count, cpart, ccount;
    size_t flags, bml, mix, gstat, status, bound, nfall, dpart, dcount;  // the ladder
    size_t bytes;
};

CertWs cert_ws(const kvq_cache *c, int batch, int max_pages)
{
    CertWs w{};
    if (c->L.bound_block <= 0) return w;
    const size_t bk = (size_t)batch * c->L.hkv, g = c->L.g;
    const size_t cap = (size_t)pow2_at_least(cert_blocks(c, max_pages));
    size_t off = 0;
    w.page_stats = off;
    off += round256(bk * max_pages * g * 8);
    w.head_ml = off;
    off += round256(bk * g * 8);
    w.blk = off;
    off += round256(bk * cap * 12 * 4);
    w.spart = off;
    off += round256(bk * g * cert_chunks(max_pages) * 4);
    w.dq = off;
    off += round256(bk * g * 4);
    w.prom = off;
    off += round256(bk * cap * 4);
    w.prom_count = off;
    off += round256(bk * 4);
    w.cpart = off;
    off += round256(bk * kCertChunks * g * (3 * c->L.d + 4) * 4);
    w.ccount = off;
    off += round256(bk * 4);
    w.flags = off;
    off += round256(bk * cap);
    w.bml = off;
    off += round256(bk * cap * g * 8);
    w.mix = off;
    off += round256(bk * g * 8);
    w.gstat = off;
    off += round256(bk * 4);
    w.status = off;
    off += round256(bk * g * 4);
    w.bound = off;
    off += round256(bk * g * 4);
    w.nfall = off;
    off += 256;
    w.dpart = off;
    off += round256(bk * kDenseSplitsMax * g * (c->L.d + 4) * 4);
    w.dcount = off;
    off += round256(bk * 4);
    w.bytes = off;
    return w;
}

// Window-decode workspace, after the decode partials and the certified-mode
// regions: per-head softmax totals, the correction partials and their
// counters (zero between calls).
struct WinWs {
    size_t head_ml, cpart, ccount, bytes;
};

WinWs win_ws(const kvq_cache *c, int batch)
{
    WinWs w{};
    const size_t bk = (size_t)batch * c->L.hkv, g = c->L.g;
    size_t off = 0;
    w.head_ml = off;
    off += round256(bk * g * 8);
    w.cpart = off;
    off += round256(bk * kCertChunks * g * (3 * c->L.d + 4) * 4);
    w.ccount = off;
    off += round256(bk * 4);
    w.bytes = off;
    return w;
}

// Dense-fallback split: at most kDenseSplitsMax splits of >= 1024 tokens
// (a multiple of 64) per (sequence, kv head).
void dense_split(int max_pages, int *n_split, int *tokens)
{
    const long long T = (long long)max_pages * kPageTokens;
    long long n = (T + 1023) / 1024;
    if (n > kDenseSplitsMax) n = kDenseSplitsMax;
    if (n < 1) n = 1;
    long long per = (T + n - 1) / n;
    per = (per + 63) / 64 * 64;
    *n_split = (int)((T + per - 1) / per);
    *tokens = (int)per;
}

// A device-accessible address for `p`: device or managed memory as is; pinned
// host memory through its device mapping.  Null for unregistered host memory.
const void *device_view(const void *p)
{
    cudaPointerAttributes a;
    if (!p || cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) return p;
    if (a.type == cudaMemoryTypeHost) return a.devicePointer;
    return nullptr;
}

kvq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA; }

}  // namespace

extern "C" {

size_t kvq_pool_bytes(const kvq_config *cfg)
{
    if (check_config(cfg) != KVQ_OK) return 0;
    const Layout L = make_layout(*cfg);
    size_t n = kHeaderBytes + (size_t)cfg->num_pages * L.page_bytes;
    if (cfg->bound_block_tokens > 0) n += (size_t)cfg->num_pages * cfg->num_kv_heads * 16;
    if (cfg->k_fmt == KVQ_HQMQ) n += (size_t)cfg->num_kv_heads * 2 * kHqmqNS * 16;
    return n;
}

kvq_status kvq_create_cache(const kvq_config *cfg, void *pool_dev, size_t pool_bytes, kvq_cache **out)
{
    if (!out) return KVQ_ERR_INVALID_ARG;
    *out = nullptr;
    const kvq_status st = check_config(cfg);
    if (st != KVQ_OK) return st;
    if (!pool_dev || !aligned(pool_dev, 256)) return KVQ_ERR_INVALID_ARG;
    if (pool_bytes < kvq_pool_bytes(cfg)) return KVQ_ERR_CAPACITY;
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, pool_dev) != cudaSuccess) {
        cudaGetLastError();
        return KVQ_ERR_INVALID_ARG;
    }
    if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged) return KVQ_ERR_INVALID_ARG;

    kvq_cache *c = new (std::nothrow) kvq_cache();
    if (!c) return KVQ_ERR_CUDA;
    c->cfg = *cfg;
    c->L = make_layout(*cfg);
    c->pool = static_cast<unsigned char *>(pool_dev);
    c->pool_bytes = pool_bytes;
    c->device = attr.device;
    c->last_stream = nullptr;
    if (cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device) != cudaSuccess) {
        delete c;
        return KVQ_ERR_CUDA;
    }
    // sign vector: s_i = -1 when the top bit of the i-th SplitMix64 output is set
    uint64_t state = cfg->rotation_seed;
    for (int i = 0; i < cfg->head_dim; i++) c->signs[i] = (splitmix64_next(state) >> 63) ? -1.0f : 1.0f;
    for (int i = cfg->head_dim; i < kMaxD; i++) c->signs[i] = 1.0f;
    for (int w = 0; w < kMaxD / 2; w++)
        c->sign_xor[w] = (c->signs[2 * w] < 0 ? 0x00008000u : 0u) | (c->signs[2 * w + 1] < 0 ? 0x80000000u : 0u);
    c->rot_scale = (float)(1.0 / sqrt((double)cfg->head_dim));
    if (cudaMemset(pool_dev, 0, kvq_pool_bytes(cfg)) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
        delete c;
        return KVQ_ERR_CUDA;
    }
    if (c->L.hq_tab) {
        const size_t n = (size_t)cfg->num_kv_heads * 2 * kHqmqNS * 4;
        float *tab = static_cast<float *>(malloc(n * sizeof(float)));
        if (!tab) {
            delete c;
            return KVQ_ERR_CUDA;
        }
        for (int h = 0; h < cfg->num_kv_heads; h++)
            for (int t = 0; t < 2; t++) hqmq_codebook(cfg->rotation_seed, h, t, tab + ((size_t)h * 2 + t) * kHqmqNS * 4);
        const cudaError_t e = cudaMemcpy(c->pool + c->L.hq_tab, tab, n * sizeof(float), cudaMemcpyHostToDevice);
        free(tab);
        if (e != cudaSuccess) {
            delete c;
            return KVQ_ERR_CUDA;
        }
    }
    *out = c;
    return KVQ_OK;
}

kvq_status kvq_destroy_cache(kvq_cache *cache)
{
    if (!cache) return KVQ_ERR_INVALID_ARG;
    if (cache->copy_stream) {
        // a copy may wait for a step's mark that no later kernel will set:
        // raise both marks to the last step first
        if (cache->io_marks) {
            volatile unsigned int *m = cache->io_marks;
            m[0] = m[1] = (unsigned int)cache->io_seq;
        }
        cudaStreamSynchronize(cache->copy_stream);
        cudaStreamDestroy(cache->copy_stream);
    }
    if (cache->io_flags) cudaFree(cache->io_flags);
    if (cache->io_marks) cudaFreeHost(cache->io_marks);
    for (int b = 0; b < 2; b++) {
        if (cache->ev_copied[b]) cudaEventDestroy(cache->ev_copied[b]);
        if (cache->ev_consumed[b]) cudaEventDestroy(cache->ev_consumed[b]);
    }
    delete cache;
    return KVQ_OK;
}

kvq_status kvq_append(kvq_cache *c, const void *k, const void *v, const int32_t *slot_mapping, int32_t n_tok,
                      void *stream)
{
    if (!c || n_tok < 0) return KVQ_ERR_INVALID_ARG;
    if (n_tok == 0) return KVQ_OK;
    if (!k || !v || !slot_mapping || !aligned(k, 16) || !aligned(v, 16) || !aligned(slot_mapping, 4))
        return KVQ_ERR_INVALID_ARG;
    AppendParams p{};
    p.k = static_cast<const __half *>(k);
    p.v = static_cast<const __half *>(v);
    p.slots = slot_mapping;
    p.n_tok = n_tok;
    p.pool = c->pool;
    p.L = c->L;
    p.clip = c->cfg.clip_ratio;
    p.rot_scale = c->rot_scale;
    p.rotate = c->cfg.rotate;
    p.scale_search = c->cfg.scale_search;
    memcpy(p.sign_xor, c->sign_xor, sizeof(p.sign_xor));
    c->last_stream = stream;
    if (c->L.hq_tab) return cuda_status(launch_hqmq_append(p, c->num_sms, static_cast<cudaStream_t>(stream)));
    if (c->L.k_fmt == KVQ_NVFP4)
        return cuda_status(launch_nvfp4_append(p, c->num_sms, static_cast<cudaStream_t>(stream)));
    return cuda_status(launch_append(p, c->num_sms, static_cast<cudaStream_t>(stream)));
}

kvq_status kvq_reset_pages(kvq_cache *c, const int32_t *page_ids, int32_t n, void *stream)
{
    if (!c || n < 0 || (n > 0 && !page_ids)) return KVQ_ERR_INVALID_ARG;
    if (n == 0 || c->L.desc_off == 0) return KVQ_OK;
    c->last_stream = stream;
    return cuda_status(launch_reset_pages(c->pool, c->L, page_ids, n, static_cast<cudaStream_t>(stream)));
}

size_t kvq_decode_windows_workspace_bytes(const kvq_cache *c, int32_t batch, int32_t max_pages_per_seq)
{
    if (!c || batch < 0 || max_pages_per_seq < 1) return 0;
    const SplitPlan s = plan_splits(c, batch, max_pages_per_seq);
    const size_t part = (size_t)batch * c->L.hkv * s.n_splits * c->L.g * (c->L.d + 4) * sizeof(float);
    return counters_bytes(batch, c->L.hkv) + round256(part) + cert_ws(c, batch, max_pages_per_seq).bytes +
           win_ws(c, batch).bytes;
}

size_t kvq_decode_workspace_bytes(const kvq_cache *c, int32_t batch, int32_t max_pages_per_seq)
{
    if (!c || batch < 0 || max_pages_per_seq < 1) return 0;
    const SplitPlan s = plan_splits(c, batch, max_pages_per_seq);
    const size_t part = (size_t)batch * c->L.hkv * s.n_splits * c->L.g * (c->L.d + 4) * sizeof(float);
    return counters_bytes(batch, c->L.hkv) + round256(part) + cert_ws(c, batch, max_pages_per_seq).bytes;
}

}  // extern "C"

namespace {

DecodeParams decode_params(kvq_cache *c, const SplitPlan &s, const void *q, const int32_t *block_table,
                           int32_t max_pages, const int32_t *ctx_lens, int32_t batch, float scale, void *workspace,
                           void *out)
{
    DecodeParams p{};
    p.pool = c->pool;
    p.q = static_cast<const __half *>(q);
    p.block_table = block_table;
    p.ctx_lens = ctx_lens;
    p.max_pages = max_pages;
    p.batch = batch;
    p.L = c->L;
    p.qscale = scale * 1.4426950408889634f;  // log2(e)
    p.rot_scale = c->rot_scale;
    p.rotate = c->cfg.rotate;
    memcpy(p.signs, c->signs, sizeof(p.signs));
    for (int i = 0; i < kMaxD; i++)
        if (c->signs[i] < 0.0f) p.sign_bits[i / 32] |= 1u << (i % 32);
    p.pages_per_split = s.pages_per_split;
    p.pages_per_warp = s.pages_per_warp;
    p.n_splits = s.n_splits;
    p.counters = static_cast<unsigned int *>(workspace);
    p.part = reinterpret_cast<float *>(static_cast<unsigned char *>(workspace) + counters_bytes(batch, c->L.hkv));
    p.out = static_cast<float *>(out);
    p.clip = c->cfg.clip_ratio;
    p.expire_first_wait = c->expire_first_wait;
    return p;
}

// The certified-mode workspace regions start after the decode partials.
unsigned char *cert_base(const kvq_cache *c, const SplitPlan &s, int batch, void *workspace)
{
    return static_cast<unsigned char *>(workspace) + counters_bytes(batch, c->L.hkv) +
           round256((size_t)batch * c->L.hkv * s.n_splits * c->L.g * (c->L.d + 4) * 4);
}

CertParams cert_params(const kvq_cache *c, const DecodeParams &p, int max_pages, float scale, unsigned char *base,
                       const CertWs &w, const void *k2, const void *v2)
{
    CertParams cp{};
    cp.pool = c->pool;
    cp.q = p.q;
    cp.block_table = p.block_table;
    cp.ctx_lens = p.ctx_lens;
    cp.max_pages = max_pages;
    cp.L = c->L;
    cp.scale = scale;
    cp.qscale = p.qscale;
    cp.rot_scale = c->rot_scale;
    cp.rotate = c->cfg.rotate;
    memcpy(cp.signs, c->signs, sizeof(cp.signs));
    cp.sort_cap = pow2_at_least(cert_blocks(c, max_pages));
    cp.page_stats = p.page_stats;
    cp.head_ml = p.head_ml;
    cp.blk = reinterpret_cast<float *>(base + w.blk);
    cp.spart = reinterpret_cast<float *>(base + w.spart);
    cp.dq = reinterpret_cast<float *>(base + w.dq);
    cp.n_chunk_cap = (int)cert_chunks(max_pages);
    cp.prom = reinterpret_cast<int32_t *>(base + w.prom);
    cp.prom_count = reinterpret_cast<int32_t *>(base + w.prom_count);
    cp.k2 = static_cast<const __half *>(k2);
    cp.v2 = static_cast<const __half *>(v2);
    cp.cpart = reinterpret_cast<float *>(base + w.cpart);
    cp.ccount = reinterpret_cast<unsigned int *>(base + w.ccount);
    cp.out = p.out;
    return cp;
}

// Certified-mode limits shared by both modes: bound blocks of 16 * 2^k <= 512
// tokens, at most kCertMaxBlocks per sequence.
kvq_status cert_shape_ok(const kvq_cache *c, int max_pages)
{
    if (c->L.bound_block <= 0) return KVQ_ERR_INVALID_ARG;
    if (cert_blocks(c, max_pages) > kCertMaxBlocks) return KVQ_ERR_UNSUPPORTED;
    const int ppb = c->L.bound_block / kPageTokens;  // pages per block: a power of two <= 32
    if (ppb > 32 || (ppb & (ppb - 1))) return KVQ_ERR_UNSUPPORTED;
    return KVQ_OK;
}

// Stream memory operations (driver entry points, resolved once): the host
// step's copy stream waits for, and announces with, 32-bit flags in device
// memory.  ok is false where they cannot be had (the host step then takes
// events).
typedef CUresult (*StreamValueFn)(CUstream, CUdeviceptr, cuuint32_t, unsigned int);
struct StreamMemOps {
    StreamValueFn wait = nullptr, write = nullptr;
    bool ok = false;
};
const StreamMemOps &stream_mem_ops()
{
    static const StreamMemOps ops = [] {
        StreamMemOps o;
        void *w = nullptr, *x = nullptr;
        cudaDriverEntryPointQueryResult q1 = cudaDriverEntryPointSymbolNotFound, q2 = q1;
        if (cudaGetDriverEntryPointByVersion("cuStreamWaitValue32", &w, 12000, cudaEnableDefault, &q1) == cudaSuccess &&
            cudaGetDriverEntryPointByVersion("cuStreamWriteValue32", &x, 12000, cudaEnableDefault, &q2) == cudaSuccess &&
            q1 == cudaDriverEntryPointSuccess && q2 == cudaDriverEntryPointSuccess && w && x) {
            o.wait = reinterpret_cast<StreamValueFn>(w);
            o.write = reinterpret_cast<StreamValueFn>(x);
            o.ok = true;
        }
        cudaGetLastError();
        return o;
    }();
    return ops;
}

kvq_status decode_impl(kvq_cache *c, const void *k_new, const void *v_new, const int32_t *slot_mapping,
                       const void *q, const int32_t *block_table, int32_t max_pages_per_seq, const int32_t *ctx_lens,
                       int32_t batch, float softmax_scale, const kvq_tier2 *tier2, void *workspace, size_t ws_bytes,
                       void *out, int32_t *promoted_out, void *stream, const unsigned int *rec_ready = nullptr,
                       unsigned int *rec_consumed = nullptr, unsigned int rec_seq = 0)
{
    if (!c || batch < 0 || max_pages_per_seq < 1) return KVQ_ERR_INVALID_ARG;
    if (batch == 0) return KVQ_OK;
    if (!q || !block_table || !ctx_lens || !out || !workspace) return KVQ_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(workspace, 256)) return KVQ_ERR_INVALID_ARG;
    if (k_new && (!v_new || !slot_mapping || !aligned(k_new, 16) || !aligned(v_new, 16))) return KVQ_ERR_INVALID_ARG;
    if (c->L.hq_tab || c->L.k_fmt == KVQ_NVFP4) {  // HQMQ, NVFP4: own decode kernels, no tier 2
        if (tier2 || (k_new && c->L.hq_tab)) return KVQ_ERR_UNSUPPORTED;  // NVFP4 fuses the step's append
        if (ws_bytes < kvq_decode_workspace_bytes(c, batch, max_pages_per_seq)) return KVQ_ERR_CAPACITY;
        const SplitPlan s = plan_splits(c, batch, max_pages_per_seq);
        const float scale = softmax_scale > 0.0f ? softmax_scale : (float)(1.0 / sqrt((double)c->L.d));
        DecodeParams p = decode_params(c, s, q, block_table, max_pages_per_seq, ctx_lens, batch, scale, workspace, out);
        p.new_k = static_cast<const __half *>(k_new);
        p.new_v = static_cast<const __half *>(v_new);
        p.new_slots = slot_mapping;
        c->last_stream = stream;
        const dim3 grid(s.n_splits, c->L.hkv, batch);
        return cuda_status(c->L.hq_tab ? launch_hqmq_decode(p, grid, static_cast<cudaStream_t>(stream))
                                       : launch_nvfp4_decode(p, grid, static_cast<cudaStream_t>(stream)));
    }
    if (!decode_supported(c->L)) return KVQ_ERR_UNSUPPORTED;
    // certified mode: checks and the tier-2 device view
    int kmax = 0;
    const void *k2 = nullptr, *v2 = nullptr;
    if (tier2) {
        if (k_new || c->L.bound_block <= 0) return KVQ_ERR_INVALID_ARG;
        if (!(tier2->promote_frac >= 0.0f && tier2->promote_frac <= 1.0f)) return KVQ_ERR_INVALID_ARG;
        const kvq_status sh = cert_shape_ok(c, max_pages_per_seq);
        if (sh != KVQ_OK) return sh;
        kmax = promote_count(tier2->promote_frac, cert_blocks(c, max_pages_per_seq));
        if (kmax > 0) {
            k2 = device_view(tier2->k_host);
            v2 = device_view(tier2->v_host);
            if (!k2 || !v2 || !aligned(k2, 16) || !aligned(v2, 16)) return KVQ_ERR_INVALID_ARG;
        }
    }
    if (ws_bytes < kvq_decode_workspace_bytes(c, batch, max_pages_per_seq)) return KVQ_ERR_CAPACITY;
    const SplitPlan s = plan_splits(c, batch, max_pages_per_seq);
    const float scale = softmax_scale > 0.0f ? softmax_scale : (float)(1.0 / sqrt((double)c->L.d));
    DecodeParams p = decode_params(c, s, q, block_table, max_pages_per_seq, ctx_lens, batch, scale, workspace, out);
    p.new_k = static_cast<const __half *>(k_new);
    p.new_v = static_cast<const __half *>(v_new);
    p.new_slots = slot_mapping;
    p.rec_ready = rec_ready;
    p.rec_consumed = rec_consumed;
    p.rec_seq = rec_seq;
    c->last_stream = stream;
    const dim3 grid(s.n_splits, c->L.hkv, batch);
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned char *base = cert_base(c, s, batch, workspace);
    const CertWs w = cert_ws(c, batch, max_pages_per_seq);
    if (kmax > 0) {
        p.page_stats = reinterpret_cast<float2 *>(base + w.page_stats);
        p.head_ml = reinterpret_cast<float2 *>(base + w.head_ml);
    }
    kvq_status rc = cuda_status(launch_decode(p, grid, st));
    if (rc != KVQ_OK || kmax == 0) return rc;

    CertParams cp = cert_params(c, p, max_pages_per_seq, scale, base, w, k2, v2);
    cp.frac = tier2->promote_frac;
    cp.kmax_out = kmax;
    cp.n_chunks = kmax < kCertChunks ? kmax : kCertChunks;
    cp.promoted_out = promoted_out;
    rc = cuda_status(launch_cert_blocks(cp, batch, st));
    if (rc != KVQ_OK) return rc;
    rc = cuda_status(launch_cert_select(cp, batch, st));
    if (rc != KVQ_OK) return rc;
    return cuda_status(launch_cert_promote(cp, batch, st));
}

bool in_unit(float x) { return x >= 0.0f && x <= 1.0f; }  // false for NaN
bool non_negative(float x) { return x >= 0.0f; }          // +inf allowed, NaN not

kvq_status ladder_impl(kvq_cache *c, const void *q, const int32_t *block_table, int32_t max_pages,
                       const int32_t *ctx_lens, int32_t batch, float softmax_scale, const void *k_tier2,
                       const void *v_tier2, const kvq_ladder *pol, void *workspace, size_t ws_bytes, void *out,
                       const kvq_ladder_report *rep, void *stream)
{
    if (!c || batch < 0 || max_pages < 1 || !pol) return KVQ_ERR_INVALID_ARG;
    if (batch == 0) return KVQ_OK;
    if (!q || !block_table || !ctx_lens || !out || !workspace) return KVQ_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(workspace, 256)) return KVQ_ERR_INVALID_ARG;
    if (!decode_supported(c->L)) return KVQ_ERR_UNSUPPORTED;
    const kvq_status sh = cert_shape_ok(c, max_pages);
    if (sh != KVQ_OK) return sh;
    if (!in_unit(pol->tau_cov) || !in_unit(pol->max_frac) || !in_unit(pol->layer_frac) ||
        !non_negative(pol->key_tol) || !non_negative(pol->v_tol) || !non_negative(pol->rank_tol) ||
        !non_negative(pol->cert_tol))
        return KVQ_ERR_INVALID_ARG;
    const int nb_max = cert_blocks(c, max_pages);
    if (rep && rep->block_flags && rep->flags_cols < nb_max) return KVQ_ERR_INVALID_ARG;
    const void *k2 = device_view(k_tier2), *v2 = device_view(v_tier2);
    if (!k2 || !v2 || !aligned(k2, 16) || !aligned(v2, 16)) return KVQ_ERR_INVALID_ARG;
    if (ws_bytes < kvq_decode_workspace_bytes(c, batch, max_pages)) return KVQ_ERR_CAPACITY;

    const SplitPlan s = plan_splits(c, batch, max_pages);
    const float scale = softmax_scale > 0.0f ? softmax_scale : (float)(1.0 / sqrt((double)c->L.d));
    DecodeParams p = decode_params(c, s, q, block_table, max_pages, ctx_lens, batch, scale, workspace, out);
    unsigned char *base = cert_base(c, s, batch, workspace);
    const CertWs w = cert_ws(c, batch, max_pages);
    p.page_stats = reinterpret_cast<float2 *>(base + w.page_stats);
    p.head_ml = reinterpret_cast<float2 *>(base + w.head_ml);
    c->last_stream = stream;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    kvq_status rc = cuda_status(launch_decode(p, dim3(s.n_splits, c->L.hkv, batch), st));
    if (rc != KVQ_OK) return rc;

    CertParams cp = cert_params(c, p, max_pages, scale, base, w, k2, v2);
    cp.ladder = 1;
    cp.frac = pol->max_frac;
    cp.n_chunks = kCertChunks;
    cp.tau_cov = pol->tau_cov;
    cp.key_tol = pol->key_tol;
    cp.v_tol = pol->v_tol;
    cp.rank_tol = pol->rank_tol;
    cp.cert_tol = pol->cert_tol;
    // more than layer_frac * batch * Hq heads <=> more than its floor (an integer count)
    cp.layer_thresh = (int)floor((double)pol->layer_frac * (double)batch * (double)c->L.hq);
    cp.flags = base + w.flags;
    cp.bml = reinterpret_cast<float2 *>(base + w.bml);
    cp.mix = reinterpret_cast<float2 *>(base + w.mix);
    cp.gstat = reinterpret_cast<int32_t *>(base + w.gstat);
    cp.status = reinterpret_cast<int32_t *>(base + w.status);
    cp.bound = reinterpret_cast<float *>(base + w.bound);
    cp.nfall = reinterpret_cast<unsigned int *>(base + w.nfall);
    if (rep) {
        cp.k_star_out = rep->k_star;
        cp.flags_out = rep->block_flags;
        cp.nb_out = rep->block_flags ? rep->flags_cols : 0;
        cp.bound_out = rep->bound;
        cp.status_out = rep->status;
    }
    dense_split(max_pages, &cp.n_dsplit, &cp.dsplit_tokens);
    cp.batch = batch;
    cp.dense_ctas = c->num_sms;  // one 256-thread CTA per SM fits the kernel's registers
    cp.dpart = reinterpret_cast<float *>(base + w.dpart);
    cp.dcount = reinterpret_cast<unsigned int *>(base + w.dcount);
    rc = cuda_status(launch_cert_blocks(cp, batch, st));
    if (rc == KVQ_OK) rc = cuda_status(launch_ladder_select(cp, batch, st));
    if (rc == KVQ_OK) rc = cuda_status(launch_cert_promote(cp, batch, st));
    if (rc == KVQ_OK) rc = cuda_status(launch_ladder_finish(cp, batch, st));
    return rc;
}

}  // namespace

extern "C" {

kvq_status kvq_decode_windows(kvq_cache *c, const void *q, const int32_t *block_table, int32_t max_pages_per_seq,
                              const int32_t *ctx_lens, int32_t batch, float softmax_scale, const void *k_win,
                              const void *v_win, int32_t sink, int32_t recent, void *workspace, size_t ws_bytes,
                              void *out, void *stream)
{
    if (!c || batch < 0 || max_pages_per_seq < 1 || sink < 0 || recent < 0) return KVQ_ERR_INVALID_ARG;
    if (batch == 0) return KVQ_OK;
    if (!q || !block_table || !ctx_lens || !out || !workspace) return KVQ_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(workspace, 256)) return KVQ_ERR_INVALID_ARG;
    if (!decode_supported(c->L)) return KVQ_ERR_UNSUPPORTED;
    const void *k2 = nullptr, *v2 = nullptr;
    if (sink + recent > 0) {
        k2 = device_view(k_win);
        v2 = device_view(v_win);
        if (!k2 || !v2 || !aligned(k2, 16) || !aligned(v2, 16)) return KVQ_ERR_INVALID_ARG;
    }
    if (ws_bytes < kvq_decode_windows_workspace_bytes(c, batch, max_pages_per_seq)) return KVQ_ERR_CAPACITY;
    const SplitPlan s = plan_splits(c, batch, max_pages_per_seq);
    const float scale = softmax_scale > 0.0f ? softmax_scale : (float)(1.0 / sqrt((double)c->L.d));
    DecodeParams p = decode_params(c, s, q, block_table, max_pages_per_seq, ctx_lens, batch, scale, workspace, out);
    // the window regions follow every certified-mode region, so calls of the
    // two kinds can share one workspace (each leaves its own counters zero)
    unsigned char *base = cert_base(c, s, batch, workspace) + cert_ws(c, batch, max_pages_per_seq).bytes;
    const WinWs w = win_ws(c, batch);
    if (sink + recent > 0) {
        p.head_ml = reinterpret_cast<float2 *>(base + w.head_ml);
        p.win_sink = sink;  // the quantised pass leaves the window tokens out
        p.win_recent = recent;
    }
    c->last_stream = stream;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    kvq_status rc = cuda_status(launch_decode(p, dim3(s.n_splits, c->L.hkv, batch), st));
    if (rc != KVQ_OK || sink + recent == 0) return rc;
    CertParams cp{};
    cp.pool = c->pool;
    cp.q = p.q;
    cp.block_table = block_table;
    cp.ctx_lens = ctx_lens;
    cp.max_pages = max_pages_per_seq;
    cp.L = c->L;
    cp.scale = scale;
    cp.qscale = p.qscale;
    cp.rot_scale = c->rot_scale;
    cp.rotate = c->cfg.rotate;
    memcpy(cp.signs, c->signs, sizeof(cp.signs));
    cp.head_ml = p.head_ml;
    {  // one wave over all (sequence, kv head) pairs
        const long long groups = (long long)batch * c->L.hkv;
        long long n = 2LL * c->num_sms / groups;  // the window instantiation keeps two CTAs per SM
        cp.n_chunks = (int)(n < 1 ? 1 : (n > kCertChunks ? kCertChunks : n));
    }
    cp.k2 = static_cast<const __half *>(k2);
    cp.v2 = static_cast<const __half *>(v2);
    cp.sink = sink;
    cp.recent = recent;
    cp.cpart = reinterpret_cast<float *>(base + w.cpart);
    cp.ccount = reinterpret_cast<unsigned int *>(base + w.ccount);
    cp.out = p.out;
    return cuda_status(launch_windows(cp, batch, st));
}

kvq_status kvq_decode_certified(kvq_cache *c, const void *q, const int32_t *block_table, int32_t max_pages_per_seq,
                                const int32_t *ctx_lens, int32_t batch, float softmax_scale, const void *k_tier2,
                                const void *v_tier2, const kvq_ladder *policy, void *workspace, size_t ws_bytes,
                                void *out, const kvq_ladder_report *report, void *stream)
{
    return ladder_impl(c, q, block_table, max_pages_per_seq, ctx_lens, batch, softmax_scale, k_tier2, v_tier2, policy,
                       workspace, ws_bytes, out, report, stream);
}

kvq_status kvq_decode_attn(kvq_cache *c, const void *q, const int32_t *block_table, int32_t max_pages_per_seq,
                           const int32_t *ctx_lens, int32_t batch, float softmax_scale, const kvq_tier2 *tier2,
                           void *workspace, size_t ws_bytes, void *out, int32_t *promoted_out, void *stream)
{
    return decode_impl(c, nullptr, nullptr, nullptr, q, block_table, max_pages_per_seq, ctx_lens, batch,
                       softmax_scale, tier2, workspace, ws_bytes, out, promoted_out, stream);
}

kvq_status kvq_decode_step(kvq_cache *c, const void *k_new, const void *v_new, const int32_t *slot_mapping,
                           const void *q, const int32_t *block_table, int32_t max_pages_per_seq,
                           const int32_t *ctx_lens, int32_t batch, float softmax_scale, void *workspace,
                           size_t ws_bytes, void *out, void *stream)
{
    if (!k_new) return KVQ_ERR_INVALID_ARG;
    if (c && c->cfg.scale_search) return KVQ_ERR_UNSUPPORTED;  // the fused append does not search scales
    return decode_impl(c, k_new, v_new, slot_mapping, q, block_table, max_pages_per_seq, ctx_lens, batch,
                       softmax_scale, nullptr, workspace, ws_bytes, out, nullptr, stream);
}

}  // extern "C"

namespace {

struct StepRecord {
    size_t q, k, v, slot, ctx, bytes;
};

size_t up16(size_t n) { return (n + 15) / 16 * 16; }

StepRecord step_record(const kvq_cache *c, int batch)
{
    StepRecord r{};
    const size_t b = (size_t)batch, d = (size_t)c->L.d;
    r.q = 0;
    r.k = up16(b * c->L.hq * d * 2);
    r.v = r.k + up16(b * c->L.hkv * d * 2);
    r.slot = r.v + up16(b * c->L.hkv * d * 2);
    r.ctx = r.slot + up16(b * 4);
    r.bytes = r.ctx + up16(b * 4);
    return r;
}

bool pinned_host(const void *p)
{
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeHost;
}

// The device view of page-locked host memory; null for anything else.
void *pinned_device_view(const void *p)
{
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return a.type == cudaMemoryTypeHost ? a.devicePointer : nullptr;
}

}  // namespace

extern "C" {

size_t kvq_step_record_bytes(const kvq_cache *c, int32_t batch)
{
    if (!c || batch < 1) return 0;
    return step_record(c, batch).bytes;
}

kvq_status kvq_debug_expire_first_wait(kvq_cache *c, int32_t on)
{
    if (!c || on < 0 || on > 2) return KVQ_ERR_INVALID_ARG;
    c->expire_first_wait = on;
    return KVQ_OK;
}

kvq_status kvq_decode_step_host(kvq_cache *c, const void *host_in, void *dev_rec, const int32_t *block_table,
                                int32_t max_pages_per_seq, int32_t batch, float softmax_scale, void *workspace,
                                size_t ws_bytes, void *host_out, void *stream)
{
    if (!c || batch < 1 || !host_in || !dev_rec || !host_out || !aligned(dev_rec, 16)) return KVQ_ERR_INVALID_ARG;
    if (!pinned_host(host_in)) return KVQ_ERR_INVALID_ARG;
    void *o = pinned_device_view(host_out);
    if (!o || !aligned(o, 16)) return KVQ_ERR_INVALID_ARG;
    if (c->cfg.scale_search || c->L.hq_tab) return KVQ_ERR_UNSUPPORTED;
    if (!c->copy_stream) {
        // the stream and its four events are created into locals and kept
        // only if all five exist, so a failure here leaves the handle as it
        // was and the next call tries again
        cudaStream_t cs = nullptr;
        cudaEvent_t ev[4] = {nullptr, nullptr, nullptr, nullptr};
        bool ok = cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) == cudaSuccess;
        for (int i = 0; ok && i < 4; i++) ok = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) == cudaSuccess;
        if (!ok) {
            for (int i = 0; i < 4; i++)
                if (ev[i]) cudaEventDestroy(ev[i]);
            if (cs) cudaStreamDestroy(cs);
            return KVQ_ERR_CUDA;
        }
        c->ev_copied[0] = ev[0];
        c->ev_copied[1] = ev[1];
        c->ev_consumed[0] = ev[2];
        c->ev_consumed[1] = ev[3];
        c->copy_stream = cs;
    }
    // The integer decode takes the flag handshake: nothing but the steps'
    // kernels on `stream`, so consecutive steps overlap through the dependent
    // launch.  NVFP4 (its own decode kernel) takes events between the steps.
    const StreamMemOps &ops = stream_mem_ops();
    const bool flags = ops.ok && c->L.k_fmt != KVQ_NVFP4;
    if (flags && !c->io_flags) {
        // ready flags in device memory; consumed marks in mapped page-locked
        // host memory, which the host reads to skip the copy's wait when the
        // mark is already there
        unsigned int *f = nullptr, *m = nullptr, *md = nullptr;
        bool ok = cudaMalloc(&f, 2 * sizeof(unsigned int)) == cudaSuccess &&
                  cudaMemset(f, 0, 2 * sizeof(unsigned int)) == cudaSuccess &&
                  cudaHostAlloc(&m, 2 * sizeof(unsigned int), cudaHostAllocMapped) == cudaSuccess &&
                  cudaHostGetDevicePointer(&md, m, 0) == cudaSuccess;
        if (!ok) {
            if (f) cudaFree(f);
            if (m) cudaFreeHost(m);
            return KVQ_ERR_CUDA;
        }
        m[0] = m[1] = 0u;
        c->io_flags = f;
        c->io_marks = m;
        c->io_marks_dev = md;
        c->io_seq = 0;
    }
    const StepRecord r = step_record(c, batch);
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool relayout = r.bytes != c->io_bytes || dev_rec != c->io_buf;
    if (relayout) {
        // another layout: no half may still be in use, so the copy waits for
        // every kernel enqueued on `stream` so far
        if (cudaEventRecord(c->ev_consumed[0], st) != cudaSuccess ||
            cudaStreamWaitEvent(c->copy_stream, c->ev_consumed[0], 0) != cudaSuccess)
            return KVQ_ERR_CUDA;
        c->io_bytes = r.bytes;
        c->io_buf = dev_rec;
    }
    const int b = c->io_next;
    unsigned char *d = static_cast<unsigned char *>(dev_rec) + (size_t)b * r.bytes;
    const int32_t *ctx = reinterpret_cast<const int32_t *>(d + r.ctx);
    const int32_t *slots = reinterpret_cast<const int32_t *>(d + r.slot);
    if (flags) {
        // Step n copies into half n & 1 once the kernel of step n - 1 has
        // started, which it does only after the kernel of step n - 2 (the
        // half's last reader) is complete: that kernel marks consumed[half]
        // = n - 2.  The copy then raises ready[half] to n, which the
        // kernel of step n waits for.  Both compare in modular order.
        // (the step count is 64-bit; the flags hold its low 32 bits)
        unsigned int *ready = c->io_flags, *consumed = c->io_marks_dev;
        const unsigned long long n64 = ++c->io_seq;
        const unsigned int n = (unsigned int)n64;
        const volatile unsigned int *seen = c->io_marks;
        // any failure from here on makes the next call start afresh (as after
        // a layout change: its copy waits for every kernel enqueued before it)
        bool fail = !relayout && n64 >= 3 && (int)(seen[b] - (n - 2u)) < 0 &&
                    ops.wait(c->copy_stream, (CUdeviceptr)(consumed + b), n - 2u, CU_STREAM_WAIT_VALUE_GEQ) != CUDA_SUCCESS;
        fail = fail || cudaMemcpyAsync(d, host_in, r.bytes, cudaMemcpyHostToDevice, c->copy_stream) != cudaSuccess ||
               ops.write(c->copy_stream, (CUdeviceptr)(ready + b), n, CU_STREAM_WRITE_VALUE_DEFAULT) != CUDA_SUCCESS;
        if (fail) {
            c->io_bytes = 0;
            return KVQ_ERR_CUDA;
        }
        c->io_next = b ^ 1;
        unsigned int *mark = n64 >= 2 ? consumed + (b ^ 1) : nullptr;
        const kvq_status rc = decode_impl(c, d + r.k, d + r.v, slots, d + r.q, block_table, max_pages_per_seq, ctx,
                                          batch, softmax_scale, nullptr, workspace, ws_bytes, o, nullptr, stream,
                                          ready + b, mark, n);
        if (rc != KVQ_OK) c->io_bytes = 0;
        return rc;
    }
    // the copy of this step's record overlaps the previous step's kernel: it
    // waits only for the kernel that last read the same buffer
    if (cudaStreamWaitEvent(c->copy_stream, c->ev_consumed[b], 0) != cudaSuccess ||
        cudaMemcpyAsync(d, host_in, r.bytes, cudaMemcpyHostToDevice, c->copy_stream) != cudaSuccess ||
        cudaEventRecord(c->ev_copied[b], c->copy_stream) != cudaSuccess ||
        cudaStreamWaitEvent(st, c->ev_copied[b], 0) != cudaSuccess)
        return KVQ_ERR_CUDA;
    const kvq_status rc = decode_impl(c, d + r.k, d + r.v, slots, d + r.q, block_table, max_pages_per_seq, ctx, batch,
                                      softmax_scale, nullptr, workspace, ws_bytes, o, nullptr, stream);
    if (rc != KVQ_OK) return rc;
    if (cudaEventRecord(c->ev_consumed[b], st) != cudaSuccess) return KVQ_ERR_CUDA;
    c->io_next = b ^ 1;
    return KVQ_OK;
}

kvq_status kvq_dequant_debug(kvq_cache *c, const int32_t *slots, int32_t n, float *k_out, float *v_out,
                             uint8_t *codes_out, uint16_t *meta_out, void *stream)
{
    if (!c || n < 0) return KVQ_ERR_INVALID_ARG;
    if (c->L.hq_tab || c->L.k_fmt == KVQ_NVFP4) return KVQ_ERR_UNSUPPORTED;  // integer formats only
    if (n == 0) return KVQ_OK;
    if (!slots) return KVQ_ERR_INVALID_ARG;
    DequantParams p{};
    p.pool = c->pool;
    p.slots = slots;
    p.n = n;
    p.L = c->L;
    p.k_out = k_out;
    p.v_out = v_out;
    p.codes_out = codes_out;
    p.meta_out = meta_out;
    c->last_stream = stream;
    return cuda_status(launch_dequant(p, static_cast<cudaStream_t>(stream)));
}

kvq_status kvq_sync_status(kvq_cache *c)
{
    if (!c) return KVQ_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(c->last_stream)) != cudaSuccess) return KVQ_ERR_CUDA;
    unsigned int st = 0;
    if (cudaMemcpy(&st, c->pool, sizeof(st), cudaMemcpyDeviceToHost) != cudaSuccess) return KVQ_ERR_CUDA;
    if (st != 0 && cudaMemset(c->pool, 0, sizeof(st)) != cudaSuccess) return KVQ_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return KVQ_ERR_CUDA;
    return static_cast<kvq_status>(st);
}

const char *kvq_status_string(kvq_status s)
{
    switch (s) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID_ARG: return "invalid argument";
    case KVQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case KVQ_ERR_CAPACITY: return "buffer smaller than required";
    case KVQ_ERR_OUT_OF_RANGE: return "slot or page index outside the pool";
    case KVQ_ERR_CUDA: return "CUDA runtime error";
    case KVQ_ERR_TIMEOUT: return "bounded device wait ran out";
    default: return "unknown status";
    }
}

}  // extern "C"
