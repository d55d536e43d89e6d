/*
 * kvq.h -- C ABI of the B200 low-bit KV cache: quantise-on-append of K/V and
 * split-K decode attention over the packed, paged cache.
 *
 * What the calls compute (page titles and sections):
 *  - Rotation: R = c_d * H_d * diag(s), a fixed random sign vector s followed by
 *    the (Sylvester) Walsh-Hadamard transform, c_d = fp32(1/sqrt(d))
 *    ["When Quantization Is Free", Methodology 1 (random-sign rotation, SRHT);
 *    "OSCAR", 2.2 (Hadamard factor of the rotation)].
 *  - Codec: per-group asymmetric int4 (group 32) and int2 (group = head_dim,
 *    optional clip ratio) with fp16 scale and fp16 zero; symmetric int8 per
 *    token-head with an fp16 scale ["When Quantization Is Free", Methodology 2
 *    (per-group scaling, rounding, nibble packing); "Runtime-Certified
 *    Bounded-Error Quantized Attention", Methodology 1 (INT8 keys, INT4 values,
 *    scales/offsets); "OSCAR", 2.2 (INT2 history, clipping thresholds)].
 *  - Decode: softmax attention of one new query per sequence over the paged
 *    cache, dequantised in registers, merged across context splits by the
 *    log-sum-exp rule, inverse-rotated ["OSCAR", 2.2b (fused kernel: unpack,
 *    dequantise, inverse rotation, attention over a paged cache)].
 *  - Sink and recent windows: the first and the latest tokens at fp16, the
 *    middle history quantised ["OSCAR", 2.2b, mixed-precision layout].
 *  - Certified mode: per-block key/value error bounds, top-fraction promotion
 *    of blocks to their fp16 originals held in pinned host memory, and the
 *    adaptive ladder (coverage-driven key promotion, value promotion, the
 *    ranking-consistency check, per-head and whole-call fp16 fallbacks)
 *    ["Runtime-Certified Bounded-Error Quantized Attention", Methodology 1-3].
 *
 * Conventions for every call:
 *  - All tensors are caller-owned device memory unless stated (the library
 *    never allocates device memory).  fp16 tensors are passed as void*.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Every call is asynchronous on that stream and never synchronises, except
 *    kvq_create_cache (zero-fills the pool) and kvq_sync_status.
 *  - Argument checks run on the host before any launch; a failed check returns
 *    an error status and launches nothing.  A failed launch returns
 *    KVQ_ERR_CUDA.  Conditions only the device can see (a block-table entry or
 *    slot outside the pool, a bounded wait that ran out) are recorded in a
 *    status word inside the pool; kvq_sync_status reports and clears it.
 *  - Calls on one cache are not thread-safe with respect to each other.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KVQ_OK = 0,
    KVQ_ERR_INVALID_ARG = 1,  /* NULL pointer, bad size, misaligned buffer     */
    KVQ_ERR_UNSUPPORTED = 2,  /* valid but not built (format/head_dim/GQA mix)  */
    KVQ_ERR_CAPACITY = 3,     /* pool or workspace smaller than required        */
    KVQ_ERR_OUT_OF_RANGE = 4, /* device saw a slot/page index outside the pool  */
    KVQ_ERR_CUDA = 5,         /* a CUDA runtime call or launch failed           */
    KVQ_ERR_TIMEOUT = 6       /* a bounded device-side wait ran out             */
} kvq_status;

typedef enum {
    KVQ_INT4_ASYM = 0, /* 4-bit codes, group 32, fp16 scale + fp16 zero         */
    KVQ_INT8_SYM = 1,  /* 8-bit signed codes, one fp16 scale per token-head     */
    KVQ_INT2_ASYM = 2, /* 2-bit codes, group = head_dim, fp16 scale + fp16 zero */
    KVQ_HQMQ = 3,      /* Hurwitz-quaternion codes of 4-element blocks (group 4,
                          head_dim 128, keys and values both), see below       */
    KVQ_NVFP4 = 4      /* e2m1 codes, one E4M3 scale per 16 elements (group 16,
                          head_dim 128, keys and values both), see below       */
} kvq_fmt;

/* NVFP4 ["Search Your Block Floating Point Scales!", NVFP4 and ScaleSearch].
 * Per block of 16 rotated elements: scale byte = E4M3 (OCP E4M3FN) of
 * max|x| / 6 (fp32 division; nearest, ties to the even code, above 448 to
 * 448); code of x = e2m1 of x / scale (fp32 division): the nearest of
 * +-{0, 0.5, 1, 1.5, 2, 3, 4, 6}, ties to the even magnitude index, beyond
 * 6 to 6, zero (and NaN) code 0, bit 3 the sign; all codes 0 when the scale
 * is 0.  With scale_search = 1 the scale bytes b0 + f, f tried as 0, -1, 1,
 * -2, 2, 3, 4, 5, 6 (positive finite codes only; b0 nonzero and finite),
 * each quantise the block and the least squared error wins, a later one only
 * if strictly smaller; the error is fp32, per run of four elements ((e0^2 +
 * e1^2) + e2^2) + e3^2 with e = x - value, then (r0 + r1) + (r2 + r3).
 * Storage (token-major rows): 64 code bytes (byte j = code[2j] |
 * code[2j+1] << 4), then per region 16 meta rows of the 8 scale bytes.  A
 * value decodes to e2m1 x scale, exact in fp16.  kvq_append, kvq_decode_attn
 * (without tier 2) and kvq_decode_attn_static serve NVFP4 caches, and
 * kvq_decode_step / kvq_decode_step_host when scale_search is 0 (the fused
 * append codes the new token with the default scales); the other decode
 * calls return KVQ_ERR_UNSUPPORTED. */

/* HQMQ ["Hurwitz Quaternion Multiplicative Quantization for KV Cache
 * Compression", 1-3].  A rotated row is cut into d/4 blocks x (a quaternion);
 * a block is coded as radius x direction, the direction as the codeword of
 * largest inner product among the 24 x 1024 products q_p q_s of a unit
 * Hurwitz quaternion q_p (the binary tetrahedral group, p = 0..23) and a
 * secondary unit quaternion q_s (s = 0..1023, drawn per kv head and K|V, no
 * calibration).  Blocks whose radius exceeds tau = 3 x the row's lower median
 * radius are outliers (Med3x): the two largest keep their four fp16 values;
 * further ones are coded with a clipped radius.
 *   units: p = 0..7 are +1, -1, +i, -i, +j, -j, +k, -k; p = 8..23 are
 *     (+-1 +-i +-j +-k)/2, component c negative iff bit c of p - 8 is set;
 *   codebook S of (kv head h, tensor t in {0 = K, 1 = V}): SplitMix64 from
 *     state rotation_seed ^ ((2h + t + 1) * 0xD1B54A32D192ED03); a candidate
 *     takes four outputs, component = (out >> 40) / 2^23 - 1 (fp32), and is
 *     kept when 1e-4 < |a|^2 <= 1 (fp32, squares summed in order), then
 *     divided by fp32 sqrt(|a|^2); the first 1024 kept are S[0..1024);
 *   row (fp32, each operation rounded, in this order): r_b = sqrt(((x0^2 +
 *     x1^2) + x2^2) + x3^2); tau = 3 x the 16th smallest r_b; outliers: up to
 *     two blocks with r_b > tau, largest first (lower block on ties); step =
 *     fp16 rounded up of tau / 31; radius code = min(31, rint(r_b / step)) (0
 *     when step = 0); direction u = x / r_b; for each s in order, w = u
 *     conj(q_s) (Hamilton product; each component is its first product,
 *     rounded, then the other three added in order by fused multiply-adds,
 *     a subtracted product as one with its first factor negated) scores
 *     max_i |w_i| (first i, sign of w_i) or, when
 *     strictly larger, (((|w0| + |w1|) + |w2|) + |w3|) / 2 (signs of w); the
 *     first s of highest score wins; index = 24 s + p (0 when r_b = 0);
 *   storage: a token's code row is d/4 fields of 20 bits (index | radius code
 *     << 15) as one little-endian bit stream (80 bytes at d = 128), 16 rows
 *     per region, token-major; meta row (24 bytes) = fp16 step, 2 zero bytes,
 *     the 32-bit outlier mask (bit b = block b), two outlier slots of four
 *     fp16 values in block order (unused slots zero).  The codebooks sit in
 *     the pool after the pages (and descriptors): [Hkv][2][1024] x 4 fp32.
 * A block decodes to (radius code x step) x q_p q_s, an outlier to its fp16
 * values.  HQMQ caches have no descriptors and no scale search; kvq_append,
 * kvq_decode_attn (without tier 2) and kvq_decode_attn_static serve them,
 * the other decode calls return KVQ_ERR_UNSUPPORTED. */

typedef struct {
    int32_t num_q_heads;        /* Hq; Hq / Hkv (the GQA group) must be 1..8          */
    int32_t num_kv_heads;       /* Hkv                                                */
    int32_t head_dim;           /* d: 64 or 128                                       */
    int32_t k_fmt, v_fmt;       /* kvq_fmt of keys / values (values: int4, int2, or
                                   HQMQ / NVFP4 with keys of the same format)        */
    int32_t k_group, v_group;   /* int4: 32; int2, int8: head_dim; HQMQ: 4; NVFP4: 16 */
    float clip_ratio;           /* (0, 1]; scales both ends of int2/int4 groups       */
    uint64_t rotation_seed;     /* SplitMix64 state that draws the sign vector        */
    int32_t rotate;             /* 1 = sign + Hadamard rotation, 0 = identity,
                                   2 = sign + Hadamard + bit-reversal permutation of
                                   the channels ["OSCAR", 2.2(a): R = H_Had P_br,
                                   without the data-derived U; the channel j of
                                   the rotated row is channel br(j) of H's output,
                                   br reversing the log2(head_dim) index bits;
                                   integer formats only]                            */
    int32_t page_tokens;        /* tokens per page; must be 16                        */
    int32_t num_pages;          /* pages in the pool                                  */
    int32_t bound_block_tokens; /* 0 = no error descriptors; else a multiple of 16    */
    int32_t scale_search;       /* 1 = ScaleSearch of each scale (see kvq_append)     */
} kvq_config;

typedef struct kvq_cache kvq_cache; /* opaque; owned by the library */

/* Tier-2 store of the certified mode ["Runtime-Certified Bounded-Error
 * Quantized Attention", Methodology 1]: the original fp16 K and V rows (not
 * rotated) indexed by slot, [num_pages*16][Hkv][d] each, 16-byte aligned.
 * Pinned host memory (cudaHostAlloc / cudaMallocHost / cudaHostRegister) is
 * read by the kernels through its device mapping, as the pages place it;
 * device memory is accepted as well.  Pageable host memory is rejected with
 * KVQ_ERR_INVALID_ARG.  The caller keeps the rows current (they are the
 * ground truth the pages call tier 2). */
typedef struct {
    const void *k_host;
    const void *v_host;
    float promote_frac; /* fraction of bound blocks per (seq, kv head) promoted */
} kvq_tier2;

/* Bytes of device memory the pool of `cfg` needs; 0 if cfg is invalid.
 * Layout: [256-byte header][num_pages pages][descriptors].  A page holds
 * num_kv_heads chunks [K codes][K meta][V codes][V meta] of 16 tokens.  Codes
 * of a token are its sequential bit stream (int4: byte j = code[2j] |
 * code[2j+1] << 4; int2: four codes per byte from the low bits up; int8:
 * two's complement) cut into 16-byte chunks stored chunk-major, chunk c of
 * token t at (c*16 + t)*16, so one 16-byte load is a whole int4 group.  Meta
 * rows are fp16 scales then fp16 zeros (int8: one scale).  Descriptors (when
 * bound_block_tokens > 0): per (page, kv head) four fp32 {max key error, max
 * value error, max |value|, 0}.  HQMQ pools add the codebooks (see
 * KVQ_HQMQ). */
size_t kvq_pool_bytes(const kvq_config *cfg);

/* Create a cache over caller-owned device memory `pool_dev` of `pool_bytes`
 * (>= kvq_pool_bytes, 256-byte aligned).  Zero-fills the pool (synchronous),
 * draws the sign vector from rotation_seed and, for HQMQ, writes the
 * codebooks.  *out receives the handle. */
kvq_status kvq_create_cache(const kvq_config *cfg, void *pool_dev, size_t pool_bytes, kvq_cache **out);

/* Release the handle (the pool memory stays the caller's). */
kvq_status kvq_destroy_cache(kvq_cache *cache);

/* Quantise-on-append ["When Quantization Is Free", Methodology 2]: rotate,
 * quantise and pack n_tok tokens of k and v (fp16, [n_tok][Hkv][d], 16-byte
 * aligned) into the slots slot_mapping[0..n_tok) (int32, device).  A negative
 * slot skips the token; a slot >= num_pages*16 is skipped and recorded as
 * KVQ_ERR_OUT_OF_RANGE in the status word.  With descriptors on, each row's
 * max |k - khat|, max |v - vhat| and max |v| are max-reduced into its page's
 * descriptor (reset a page with kvq_reset_pages before reusing it).
 * With cfg.scale_search = 1 each group's fp16 scale is searched
 * ["Search Your Block Floating Point Scales!", ScaleSearch]: the scales whose
 * bit patterns are the default scale's plus f, f in [-2, 6] (positive finite
 * only), each quantise the group and the one with the least squared
 * reconstruction error is stored (fp32 sums: per run of 64 consecutive
 * elements, even and odd elements apart in element order, then added, the
 * runs added in order; candidates tried as 0, -1, 1, -2, 2, 3, 4, 5, 6, a
 * later one kept only if strictly better); the zero is unchanged.
 * HQMQ caches code each row as KVQ_HQMQ states (a search over 24,576
 * codewords per block: compute-bound, about 1.5 M fp32 operations a row). */
kvq_status kvq_append(kvq_cache *cache, const void *k, const void *v, const int32_t *slot_mapping, int32_t n_tok,
                      void *stream);

/* Zero the descriptors of n pages listed in page_ids (int32, device). */
kvq_status kvq_reset_pages(kvq_cache *cache, const int32_t *page_ids, int32_t n, void *stream);

/* Workspace bytes kvq_decode_attn needs for `batch` sequences with block
 * tables of max_pages_per_seq entries (with bound blocks configured, this
 * includes the certified mode's page statistics, promoted-block lists and
 * partials).  The workspace must be zero-filled before its first use; every
 * decode call leaves it ready for the next one. */
size_t kvq_decode_workspace_bytes(const kvq_cache *cache, int32_t batch, int32_t max_pages_per_seq);

/* Decode attention ["OSCAR", 2.2b]: for each sequence b and query head h,
 * out[b][h] = R^T softmax(scale * (R q[b][h]) . khat_t) . vhat_t over the
 * ctx_lens[b] tokens whose pages block_table[b][0..] lists (16 tokens a page),
 * with kv head h / (Hq/Hkv).
 *   q:           fp16 [batch][Hq][d] (device)
 *   block_table: int32 [batch][max_pages_per_seq] (device)
 *   ctx_lens:    int32 [batch] (device), 0 <= ctx_lens[b] <= 16*max_pages_per_seq
 *   softmax_scale: <= 0 means 1/sqrt(d)
 *   tier2:       NULL, or the certified-mode store (needs bound_block_tokens
 *                of 16 * 2^k tokens, at most 512, and a block count
 *                16*max_pages_per_seq/bound_block_tokens of at most 16384,
 *                else KVQ_ERR_UNSUPPORTED; promote_frac in [0, 1]).  The quantised decode then records per-page
 *                softmax statistics; per (sequence, kv head) a bound is formed
 *                for every block [Methodology 2: a key term from the score
 *                perturbation, a value term from the value error, weighted by
 *                the block's softmax mass], the ceil(promote_frac * n_blocks)
 *                highest blocks (ties: lower block first) are recomputed from
 *                the tier-2 rows, and their quantised contribution to the
 *                output is replaced by the exact one [Methodology 3].  Three
 *                launches on `stream`.
 *   workspace:   >= kvq_decode_workspace_bytes, zero-filled before first use;
 *                one workspace must not serve two decode calls that overlap
 *   out:         fp32 [batch][Hq][d] (device, 16-byte aligned); fp32 so the
 *                result keeps the kernel's accuracy (an fp16 store alone
 *                would round outputs of magnitude 32 by up to 0.008)
 *   promoted_out (certified mode, optional): int32 [batch][Hkv][kmax] block
 *                indices promoted, highest bound first, -1 padded, where
 *                kmax = ceil(promote_frac * ceil(16*max_pages_per_seq / block)).
 * An empty context gives a zero output row.
 * Kernels of this call (and of kvq_decode_step) are launched as programmatic
 * dependents of the stream's previous kernel: each waits for that kernel to
 * complete, with its writes visible, before touching memory, so stream order
 * holds as for a plain launch; only the launch latency is overlapped. */
kvq_status kvq_decode_attn(kvq_cache *cache, const void *q, const int32_t *block_table, int32_t max_pages_per_seq,
                           const int32_t *ctx_lens, int32_t batch, float softmax_scale, const kvq_tier2 *tier2,
                           void *workspace, size_t ws_bytes, void *out, int32_t *promoted_out, void *stream);

/* Workspace bytes kvq_decode_windows needs (zero-filled before first use;
 * every call leaves it ready for the next). */
size_t kvq_decode_windows_workspace_bytes(const kvq_cache *cache, int32_t batch, int32_t max_pages_per_seq);

/* Decode with 16-bit sink and recent windows ["OSCAR", 2.2b: the paged cache
 * keeps the first (sink) and the most recent tokens at full precision and
 * the middle history low-bit]: as kvq_decode_attn, except that each
 * sequence's first `sink` tokens and last `recent` tokens attend with their
 * fp16 rows from a compact window store, the rest with the quantised cache.
 *   k_win, v_win: fp16 [batch][sink + recent][Hkv][d] (not rotated; device
 *                 memory or pinned host memory, 16-byte aligned): row t holds
 *                 token t for t < sink; row sink + t % recent holds token t
 *                 of the recent window.  The caller keeps the store current
 *                 (write each new token's row at sink + t % recent when it is
 *                 appended; rows of tokens outside both windows are not read).
 *   sink, recent: >= 0; a token in both windows is read from its sink row.
 * The quantised decode runs first over the tokens between the windows (the
 * window tokens are in the pool too, but masked out of that pass); then up
 * to 16 CTAs per (sequence, kv head) attend over the window rows and merge
 * their partial into the output by the log-sum-exp rule.  Two launches; one
 * when both windows are empty.  Workspace: kvq_decode_windows_workspace_bytes. */
kvq_status kvq_decode_windows(kvq_cache *cache, const void *q, const int32_t *block_table, int32_t max_pages_per_seq,
                              const int32_t *ctx_lens, int32_t batch, float softmax_scale, const void *k_win,
                              const void *v_win, int32_t sink, int32_t recent, void *workspace, size_t ws_bytes,
                              void *out, void *stream);

/* Policy of the certified ladder ["Runtime-Certified Bounded-Error Quantized
 * Attention", Methodology 3: adaptive Top-K, ranking-consistency check,
 * four-rung fallback ladder].  Tolerances may be +INFINITY (that rung or
 * check off); NaN or a value outside its range is KVQ_ERR_INVALID_ARG. */
typedef struct {
    float tau_cov;    /* [0, 1]: estimated block mass the exact keys must cover, for every head   */
    float max_frac;   /* [0, 1]: budget, at most ceil(max_frac * n_blocks) key-promoted blocks     */
    float key_tol;    /* >= 0: rung 1 grows the key set until the predicted key term is <= key_tol */
    float v_tol;      /* >= 0: rung 2 promotes values of blocks with max_h Phat_h(b)*eta_b > v_tol */
    float rank_tol;   /* >= 0: slack of the ranking-consistency check                              */
    float cert_tol;   /* >= 0: heads whose certified bound exceeds it fall back to fp16 (rung 3)   */
    float layer_frac; /* [0, 1]: every head falls back when more than layer_frac*batch*Hq do (rung 4) */
} kvq_ladder;

/* Status bits of a head (kvq_ladder_report.status). */
enum {
    KVQ_LADDER_EXPANDED = 1,    /* rung 1 added blocks beyond the coverage set (group-wide)   */
    KVQ_LADDER_CAPPED = 2,      /* the budget cut the key set short (group-wide)              */
    KVQ_LADDER_VALUES = 4,      /* rung 2 promoted values in this kv head's group             */
    KVQ_LADDER_RANK_FAIL = 8,   /* the ranking-consistency check failed for this head         */
    KVQ_LADDER_BOUND_FAIL = 16, /* the certified bound exceeded cert_tol                      */
    KVQ_LADDER_HEAD_DENSE = 32, /* rung 3: this head was recomputed as fp16 attention         */
    KVQ_LADDER_LAYER_DENSE = 64 /* rung 4: every head of the call was recomputed in fp16      */
};

/* Optional device outputs of kvq_decode_certified (any pointer may be NULL). */
typedef struct {
    int32_t *k_star;      /* [batch][Hkv]: key-promoted blocks                              */
    uint8_t *block_flags; /* [batch][Hkv][flags_cols]: bit 0 key exact, bit 1 value exact;
                             flags_cols >= ceil(16*max_pages_per_seq / bound_block_tokens) */
    int32_t flags_cols;
    float *bound;         /* [batch][Hq]: certified bound of the mixed output (before any
                             fallback), an upper bound on the inf-norm of its error in the
                             rotated domain                                                 */
    int32_t *status;      /* [batch][Hq]: KVQ_LADDER_* bits                                 */
} kvq_ladder_report;

/* Certified decode with the adaptive ladder ["Runtime-Certified Bounded-Error
 * Quantized Attention", Methodology 1-3].  Per sequence and kv head, with
 * Phat_h(b) the softmax mass of bound block b under the quantised scores of
 * query head h, Delta_h(b) = scale*||R q_h||_1*eps_b the largest score error
 * of the block, and eta_b, nu_b its largest value error and |value| (the
 * descriptors):
 *  1. blocks are ranked by max_h Phat_h(b) (ties: lower block first);
 *  2. K_cov = the fewest leading blocks whose Phat reaches tau_cov for every
 *     head of the group;
 *  3. rung 1: K_key = the fewest leading blocks whose exact keys bring every
 *     head's predicted key term sum_b Phat nu_b (e^{D_b + A} - 1), A = ln
 *     sum_b Phat e^{D_b} (D = 0 for exact-key blocks, Delta otherwise) to
 *     key_tol; the first K* = min(budget, max(K_cov, K_key)) blocks are
 *     recomputed with their tier-2 keys;
 *  4. rung 2: blocks with max_h Phat_h(b)*eta_b > v_tol use their tier-2 values;
 *  5. the output is attention with those keys/values exact, the rest dequantised;
 *  6. per head, the key-promoted blocks ordered by Phat_h fail the ranking
 *     check when a later one has an exact mass above (1 + rank_tol) times an
 *     earlier one's;
 *  7. per head, the certified bound of that output is the key term and the
 *     mass-weighted value error of the blocks with quantised values, both
 *     over the output's own softmax masses;
 *  8. rung 3: a head whose check fails or whose bound exceeds cert_tol is
 *     recomputed as fp16 attention over its tier-2 rows;
 *  9. rung 4: if more than layer_frac*batch*Hq heads fall back, all do.
 * Decisions are taken in fp32 from the quantised pass's statistics.
 *   k_tier2, v_tier2: the tier-2 store as for kvq_tier2 (pinned host or
 *                device memory, [num_pages*16][Hkv][d] fp16, 16-byte aligned;
 *                pageable host memory: KVQ_ERR_INVALID_ARG)
 *   Other arguments as kvq_decode_attn, with the certified-mode limits on
 *   the bound blocks (KVQ_ERR_UNSUPPORTED beyond them).  Six launches on
 *   `stream`; the fp16 fallback kernel exits at once when no head needs it. */
kvq_status kvq_decode_certified(kvq_cache *cache, const void *q, const int32_t *block_table,
                                int32_t max_pages_per_seq, const int32_t *ctx_lens, int32_t batch,
                                float softmax_scale, const void *k_tier2, const void *v_tier2,
                                const kvq_ladder *policy, void *workspace, size_t ws_bytes, void *out,
                                const kvq_ladder_report *report, void *stream);

/* One decode step: quantise-on-append of each sequence's new token followed
 * by decode attention over the grown context, in one launch.  k_new, v_new:
 * fp16 [batch][Hkv][d] (16-byte aligned), the token at position
 * ctx_lens[b] - 1; slot_mapping[b] must be that position's slot, i.e.
 * block_table[b][(ctx_lens[b]-1)/16]*16 + (ctx_lens[b]-1)%16 (otherwise the
 * token is not stored and KVQ_ERR_OUT_OF_RANGE is recorded).  The stored
 * codes are byte-identical to kvq_append's and the output equals kvq_append
 * followed by kvq_decode_attn.  Other arguments as kvq_decode_attn (no
 * certified mode).  A cache configured with scale_search returns
 * KVQ_ERR_UNSUPPORTED (use kvq_append, then kvq_decode_attn). */
kvq_status kvq_decode_step(kvq_cache *cache, const void *k_new, const void *v_new, const int32_t *slot_mapping,
                           const void *q, const int32_t *block_table, int32_t max_pages_per_seq,
                           const int32_t *ctx_lens, int32_t batch, float softmax_scale, void *workspace,
                           size_t ws_bytes, void *out, void *stream);

/* Bytes of the host record of kvq_decode_step_host for `batch` sequences:
 * q fp16 [batch][Hq][d], then k_new fp16 [batch][Hkv][d], v_new fp16
 * [batch][Hkv][d], slot_mapping int32 [batch], ctx_lens int32 [batch], each
 * section starting at a multiple of 16 bytes.  0 for a NULL cache or
 * batch < 1. */
size_t kvq_step_record_bytes(const kvq_cache *cache, int32_t batch);

/* One decode step from and to host memory: kvq_decode_step on a copy of
 * the pinned host record `host_in` (kvq_step_record_bytes long, layout
 * above), whose kernel writes the fp32 output [batch][Hq][d] straight to
 * pinned `host_out` (16-byte aligned) through its device mapping (no copy
 * back).  `dev_rec` is device memory for two records (2 x
 * kvq_step_record_bytes, 16-byte aligned), used alternately: the record is
 * copied on a stream of the library's own, waiting only for the step that
 * last used the same half, so the copy overlaps the previous step's kernel;
 * the kernel, on `stream`, waits for its copy.  For the integer formats the
 * two sides meet through 32-bit flags in device memory (stream memory
 * operations on the copy stream; the kernel waits for its record's flag,
 * bounded, else KVQ_ERR_TIMEOUT, and marks the previous record consumed), so
 * that `stream` holds nothing between the steps' kernels and they overlap
 * through the dependent launch; NVFP4 caches use events.  All steps of a
 * cache go on the same `stream`.  Synchronise `stream` before reading
 * host_out; host_in too must stay unchanged until then (its copy runs
 * asynchronously).  One thread at a time per cache.  block_table stays in
 * device memory.  Host buffers
 * that are not page-locked (cudaHostAlloc / cudaHostRegister) return
 * KVQ_ERR_INVALID_ARG, as do the cases kvq_decode_step rejects. */
kvq_status kvq_decode_step_host(kvq_cache *cache, const void *host_in, void *dev_rec, const int32_t *block_table,
                                int32_t max_pages_per_seq, int32_t batch, float softmax_scale, void *workspace,
                                size_t ws_bytes, void *host_out, void *stream);

/* Decode attention that allocates nothing and takes no workspace, for
 * callers that cannot allocate device memory: an engine that reserves all of
 * the GPU's memory up front for its own pools (so any later cudaMalloc fails
 * or would steal from the KV pool), or code that must not allocate once it is
 * serving (allocation can block and synchronise the device).  The pages have
 * no counterpart of this call; it exists for such integrations.
 *
 * Same arguments and result as kvq_decode_attn without the workspace and
 * certified-mode arguments.  The workspace is a 4 MiB array in the library's
 * own device memory (one per GPU that loads the library, held until process
 * exit); a call whose kvq_decode_workspace_bytes(cache, batch,
 * max_pages_per_seq) exceeds 4 MiB returns KVQ_ERR_CAPACITY and launches
 * nothing.  The cache's device must be current.  The first call on a device
 * looks up the array's device address (cudaGetSymbolAddress), so make that
 * first call before any stream capture.  Each call clears the array's split
 * counters on `stream` (cudaMemsetAsync) and then launches the decode; every
 * call shares the one array and it keeps the last call's contents, so calls
 * that can overlap on the GPU (different streams, or concurrent host threads)
 * race on it and must be serialised by the caller. */
kvq_status kvq_decode_attn_static(kvq_cache *cache, const void *q, const int32_t *block_table,
                                  int32_t max_pages_per_seq, const int32_t *ctx_lens, int32_t batch,
                                  float softmax_scale, void *out, void *stream);

/* Read back n stored rows (slots[0..n), int32 device) per kv head:
 *   k_out, v_out: fp32 [n][Hkv][d] rotated-domain dequantised values
 *                 (code*scale + zero, one rounding), may be NULL;
 *   codes_out:    uint8 [n][Hkv][2][d] codes in channel order (K then V;
 *                 int8 as two's complement), may be NULL;
 *   meta_out:     uint16 [n][Hkv][2][8] fp16 scales in [0,4) and zeros in
 *                 [4,8) (unused entries 0), may be NULL. */
kvq_status kvq_dequant_debug(kvq_cache *cache, const int32_t *slots, int32_t n, float *k_out, float *v_out,
                             uint8_t *codes_out, uint16_t *meta_out, void *stream);

/* Test hooks of the decode kernels that kvq_decode_attn and kvq_decode_step
 * launch (the pages have no counterpart of them).  They let a test drive
 * paths that otherwise need a copy that never completes or a block table
 * changed by the previous kernel, without hanging or faulting the GPU.
 *   on = 1: each warp's first page wait counts as expired: the warp records
 *           KVQ_ERR_TIMEOUT in the status word, waits (bounded, the normal
 *           one-second limit) for the page copies it has already started,
 *           and attends no page, so the output is not the attention;
 *   on = 2: the page copies a warp starts from the block-table entries it
 *           read before the previous kernel finished count as wrong guesses:
 *           it waits them out and copies those pages again (the output is
 *           the attention);
 *   on = 0: normal operation.
 * Returns KVQ_ERR_INVALID_ARG for a null cache or on outside {0, 1, 2}. */
kvq_status kvq_debug_expire_first_wait(kvq_cache *cache, int32_t on);

/* Synchronise the cache's last stream use and return (then clear) the device
 * status word: KVQ_OK, KVQ_ERR_OUT_OF_RANGE or KVQ_ERR_TIMEOUT. */
kvq_status kvq_sync_status(kvq_cache *cache);

/* Static description of a status code. */
const char *kvq_status_string(kvq_status status);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
