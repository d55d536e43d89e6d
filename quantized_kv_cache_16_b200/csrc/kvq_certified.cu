// kvq_certified.cu -- the certified decode mode ["Runtime-Certified
// Bounded-Error Quantized Attention", Methodology 1-3].
//
// The quantised decode kernel runs first and, besides its output, records
// for every page and query head the pair (m, l): its running max and the sum
// of 2^(s - m) over the page's tokens (log2 units).  Then:
//
//   blocks  (one thread per page and query head, many CTAs) and
//   select  (one CTA per sequence and kv head) per query head, from the
//           totals M, L of the quantised softmax (written by the decode
//           kernel's final merge): the mass P_b of every bound block,
//           and with the block descriptors (eps: max key error, eta: max
//           value error, nu: max |value|, all in the rotated domain)
//             Delta_b = scale * ||q_r||_1 * eps_b
//             A       = ln sum_b P_b e^(Delta_b)
//             bound_b = P_b * ((e^(Delta_b + A) - 1) * nu_b + eta_b);
//           a block's score is the largest bound over the group's heads; the
//           top ceil(frac * n_blocks) blocks (ties: lower block first) are
//           promoted.  The pages give the key term as a total-variation bound
//           on the softmax shift and the value term as the mass-weighted
//           value error, without a formula; this is the rigorous reading.
//   promote (up to kCertChunks CTAs per sequence and kv head) reads the
//           promoted blocks' exact fp16 rows from tier 2 (pinned host memory
//           mapped into the device's address space), rotates them, and forms
//           two partials per head over those tokens: with the exact rows and
//           with the dequantised rows.  The last CTA replaces the quantised
//           contribution of the promoted blocks by the exact one:
//             o = (L 2^(M-R) o_q + R^T(acc_e 2^(m_e-R) - acc_q 2^(m_q-R)))
//                 / (L 2^(M-R) + l_e 2^(m_e-R) - l_q 2^(m_q-R)).
#include <math.h>

#include "kvq_cert.cuh"

namespace kvq {
namespace {

using namespace cert;

constexpr int kBlkThreads = 256;  // pages per CTA of the blocks kernel

// Pass 1, one thread per (page, query head), pages of a bound block in
// consecutive lanes: the page's softmax mass l 2^(m - M) / L and its
// descriptor, reduced over the block's ppb lanes (ppb a power of two <= 32);
// the block's first lane stores the head's mass (head 0 also the block's
// descriptors) and P_b e^(Delta_b); the CTA's sum of those goes to spart.
template <int D>
__global__ void __launch_bounds__(kBlkThreads) cert_blocks_kernel(const __grid_constant__ CertParams p)
{
    pdl_enter();
    constexpr int E = D / 32;
    const Layout &L = p.L;
    const int chunk = blockIdx.x, b = blockIdx.z;
    const int g = L.g, kvh = blockIdx.y / g, h = blockIdx.y - kvh * g;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    __shared__ float dq_s;
    __shared__ float red[kBlkThreads / 32];

    const int T = clamp_ctx(p.ctx_lens[b], p.max_pages);
    const int n_pages = (T + kPageTokens - 1) / kPageTokens;
    if (chunk * kBlkThreads >= n_pages) return;  // the whole CTA lies past the context
    const int ppb = L.bound_block / kPageTokens;
    const long long bk = (long long)b * L.hkv + kvh;
    if (warp == 0) {  // scale * ||q_r||_1 of this head: Delta_b = dq * eps_b
        float x[E];
        rotated_query<D>(p, b, kvh * g + h, lane, x);
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < E; e++) a += fabsf(x[e]);
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) a += __shfl_xor_sync(kFull, a, m);
        if (lane == 0) {
            dq_s = p.scale * a;
            if (chunk == 0) p.dq[bk * g + h] = p.scale * a;
        }
    }
    const int pi = chunk * kBlkThreads + tid;
    const float2 ml = p.head_ml[bk * g + h];
    float P = 0.f, eps = 0.f, eta = 0.f, nu = 0.f;
    if (pi < n_pages) {
        const int pg = p.block_table[(long long)b * p.max_pages + pi];
        const float2 s = p.page_stats[(bk * p.max_pages + pi) * g + h];
        if (pg >= 0 && pg < L.num_pages) {  // others were recorded by the decode kernel
            const float4 dsc =
                *reinterpret_cast<const float4 *>(p.pool + L.desc_off + ((long long)pg * L.hkv + kvh) * 16);
            eps = dsc.x;
            eta = dsc.y;
            nu = dsc.z;
        }
        if (s.y > 0.f && ml.y > 0.f) P = s.y * ex2(s.x - ml.x) / ml.y;
    }
    for (int m = 1; m < ppb; m <<= 1) {  // uniform trip count
        P += __shfl_xor_sync(kFull, P, m);
        eps = fmaxf(eps, __shfl_xor_sync(kFull, eps, m));
        eta = fmaxf(eta, __shfl_xor_sync(kFull, eta, m));
        nu = fmaxf(nu, __shfl_xor_sync(kFull, nu, m));
    }
    __syncthreads();  // dq_s
    float contrib = 0.f;
    if (pi < n_pages && (pi & (ppb - 1)) == 0) {
        float *rec = p.blk + (bk * p.sort_cap + pi / ppb) * kBlkRec;
        rec[h] = P;
        if (h == 0) {
            rec[8] = eps;
            rec[9] = eta;
            rec[10] = nu;
        }
        contrib = P * expf(dq_s * eps);
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) contrib += __shfl_xor_sync(kFull, contrib, m);
    if (lane == 0) red[warp] = contrib;
    __syncthreads();
    if (tid == 0) {
        float sum = 0.f;
        for (int w = 0; w < kBlkThreads / 32; w++) sum += red[w];
        p.spart[(bk * g + h) * p.n_chunk_cap + chunk] = sum;
    }
}

template <int D>
__global__ void __launch_bounds__(kSelThreads) cert_select_kernel(const __grid_constant__ CertParams p)
{
    pdl_enter();
    const Layout &L = p.L;
    const int kvh = blockIdx.x, b = blockIdx.y;
    const int tid = threadIdx.x;
    const int g = L.g;
    extern __shared__ unsigned long long keys[];
    __shared__ float dq[kMaxGqa];  // scale * ||q_r||_1: Delta_b = dq * eps_b
    __shared__ float A[kMaxGqa];

    const int T = clamp_ctx(p.ctx_lens[b], p.max_pages);
    const int n_pages = (T + kPageTokens - 1) / kPageTokens;
    const int block = L.bound_block;
    const int nb = (T + block - 1) / block;
    const long long bk = (long long)b * L.hkv + kvh;

    // A = ln sum_b P_b e^(Delta_b) per head: the blocks kernel's chunk sums,
    // added in a fixed order
    // (warp h: lanes over the chunks, then a fixed-order tree)
    const int n_chunks = (n_pages + kBlkThreads - 1) / kBlkThreads;
    {
        const int warp = tid >> 5, lane = tid & 31;
        if (warp < g) {
            const float *sp = p.spart + (bk * g + warp) * p.n_chunk_cap;
            float sum = 0.f;
            for (int ch = lane; ch < n_chunks; ch += 32) sum += sp[ch];
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) sum += __shfl_xor_sync(kFull, sum, m);
            if (lane == 0) {
                A[warp] = sum > 0.f ? logf(sum) : 0.f;
                dq[warp] = nb > 0 ? p.dq[bk * g + warp] : 0.f;
            }
        }
    }
    __syncthreads();
    const float *blk = p.blk + bk * (long long)p.sort_cap * kBlkRec;

    // pass 2, one thread per block: score -> sort key (score bits, then the
    // complement of the index so that equal scores order the lower block first)
    int np2 = 1;
    while (np2 < nb) np2 <<= 1;
    for (int bb = tid; bb < np2; bb += kSelThreads) {
        unsigned long long key = 0ull;
        if (bb < nb) {
            const float *rec = blk + (long long)bb * kBlkRec;
            const float4 p0 = *reinterpret_cast<const float4 *>(rec), p1 = *reinterpret_cast<const float4 *>(rec + 4);
            const float4 d = *reinterpret_cast<const float4 *>(rec + 8);
            const float P[kMaxGqa] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
            float sc = 0.f;
#pragma unroll
            for (int h = 0; h < kMaxGqa; h++)
                if (h < g && P[h] > 0.f) sc = fmaxf(sc, P[h] * fmaf(expm1f(fmaf(dq[h], d.x, A[h])), d.z, d.y));
            key = sort_key(sc, bb);
        }
        keys[bb] = key;
    }
    sort_keys_desc<kSelThreads>(keys, np2, tid);

    // the top ceil(frac * nb) blocks (fp64, guarded so an exact product is not bumped up)
    int kp = 0;
    if (p.frac > 0.f && nb > 0) {
        kp = (int)ceil((double)p.frac * (double)nb - 1e-9);
        kp = kp < 0 ? 0 : (kp > nb ? nb : kp);
    }
    int32_t *prom = p.prom + bk * p.sort_cap;
    for (int r = tid; r < kp; r += kSelThreads) prom[r] = key_index(keys[r]) | kPromKey | kPromVal;
    if (p.promoted_out)
        for (int r = tid; r < p.kmax_out; r += kSelThreads)
            p.promoted_out[bk * p.kmax_out + r] = r < kp ? key_index(keys[r]) : -1;
    if (tid == 0) p.prom_count[bk] = kp;
}

// Recomputation of the promoted blocks, up to n_chunks CTAs per (sequence,
// kv head), G >= the GQA group (a power of two).  Exact rows stay in the
// original domain: an exact key's score is q.k there (equal to (Rq).(Rk),
// R orthogonal) and exact values are summed unrotated; only the dequantised
// rows live in the rotated domain.
// WIN: the exact tokens are a sequence's sink and recent windows instead of
// promoted blocks; their fp16 rows come from the compact window store (row
// t for t < sink, row sink + t % recent for a recent token), and each CTA
// takes a contiguous share of the window tokens.  The quantised pass left
// those tokens out, so there is no quantised side to take away: the merge
// adds the exact partial to the quantised one (a plain log-sum-exp merge;
// the quantised side's mass is 0).
template <int D, int G, bool WIN>
__global__ void __launch_bounds__(kPromThreads, WIN ? 2 : 1) cert_promote_kernel(const __grid_constant__ CertParams p)
{
    pdl_enter();
    constexpr int E = D / 32;
    const Layout &L = p.L;
    const int chunk_id = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = L.g;
    const long long bk = (long long)b * L.hkv + kvh;
    const int T = clamp_ctx(p.ctx_lens[b], p.max_pages);
    // window tokens: [0, ns) and [lo_r, T), nwin in all, `per` a CTA
    int kp, ns = 0, lo_r = 0, nwin = 0, per = 0;
    if constexpr (WIN) {
        ns = min(p.sink, T);
        lo_r = p.recent > 0 ? max(p.sink, T - p.recent) : T;
        lo_r = min(lo_r, T);
        nwin = ns + (T - lo_r);
        constexpr int span = kPromWarps * kTokBatch;
        kp = min(p.n_chunks, (nwin + span - 1) / span);
        per = kp > 0 ? (nwin + kp - 1) / kp : 0;
    } else {
        kp = p.prom_count[bk];
    }
    const int n_act = min(kp, p.n_chunks);
    if (chunk_id >= n_act) return;

    extern __shared__ float wacc[];  // [kPromWarps][g][3][D]
    __shared__ float sq[G * kMaxD], so[G * kMaxD];
    __shared__ float wm[kPromWarps * G * 2], wl[kPromWarps * G * 2];
    // per warp and head, (m, l) of a key-promoted block's exact scores over
    // the warp's share of its tokens (the ladder's ranking check); two
    // buffers, a barrier every block
    __shared__ float2 bsm[2][kPromWarps][G];
    __shared__ int sflag;

    const int block = L.bound_block;
    const int32_t *bt = p.block_table + (long long)b * p.max_pages;
    const int32_t *prom = WIN ? nullptr : p.prom + bk * p.sort_cap;

    // queries in log2 units: rotated (against dequantised keys) and original
    // (against exact keys)
    if (warp < g) {
        float x[E];
        rotated_query<D>(p, b, kvh * g + warp, lane, x);
        const __half *qh = p.q + ((long long)b * L.hq + kvh * g + warp) * D + lane * E;
#pragma unroll
        for (int e = 0; e < E; e++) {
            sq[warp * D + lane * E + e] = x[e] * p.qscale;
            so[warp * D + lane * E + e] = __half2float(qh[e]) * p.qscale;
        }
    }
    __syncthreads();
    float qr[G][E];  // the original-domain query stays in shared memory (one vector load per use)
#pragma unroll
    for (int h = 0; h < G; h++)
#pragma unroll
        for (int e = 0; e < E; e++) qr[h][e] = h < g ? sq[h * D + lane * E + e] : 0.f;

    // partials over this CTA's promoted tokens: [0] the mixed softmax (exact
    // keys and values where promoted), [1] the quantised one.  The mixed
    // side sums exact values (original domain, ae) and dequantised ones
    // (rotated domain, ar) apart; aq is the quantised side's sum.
    float m[G][2], l[G][2], ae[G][E], ar[G][E], aq[G][E];
#pragma unroll
    for (int h = 0; h < G; h++) {
#pragma unroll
        for (int w = 0; w < 2; w++) {
            m[h][w] = -INFINITY;
            l[h][w] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < E; e++) ae[h][e] = ar[h][e] = aq[h][e] = 0.f;
    }

    int parity = 0;
    for (int r = chunk_id; r < kp; r += n_act, parity ^= 1) {
        // this segment: positions (WIN: window indices) [t0, t1)
        int blk_id = 0, t0, t1;
        bool kx = true, vx = true;
        if constexpr (WIN) {
            t0 = r * per;
            t1 = min(nwin, t0 + per);
        } else {
            const int ent = prom[r];
            blk_id = ent & kPromIdx;
            kx = (ent & kPromKey) != 0;
            vx = (ent & kPromVal) != 0;
            t0 = blk_id * block;
            t1 = min(t0 + block, T);
        }
        float bm[G], bl[G];
#pragma unroll
        for (int h = 0; h < G; h++) {
            bm[h] = -INFINITY;
            bl[h] = 0.f;
        }
        for (int tb = t0 + warp * kTokBatch; tb < t1; tb += kPromWarps * kTokBatch) {
            // issue the batch's exact-row loads (host link) before any math
            RawRow<E> kraw[kTokBatch], vraw[kTokBatch];
            int pgs[kTokBatch], toks[kTokBatch];
#pragma unroll
            for (int u = 0; u < kTokBatch; u++) {
                int t = -1, pg = -1;
                if (tb + u < t1) {
                    t = tb + u;
                    if constexpr (WIN) t = t < ns ? t : lo_r + (t - ns);
                    pg = bt[t / kPageTokens];
                    if (pg >= L.num_pages) pg = -1;
                }
                pgs[u] = pg;
                toks[u] = t % kPageTokens;
                if (pg >= 0) {
                    long long row;
                    if constexpr (WIN) {
                        const int wrow = t < p.sink ? t : p.sink + t % p.recent;
                        row = (((long long)b * (p.sink + p.recent) + wrow) * L.hkv + kvh) * D + lane * E;
                    } else {
                        row = ((long long)(pg * kPageTokens + t % kPageTokens) * L.hkv + kvh) * D + lane * E;
                    }
                    if (kx) kraw[u].load(p.k2 + row);
                    if (vx) vraw[u].load(p.v2 + row);
                }
            }
            unsigned vmask = 0;  // tokens of the batch that are there
#pragma unroll
            for (int u = 0; u < kTokBatch; u++) vmask |= (pgs[u] >= 0 ? 1u : 0u) << u;
            static_assert(kTokBatch == 8, "a batch of 8 tokens x 4 heads fills one transpose-reduce");
            // heads in groups of four (a group past g holds zeros); lane j of
            // a reduction holds token j >> 2, head 4 hg + (j & 3)
            constexpr int NHG = G > 4 ? G / 4 : 1;
            const int uj = lane >> 2, hlj = lane & 3;
#pragma unroll
            for (int hg = 0; hg < NHG; hg++) {
                // 1. partial dot products, index u * 4 + head: [0] the mixed
                // side (exact keys where promoted), [1] the quantised side
                float d0[32], d1[32];
#pragma unroll
                for (int i = 0; i < 32; i++) d0[i] = d1[i] = 0.f;
#pragma unroll
                for (int u = 0; u < kTokBatch; u++) {
                    if (!((vmask >> u) & 1u)) continue;  // warp-uniform
                    float ke[E] = {}, kq[E] = {};
                    if (kx) kraw[u].widen(ke);
                    if constexpr (!WIN) {
                        const unsigned char *chunk =
                            p.pool + kHeaderBytes + (long long)pgs[u] * L.page_bytes + (long long)kvh * L.chunk_bytes;
                        dequant_lane<E>(chunk, L.k_codes, L.k_meta, L.k_row_meta, L.k_fmt, toks[u], lane, kq);
                    }
#pragma unroll
                    for (int hl = 0; hl < 4; hl++) {
                        const int h = hg * 4 + hl;
                        if (h >= g) break;
                        float qo[E];
                        if constexpr (E == 4) {
                            const float4 v4 = *reinterpret_cast<const float4 *>(so + h * D + lane * E);
                            qo[0] = v4.x;
                            qo[E > 1 ? 1 : 0] = v4.y;
                            qo[E > 2 ? 2 : 0] = v4.z;
                            qo[E > 3 ? 3 : 0] = v4.w;
                        } else {
#pragma unroll
                            for (int e = 0; e < E; e++) qo[e] = so[h * D + lane * E + e];
                        }
                        float a0 = 0.f, a1 = 0.f;
#pragma unroll
                        for (int e = 0; e < E; e++) {
                            a0 = fmaf(qo[e], ke[e], a0);
                            if constexpr (!WIN) a1 = fmaf(qr[h][e], kq[e], a1);
                        }
                        d0[u * 4 + hl] = a0;
                        d1[u * 4 + hl] = a1;
                    }
                }
                // 2. the totals, one (token, head) per lane
                const bool live = ((vmask >> uj) & 1u) && hg * 4 + hlj < g;
                float s1 = -INFINITY;
                if constexpr (!WIN) {
                    s1 = transpose_reduce32(d1, lane);
                    if (!live) s1 = -INFINITY;
                }
                float s0 = s1;
                if (kx) {
                    s0 = transpose_reduce32(d0, lane);
                    if (!live) s0 = -INFINITY;
                }
                // 3. per side and head: the batch max, the weights relative to
                // the new running max, the batch sum; then rescale (m, l, sums)
                float pw[2] = {0.f, 0.f};
#pragma unroll
                for (int w = 0; w < 2; w++) {
                    if (WIN && w == 1) break;
                    const float sw = w ? s1 : s0;
                    float bmax = sw;
#pragma unroll
                    for (int o = 4; o < 32; o <<= 1) bmax = fmaxf(bmax, __shfl_xor_sync(kFull, bmax, o));
                    float mo = m[hg * 4][w];
#pragma unroll
                    for (int k = 1; k < 4; k++)
                        if (hg * 4 + k < G && hlj == k) mo = m[hg * 4 + k][w];
                    const float mnew = fmaxf(mo, bmax);
                    const float pj = sw == -INFINITY ? 0.f : ex2(sw - mnew);
                    float psum = pj;
#pragma unroll
                    for (int o = 4; o < 32; o <<= 1) psum += __shfl_xor_sync(kFull, psum, o);
                    pw[w] = pj;
#pragma unroll
                    for (int k = 0; k < 4; k++) {  // lane k holds head 4 hg + k's figures
                        const int h = hg * 4 + k;
                        if (h >= g) break;
                        const float mn = __shfl_sync(kFull, mnew, k), ps = __shfl_sync(kFull, psum, k);
                        const float al = m[h][w] == -INFINITY ? 0.f : ex2(m[h][w] - mn);
                        l[h][w] = fmaf(l[h][w], al, ps);
#pragma unroll
                        for (int e = 0; e < E; e++) {
                            if (w == 0) {
                                ae[h][e] *= al;
                                ar[h][e] *= al;
                            } else {
                                aq[h][e] *= al;
                            }
                        }
                        if (p.ladder && kx && w == 0) {  // the block's own (max, sum) for the check
                            const float bmx = __shfl_sync(kFull, bmax, k);
                            if (bmx != -INFINITY) {
                                const float nbm = fmaxf(bm[h], bmx);
                                bl[h] = fmaf(bl[h], ex2(bm[h] - nbm), ps * ex2(mn - nbm));
                                bm[h] = nbm;
                            }
                        }
                        m[h][w] = mn;
                    }
                }
                // 4. values: every lane takes each (token, head) weight in turn
#pragma unroll
                for (int u = 0; u < kTokBatch; u++) {
                    if (!((vmask >> u) & 1u)) continue;  // warp-uniform
                    float ve[E] = {}, vq[E] = {};
                    if (vx) vraw[u].widen(ve);
                    if (!WIN || !vx) {
                        const unsigned char *chunk =
                            p.pool + kHeaderBytes + (long long)pgs[u] * L.page_bytes + (long long)kvh * L.chunk_bytes;
                        dequant_lane<E>(chunk, L.v_codes, L.v_meta, L.v_row_meta, L.v_fmt, toks[u], lane, vq);
                    }
#pragma unroll
                    for (int hl = 0; hl < 4; hl++) {
                        const int h = hg * 4 + hl;
                        if (h >= g) break;
                        const float w0 = __shfl_sync(kFull, pw[0], u * 4 + hl);
#pragma unroll
                        for (int e = 0; e < E; e++) {
                            if (vx) ae[h][e] = fmaf(w0, ve[e], ae[h][e]);
                            else ar[h][e] = fmaf(w0, vq[e], ar[h][e]);
                        }
                        if constexpr (!WIN) {
                            const float w1 = __shfl_sync(kFull, pw[1], u * 4 + hl);
#pragma unroll
                            for (int e = 0; e < E; e++) aq[h][e] = fmaf(w1, vq[e], aq[h][e]);
                        }
                    }
                }
            }
        }
        if (p.ladder) {  // CTA-uniform
            if (kx && lane == 0)
#pragma unroll
                for (int h = 0; h < G; h++)
                    if (h < g) bsm[parity][warp][h] = make_float2(bm[h], bl[h]);
            __syncthreads();
            if (kx && warp == 0 && lane < g) {
                float M = -INFINITY, Ls = 0.f;
#pragma unroll
                for (int w = 0; w < kPromWarps; w++) M = fmaxf(M, bsm[parity][w][lane].x);
#pragma unroll
                for (int w = 0; w < kPromWarps; w++) {
                    const float2 v = bsm[parity][w][lane];
                    if (v.x != -INFINITY) Ls = fmaf(v.y, ex2(v.x - M), Ls);
                }
                p.bml[((long long)bk * p.sort_cap + blk_id) * g + lane] = make_float2(M, Ls);
            }
        }
    }

    // warps -> shared memory -> one partial per head: rows ae, ar, aq, then
    // (m, l) of the mixed and of the quantised side
#pragma unroll
    for (int h = 0; h < G; h++)
        if (h < g) {
#pragma unroll
            for (int e = 0; e < E; e++) {
                wacc[((warp * g + h) * 3 + 0) * D + lane * E + e] = ae[h][e];
                wacc[((warp * g + h) * 3 + 1) * D + lane * E + e] = ar[h][e];
                wacc[((warp * g + h) * 3 + 2) * D + lane * E + e] = aq[h][e];
            }
            if (lane == 0)
#pragma unroll
                for (int w = 0; w < 2; w++) {
                    wm[(warp * G + h) * 2 + w] = m[h][w];
                    wl[(warp * G + h) * 2 + w] = l[h][w];
                }
        }
    __syncthreads();
    constexpr int REC = 3 * D + 4;
    float *cp = p.cpart + (bk * p.n_chunks + chunk_id) * (long long)g * REC;
    for (int idx = tid; idx < g * 3 * D; idx += kPromThreads) {
        const int h = idx / (3 * D), rem = idx - h * 3 * D;
        const int row = rem / D, ch = rem - row * D;
        const int w = row == 2 ? 1 : 0;  // rows 0, 1: the mixed side; row 2: the quantised side
        float M = -INFINITY;
#pragma unroll
        for (int ww = 0; ww < kPromWarps; ww++) M = fmaxf(M, wm[(ww * G + h) * 2 + w]);
        float a = 0.f, Ls = 0.f;
        if (M != -INFINITY)
#pragma unroll
            for (int ww = 0; ww < kPromWarps; ww++) {
                const float mw = wm[(ww * G + h) * 2 + w];
                const float f = mw == -INFINITY ? 0.f : ex2(mw - M);
                a = fmaf(f, wacc[((ww * g + h) * 3 + row) * D + ch], a);
                Ls = fmaf(f, wl[(ww * G + h) * 2 + w], Ls);
            }
        cp[h * REC + row * D + ch] = a;
        if (ch == 0 && row != 1) {
            cp[h * REC + 3 * D + 2 * w] = M;
            cp[h * REC + 3 * D + 2 * w + 1] = Ls;
        }
    }

    // the last CTA of this (sequence, kv head) applies the correction
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(p.ccount + bk, 1u);
        sflag = prev == (unsigned)(n_act - 1);
    }
    __syncthreads();
    if (!sflag) return;
    __threadfence();
    if (tid == 0) p.ccount[bk] = 0u;
    const float *cbase = p.cpart + bk * p.n_chunks * (long long)g * REC;
    for (int h = warp; h < g; h += kPromWarps) {
        // lane c: (max, sum) of chunk c's two sides, loaded in parallel
        float Mx[2], Ls[2], fch[2];
#pragma unroll
        for (int w = 0; w < 2; w++) {
            float2 mlc = make_float2(-INFINITY, 0.f);
            if (lane < n_act) mlc = __ldcg(reinterpret_cast<const float2 *>(cbase + (lane * g + h) * REC + 3 * D + 2 * w));
            float M = mlc.x;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, o));
            Mx[w] = M;
            fch[w] = (mlc.x == -INFINITY || M == -INFINITY) ? 0.f : ex2(mlc.x - M);
            float lsum = fch[w] * mlc.y;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) lsum += __shfl_xor_sync(kFull, lsum, o);
            Ls[w] = lsum;
        }
        // the three sums over the chunks, one row at a time (loads unrolled)
        float a[3][E];
#pragma unroll
        for (int row = 0; row < 3; row++) {
            const int w = row == 2 ? 1 : 0;
            float rows[kCertChunks][E];
#pragma unroll
            for (int c = 0; c < kCertChunks; c++)
#pragma unroll
                for (int e = 0; e < E; e++)
                    rows[c][e] = c < n_act ? __ldcg(cbase + (c * g + h) * REC + row * D + lane * E + e) : 0.f;
#pragma unroll
            for (int e = 0; e < E; e++) a[row][e] = 0.f;
#pragma unroll
            for (int c = 0; c < kCertChunks; c++) {
                const float fc = __shfl_sync(kFull, fch[w], c);
#pragma unroll
                for (int e = 0; e < E; e++) a[row][e] = fmaf(fc, rows[c][e], a[row][e]);
            }
        }
        const float2 ml = p.head_ml[bk * g + h];  // the quantised pass: (M, L)
        float R = fmaxf(Mx[0], Mx[1]);
        if (ml.y > 0.f) R = fmaxf(R, ml.x);
        const float f0 = ml.y > 0.f ? ml.y * ex2(ml.x - R) : 0.f;
        const float fe = Mx[0] == -INFINITY ? 0.f : ex2(Mx[0] - R);
        const float fq = Mx[1] == -INFINITY ? 0.f : ex2(Mx[1] - R);
        const float den = f0 + Ls[0] * fe - Ls[1] * fq;
        if (p.ladder && lane == 0) p.mix[bk * g + h] = make_float2(R, den);
        // dequantised sums (rotated domain) back to the original domain
        float dlt[E];
#pragma unroll
        for (int e = 0; e < E; e++) dlt[e] = a[1][e] * fe - a[2][e] * fq;
        if (p.rotate) {
            if (p.rotate == 2) warp_bitrev<D>(dlt, lane);  // undo P_br first
            fwht_warp<D>(dlt, lane);
#pragma unroll
            for (int e = 0; e < E; e++) dlt[e] *= p.rot_scale * p.signs[lane * E + e];
        }
        float *o = p.out + ((long long)b * L.hq + kvh * g + h) * D + lane * E;
#pragma unroll
        for (int e = 0; e < E; e++) o[e] = den > 0.f ? (f0 * o[e] + a[0][e] * fe + dlt[e]) / den : 0.f;
    }
}

}  // namespace

cudaError_t launch_cert_blocks(const CertParams &p, int batch, cudaStream_t s)
{
    const dim3 bgrid(p.n_chunk_cap, p.L.hkv * p.L.g, batch);
    return p.L.d == 128 ? launch_pdl(cert_blocks_kernel<128>, bgrid, kBlkThreads, 0, s, p)
                        : launch_pdl(cert_blocks_kernel<64>, bgrid, kBlkThreads, 0, s, p);
}

cudaError_t launch_cert_select(const CertParams &p, int batch, cudaStream_t s)
{
    static DeviceOnce once[2];
    const int di = p.L.d == 64 ? 0 : 1;
    const size_t smem = (size_t)p.sort_cap * sizeof(unsigned long long);
    if (once[di].needed()) {
        const cudaError_t e =
            di ? cudaFuncSetAttribute(cert_select_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      kCertMaxBlocks * (int)sizeof(unsigned long long))
               : cudaFuncSetAttribute(cert_select_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      kCertMaxBlocks * (int)sizeof(unsigned long long));
        if (e != cudaSuccess) return e;
        once[di].mark();
    }
    const dim3 grid(p.L.hkv, batch);
    return di ? launch_pdl(cert_select_kernel<128>, grid, kSelThreads, smem, s, p)
              : launch_pdl(cert_select_kernel<64>, grid, kSelThreads, smem, s, p);
}

template <int D, int G, bool WIN>
cudaError_t launch_promote_t(const CertParams &p, int batch, cudaStream_t s)
{
    static DeviceOnce once;
    if (once.needed()) {
        const int cap = kPromWarps * G * 3 * D * (int)sizeof(float);
        const cudaError_t e =
            cudaFuncSetAttribute(cert_promote_kernel<D, G, WIN>, cudaFuncAttributeMaxDynamicSharedMemorySize, cap);
        if (e != cudaSuccess) return e;
        once.mark();
    }
    const size_t smem = (size_t)kPromWarps * p.L.g * 3 * D * sizeof(float);
    const dim3 grid(p.n_chunks, p.L.hkv, batch);
    return launch_pdl(cert_promote_kernel<D, G, WIN>, grid, kPromThreads, smem, s, p);
}

template <int D, bool WIN>
cudaError_t launch_promote_d(const CertParams &p, int batch, cudaStream_t s)
{
    const int g = p.L.g;
    if (g <= 1) return launch_promote_t<D, 1, WIN>(p, batch, s);
    if (g <= 2) return launch_promote_t<D, 2, WIN>(p, batch, s);
    if (g <= 4) return launch_promote_t<D, 4, WIN>(p, batch, s);
    return launch_promote_t<D, 8, WIN>(p, batch, s);
}

cudaError_t launch_cert_promote(const CertParams &p, int batch, cudaStream_t s)
{
    return p.L.d == 128 ? launch_promote_d<128, false>(p, batch, s) : launch_promote_d<64, false>(p, batch, s);
}

cudaError_t launch_windows(const CertParams &p, int batch, cudaStream_t s)
{
    return p.L.d == 128 ? launch_promote_d<128, true>(p, batch, s) : launch_promote_d<64, true>(p, batch, s);
}

}  // namespace kvq
