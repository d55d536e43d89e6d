// kvq_ladder.cu -- the adaptive ladder of the certified decode
// ["Runtime-Certified Bounded-Error Quantized Attention", Methodology 3:
// adaptive Top-K, ranking-consistency check, four-rung fallback ladder].
//
// Launch order on the stream (all programmatic dependents):
//   decode (page statistics) -> cert_blocks (block masses and descriptors)
//   -> ladder_select -> cert_promote -> ladder_finish -> ladder_dense.
//
//   select  (one CTA per sequence and kv head) ranks the blocks by
//           r(b) = max_h Phat_h(b), the group's largest estimated mass (ties:
//           lower block first), and from CTA-wide scans over that order
//           finds K_cov, the fewest leading blocks whose mass reaches tau_cov
//           for every head, and K_key (rung 1), the fewest whose exact keys
//           bring every head's predicted key term
//             E(K) = expm1(A) sum_b Phat nu + e^A sum_{i>=K} Phat nu expm1(Delta)
//             A    = log1p((sum_b Phat - 1) + sum_{i>=K} Phat expm1(Delta))
//           to key_tol.  K* = min(budget, max(K_cov, K_key)) leading blocks
//           get exact keys; blocks with max_h Phat_h(b) eta_b > v_tol get
//           exact values (rung 2).  The promote kernel recomputes those blocks.
//   finish  (one CTA per sequence and kv head) forms, per head, the masses
//           P' of the mixed softmax (exact scores in key-promoted blocks) and
//           the certified bound of the mixed output
//             bound = (expm1(A') S_nu + e^A' S_nu,D + S_eta) / S_P,
//             A' = log1p(S_D / S_P)
//           (sums over blocks of P', P' expm1(D), P' nu, P' nu expm1(D) and,
//           over blocks with quantised values, P' eta; D = 0 in key-promoted
//           blocks, Delta elsewhere), and runs the ranking-consistency check:
//           the key-promoted blocks sorted by Phat_h fail when a block placed
//           lower has an exact mass above (1 + rank_tol) times that of one
//           placed higher.  A failed check or a bound above cert_tol sends the
//           head to the fp16 fallback (rung 3) and counts it.
//   dense   recomputes fp16 attention over the tier-2 rows for those heads,
//           or for every head when more than layer_thresh heads fell back
//           (rung 4), split over the context with a last-CTA merge.
#include <math.h>

#include "kvq_cert.cuh"

namespace kvq {
namespace {

using namespace cert;

constexpr int kNoK = 0x7fffffff;

template <int D>
__global__ void __launch_bounds__(kSelThreads) ladder_select_kernel(const __grid_constant__ CertParams p)
{
    pdl_enter();
    const Layout &L = p.L;
    const int kvh = blockIdx.x, b = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = L.g;
    extern __shared__ unsigned long long keys[];  // [sort_cap], then flags [sort_cap] bytes
    unsigned char *fl = reinterpret_cast<unsigned char *>(keys + p.sort_cap);
    __shared__ float dqs[kMaxGqa];
    __shared__ float scan_sm[(kSelThreads / 32) * 2 * kMaxGqa];
    __shared__ int kcov_s, kkey_s, nval_s;
    __shared__ int wcnt[kSelThreads / 32];

    if (blockIdx.x == 0 && blockIdx.y == 0 && tid == 0) *p.nfall = 0u;  // this call's fallback count
    const int T = clamp_ctx(p.ctx_lens[b], p.max_pages);
    const int nb = (T + L.bound_block - 1) / L.bound_block;
    const long long bk = (long long)b * L.hkv + kvh;
    if (tid < kMaxGqa) dqs[tid] = (tid < g && nb > 0) ? p.dq[bk * g + tid] : 0.f;
    if (tid == 0) {
        kcov_s = kNoK;
        kkey_s = kNoK;
        nval_s = 0;
    }
    const float *blk = p.blk + bk * (long long)p.sort_cap * kBlkRec;

    // 1. ranking keys: the group's largest estimated mass
    int np2 = 1;
    while (np2 < nb) np2 <<= 1;
    for (int bb = tid; bb < np2; bb += kSelThreads) {
        unsigned long long key = 0ull;
        if (bb < nb) {
            const float *rec = blk + (long long)bb * kBlkRec;
            float r = 0.f;
            for (int h = 0; h < g; h++) r = fmaxf(r, rec[h]);
            key = sort_key(r, bb);
        }
        keys[bb] = key;
    }
    sort_keys_desc<kSelThreads>(keys, np2, tid);

    // 2. per-thread sums over a contiguous run of ranks [i0, i1)
    const int per = (nb + kSelThreads - 1) / kSelThreads;
    const int i0 = min(nb, tid * per), i1 = min(nb, i0 + per);
    // per head h: fw[2h], fw[2h+1] = Phat, Phat nu (prefix sums); rv[2h], rv[2h+1] =
    // Phat expm1(Delta), Phat nu expm1(Delta) (suffix sums)
    float fw[2 * kMaxGqa], rv[2 * kMaxGqa];
#pragma unroll
    for (int n = 0; n < 2 * kMaxGqa; n++) fw[n] = rv[n] = 0.f;
    for (int i = i0; i < i1; i++) {
        const float *rec = blk + (long long)key_index(keys[i]) * kBlkRec;
        const float eps = rec[8], nu = rec[10];
#pragma unroll
        for (int h = 0; h < kMaxGqa; h++) {
            if (h >= g) break;
            const float a = rec[h], dm = expm1f(dqs[h] * eps);
            fw[2 * h] += a;
            fw[2 * h + 1] += a * nu;
            rv[2 * h] += a * dm;
            rv[2 * h + 1] += a * nu * dm;
        }
    }
    float fw_tot[2 * kMaxGqa], rv_tot[2 * kMaxGqa], own[2 * kMaxGqa];
#pragma unroll
    for (int n = 0; n < 2 * kMaxGqa; n++) own[n] = rv[n];
    block_scan<kSelThreads, 2 * kMaxGqa, false, SumOp>(fw, fw_tot, scan_sm, tid, 2 * g);
    block_scan<kSelThreads, 2 * kMaxGqa, true, SumOp>(rv, rv_tot, scan_sm, tid, 2 * g);
    // fw: sums over ranks < i0; rv + own: sums over ranks >= i0

    // 3. walk K = i0+1 .. i1 (thread 0 also K = 0): the coverage and the
    // predicted key term with the first K ranked blocks' keys exact
    float C[kMaxGqa], sD[kMaxGqa], sND[kMaxGqa];
#pragma unroll
    for (int h = 0; h < kMaxGqa; h++) {
        C[h] = fw[2 * h];
        sD[h] = rv[2 * h] + own[2 * h];
        sND[h] = rv[2 * h + 1] + own[2 * h + 1];
    }
    int my_cov = kNoK, my_key = kNoK;
    auto eval = [&](int K) {
        bool cov_ok = true, key_ok = true;
#pragma unroll
        for (int h = 0; h < kMaxGqa; h++) {
            if (h >= g) break;
            cov_ok = cov_ok && C[h] >= p.tau_cov;
            const float A = log1pf((fw_tot[2 * h] - 1.f) + fmaxf(sD[h], 0.f));
            const float E = expm1f(A) * fw_tot[2 * h + 1] + expf(A) * fmaxf(sND[h], 0.f);
            key_ok = key_ok && E <= p.key_tol;
        }
        if (cov_ok && my_cov == kNoK) my_cov = K;
        if (key_ok && my_key == kNoK) my_key = K;
    };
    if (tid == 0) eval(0);
    for (int K = i0 + 1; K <= i1 && (my_cov == kNoK || my_key == kNoK); K++) {
        const float *rec = blk + (long long)key_index(keys[K - 1]) * kBlkRec;  // rank K-1 joins the prefix
        const float eps = rec[8], nu = rec[10];
#pragma unroll
        for (int h = 0; h < kMaxGqa; h++) {
            if (h >= g) break;
            const float a = rec[h], dm = expm1f(dqs[h] * eps);
            C[h] += a;
            sD[h] -= a * dm;
            sND[h] -= a * nu * dm;
        }
        eval(K);
    }
    if (my_cov != kNoK) atomicMin(&kcov_s, my_cov);
    if (my_key != kNoK) atomicMin(&kkey_s, my_key);
    for (int bb = tid; bb < nb; bb += kSelThreads) fl[bb] = 0;
    __syncthreads();

    // tau_cov >= 1 asks for all of the mass: every block, whatever the
    // rounded running sum of the estimated masses reaches first
    const int k_cov = p.tau_cov >= 1.f ? nb : p.tau_cov > 0.f ? (kcov_s == kNoK ? nb : kcov_s) : 0;
    const int k_key = kkey_s == kNoK ? nb : kkey_s;
    int k_cap = 0;
    if (p.frac > 0.f && nb > 0) {
        k_cap = (int)ceil((double)p.frac * (double)nb - 1e-9);
        k_cap = k_cap < 0 ? 0 : (k_cap > nb ? nb : k_cap);
    }
    const int want = max(k_cov, k_key);
    const int k_star = min(want, k_cap);

    // 4. flags: exact keys for the first K* ranked blocks, exact values
    // where the estimated value-error contribution exceeds v_tol
    for (int i = tid; i < k_star; i += kSelThreads) fl[key_index(keys[i])] = 1;
    __syncthreads();
    int any_val = 0;
    for (int bb = tid; bb < nb; bb += kSelThreads) {
        const float *rec = blk + (long long)bb * kBlkRec;
        float w = 0.f;
        for (int h = 0; h < g; h++) w = fmaxf(w, rec[h] * rec[9]);
        if (w > p.v_tol) {
            fl[bb] |= 2;
            any_val = 1;
        }
    }
    any_val = __syncthreads_or(any_val);

    // 5. the promotion list: the K* key blocks in rank order (with their value
    // flag), then the value-only blocks in block order
    int32_t *prom = p.prom + bk * p.sort_cap;
    for (int i = tid; i < k_star; i += kSelThreads) {
        const int bb = key_index(keys[i]);
        prom[i] = bb | kPromKey | ((fl[bb] & 2) ? kPromVal : 0);
    }
    for (int base = 0; base < nb; base += kSelThreads) {
        const int bb = base + tid;
        const bool take = bb < nb && fl[bb] == 2;
        const unsigned ballot = __ballot_sync(kFull, take);
        if (lane == 0) wcnt[warp] = __popc(ballot);
        __syncthreads();
        int before = nval_s;
        for (int w = 0; w < warp; w++) before += wcnt[w];
        if (take) prom[k_star + before + __popc(ballot & ((1u << lane) - 1u))] = bb | kPromVal;
        __syncthreads();
        if (tid == 0)
            for (int w = 0; w < kSelThreads / 32; w++) nval_s += wcnt[w];
        __syncthreads();
    }

    unsigned char *gfl = p.flags + bk * p.sort_cap;
    for (int bb = tid; bb < nb; bb += kSelThreads) gfl[bb] = fl[bb];
    if (p.flags_out)
        for (int bb = tid; bb < p.nb_out; bb += kSelThreads) p.flags_out[bk * p.nb_out + bb] = bb < nb ? fl[bb] : 0;
    if (tid == 0) {
        p.prom_count[bk] = k_star + nval_s;
        const int st = (k_star > k_cov ? kStExpanded : 0) | (want > k_cap ? kStCapped : 0) | (any_val ? kStValues : 0);
        p.gstat[bk] = st | (k_star << 16);
        if (p.k_star_out) p.k_star_out[bk] = k_star;
    }
}

template <int D>
__global__ void __launch_bounds__(kSelThreads) ladder_finish_kernel(const __grid_constant__ CertParams p)
{
    pdl_enter();
    const Layout &L = p.L;
    const int kvh = blockIdx.x, b = blockIdx.y;
    const int tid = threadIdx.x;
    const int g = L.g;
    extern __shared__ unsigned long long keys[];  // [sort_cap]
    __shared__ float Rs[kMaxGqa], dens[kMaxGqa], fq[kMaxGqa], dqs[kMaxGqa];
    __shared__ float scan_sm[(kSelThreads / 32) * 5 * kMaxGqa];
    __shared__ int fail_s[kMaxGqa];

    const int T = clamp_ctx(p.ctx_lens[b], p.max_pages);
    const int nb = (T + L.bound_block - 1) / L.bound_block;
    const long long bk = (long long)b * L.hkv + kvh;
    const int gs = p.gstat[bk], k_star = gs >> 16, cnt = p.prom_count[bk];
    if (tid < kMaxGqa) {
        float R = 0.f, den = 0.f, f = 0.f, dq = 0.f;
        if (tid < g && nb > 0) {
            const float2 ml = p.head_ml[bk * g + tid];  // quantised softmax (M, L), log2 units
            const float2 mx = cnt > 0 ? p.mix[bk * g + tid] : ml;  // mixed softmax (R, den)
            R = mx.x;
            den = mx.y;
            f = (ml.y > 0.f && mx.y > 0.f) ? ml.y * ex2(ml.x - mx.x) / mx.y : 0.f;
            dq = p.dq[bk * g + tid];
        }
        Rs[tid] = R;
        dens[tid] = den;
        fq[tid] = f;
        dqs[tid] = dq;
        fail_s[tid] = 0;
    }
    __syncthreads();

    // masses P' of the mixed softmax and the sums of the bound, per head
    const float *blk = p.blk + bk * (long long)p.sort_cap * kBlkRec;
    const unsigned char *gfl = p.flags + bk * p.sort_cap;
    const float2 *bml = p.bml + bk * (long long)p.sort_cap * g;
    float S[5 * kMaxGqa];  // per head h, S[5h..5h+4]: P', P' expm1(D), P' nu, P' nu expm1(D), P' eta (quantised values)
#pragma unroll
    for (int n = 0; n < 5 * kMaxGqa; n++) S[n] = 0.f;
    for (int bb = tid; bb < nb; bb += kSelThreads) {
        const float *rec = blk + (long long)bb * kBlkRec;
        const float eps = rec[8], eta = rec[9], nu = rec[10];
        const int f = gfl[bb];
#pragma unroll
        for (int h = 0; h < kMaxGqa; h++) {
            if (h >= g) break;
            float P, dm;
            if (f & 1) {
                const float2 v = bml[(long long)bb * g + h];
                P = dens[h] > 0.f ? v.y * ex2(v.x - Rs[h]) / dens[h] : 0.f;
                dm = 0.f;
            } else {
                P = rec[h] * fq[h];
                dm = expm1f(dqs[h] * eps);
            }
            S[5 * h] += P;
            S[5 * h + 1] += P * dm;
            S[5 * h + 2] += P * nu;
            S[5 * h + 3] += P * nu * dm;
            if (!(f & 2)) S[5 * h + 4] += P * eta;
        }
    }
    float tot[5 * kMaxGqa];
    block_scan<kSelThreads, 5 * kMaxGqa, false, SumOp>(S, tot, scan_sm, tid, 5 * g);

    // ranking-consistency check per head over the key-promoted blocks
    if (isfinite(p.rank_tol) && k_star >= 2 && k_star <= 32) {
        // few blocks: one warp per head, lane i holds the i-th block and
        // compares it with every block placed after it in the Phat order
        const int32_t *prom = p.prom + bk * p.sort_cap;
        const int warp = tid >> 5, lane = tid & 31;
        for (int h = warp; h < g; h += kSelThreads / 32) {
            float ph = 0.f, pe = 0.f;
            int bb = 0;
            if (lane < k_star) {
                bb = prom[lane] & kPromIdx;
                ph = blk[(long long)bb * kBlkRec + h];
                const float2 v = bml[(long long)bb * g + h];
                pe = v.y * ex2(v.x - Rs[h]);
            }
            int fail = 0;
            for (int j = 0; j < k_star; j++) {
                const float phj = __shfl_sync(kFull, ph, j), pej = __shfl_sync(kFull, pe, j);
                const int bj = __shfl_sync(kFull, bb, j);
                const bool after = phj < ph || (phj == ph && bj > bb);
                if (lane < k_star && after && pej > (1.f + p.rank_tol) * pe) fail = 1;
            }
            fail = __any_sync(kFull, fail);
            if (lane == 0) fail_s[h] = fail;
        }
        __syncthreads();
    } else if (isfinite(p.rank_tol) && k_star >= 2) {
        int np2 = 1;
        while (np2 < k_star) np2 <<= 1;
        const int32_t *prom = p.prom + bk * p.sort_cap;
        const int per = (k_star + kSelThreads - 1) / kSelThreads;
        const int i0 = min(k_star, tid * per), i1 = min(k_star, i0 + per);
        for (int h = 0; h < g; h++) {
            for (int i = tid; i < np2; i += kSelThreads) {
                unsigned long long key = 0ull;
                if (i < k_star) {
                    const int bb = prom[i] & kPromIdx;
                    key = sort_key(blk[(long long)bb * kBlkRec + h], bb);
                }
                keys[i] = key;
            }
            sort_keys_desc<kSelThreads>(keys, np2, tid);
            // exact masses in the Phat order; a later block may not exceed
            // (1 + rank_tol) times an earlier one
            float run[1] = {-INFINITY}, all[1];
            for (int i = i0; i < i1; i++) {
                const float2 v = bml[(long long)key_index(keys[i]) * g + h];
                run[0] = fmaxf(run[0], v.y * ex2(v.x - Rs[h]));
            }
            block_scan<kSelThreads, 1, true, MaxOp>(run, all, scan_sm, tid);  // max over positions >= i1
            float after = run[0];
            int fail = 0;
            for (int i = i1 - 1; i >= i0; i--) {
                const float2 v = bml[(long long)key_index(keys[i]) * g + h];
                const float pe = v.y * ex2(v.x - Rs[h]);
                if (after > (1.f + p.rank_tol) * pe) fail = 1;
                after = fmaxf(after, pe);
            }
            fail = __syncthreads_or(fail);
            if (tid == 0) fail_s[h] = fail;
        }
        __syncthreads();
    }

    // decisions: a failed check or a bound above cert_tol sends the head to
    // the fp16 fallback
    if (tid < g) {
        const int h = tid;
        const float SP = tot[5 * h];
        float bnd = 0.f;
        if (SP > 0.f) {
            const float A = log1pf(tot[5 * h + 1] / SP);
            bnd = (expm1f(A) * tot[5 * h + 2] + expf(A) * tot[5 * h + 3] + tot[5 * h + 4]) / SP;
        }
        const bool fr = fail_s[h] != 0, fb = bnd > p.cert_tol;
        int st = (gs & 0xFFFF) | (fr ? kStRankFail : 0) | (fb ? kStBoundFail : 0);
        if (fr || fb) {
            st |= kStHeadDense;
            atomicAdd(p.nfall, 1u);
        }
        const long long head = (long long)b * L.hq + kvh * g + h;
        p.status[head] = st;
        p.bound[head] = bnd;
        if (p.status_out) p.status_out[head] = st;
        if (p.bound_out) p.bound_out[head] = bnd;
    }
}

// fp16 attention over the tier-2 rows (original domain, no rotation) for the
// heads that fell back.  Work items (context split, kv head, sequence) are
// handed out over a persistent grid; a group's splits are merged by the CTA
// that finishes its last one.
template <int D>
__device__ __forceinline__ void dense_item(const CertParams &p, int split, int kvh, int b, unsigned mask, bool layer,
                                           float *wacc, float *wm, float *wl, int *sflag)
{
    constexpr int E = D / 32;
    const Layout &L = p.L;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = L.g;
    const long long bk = (long long)b * L.hkv + kvh;
    const int T = clamp_ctx(p.ctx_lens[b], p.max_pages);
    const int t0 = split * p.dsplit_tokens, t1 = min(T, t0 + p.dsplit_tokens);
    const int32_t *bt = p.block_table + (long long)b * p.max_pages;

    float qr[kMaxGqa][E];
#pragma unroll
    for (int h = 0; h < kMaxGqa; h++)
#pragma unroll
        for (int e = 0; e < E; e++)
            qr[h][e] = h < g ? __half2float(p.q[((long long)b * L.hq + kvh * g + h) * D + lane * E + e]) * p.qscale : 0.f;
    float m[kMaxGqa], l[kMaxGqa], acc[kMaxGqa][E];
#pragma unroll
    for (int h = 0; h < kMaxGqa; h++) {
        m[h] = -INFINITY;
        l[h] = 0.f;
#pragma unroll
        for (int e = 0; e < E; e++) acc[h][e] = 0.f;
    }
    for (int tb = t0 + warp * kTokBatch; tb < t1; tb += kPromWarps * kTokBatch) {
        RawRow<E> kraw[kTokBatch], vraw[kTokBatch];
        bool ok[kTokBatch];
#pragma unroll
        for (int u = 0; u < kTokBatch; u++) {
            const int t = tb + u;
            int pg = -1;
            if (t < t1) {
                pg = bt[t / kPageTokens];
                if (pg >= L.num_pages) pg = -1;
            }
            ok[u] = pg >= 0;
            if (ok[u]) {
                const long long row = ((long long)(pg * kPageTokens + t % kPageTokens) * L.hkv + kvh) * D + lane * E;
                kraw[u].load(p.k2 + row);
                vraw[u].load(p.v2 + row);
            }
        }
#pragma unroll
        for (int u = 0; u < kTokBatch; u++) {
            if (!ok[u]) continue;  // warp-uniform
            float k[E], v[E];
            kraw[u].widen(k);
            vraw[u].widen(v);
#pragma unroll
            for (int h = 0; h < kMaxGqa; h++) {
                if (h >= g) break;
                float s = 0.f;
#pragma unroll
                for (int e = 0; e < E; e++) s = fmaf(qr[h][e], k[e], s);
#pragma unroll
                for (int mm = 16; mm >= 1; mm >>= 1) s += __shfl_xor_sync(kFull, s, mm);
                online_update<E>(m[h], l[h], acc[h], s, v);
            }
        }
    }

    // warps -> one partial per head
    __syncthreads();  // the previous item's shared-memory reads are done
#pragma unroll
    for (int h = 0; h < kMaxGqa; h++)
        if (h < g) {
#pragma unroll
            for (int e = 0; e < E; e++) wacc[(warp * g + h) * D + lane * E + e] = acc[h][e];
            if (lane == 0) {
                wm[warp * kMaxGqa + h] = m[h];
                wl[warp * kMaxGqa + h] = l[h];
            }
        }
    __syncthreads();
    constexpr int REC = D + 4;
    float *dp = p.dpart + (bk * p.n_dsplit + split) * (long long)g * REC;
    for (int idx = tid; idx < g * D; idx += kPromThreads) {
        const int h = idx / D, ch = idx - h * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kPromWarps; w++) M = fmaxf(M, wm[w * kMaxGqa + h]);
        float a = 0.f, Ls = 0.f;
        if (M != -INFINITY)
#pragma unroll
            for (int w = 0; w < kPromWarps; w++) {
                const float mw = wm[w * kMaxGqa + h];
                const float f = mw == -INFINITY ? 0.f : ex2(mw - M);
                a = fmaf(f, wacc[(w * g + h) * D + ch], a);
                Ls = fmaf(f, wl[w * kMaxGqa + h], Ls);
            }
        dp[h * REC + ch] = a;
        if (ch == 0) {
            dp[h * REC + D] = M;
            dp[h * REC + D + 1] = Ls;
        }
    }

    // the CTA that finishes the group's last split merges them
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(p.dcount + bk, 1u);
        *sflag = prev == (unsigned)(p.n_dsplit - 1);
    }
    __syncthreads();
    if (!*sflag) return;
    __threadfence();
    if (tid == 0) p.dcount[bk] = 0u;
    const float *base = p.dpart + bk * p.n_dsplit * (long long)g * REC;
    for (int h = warp; h < g; h += kPromWarps) {
        if (!(mask & (1u << h))) continue;
        float M = -INFINITY;
        for (int c = 0; c < p.n_dsplit; c++) M = fmaxf(M, __ldcg(base + (c * g + h) * REC + D));
        float Ls = 0.f, a[E];
#pragma unroll
        for (int e = 0; e < E; e++) a[e] = 0.f;
        if (M != -INFINITY)
            for (int c = 0; c < p.n_dsplit; c++) {
                const float mc = __ldcg(base + (c * g + h) * REC + D);
                if (mc == -INFINITY) continue;
                const float f = ex2(mc - M);
                Ls = fmaf(f, __ldcg(base + (c * g + h) * REC + D + 1), Ls);
#pragma unroll
                for (int e = 0; e < E; e++) a[e] = fmaf(f, __ldcg(base + (c * g + h) * REC + lane * E + e), a[e]);
            }
        const long long head = (long long)b * L.hq + kvh * g + h;
        float *o = p.out + head * D + lane * E;
#pragma unroll
        for (int e = 0; e < E; e++) o[e] = Ls > 0.f ? a[e] / Ls : 0.f;
        if (layer && lane == 0) {
            p.status[head] |= kStLayerDense;
            if (p.status_out) p.status_out[head] |= kStLayerDense;
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kPromThreads) ladder_dense_kernel(const __grid_constant__ CertParams p)
{
    pdl_enter();
    const Layout &L = p.L;
    extern __shared__ float wacc[];  // [kPromWarps][g][D]
    __shared__ float wm[kPromWarps * kMaxGqa], wl[kPromWarps * kMaxGqa];
    __shared__ int sflag;
    const unsigned nfall = __ldcg(p.nfall);
    if (nfall == 0u) return;  // no head fell back (the common case)
    const bool layer = nfall > (unsigned)p.layer_thresh;
    const int per_b = p.n_dsplit * L.hkv;
    const int n_items = per_b * p.batch;
    for (int it = blockIdx.x; it < n_items; it += gridDim.x) {  // uniform over the CTA
        const int b = it / per_b, r = it - b * per_b;
        const int kvh = r / p.n_dsplit, split = r - kvh * p.n_dsplit;
        unsigned mask = 0;
        for (int h = 0; h < L.g; h++)
            if (layer || (__ldcg(p.status + (long long)b * L.hq + kvh * L.g + h) & kStHeadDense)) mask |= 1u << h;
        if (mask) dense_item<D>(p, split, kvh, b, mask, layer, wacc, wm, wl, &sflag);
    }
}

}  // namespace

cudaError_t launch_ladder_select(const CertParams &p, int batch, cudaStream_t s)
{
    static DeviceOnce once[2];
    const int di = p.L.d == 64 ? 0 : 1;
    if (once[di].needed()) {
        const int cap = kCertMaxBlocks * (int)(sizeof(unsigned long long) + 1);
        const cudaError_t e =
            di ? cudaFuncSetAttribute(ladder_select_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, cap)
               : cudaFuncSetAttribute(ladder_select_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, cap);
        if (e != cudaSuccess) return e;
        once[di].mark();
    }
    const size_t smem = (size_t)p.sort_cap * (sizeof(unsigned long long) + 1);
    const dim3 grid(p.L.hkv, batch);
    return di ? launch_pdl(ladder_select_kernel<128>, grid, kSelThreads, smem, s, p)
              : launch_pdl(ladder_select_kernel<64>, grid, kSelThreads, smem, s, p);
}

cudaError_t launch_ladder_finish(const CertParams &p, int batch, cudaStream_t s)
{
    static DeviceOnce once[2];
    const int di = p.L.d == 64 ? 0 : 1;
    if (once[di].needed()) {
        const int cap = kCertMaxBlocks * (int)sizeof(unsigned long long);
        const int dcap = kPromWarps * kMaxGqa * kMaxD * (int)sizeof(float);
        cudaError_t e =
            di ? cudaFuncSetAttribute(ladder_finish_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, cap)
               : cudaFuncSetAttribute(ladder_finish_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, cap);
        if (e != cudaSuccess) return e;
        e = di ? cudaFuncSetAttribute(ladder_dense_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, dcap)
               : cudaFuncSetAttribute(ladder_dense_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, dcap);
        if (e != cudaSuccess) return e;
        once[di].mark();
    }
    const size_t smem = (size_t)p.sort_cap * sizeof(unsigned long long);
    const dim3 grid(p.L.hkv, batch);
    cudaError_t e = di ? launch_pdl(ladder_finish_kernel<128>, grid, kSelThreads, smem, s, p)
                       : launch_pdl(ladder_finish_kernel<64>, grid, kSelThreads, smem, s, p);
    if (e != cudaSuccess) return e;
    const size_t dsmem = (size_t)kPromWarps * p.L.g * p.L.d * sizeof(float);
    const int items = p.n_dsplit * p.L.hkv * batch;
    const dim3 dgrid(items < p.dense_ctas ? items : p.dense_ctas);
    return di ? launch_pdl(ladder_dense_kernel<128>, dgrid, kPromThreads, dsmem, s, p)
              : launch_pdl(ladder_dense_kernel<64>, dgrid, kPromThreads, dsmem, s, p);
}

}  // namespace kvq
