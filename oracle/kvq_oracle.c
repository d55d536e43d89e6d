/*
 * kvq_oracle.c -- CPU oracle for the low-bit KV cache (TEST INFRASTRUCTURE).
 *
 * This file is the plain, slow, obviously-correct statement of what the hot
 * path computes.  Only the tests, the package smoke check and the benchmark's
 * CPU-baseline leg may load it.  It shares no code, header, table or constant
 * generator with the CUDA library: the byte layout, the sign generator and the
 * rotation constant are all restated here from their written definitions.
 *
 * Sources (cited by page title and section):
 *   [SRFT]  "When Quantization Is Free: An int4 KV Cache That Outruns fp16 on
 *           Apple Silicon" -- Methodology 1 (random-sign rotation, SRHT as the
 *           Hadamard alternative), Methodology 2 (fused kernel: sign in
 *           registers, butterfly passes, per-group scaling, rounding, nibble
 *           packing).
 *   [CERT]  "Runtime-Certified Bounded-Error Quantized Attention" --
 *           Methodology 1 (tier 1: INT8 keys / INT4 values with scales,
 *           offsets and per-block error descriptors; tier 2: fp16 originals in
 *           pinned host RAM), Methodology 2 (key term E_key from the per-token
 *           score perturbation, value term E_val from per-block reconstruction
 *           errors weighted by block mass), Methodology 3 (top-K* promotion of
 *           blocks to fp16).
 *   [OSCAR] "OSCAR: Offline Spectral Covariance-Aware Rotation for 2-bit KV
 *           cache quantization" -- 2.2 Algorithm design (Hadamard factor of the
 *           rotation, clipping thresholds; paged INT2 history; fused kernel
 *           doing unpack, dequantization, inverse rotation and attention).
 *
 * Precision: the codec (rotation, statistics, scale/zero, codes) is fp32 with
 * every operation rounded separately (build with -ffp-contract=off), because
 * the quantised codes are integers decided by floating point and both sides
 * must take that decision in the same precision.  Attention is fp64.
 *
 * Readings of points the pages leave open are listed next to the code that
 * takes them.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define KVQO_INT4_ASYM 0
#define KVQO_INT8_SYM 1
#define KVQO_INT2_ASYM 2
#define KVQO_HQMQ 3        /* Hurwitz-quaternion multiplicative VQ of 4-element blocks */
#define KVQO_NVFP4 4       /* e2m1 codes, one E4M3 scale per 16 elements */
#define KVQO_HQMQ_NS 1024  /* secondary codebook size per (kv head, K|V) */
#define KVQO_HQMQ_NO 2     /* fp16 outlier blocks a row can keep (Med3x) */

#define KVQO_PAGE_TOKENS 16
#define KVQO_HEADER_BYTES 256
#define KVQO_MAXD 256

typedef struct {
    int32_t num_q_heads;
    int32_t num_kv_heads;
    int32_t head_dim;
    int32_t k_fmt;
    int32_t v_fmt;
    int32_t k_group;
    int32_t v_group;
    float clip_ratio;
    uint64_t rotation_seed;
    int32_t rotate;
    int32_t page_tokens;
    int32_t num_pages;
    int32_t bound_block_tokens;
    int32_t scale_search; /* 1: ScaleSearch over the scale's fp16 bit pattern */
} kvqo_config;

/* ------------------------------------------------------------------------- */
/* IEEE binary16 conversions, written from the format definition.            */
/* ------------------------------------------------------------------------- */

/* binary16 bits -> fp32 value (exact). */
float kvqo_h2f(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    float v;
    if (e == 0)
        v = ldexpf((float)m, -24); /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexpf((float)(m | 0x400), e - 25); /* (1024+m) * 2^(e-15-10) */
    return sign ? -v : v;
}

/* round-half-to-even of a non-negative double that holds few bits. */
static double rhe(double q)
{
    double n = floor(q);
    double f = q - n;
    if (f > 0.5) return n + 1.0;
    if (f < 0.5) return n;
    return (fmod(n, 2.0) == 0.0) ? n : n + 1.0;
}

/* Magnitude |x| (finite, >= 0) -> binary16 bits of the value on the fp16 grid
 * selected by `mode`: 0 = nearest-even, 1 = up (away from zero for the
 * magnitude), 2 = down (toward zero).  Overflow handling is left to the
 * caller. */
static uint32_t mag_to_h(double a, int mode)
{
    double step;
    int e = 0;
    if (a < ldexp(1.0, -14)) {
        step = ldexp(1.0, -24); /* subnormal grid */
    } else {
        int E;
        frexp(a, &E); /* a = f * 2^E, f in [0.5,1) */
        e = E - 1;    /* 2^e <= a < 2^(e+1) */
        step = ldexp(1.0, e - 10);
    }
    double q = a / step; /* exact: a has at most 24 significant bits */
    double n;
    if (mode == 0) n = rhe(q);
    else if (mode == 1) n = ceil(q);
    else n = floor(q);
    if (a < ldexp(1.0, -14)) return (uint32_t)n; /* n == 1024 is the smallest normal */
    /* n in [1024, 2048]; n == 2048 carries into the exponent correctly */
    return (uint32_t)(((e + 15) << 10) + ((int)n - 1024));
}

/* fp32 -> binary16, round to nearest, ties to even. */
uint16_t kvqo_f2h_rn(float x)
{
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    if (isnan(x)) return 0x7e00;
    double a = fabs((double)x);
    if (a >= 65520.0) return sign | 0x7c00; /* at or past max + half ulp */
    return sign | (uint16_t)mag_to_h(a, 0);
}

/* fp32 -> binary16, round toward +infinity. */
uint16_t kvqo_f2h_ru(float x)
{
    if (isnan(x)) return 0x7e00;
    double a = fabs((double)x);
    if (!signbit(x)) {
        if (a > 65504.0) return 0x7c00;
        return (uint16_t)mag_to_h(a, 1);
    }
    if (a > 65504.0) return 0xfbff; /* -65504 is the least fp16 >= x */
    return 0x8000 | (uint16_t)mag_to_h(a, 2);
}

/* ------------------------------------------------------------------------- */
/* Rotation R = c_d * H_d * diag(s)                                          */
/* ------------------------------------------------------------------------- */

/* SplitMix64 (Steele, Lea, Flood; Vigna's reference generator): the state
 * advances by the golden-ratio increment and each output is the state passed
 * through the two xor-shift-multiply rounds. */
static uint64_t splitmix64_next(uint64_t *state)
{
    uint64_t z = (*state += 0x9E3779B97F4A7C15ULL);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t kvqo_splitmix64_output(uint64_t seed, int index)
{
    uint64_t st = seed, z = 0;
    for (int i = 0; i <= index; i++) z = splitmix64_next(&st);
    return z;
}

/* [SRFT] Methodology 1: a fixed random sign vector s.  Reading: one vector per
 * cache, s_i = -1 when the top bit of the i-th SplitMix64 output (state seeded
 * with rotation_seed) is set, else +1; the same s serves every head, K and V. */
void kvqo_signs(uint64_t seed, int d, float *s)
{
    uint64_t st = seed;
    for (int i = 0; i < d; i++) s[i] = (splitmix64_next(&st) >> 63) ? -1.0f : 1.0f;
}

/* c_d = 1/sqrt(d) rounded to fp32. */
float kvqo_rot_scale_f32(int d) { return (float)(1.0 / sqrt((double)d)); }

/* [OSCAR] 2.2(a): P_br, the bit-reversal permutation of the channel index.
 * With rotate = 2 the rotation is R = H_Had P_br in the page's row-vector
 * form x R (U, the data-derived eigenbasis, left out): the Hadamard output t
 * is permuted after the scale, y_j = t_{br(j)}, br(j) = j with its log2(d)
 * bits in reverse order.  br is its own inverse. */
int kvqo_bitrev(int j, int d)
{
    int r = 0;
    for (int b = 1; b < d; b <<= 1) {
        r = (r << 1) | (j & 1);
        j >>= 1;
    }
    return r;
}

static void bitrev_f32(float *y, int d)
{
    for (int j = 0; j < d; j++) {
        const int k = kvqo_bitrev(j, d);
        if (k > j) {
            const float t = y[j];
            y[j] = y[k];
            y[k] = t;
        }
    }
}

static void bitrev_f64(double *y, int d)
{
    for (int j = 0; j < d; j++) {
        const int k = kvqo_bitrev(j, d);
        if (k > j) {
            const double t = y[j];
            y[j] = y[k];
            y[k] = t;
        }
    }
}

/* [SRFT] Methodology 1-2 with the Hadamard choice (SRHT), [OSCAR] 2.2
 * (H_Had factor): y = c_d * H_d * diag(s) * x in fp32.  H_d is the Sylvester
 * (natural-order) Hadamard matrix applied as log2(d) butterfly stages with
 * half-width h = 1, 2, 4, ..., d/2; each stage maps the pair (j, j+h), j&h==0,
 * to (a+b, a-b).  Stages run in that order and every operation rounds on its
 * own; the codec's integer decisions depend on this exact order. */
void kvqo_rotate_f32(const float *x, const float *s, int d, int rotate, float *y)
{
    if (!rotate) {
        for (int i = 0; i < d; i++) y[i] = x[i];
        return;
    }
    for (int i = 0; i < d; i++) y[i] = x[i] * s[i];
    for (int h = 1; h < d; h <<= 1)
        for (int j = 0; j < d; j++)
            if (!(j & h)) {
                float a = y[j], b = y[j + h];
                y[j] = a + b;
                y[j + h] = a - b;
            }
    float c = kvqo_rot_scale_f32(d);
    for (int i = 0; i < d; i++) y[i] = y[i] * c;
    if (rotate == 2) bitrev_f32(y, d);
}

static void fwht_f64(double *y, int d)
{
    for (int h = 1; h < d; h <<= 1)
        for (int j = 0; j < d; j++)
            if (!(j & h)) {
                double a = y[j], b = y[j + h];
                y[j] = a + b;
                y[j + h] = a - b;
            }
}

/* fp64 forward rotation R x (used for queries and for the exact fp16 rows). */
void kvqo_rotate_f64(const double *x, const float *s, int d, int rotate, double *y)
{
    if (!rotate) {
        for (int i = 0; i < d; i++) y[i] = x[i];
        return;
    }
    for (int i = 0; i < d; i++) y[i] = x[i] * (double)s[i];
    fwht_f64(y, d);
    double c = 1.0 / sqrt((double)d);
    for (int i = 0; i < d; i++) y[i] *= c;
    if (rotate == 2) bitrev_f64(y, d);
}

/* fp64 inverse rotation R^T x = diag(s) * H_d * c_d * x ([OSCAR] 2.2b: the
 * fused kernel applies the inverse rotation to the attention output); with
 * rotate = 2 the bit reversal is undone first. */
void kvqo_inv_rotate_f64(const double *x, const float *s, int d, int rotate, double *y)
{
    if (!rotate) {
        for (int i = 0; i < d; i++) y[i] = x[i];
        return;
    }
    for (int i = 0; i < d; i++) y[i] = x[i];
    if (rotate == 2) bitrev_f64(y, d);
    fwht_f64(y, d);
    double c = 1.0 / sqrt((double)d);
    for (int i = 0; i < d; i++) y[i] = y[i] * c * (double)s[i];
}

/* ------------------------------------------------------------------------- */
/* Codec for one token-head row                                              */
/* ------------------------------------------------------------------------- */

static int fmt_bits(int fmt) { return fmt == KVQO_INT4_ASYM ? 4 : fmt == KVQO_INT8_SYM ? 8 : 2; }

/* Quantise one rotated row y[0..d).
 *
 * Asymmetric formats (int4, int2) -- [SRFT] Methodology 2 (per-group
 * statistics, rounding), [CERT] Methodology 1 (scales/offsets):
 *   lo = min, hi = max over the group; with clip ratio r < 1 ([OSCAR] 2.2a,
 *   clipping thresholds) both ends are scaled by r (reading: toward zero);
 *   scale_h = fp16_rn((hi - lo) / (2^b - 1)); zero_h = fp16_rn(lo);
 *   inv = 1 / float(scale_h) (0 when scale_h == 0);
 *   code = clamp(rint((y - float(zero_h)) * inv), 0, 2^b - 1), ties to even.
 * Reading: "zero" is an additive fp16 offset equal to the group minimum.
 *
 * Symmetric int8 ([SRFT] Methodology 2, absmax; [CERT] Methodology 1, INT8
 * keys): a = max |y| over the row (the config fixes one scale per token-head);
 *   scale_h = fp16_ru(a / 127) -- rounding up keeps |y| * inv <= 127;
 *   code = clamp(rint(y * inv), -127, 127).
 *
 * Outputs: code[d], scale_h[ng], zero_h[ng] (zero unused for int8), and the
 * fp32 descriptors max|y - yhat| and max|y| with yhat = float(code)*scale
 * (+ zero), each operation rounded on its own. */
/* ScaleSearch ["Search Your Block Floating Point Scales!", ScaleSearch]: the
 * page searches integer offsets f in [-2, 6] on the bit pattern of the
 * default block scale and keeps the scale of least squared error.  Here the
 * scale is the codec's fp16 scale: candidate f has the bits of the default
 * scale plus f (only positive finite fp16 values), the zero stays.  Each
 * candidate quantises the group as the codec does and sums the squared
 * reconstruction errors in fp32, in a fixed order: the group is cut into
 * runs of 64 consecutive elements (one run if it is shorter); in a run, the
 * even and the odd elements are summed apart, in element order, and the
 * two added; the runs' sums are added in order.  Candidates are tried in
 * the order 0, -1, 1, -2, 2, 3, 4, 5, 6 and one replaces the best so far
 * only with a strictly smaller error, so ties keep the one nearer the
 * default.  Returns the chosen scale bits. */
static const int kvqo_search_order[9] = {0, -1, 1, -2, 2, 3, 4, 5, 6};

static float group_sq_error(const float *yg, int n, float sf, float zf, float lo_code, float hi_code)
{
    float inv = (sf == 0.0f) ? 0.0f : 1.0f / sf;
    int run = n < 64 ? n : 64;
    float total = 0.0f;
    for (int r0 = 0; r0 < n; r0 += run) {
        float ev = 0.0f, od = 0.0f;
        for (int i = r0; i < r0 + run; i++) {
            float v = (yg[i] - zf) * inv;
            float c = rintf(v);
            if (c < lo_code) c = lo_code;
            if (c > hi_code) c = hi_code;
            float yhat = c * sf + zf;
            float e = yg[i] - yhat;
            float e2 = e * e;
            if ((i - r0) % 2 == 0) ev = ev + e2;
            else od = od + e2;
        }
        float rs = ev + od;
        total = (r0 == 0) ? rs : total + rs;
    }
    return total;
}

static uint16_t search_scale(const float *yg, int n, uint16_t sh0, float zf, float lo_code, float hi_code)
{
    if (sh0 == 0 || sh0 >= 0x7C00u) return sh0;
    uint16_t best = sh0;
    float best_err = 0.0f;
    for (int k = 0; k < 9; k++) {
        int bits = (int)sh0 + kvqo_search_order[k];
        if (bits <= 0 || bits >= 0x7C00) continue;
        float err = group_sq_error(yg, n, kvqo_h2f((uint16_t)bits), zf, lo_code, hi_code);
        if (k == 0 || err < best_err) {
            best = (uint16_t)bits;
            best_err = err;
        }
    }
    return best;
}

static void quantize_row(int fmt, int group, float clip, int search, const float *y, int d, int16_t *code,
                         uint16_t *scale_h, uint16_t *zero_h, float *err_max, float *abs_max)
{
    float emax = 0.0f, amax = 0.0f;
    if (fmt == KVQO_INT8_SYM) {
        float a = 0.0f;
        for (int i = 0; i < d; i++) a = fmaxf(a, fabsf(y[i]));
        float sf_raw = a / 127.0f;
        uint16_t sh = kvqo_f2h_ru(sf_raw);
        if (search) sh = search_scale(y, d, sh, 0.0f, -127.0f, 127.0f);
        float sf = kvqo_h2f(sh);
        float inv = (sf == 0.0f) ? 0.0f : 1.0f / sf;
        for (int i = 0; i < d; i++) {
            float v = y[i] * inv;
            float r = rintf(v);
            if (r < -127.0f) r = -127.0f;
            if (r > 127.0f) r = 127.0f;
            code[i] = (int16_t)r;
            float yhat = (float)code[i] * sf;
            emax = fmaxf(emax, fabsf(y[i] - yhat));
            amax = fmaxf(amax, fabsf(y[i]));
        }
        scale_h[0] = sh;
        zero_h[0] = 0;
    } else {
        int bits = fmt_bits(fmt);
        float qmax = (float)((1 << bits) - 1);
        int ng = d / group;
        for (int g = 0; g < ng; g++) {
            const float *yg = y + g * group;
            float lo = yg[0], hi = yg[0];
            for (int i = 1; i < group; i++) {
                lo = fminf(lo, yg[i]);
                hi = fmaxf(hi, yg[i]);
            }
            if (clip < 1.0f) {
                lo = lo * clip;
                hi = hi * clip;
            }
            float sf_raw = (hi - lo) / qmax;
            uint16_t sh = kvqo_f2h_rn(sf_raw);
            uint16_t zh = kvqo_f2h_rn(lo);
            if (search) sh = search_scale(yg, group, sh, kvqo_h2f(zh), 0.0f, qmax);
            float sf = kvqo_h2f(sh), zf = kvqo_h2f(zh);
            float inv = (sf == 0.0f) ? 0.0f : 1.0f / sf;
            for (int i = 0; i < group; i++) {
                float v = (yg[i] - zf) * inv;
                float r = rintf(v);
                if (r < 0.0f) r = 0.0f;
                if (r > qmax) r = qmax;
                int16_t c = (int16_t)r;
                code[g * group + i] = c;
                float yhat = (float)c * sf + zf;
                emax = fmaxf(emax, fabsf(yg[i] - yhat));
                amax = fmaxf(amax, fabsf(yg[i]));
            }
            scale_h[g] = sh;
            zero_h[g] = zh;
        }
    }
    *err_max = emax;
    *abs_max = amax;
}

/* ------------------------------------------------------------------------- */
/* HQMQ: Hurwitz quaternion multiplicative quantisation ([HQMQ] 1-3)          */
/* ------------------------------------------------------------------------- */

/* The 24 unit Hurwitz quaternions (the binary tetrahedral group 2T) in code
 * order: p = 0..7 are +1, -1, +i, -i, +j, -j, +k, -k; p = 8..23 are
 * (+-1 +-i +-j +-k)/2 with component c negative iff bit c of p - 8 is set. */
void kvqo_hqmq_unit(int p, float q[4])
{
    for (int i = 0; i < 4; i++) q[i] = 0.0f;
    if (p < 8) {
        q[p / 2] = (p & 1) ? -1.0f : 1.0f;
    } else {
        for (int i = 0; i < 4; i++) q[i] = (((p - 8) >> i) & 1) ? -0.5f : 0.5f;
    }
}

/* Hamilton product r = a b in fp32 as fused multiply-add chains: each
 * component starts from its first product (rounded) and adds the other three
 * products in order, each with one rounding (fmaf); a subtracted product is
 * added with its first factor negated. */
static void qmul_f32(const float a[4], const float b[4], float r[4])
{
    r[0] = fmaf(-a[3], b[3], fmaf(-a[2], b[2], fmaf(-a[1], b[1], a[0] * b[0])));
    r[1] = fmaf(-a[3], b[2], fmaf(a[2], b[3], fmaf(a[1], b[0], a[0] * b[1])));
    r[2] = fmaf(a[3], b[1], fmaf(a[2], b[0], fmaf(-a[1], b[3], a[0] * b[2])));
    r[3] = fmaf(a[3], b[0], fmaf(-a[2], b[1], fmaf(a[1], b[2], a[0] * b[3])));
}

/* Secondary codebook S of (kv head, tensor): NS unit quaternions drawn
 * without calibration ([HQMQ] 1: random unit quaternions per layer, head
 * and role).  SplitMix64 stream of state seed ^ ((2 kvh + tensor + 1) *
 * 0xD1B54A32D192ED03); a candidate takes four outputs, component =
 * (out >> 40) / 2^23 - 1 (exact in fp32, in [-1, 1)), and is kept when
 * 1e-4 < |a|^2 <= 1 (squares summed in order), divided by sqrt(|a|^2). */
void kvqo_hqmq_codebook(uint64_t seed, int kvh, int tensor, float *S)
{
    uint64_t st = seed ^ ((uint64_t)(2 * kvh + tensor + 1) * 0xD1B54A32D192ED03ULL);
    int n = 0;
    while (n < KVQO_HQMQ_NS) {
        float a[4];
        for (int i = 0; i < 4; i++) a[i] = (float)(splitmix64_next(&st) >> 40) / 8388608.0f - 1.0f;
        float n2 = a[0] * a[0] + a[1] * a[1] + a[2] * a[2] + a[3] * a[3];
        if (!(n2 > 1e-4f && n2 <= 1.0f)) continue;
        float r = sqrtf(n2);
        for (int i = 0; i < 4; i++) S[4 * n + i] = a[i] / r;
        n++;
    }
}

/* Codeword index of a unit direction u ([HQMQ] 1: the codeword of largest
 * inner product in C = {q_p q_s}).  <u, q_p q_s> = <u conj(q_s), q_p>, so for
 * each s, w = u conj(q_s) and the best unit of 2T is closed-form: an axis
 * unit scores max_i |w_i| (first i on ties, sign of w_i), a half unit
 * (((|w0| + |w1|) + |w2|) + |w3|) / 2 (signs of w); the half unit wins only
 * when strictly higher, and over s the first highest score wins.
 * Index = 24 s + p. */
static int hqmq_encode_dir(const float u[4], const float *S)
{
    int best = 0;
    float best_sc = -INFINITY;
    for (int si = 0; si < KVQO_HQMQ_NS; si++) {
        const float cb[4] = {S[4 * si], -S[4 * si + 1], -S[4 * si + 2], -S[4 * si + 3]};
        float w[4], aw[4];
        qmul_f32(u, cb, w);
        for (int i = 0; i < 4; i++) aw[i] = fabsf(w[i]);
        int ia = 0;
        float ma = aw[0];
        for (int i = 1; i < 4; i++)
            if (aw[i] > ma) {
                ma = aw[i];
                ia = i;
            }
        float mh = (aw[0] + aw[1] + aw[2] + aw[3]) * 0.5f;
        int pp;
        float sc;
        if (mh > ma) {
            sc = mh;
            pp = 8 + (w[0] < 0.0f) + 2 * (w[1] < 0.0f) + 4 * (w[2] < 0.0f) + 8 * (w[3] < 0.0f);
        } else {
            sc = ma;
            pp = 2 * ia + (w[ia] < 0.0f);
        }
        if (sc > best_sc) {
            best_sc = sc;
            best = 24 * si + pp;
        }
    }
    return best;
}

/* One HQMQ row (d/4 blocks) with Med3x outlier extraction ([HQMQ] 1 and 3):
 *   r_b = sqrt(((x0^2 + x1^2) + x2^2) + x3^2), fp32;
 *   r_med = the lower median of the row's radii, tau = 3 r_med (the page's
 *     C = 3; the "batch" is read as the row, the unit quantised at once);
 *   outliers: up to KVQO_HQMQ_NO blocks with r_b > tau, largest first (lower
 *     block on ties), kept as fp16 with their mask bit set;
 *   radius step = fp16 rounded up of tau / 31; radius code = min(31,
 *     rint(r_b / step)) (0 when the step is 0);
 *   direction code = hqmq_encode_dir(x_b / r_b) (0 when r_b = 0).
 * field[b] = index | code << 15.  The page quantises the radius without
 * saying how; a uniform 5-bit code on [0, tau] with the outliers cut off is
 * the plainest reading that gives its ~5 bits per element (15 + 5 bits per
 * 4 elements). */
static void hqmq_quantize_row(const float *y, int d, const float *S, uint32_t *field, uint16_t *step_h,
                              uint32_t *mask, uint16_t outl[KVQO_HQMQ_NO][4])
{
    int nb = d / 4;
    float r[64], srt[64];
    for (int b = 0; b < nb; b++) {
        const float *x = y + 4 * b;
        r[b] = sqrtf(x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3]);
        srt[b] = r[b];
    }
    for (int i = 1; i < nb; i++)
        for (int j = i; j > 0 && srt[j - 1] > srt[j]; j--) {
            float t = srt[j];
            srt[j] = srt[j - 1];
            srt[j - 1] = t;
        }
    float tau = 3.0f * srt[(nb - 1) / 2];
    uint32_t m = 0;
    for (int k = 0; k < KVQO_HQMQ_NO; k++) {
        int pick = -1;
        for (int b = 0; b < nb; b++)
            if (!((m >> b) & 1u) && r[b] > tau && (pick < 0 || r[b] > r[pick])) pick = b;
        if (pick >= 0) m |= 1u << pick;
    }
    uint16_t sh = kvqo_f2h_ru(tau / 31.0f);
    float sf = kvqo_h2f(sh);
    int slot = 0;
    for (int k = 0; k < KVQO_HQMQ_NO; k++)
        for (int i = 0; i < 4; i++) outl[k][i] = 0;
    for (int b = 0; b < nb; b++) {
        const float *x = y + 4 * b;
        if ((m >> b) & 1u) {
            for (int i = 0; i < 4; i++) outl[slot][i] = kvqo_f2h_rn(x[i]);
            slot++;
            field[b] = 0;
            continue;
        }
        unsigned rc = 0;
        if (sf > 0.0f) {
            float v = rintf(r[b] / sf);
            rc = v > 31.0f ? 31u : (unsigned)v;
        }
        int idx = 0;
        if (r[b] > 0.0f) {
            float u[4];
            for (int i = 0; i < 4; i++) u[i] = x[i] / r[b];
            idx = hqmq_encode_dir(u, S);
        }
        field[b] = (uint32_t)idx | (rc << 15);
    }
    *step_h = sh;
    *mask = m;
}

/* Reconstruction of block b of an HQMQ row in fp64: the outlier's fp16
 * values, or (radius code x step) times the codeword q_p q_s. */
static void hqmq_dequant_block(uint32_t field, int is_outlier, const uint16_t *outl4, const float *S, double step,
                               double out[4])
{
    if (is_outlier) {
        for (int i = 0; i < 4; i++) out[i] = kvqo_h2f(outl4[i]);
        return;
    }
    int idx = (int)(field & 0x7FFFu), rc = (int)(field >> 15);
    int si = idx / 24, pp = idx % 24;
    float qp[4];
    kvqo_hqmq_unit(pp, qp);
    const float *b = S + 4 * si;
    double a[4] = {qp[0], qp[1], qp[2], qp[3]}, c[4];
    c[0] = a[0] * b[0] - a[1] * b[1] - a[2] * b[2] - a[3] * b[3];
    c[1] = a[0] * b[1] + a[1] * b[0] + a[2] * b[3] - a[3] * b[2];
    c[2] = a[0] * b[2] - a[1] * b[3] + a[2] * b[0] + a[3] * b[1];
    c[3] = a[0] * b[3] + a[1] * b[2] - a[2] * b[1] + a[3] * b[0];
    double rh = (double)rc * step;
    for (int i = 0; i < 4; i++) out[i] = rh * c[i];
}

/* ------------------------------------------------------------------------- */
/* NVFP4 ([ScaleSearch] NVFP4 and ScaleSearch: e2m1 values, an E4M3 scale    */
/* per block of 16, default scale = round(max|x| / 6) in E4M3)               */
/* ------------------------------------------------------------------------- */

/* Value of an E4M3 byte (OCP FP8 E4M3FN: bias 7, no infinities, S.1111.111
 * is NaN, subnormals m * 2^-9). */
double kvqo_e4m3_value(uint8_t b)
{
    int e = (b >> 3) & 15, m = b & 7;
    double sg = (b & 0x80) ? -1.0 : 1.0;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) return sg * ldexp((double)m, -9);
    return sg * ldexp(1.0 + m / 8.0, e - 7);
}

/* Non-negative x to E4M3: the nearest finite code, ties to the even code,
 * anything above the largest finite value (448) to 448; NaN to NaN. */
uint8_t kvqo_e4m3_rn_sat(float x)
{
    if (isnan(x)) return 0x7F;
    int best = 0;
    double bd = INFINITY;
    for (int b = 0; b <= 0x7E; b++) {
        double dd = fabs((double)x - kvqo_e4m3_value((uint8_t)b));
        if (dd < bd || (dd == bd && !(b & 1))) {
            bd = dd;
            best = b;
        }
    }
    return (uint8_t)best;
}

static const double e2m1_mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* v to a 4-bit e2m1 code: the nearest of +-{0, 0.5, 1, 1.5, 2, 3, 4, 6},
 * ties to the even magnitude index, beyond 6 (infinity included) to 6; bit
 * 3 = sign (zero is always code 0; NaN is code 0). */
uint8_t kvqo_e2m1_rn(float v)
{
    double a = fabs((double)v);
    if (isinf(a)) return (uint8_t)((signbit(v) ? 8 : 0) | 7);
    int best = 0;
    double bd = INFINITY;
    for (int m = 0; m < 8; m++) {
        double dd = fabs(a - e2m1_mag[m]);
        if (dd < bd || (dd == bd && !(m & 1))) {
            bd = dd;
            best = m;
        }
    }
    if (best == 0) return 0;
    return (uint8_t)((signbit(v) ? 8 : 0) | best);
}

static double e2m1_value(uint8_t c) { return ((c & 8) ? -1.0 : 1.0) * e2m1_mag[c & 7]; }

/* Codes of a 16-element block under scale code sc: v = y / scale (fp32),
 * code = e2m1 of v; all zero when the scale is 0. */
static void nvfp4_codes(const float *y, uint8_t sc, uint8_t *code)
{
    float sf = (float)kvqo_e4m3_value(sc);
    for (int i = 0; i < 16; i++) code[i] = sf > 0.0f ? kvqo_e2m1_rn(y[i] / sf) : 0;
}

/* Squared reconstruction error of a block in fp32: per run of four
 * elements ((e0^2 + e1^2) + e2^2) + e3^2, then (r0 + r1) + (r2 + r3); each
 * e = y - code value x scale (that product is exact), each operation
 * rounded. */
static float nvfp4_sq_error(const float *y, uint8_t sc)
{
    uint8_t code[16];
    nvfp4_codes(y, sc, code);
    float sf = (float)kvqo_e4m3_value(sc), r[4];
    for (int q = 0; q < 4; q++) {
        float acc = 0.0f;
        for (int i = 0; i < 4; i++) {
            float e = y[4 * q + i] - (float)e2m1_value(code[4 * q + i]) * sf;
            float e2 = e * e;
            acc = i == 0 ? e2 : acc + e2;
        }
        r[q] = acc;
    }
    return (r[0] + r[1]) + (r[2] + r[3]);
}

/* One row of d elements: per block of 16, amax = max |y| (fp32), default
 * scale code = E4M3 RN (saturating) of amax / 6 (fp32 division); with
 * search ([ScaleSearch] ScaleSearch) the codes b0 + f, f tried as 0, -1, 1,
 * -2, 2, 3, 4, 5, 6 (positive finite codes only, b0 itself nonzero and
 * finite), keep the least squared error, a later one only if strictly
 * smaller. */
static void nvfp4_quantize_row(const float *y, int d, int search, uint8_t *code, uint8_t *scale)
{
    for (int g = 0; g < d / 16; g++) {
        const float *yg = y + 16 * g;
        float amax = 0.0f;
        for (int i = 0; i < 16; i++) amax = fmaxf(amax, fabsf(yg[i]));
        uint8_t b0 = kvqo_e4m3_rn_sat(amax / 6.0f), best = b0;
        if (search && b0 != 0 && b0 <= 0x7E) {
            static const int offs[9] = {0, -1, 1, -2, 2, 3, 4, 5, 6};
            float be = 0.0f;
            for (int k = 0; k < 9; k++) {
                int b = (int)b0 + offs[k];
                if (b < 1 || b > 0x7E) continue;
                float e = nvfp4_sq_error(yg, (uint8_t)b);
                if (k == 0 || e < be) {
                    be = e;
                    best = (uint8_t)b;
                }
            }
        }
        scale[g] = best;
        nvfp4_codes(yg, best, code + 16 * g);
    }
}

/* ------------------------------------------------------------------------- */
/* Paged pool layout (restated here from the written layout definition)      */
/* ------------------------------------------------------------------------- */
/* pool  = [header: 256 B][pages: num_pages x page_bytes][descriptors]
 * page  = num_kv_heads chunks, chunk = [K codes][K meta][V codes][V meta]
 * codes = 16 tokens; a token's code row is the sequential bit stream of its d
 *         codes (int4: byte j = code[2j] | code[2j+1] << 4; int2: byte j holds
 *         codes 4j..4j+3 from the low bits up; int8: two's complement bytes),
 *         stored 16 bytes at a time "chunk-major": chunk c of token t sits at
 *         (c*16 + t)*16 inside the region, so one 16-byte load is one whole
 *         int4 group of 32.
 * meta  = 16 tokens x row meta; asymmetric: ng fp16 scales then ng fp16
 *         zeros; int8: one fp16 scale.
 * descriptors (only when bound blocks are on): per (page, kv head) four fp32
 *         {max key error, max value error, max |value|, 0} over the page. */

/* HQMQ rows: d/4 blocks x 20 bits (15-bit codeword index, then a 5-bit
 * radius code) as one little-endian bit stream; meta = fp16 radius step,
 * 2 zero bytes, the 32-bit outlier mask, KVQO_HQMQ_NO outlier slots of four
 * fp16 values (in block order). */
/* NVFP4 rows: d/2 code bytes (byte j = code[2j] | code[2j+1] << 4) stored
 * token-major, meta = d/16 E4M3 scale bytes. */
static int row_code_bytes(int fmt, int d)
{
    if (fmt == KVQO_HQMQ) return d * 5 / 8;
    if (fmt == KVQO_NVFP4) return d / 2;
    return d * fmt_bits(fmt) / 8;
}
static int row_meta_bytes(int fmt, int d, int group)
{
    if (fmt == KVQO_HQMQ) return 8 + 8 * KVQO_HQMQ_NO;
    if (fmt == KVQO_NVFP4) return d / 16;
    return fmt == KVQO_INT8_SYM ? 2 : 4 * (d / group);
}
static size_t region_code_bytes(int fmt, int d) { return (size_t)KVQO_PAGE_TOKENS * row_code_bytes(fmt, d); }
static size_t region_meta_bytes(int fmt, int d, int g) { return (size_t)KVQO_PAGE_TOKENS * row_meta_bytes(fmt, d, g); }

static size_t chunk_bytes(const kvqo_config *c)
{
    int d = c->head_dim;
    return region_code_bytes(c->k_fmt, d) + region_meta_bytes(c->k_fmt, d, c->k_group) +
           region_code_bytes(c->v_fmt, d) + region_meta_bytes(c->v_fmt, d, c->v_group);
}

size_t kvqo_page_bytes(const kvqo_config *c) { return (size_t)c->num_kv_heads * chunk_bytes(c); }

size_t kvqo_desc_offset(const kvqo_config *c)
{
    return KVQO_HEADER_BYTES + (size_t)c->num_pages * kvqo_page_bytes(c);
}

/* HQMQ secondary codebooks follow the descriptors: [Hkv][2][NS] unit
 * quaternions, fp32 x 4. */
size_t kvqo_hqmq_table_offset(const kvqo_config *c)
{
    size_t n = kvqo_desc_offset(c);
    if (c->bound_block_tokens > 0) n += (size_t)c->num_pages * c->num_kv_heads * 16;
    return n;
}

size_t kvqo_pool_bytes(const kvqo_config *c)
{
    size_t n = kvqo_hqmq_table_offset(c);
    if (c->k_fmt == KVQO_HQMQ) n += (size_t)c->num_kv_heads * 2 * KVQO_HQMQ_NS * 16;
    return n;
}

/* byte offset of the region (tensor 0 = K, 1 = V) of (page, kv head) */
static size_t region_base(const kvqo_config *c, int page, int kvh, int tensor, int meta)
{
    int d = c->head_dim;
    size_t off = KVQO_HEADER_BYTES + (size_t)page * kvqo_page_bytes(c) + (size_t)kvh * chunk_bytes(c);
    if (tensor == 1) off += region_code_bytes(c->k_fmt, d) + region_meta_bytes(c->k_fmt, d, c->k_group);
    if (meta) off += region_code_bytes(tensor ? c->v_fmt : c->k_fmt, d);
    return off;
}

static void pack_row(const kvqo_config *c, uint8_t *pool, int page, int tok, int kvh, int tensor, const int16_t *code,
                     const uint16_t *scale_h, const uint16_t *zero_h)
{
    int d = c->head_dim;
    int fmt = tensor ? c->v_fmt : c->k_fmt;
    int group = tensor ? c->v_group : c->k_group;
    int rb = row_code_bytes(fmt, d);
    uint8_t stream[KVQO_MAXD];
    memset(stream, 0, sizeof(stream));
    int bits = fmt_bits(fmt);
    for (int i = 0; i < d; i++) {
        unsigned v = (unsigned)code[i] & ((1u << bits) - 1u);
        stream[(i * bits) / 8] |= (uint8_t)(v << ((i * bits) % 8));
    }
    uint8_t *codes = pool + region_base(c, page, kvh, tensor, 0);
    for (int ch = 0; ch < rb / 16; ch++) memcpy(codes + ((size_t)ch * 16 + tok) * 16, stream + ch * 16, 16);
    uint8_t *meta = pool + region_base(c, page, kvh, tensor, 1) + (size_t)tok * row_meta_bytes(fmt, d, group);
    if (fmt == KVQO_INT8_SYM) {
        memcpy(meta, &scale_h[0], 2);
    } else {
        int ng = d / group;
        for (int g = 0; g < ng; g++) {
            memcpy(meta + 2 * g, &scale_h[g], 2);
            memcpy(meta + 2 * ng + 2 * g, &zero_h[g], 2);
        }
    }
}

/* The HQMQ secondary codebook of (kv head, tensor) in the pool. */
static const float *hqmq_table(const kvqo_config *c, const uint8_t *pool, int kvh, int tensor)
{
    return (const float *)(pool + kvqo_hqmq_table_offset(c)) + ((size_t)kvh * 2 + tensor) * KVQO_HQMQ_NS * 4;
}

/* Write the HQMQ secondary codebooks into a new pool (every (kv head,
 * tensor) pair); nothing for the other formats. */
void kvqo_init_pool(const kvqo_config *c, uint8_t *pool)
{
    if (c->k_fmt != KVQO_HQMQ) return;
    for (int kvh = 0; kvh < c->num_kv_heads; kvh++)
        for (int tensor = 0; tensor < 2; tensor++)
            kvqo_hqmq_codebook(c->rotation_seed, kvh, tensor, (float *)(void *)hqmq_table(c, pool, kvh, tensor));
}

/* HQMQ rows are stored token-major: the 20-bit fields as one little-endian
 * bit stream, then the meta row (see row_meta_bytes). */
static void hqmq_pack_row(const kvqo_config *c, uint8_t *pool, int page, int tok, int kvh, int tensor,
                          const uint32_t *field, uint16_t step, uint32_t mask, uint16_t outl[KVQO_HQMQ_NO][4])
{
    int d = c->head_dim, nb = d / 4, rb = row_code_bytes(KVQO_HQMQ, d);
    uint8_t stream[KVQO_MAXD];
    memset(stream, 0, sizeof(stream));
    for (int b = 0; b < nb; b++)
        for (int bit = 0; bit < 20; bit++)
            if ((field[b] >> bit) & 1u) stream[(20 * b + bit) / 8] |= (uint8_t)(1u << ((20 * b + bit) % 8));
    memcpy(pool + region_base(c, page, kvh, tensor, 0) + (size_t)tok * rb, stream, (size_t)rb);
    uint8_t *meta = pool + region_base(c, page, kvh, tensor, 1) + (size_t)tok * row_meta_bytes(KVQO_HQMQ, d, 4);
    memset(meta, 0, (size_t)row_meta_bytes(KVQO_HQMQ, d, 4));
    memcpy(meta, &step, 2);
    memcpy(meta + 4, &mask, 4);
    for (int k = 0; k < KVQO_HQMQ_NO; k++) memcpy(meta + 8 + 8 * k, outl[k], 8);
}

/* Read an HQMQ row back: fields, step, mask, outlier slots. */
void kvqo_hqmq_read_row(const kvqo_config *c, const uint8_t *pool, int slot, int kvh, int tensor, uint32_t *field,
                        uint16_t *step, uint32_t *mask, uint16_t *outl)
{
    int d = c->head_dim, nb = d / 4, rb = row_code_bytes(KVQO_HQMQ, d);
    int page = slot / KVQO_PAGE_TOKENS, tok = slot % KVQO_PAGE_TOKENS;
    const uint8_t *stream = pool + region_base(c, page, kvh, tensor, 0) + (size_t)tok * rb;
    for (int b = 0; b < nb; b++) {
        uint32_t f = 0;
        for (int bit = 0; bit < 20; bit++)
            f |= (uint32_t)((stream[(20 * b + bit) / 8] >> ((20 * b + bit) % 8)) & 1u) << bit;
        field[b] = f;
    }
    const uint8_t *meta = pool + region_base(c, page, kvh, tensor, 1) + (size_t)tok * row_meta_bytes(KVQO_HQMQ, d, 4);
    memcpy(step, meta, 2);
    memcpy(mask, meta + 4, 4);
    memcpy(outl, meta + 8, 8 * KVQO_HQMQ_NO);
}

static void nvfp4_pack_row(const kvqo_config *c, uint8_t *pool, int page, int tok, int kvh, int tensor,
                           const uint8_t *code, const uint8_t *scale)
{
    int d = c->head_dim;
    uint8_t *row = pool + region_base(c, page, kvh, tensor, 0) + (size_t)tok * row_code_bytes(KVQO_NVFP4, d);
    for (int j = 0; j < d / 2; j++) row[j] = (uint8_t)(code[2 * j] | (code[2 * j + 1] << 4));
    memcpy(pool + region_base(c, page, kvh, tensor, 1) + (size_t)tok * row_meta_bytes(KVQO_NVFP4, d, 16), scale,
           (size_t)(d / 16));
}

/* Read an NVFP4 row back: codes (one per element) and scale bytes. */
void kvqo_nvfp4_read_row(const kvqo_config *c, const uint8_t *pool, int slot, int kvh, int tensor, uint8_t *code,
                         uint8_t *scale)
{
    int d = c->head_dim;
    int page = slot / KVQO_PAGE_TOKENS, tok = slot % KVQO_PAGE_TOKENS;
    const uint8_t *row = pool + region_base(c, page, kvh, tensor, 0) + (size_t)tok * row_code_bytes(KVQO_NVFP4, d);
    for (int j = 0; j < d / 2; j++) {
        code[2 * j] = row[j] & 15;
        code[2 * j + 1] = row[j] >> 4;
    }
    memcpy(scale, pool + region_base(c, page, kvh, tensor, 1) + (size_t)tok * row_meta_bytes(KVQO_NVFP4, d, 16),
           (size_t)(d / 16));
}

/* Read back the codes, scales and zeros of one stored row (inverse of
 * pack_row). */
void kvqo_read_row(const kvqo_config *c, const uint8_t *pool, int slot, int kvh, int tensor, int16_t *code,
                   uint16_t *scale_h, uint16_t *zero_h)
{
    int d = c->head_dim;
    int fmt = tensor ? c->v_fmt : c->k_fmt;
    int group = tensor ? c->v_group : c->k_group;
    int page = slot / KVQO_PAGE_TOKENS, tok = slot % KVQO_PAGE_TOKENS;
    int rb = row_code_bytes(fmt, d);
    uint8_t stream[KVQO_MAXD];
    const uint8_t *codes = pool + region_base(c, page, kvh, tensor, 0);
    for (int ch = 0; ch < rb / 16; ch++) memcpy(stream + ch * 16, codes + ((size_t)ch * 16 + tok) * 16, 16);
    int bits = fmt_bits(fmt);
    for (int i = 0; i < d; i++) {
        unsigned v = (stream[(i * bits) / 8] >> ((i * bits) % 8)) & ((1u << bits) - 1u);
        if (fmt == KVQO_INT8_SYM) code[i] = (int16_t)(int8_t)v;
        else code[i] = (int16_t)v;
    }
    const uint8_t *meta = pool + region_base(c, page, kvh, tensor, 1) + (size_t)tok * row_meta_bytes(fmt, d, group);
    if (fmt == KVQO_INT8_SYM) {
        memcpy(&scale_h[0], meta, 2);
        zero_h[0] = 0;
    } else {
        int ng = d / group;
        for (int g = 0; g < ng; g++) {
            memcpy(&scale_h[g], meta + 2 * g, 2);
            memcpy(&zero_h[g], meta + 2 * ng + 2 * g, 2);
        }
    }
}

/* Dequantise one stored row in the rotated domain, fp64:
 * asymmetric: code * scale + zero; int8: code * scale. */
void kvqo_dequant_row(const kvqo_config *c, const uint8_t *pool, int slot, int kvh, int tensor, double *out)
{
    int d = c->head_dim;
    int fmt = tensor ? c->v_fmt : c->k_fmt;
    int group = tensor ? c->v_group : c->k_group;
    if (fmt == KVQO_HQMQ) {
        uint32_t field[64], mask;
        uint16_t step, outl[KVQO_HQMQ_NO][4];
        kvqo_hqmq_read_row(c, pool, slot, kvh, tensor, field, &step, &mask, &outl[0][0]);
        const float *S = hqmq_table(c, pool, kvh, tensor);
        int k = 0;
        for (int b = 0; b < d / 4; b++) {
            int is_out = (mask >> b) & 1u;
            hqmq_dequant_block(field[b], is_out, is_out ? outl[k] : NULL, S, (double)kvqo_h2f(step), out + 4 * b);
            k += is_out;
        }
        return;
    }
    if (fmt == KVQO_NVFP4) {  /* e2m1 value x E4M3 scale */
        uint8_t nc[KVQO_MAXD], ns[KVQO_MAXD / 16];
        kvqo_nvfp4_read_row(c, pool, slot, kvh, tensor, nc, ns);
        for (int i = 0; i < d; i++) out[i] = e2m1_value(nc[i]) * kvqo_e4m3_value(ns[i / 16]);
        return;
    }
    int16_t code[KVQO_MAXD];
    uint16_t sh[KVQO_MAXD], zh[KVQO_MAXD];
    kvqo_read_row(c, pool, slot, kvh, tensor, code, sh, zh);
    for (int i = 0; i < d; i++) {
        if (fmt == KVQO_INT8_SYM) {
            out[i] = (double)code[i] * (double)kvqo_h2f(sh[0]);
        } else {
            int g = i / group;
            out[i] = (double)code[i] * (double)kvqo_h2f(sh[g]) + (double)kvqo_h2f(zh[g]);
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Configuration check                                                       */
/* ------------------------------------------------------------------------- */

static int fmt_ok(int fmt, int group, int d)
{
    if (fmt == KVQO_INT8_SYM) return 1;
    if (fmt == KVQO_HQMQ) return group == 4 && d == 128;
    if (fmt == KVQO_NVFP4) return group == 16 && d == 128;
    if (fmt != KVQO_INT4_ASYM && fmt != KVQO_INT2_ASYM) return 0;
    if (group <= 0 || d % group) return 0;
    return 1;
}

int kvqo_config_ok(const kvqo_config *c)
{
    int d = c->head_dim;
    if (d != 64 && d != 128) return 0;
    if (c->num_kv_heads <= 0 || c->num_q_heads <= 0 || c->num_q_heads % c->num_kv_heads) return 0;
    if (c->page_tokens != KVQO_PAGE_TOKENS || c->num_pages <= 0) return 0;
    if (!fmt_ok(c->k_fmt, c->k_group, d) || !fmt_ok(c->v_fmt, c->v_group, d)) return 0;
    if (!(c->clip_ratio > 0.0f && c->clip_ratio <= 1.0f)) return 0;
    if (c->bound_block_tokens < 0 || c->bound_block_tokens % KVQO_PAGE_TOKENS) return 0;
    if (c->scale_search != 0 && c->scale_search != 1) return 0;
    if ((c->k_fmt == KVQO_HQMQ) != (c->v_fmt == KVQO_HQMQ)) return 0;  /* both or neither */
    if (c->k_fmt == KVQO_HQMQ && (c->bound_block_tokens != 0 || c->scale_search)) return 0;
    if ((c->k_fmt == KVQO_NVFP4) != (c->v_fmt == KVQO_NVFP4)) return 0;
    if (c->k_fmt == KVQO_NVFP4 && c->bound_block_tokens != 0) return 0;
    return 1;
}

/* ------------------------------------------------------------------------- */
/* Append: rotate + quantise + pack ([SRFT] Methodology 2, the fused path)   */
/* ------------------------------------------------------------------------- */

/* k, v: fp16 bits [n_tok][num_kv_heads][head_dim].  slot_mapping[n] < 0 skips
 * token n.  Returns 0, or -1 for a slot outside the pool (nothing written for
 * that token).  Also writes, when y_out is not NULL, the fp32 rotated rows
 * [n_tok][num_kv_heads][2][head_dim] (K then V). */
int kvqo_append(const kvqo_config *c, uint8_t *pool, const uint16_t *k, const uint16_t *v,
                const int32_t *slot_mapping, int n_tok, float *y_out)
{
    if (!kvqo_config_ok(c)) return -2;
    int d = c->head_dim, hkv = c->num_kv_heads;
    float s[KVQO_MAXD], x[KVQO_MAXD], y[KVQO_MAXD];
    kvqo_signs(c->rotation_seed, d, s);
    int rc = 0;
    for (int n = 0; n < n_tok; n++) {
        int slot = slot_mapping[n];
        if (slot < 0) continue;
        if (slot >= c->num_pages * KVQO_PAGE_TOKENS) {
            rc = -1;
            continue;
        }
        int page = slot / KVQO_PAGE_TOKENS, tok = slot % KVQO_PAGE_TOKENS;
        for (int kvh = 0; kvh < hkv; kvh++) {
            for (int tensor = 0; tensor < 2; tensor++) {
                const uint16_t *src = (tensor ? v : k) + ((size_t)n * hkv + kvh) * d;
                int fmt = tensor ? c->v_fmt : c->k_fmt;
                int group = tensor ? c->v_group : c->k_group;
                for (int i = 0; i < d; i++) x[i] = kvqo_h2f(src[i]);
                kvqo_rotate_f32(x, s, d, c->rotate, y);
                if (y_out) memcpy(y_out + (((size_t)n * hkv + kvh) * 2 + tensor) * d, y, sizeof(float) * d);
                if (fmt == KVQO_HQMQ) {
                    uint32_t field[64], mask;
                    uint16_t step, outl[KVQO_HQMQ_NO][4];
                    hqmq_quantize_row(y, d, hqmq_table(c, pool, kvh, tensor), field, &step, &mask, outl);
                    hqmq_pack_row(c, pool, page, tok, kvh, tensor, field, step, mask, outl);
                    continue;
                }
                if (fmt == KVQO_NVFP4) {
                    uint8_t nc[KVQO_MAXD], ns[KVQO_MAXD / 16];
                    nvfp4_quantize_row(y, d, c->scale_search, nc, ns);
                    nvfp4_pack_row(c, pool, page, tok, kvh, tensor, nc, ns);
                    continue;
                }
                int16_t code[KVQO_MAXD];
                uint16_t sh[KVQO_MAXD], zh[KVQO_MAXD];
                float emax, amax;
                quantize_row(fmt, group, fmt == KVQO_INT8_SYM ? 1.0f : c->clip_ratio, c->scale_search, y, d, code, sh,
                             zh, &emax,
                             &amax);
                pack_row(c, pool, page, tok, kvh, tensor, code, sh, zh);
                if (c->bound_block_tokens > 0) {
                    float *desc = (float *)(pool + kvqo_desc_offset(c) + ((size_t)page * hkv + kvh) * 16);
                    if (tensor == 0) {
                        desc[0] = fmaxf(desc[0], emax);
                    } else {
                        desc[1] = fmaxf(desc[1], emax);
                        desc[2] = fmaxf(desc[2], amax);
                    }
                }
            }
        }
    }
    return rc;
}

/* Dequantise stored rows: out [n][num_kv_heads][head_dim] fp64 (rotated
 * domain); k_out or v_out may be NULL. */
void kvqo_dequant(const kvqo_config *c, const uint8_t *pool, const int32_t *slots, int n, double *k_out, double *v_out)
{
    int d = c->head_dim, hkv = c->num_kv_heads;
    for (int i = 0; i < n; i++)
        for (int kvh = 0; kvh < hkv; kvh++) {
            if (k_out) kvqo_dequant_row(c, pool, slots[i], kvh, 0, k_out + ((size_t)i * hkv + kvh) * d);
            if (v_out) kvqo_dequant_row(c, pool, slots[i], kvh, 1, v_out + ((size_t)i * hkv + kvh) * d);
        }
}

/* ------------------------------------------------------------------------- */
/* Attention (fp64)                                                          */
/* ------------------------------------------------------------------------- */

/* Softmax attention of one rotated query over T rotated keys/values, split
 * into n_split contiguous token ranges whose partial states (m, l, acc) are
 * merged by the log-sum-exp rule M = max m_i, L = sum e^{m_i-M} l_i,
 * o = sum e^{m_i-M} acc_i / L.  n_split = 1 is the plain single pass.
 * T = 0 gives the zero vector. */
void kvqo_attend(const double *qr, const double *K, const double *V, int T, int d, double scale, int n_split,
                 double *o)
{
    for (int i = 0; i < d; i++) o[i] = 0.0;
    if (T <= 0) return;
    if (n_split < 1) n_split = 1;
    if (n_split > T) n_split = T;
    double *acc = (double *)calloc((size_t)n_split * d, sizeof(double));
    double *m = (double *)malloc(sizeof(double) * n_split);
    double *l = (double *)calloc((size_t)n_split, sizeof(double));
    double *sc = (double *)malloc(sizeof(double) * T);
    for (int t = 0; t < T; t++) {
        double dot = 0.0;
        for (int i = 0; i < d; i++) dot += qr[i] * K[(size_t)t * d + i];
        sc[t] = scale * dot;
    }
    for (int sp = 0; sp < n_split; sp++) {
        int t0 = (int)((long long)T * sp / n_split), t1 = (int)((long long)T * (sp + 1) / n_split);
        double mx = -INFINITY;
        for (int t = t0; t < t1; t++) mx = fmax(mx, sc[t]);
        m[sp] = mx;
        for (int t = t0; t < t1; t++) {
            double p = exp(sc[t] - mx);
            l[sp] += p;
            for (int i = 0; i < d; i++) acc[(size_t)sp * d + i] += p * V[(size_t)t * d + i];
        }
    }
    double M = -INFINITY;
    for (int sp = 0; sp < n_split; sp++) M = fmax(M, m[sp]);
    double L = 0.0;
    for (int sp = 0; sp < n_split; sp++) L += exp(m[sp] - M) * l[sp];
    for (int sp = 0; sp < n_split; sp++) {
        double w = exp(m[sp] - M) / L;
        for (int i = 0; i < d; i++) o[i] += w * acc[(size_t)sp * d + i];
    }
    free(acc);
    free(m);
    free(l);
    free(sc);
}

static int slot_of(const int32_t *block_table, int max_pages, int b, int t)
{
    return block_table[(size_t)b * max_pages + t / KVQO_PAGE_TOKENS] * KVQO_PAGE_TOKENS + t % KVQO_PAGE_TOKENS;
}

static int decode_args_ok(const kvqo_config *c, const int32_t *block_table, int max_pages, const int32_t *ctx_lens,
                          int B)
{
    for (int b = 0; b < B; b++) {
        int T = ctx_lens[b];
        if (T < 0 || T > max_pages * KVQO_PAGE_TOKENS) return 0;
        for (int p = 0; p < (T + KVQO_PAGE_TOKENS - 1) / KVQO_PAGE_TOKENS; p++) {
            int pg = block_table[(size_t)b * max_pages + p];
            if (pg < 0 || pg >= c->num_pages) return 0;
        }
    }
    return 1;
}

/* Threads of the decode's (sequence, kv head) loop; returns the count in
 * effect (1 when the oracle is built without OpenMP).  Timing only: the
 * results do not depend on it. */
int kvqo_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/* Decode attention over the quantised cache ([OSCAR] 2.2b fused kernel:
 * unpack, dequantise, attention, inverse rotation; the split/LSE merge is the
 * flash-decoding form the hot path uses).  Per sequence b and query head h:
 *   kv head = h / (Hq/Hkv) (contiguous grouping; the pages are silent),
 *   q_r = R q, s_t = scale * q_r . khat_t for t in [0, ctx_lens[b]) read
 *   through the block table, p = softmax(s), o = R^T sum_t p_t vhat_t.
 * q: fp16 bits [B][Hq][d]; out: fp64 [B][Hq][d].  scale <= 0 means 1/sqrt(d).
 * sel (optional, [B][Hkv]) restricts the work to the flagged pairs; rows of
 * other pairs are left untouched.  Returns 0, or -1 for a bad table/length. */
int kvqo_decode(const kvqo_config *c, const uint8_t *pool, const uint16_t *q, const int32_t *block_table,
                int max_pages, const int32_t *ctx_lens, int B, double scale, int n_split, const int32_t *sel,
                double *out)
{
    if (!kvqo_config_ok(c)) return -2;
    if (!decode_args_ok(c, block_table, max_pages, ctx_lens, B)) return -1;
    int d = c->head_dim, hq = c->num_q_heads, hkv = c->num_kv_heads, g = hq / hkv;
    if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
    float s[KVQO_MAXD];
    kvqo_signs(c->rotation_seed, d, s);
    /* (sequence, kv head) pairs are independent; with OpenMP they run on the
     * threads kvqo_set_threads chose, each pair's arithmetic unchanged */
#ifdef _OPENMP
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
#endif
    for (int b = 0; b < B; b++) {
        for (int kvh = 0; kvh < hkv; kvh++) {
            int T = ctx_lens[b];
            if (sel && !sel[b * hkv + kvh]) continue;
            double *K = (double *)malloc(sizeof(double) * ((size_t)T * d + 1));
            double *V = (double *)malloc(sizeof(double) * ((size_t)T * d + 1));
            for (int t = 0; t < T; t++) {
                int slot = slot_of(block_table, max_pages, b, t);
                kvqo_dequant_row(c, pool, slot, kvh, 0, K + (size_t)t * d);
                kvqo_dequant_row(c, pool, slot, kvh, 1, V + (size_t)t * d);
            }
            for (int hh = 0; hh < g; hh++) {
                int h = kvh * g + hh;
                double qx[KVQO_MAXD], qr[KVQO_MAXD], orot[KVQO_MAXD];
                for (int i = 0; i < d; i++) qx[i] = (double)kvqo_h2f(q[((size_t)b * hq + h) * d + i]);
                kvqo_rotate_f64(qx, s, d, c->rotate, qr);
                kvqo_attend(qr, K, V, T, d, scale, n_split, orot);
                kvqo_inv_rotate_f64(orot, s, d, c->rotate, out + ((size_t)b * hq + h) * d);
            }
            free(K);
            free(V);
        }
    }
    return 0;
}

/* Unquantised reference: softmax attention in fp64 over fp16 K/V rows stored
 * per slot ([num_slots][Hkv][d]) with no rotation -- the quality yardstick
 * ([CERT] Methodology 1: the fp16 originals are the ground truth). */
int kvqo_decode_fp16(const kvqo_config *c, const uint16_t *k_slots, const uint16_t *v_slots, const uint16_t *q,
                     const int32_t *block_table, int max_pages, const int32_t *ctx_lens, int B, double scale,
                     const int32_t *sel, double *out)
{
    if (!decode_args_ok(c, block_table, max_pages, ctx_lens, B)) return -1;
    int d = c->head_dim, hq = c->num_q_heads, hkv = c->num_kv_heads, g = hq / hkv;
    if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
    for (int b = 0; b < B; b++) {
        int T = ctx_lens[b];
        for (int kvh = 0; kvh < hkv; kvh++) {
            if (sel && !sel[b * hkv + kvh]) continue;
            double *K = (double *)malloc(sizeof(double) * ((size_t)T * d + 1));
            double *V = (double *)malloc(sizeof(double) * ((size_t)T * d + 1));
            for (int t = 0; t < T; t++) {
                size_t row = ((size_t)slot_of(block_table, max_pages, b, t) * hkv + kvh) * d;
                for (int i = 0; i < d; i++) {
                    K[(size_t)t * d + i] = kvqo_h2f(k_slots[row + i]);
                    V[(size_t)t * d + i] = kvqo_h2f(v_slots[row + i]);
                }
            }
            for (int hh = 0; hh < g; hh++) {
                int h = kvh * g + hh;
                double qx[KVQO_MAXD];
                for (int i = 0; i < d; i++) qx[i] = (double)kvqo_h2f(q[((size_t)b * hq + h) * d + i]);
                kvqo_attend(qx, K, V, T, d, scale, 1, out + ((size_t)b * hq + h) * d);
            }
            free(K);
            free(V);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Certified decode ([CERT] Methodology 1-3)                                 */
/* ------------------------------------------------------------------------- */

/* Number of blocks promoted out of n_blocks: ceil(frac * n_blocks), computed
 * in fp64 with a 1e-9 guard so an exact product is not bumped up by rounding,
 * clamped to [0, n_blocks]. */
int kvqo_promote_count(double frac, int n_blocks)
{
    if (frac <= 0.0 || n_blocks <= 0) return 0;
    int k = (int)ceil(frac * (double)n_blocks - 1e-9);
    if (k < 0) k = 0;
    if (k > n_blocks) k = n_blocks;
    return k;
}

/* Per-block bound, in the rotated domain, for one query head.  Reading of
 * [CERT] Methodology 2 (the pages give the two terms but print no formula):
 *   Delta_b = scale * ||q_r||_1 * eps_b        (eps_b: max |k - khat| in b)
 *   P_b     = sum_{t in b} phat_t               (mass under quantised scores)
 *   A       = ln sum_b P_b e^{Delta_b}
 *   bound_b = P_b * ((e^{Delta_b + A} - 1) * nu_b + eta_b)
 * with eta_b = max |v - vhat| and nu_b = max |v| over the block.  Then
 * ||o_r,exact - o_r,quant||_inf <= sum_b bound_b: the key term bounds the
 * total-variation shift of the softmax (p_t/phat_t = e^{delta_t}/Z with
 * e^{-A} <= Z <= e^{A} by Jensen), the value term is the mass-weighted
 * reconstruction error. */
static void block_bounds_one_head(const double *phat, int T, int block, const double *eps, const double *eta,
                                  const double *nu, double qnorm1, double scale, double *bound)
{
    int nb = (T + block - 1) / block;
    double *P = (double *)calloc((size_t)nb + 1, sizeof(double));
    for (int t = 0; t < T; t++) P[t / block] += phat[t];
    double sumexp = 0.0;
    for (int b = 0; b < nb; b++) sumexp += P[b] * exp(scale * qnorm1 * eps[b]);
    double A = log(sumexp);
    for (int b = 0; b < nb; b++) {
        double Db = scale * qnorm1 * eps[b];
        bound[b] = P[b] * ((exp(Db + A) - 1.0) * nu[b] + eta[b]);
    }
    free(P);
}

/* Certified decode.  For every (sequence, kv head): compute per-block bounds
 * for each query head of the group, score each block by the largest of them,
 * promote the top ceil(frac * n_blocks) blocks (ties to the lower block index;
 * a partial last block counts) to their exact fp16 originals from tier 2
 * (rotated in fp64), and run attention with promoted blocks exact and all
 * others dequantised.  k_slots/v_slots: tier-2 fp16 rows [num_slots][Hkv][d].
 * promoted (optional): [B][Hkv][max_promote] block indices in descending score
 * order, -1 padded.  forced (optional, same shape): promote exactly these
 * blocks (entries < 0 or >= n_blocks ignored) instead of the top scores --
 * for checking an implementation whose selection legitimately differs on a
 * near-tie; bounds and scores are computed as usual.  score_out (optional): [B][Hkv][max_blocks].
 * bound_sum_out (optional): [B][Hq], sum_b bound_b of each head (all blocks
 * quantised).  quant_out (optional): [B][Hq][d] the plain quantised output. */
int kvqo_decode_certified(const kvqo_config *c, const uint8_t *pool, const uint16_t *k_slots,
                          const uint16_t *v_slots, const uint16_t *q, const int32_t *block_table, int max_pages,
                          const int32_t *ctx_lens, int B, double scale, double frac, const int32_t *sel,
                          double *out, int32_t *promoted, int max_promote, double *score_out, int max_blocks,
                          double *bound_sum_out, const int32_t *forced)
{
    if (!kvqo_config_ok(c) || c->bound_block_tokens <= 0) return -2;
    if (!decode_args_ok(c, block_table, max_pages, ctx_lens, B)) return -1;
    int d = c->head_dim, hq = c->num_q_heads, hkv = c->num_kv_heads, g = hq / hkv;
    int block = c->bound_block_tokens;
    if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
    float s[KVQO_MAXD];
    kvqo_signs(c->rotation_seed, d, s);
    for (int b = 0; b < B; b++) {
        int T = ctx_lens[b];
        int nb = (T + block - 1) / block;
        for (int kvh = 0; kvh < hkv; kvh++) {
            if (sel && !sel[b * hkv + kvh]) continue;
            size_t n = (size_t)T * d + 1;
            double *K = (double *)malloc(sizeof(double) * n), *V = (double *)malloc(sizeof(double) * n);
            double *eps = (double *)calloc((size_t)nb + 1, sizeof(double));
            double *eta = (double *)calloc((size_t)nb + 1, sizeof(double));
            double *nu = (double *)calloc((size_t)nb + 1, sizeof(double));
            double *score = (double *)calloc((size_t)nb + 1, sizeof(double));
            double *bound = (double *)calloc((size_t)nb + 1, sizeof(double));
            double *phat = (double *)malloc(sizeof(double) * ((size_t)T + 1));
            double *sc = (double *)malloc(sizeof(double) * ((size_t)T + 1));
            for (int t = 0; t < T; t++) {
                int slot = slot_of(block_table, max_pages, b, t);
                kvqo_dequant_row(c, pool, slot, kvh, 0, K + (size_t)t * d);
                kvqo_dequant_row(c, pool, slot, kvh, 1, V + (size_t)t * d);
            }
            /* block descriptors: max over the block's pages */
            for (int p = 0; p < (T + KVQO_PAGE_TOKENS - 1) / KVQO_PAGE_TOKENS; p++) {
                int pg = block_table[(size_t)b * max_pages + p];
                const float *desc = (const float *)(pool + kvqo_desc_offset(c) + ((size_t)pg * hkv + kvh) * 16);
                int blk = p * KVQO_PAGE_TOKENS / block;
                eps[blk] = fmax(eps[blk], (double)desc[0]);
                eta[blk] = fmax(eta[blk], (double)desc[1]);
                nu[blk] = fmax(nu[blk], (double)desc[2]);
            }
            double qr[16][KVQO_MAXD];
            for (int hh = 0; hh < g && hh < 16; hh++) {
                int h = kvh * g + hh;
                double qx[KVQO_MAXD], qn = 0.0;
                for (int i = 0; i < d; i++) qx[i] = (double)kvqo_h2f(q[((size_t)b * hq + h) * d + i]);
                kvqo_rotate_f64(qx, s, d, c->rotate, qr[hh]);
                for (int i = 0; i < d; i++) qn += fabs(qr[hh][i]);
                double mx = -INFINITY, L = 0.0;
                for (int t = 0; t < T; t++) {
                    double dot = 0.0;
                    for (int i = 0; i < d; i++) dot += qr[hh][i] * K[(size_t)t * d + i];
                    sc[t] = scale * dot;
                    mx = fmax(mx, sc[t]);
                }
                for (int t = 0; t < T; t++) L += exp(sc[t] - mx);
                for (int t = 0; t < T; t++) phat[t] = exp(sc[t] - mx) / L;
                block_bounds_one_head(phat, T, block, eps, eta, nu, qn, scale, bound);
                double bs = 0.0;
                for (int bb = 0; bb < nb; bb++) {
                    score[bb] = (hh == 0) ? bound[bb] : fmax(score[bb], bound[bb]);
                    bs += bound[bb];
                }
                if (bound_sum_out) bound_sum_out[(size_t)b * hq + h] = bs;
            }
            if (score_out)
                for (int bb = 0; bb < nb && bb < max_blocks; bb++) score_out[((size_t)b * hkv + kvh) * max_blocks + bb] = score[bb];
            /* selection: top k by score, ties to the lower index */
            int k = kvqo_promote_count(frac, nb);
            char *taken = (char *)calloc((size_t)nb + 1, 1);
            if (forced) {
                const int32_t *f = forced + ((size_t)b * hkv + kvh) * max_promote;
                for (int r = 0; r < max_promote; r++) {
                    if (f[r] >= 0 && f[r] < nb) taken[f[r]] = 1;
                    if (promoted) promoted[((size_t)b * hkv + kvh) * max_promote + r] = f[r];
                }
                k = 0;
            }
            for (int r = 0; r < k; r++) {
                int best = -1;
                for (int bb = 0; bb < nb; bb++)
                    if (!taken[bb] && (best < 0 || score[bb] > score[best])) best = bb;
                taken[best] = 1;
                if (promoted && r < max_promote) promoted[((size_t)b * hkv + kvh) * max_promote + r] = best;
            }
            if (promoted && !forced)
                for (int r = k; r < max_promote; r++) promoted[((size_t)b * hkv + kvh) * max_promote + r] = -1;
            /* promoted blocks use the exact rotated fp16 originals */
            for (int t = 0; t < T; t++) {
                if (!taken[t / block]) continue;
                int slot = slot_of(block_table, max_pages, b, t);
                double xk[KVQO_MAXD], xv[KVQO_MAXD];
                size_t row = ((size_t)slot * hkv + kvh) * d;
                for (int i = 0; i < d; i++) {
                    xk[i] = kvqo_h2f(k_slots[row + i]);
                    xv[i] = kvqo_h2f(v_slots[row + i]);
                }
                kvqo_rotate_f64(xk, s, d, c->rotate, K + (size_t)t * d);
                kvqo_rotate_f64(xv, s, d, c->rotate, V + (size_t)t * d);
            }
            for (int hh = 0; hh < g; hh++) {
                int h = kvh * g + hh;
                double orot[KVQO_MAXD];
                kvqo_attend(qr[hh], K, V, T, d, scale, 1, orot);
                kvqo_inv_rotate_f64(orot, s, d, c->rotate, out + ((size_t)b * hq + h) * d);
            }
            free(taken);
            free(K);
            free(V);
            free(eps);
            free(eta);
            free(nu);
            free(score);
            free(bound);
            free(phat);
            free(sc);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Certified decode with the adaptive ladder ([CERT] Methodology 3)          */
/* ------------------------------------------------------------------------- */

/* Policy of the ladder.  Readings of [CERT] Methodology 3 ("adaptive Top-K",
 * "ranking-consistency check", "four-rung fallback ladder"), which name the
 * steps but print no formula:
 *   tau_cov    coverage target of the estimated block mass (e.g. 0.995);
 *   max_frac   budget: at most ceil(max_frac * n_blocks) key-promoted blocks;
 *   key_tol    rung 1 target for the predicted key term (inf: rung 1 off);
 *   v_tol      rung 2 threshold on a block's estimated value error
 *              contribution max_h Phat_h(b) * eta_b (inf: rung 2 off);
 *   rank_tol   relative slack rho of the ranking-consistency check (inf: off);
 *   cert_tol   a head whose certified bound exceeds it falls back (rung 3);
 *   layer_frac rung 4: every head of the call falls back when more than
 *              layer_frac * B * Hq heads fall back on their own. */
typedef struct {
    double tau_cov, max_frac, key_tol, v_tol, rank_tol, cert_tol, layer_frac;
} kvqo_ladder;

/* Outputs (every pointer but out optional).  [B][Hq][d]: out (final), mixed
 * (before any fallback), dense (fp16 attention).  [B][Hq]: err (measured
 * rotated-domain inf-norm error of mixed against exact attention), bound,
 * status (bits below).  [B][Hkv]: k_star, k_cov, k_key.  [B][Hkv][max_blocks]:
 * flags (bit 0 key exact, bit 1 value exact), rscore (the ranking score r);
 * rank_margin [B][Hq]: max over ordered pairs of (later exact mass / earlier
 * exact mass) - 1 (0 with fewer than two key-promoted blocks, inf when an
 * earlier block has zero exact mass and a later one does not).
 * [B][Hkv][max_blocks + 1]: cov (min over the group's heads of the coverage of
 * the first K ranked blocks), ekey (max over the heads of the predicted key
 * term with the first K ranked blocks' keys exact). */
typedef struct {
    double *out, *mixed, *dense, *err, *bound;
    int32_t *status, *k_star, *k_cov, *k_key;
    uint8_t *flags;
    double *rscore, *cov, *ekey;
    int32_t max_blocks;
    double *rank_margin; /* [B][Hq]: the smallest rank_tol the head's check passes with */
} kvqo_ladder_out;

#define KVQO_LADDER_EXPANDED 1    /* rung 1 added blocks beyond the coverage set */
#define KVQO_LADDER_CAPPED 2      /* the budget stopped coverage or rung 1     */
#define KVQO_LADDER_VALUES 4      /* rung 2 promoted values in this group      */
#define KVQO_LADDER_RANK_FAIL 8   /* ranking-consistency check failed          */
#define KVQO_LADDER_BOUND_FAIL 16 /* certified bound above cert_tol            */
#define KVQO_LADDER_HEAD_DENSE 32 /* rung 3: this head recomputed in fp16      */
#define KVQO_LADDER_LAYER_DENSE 64 /* rung 4: every head recomputed in fp16    */

typedef struct {
    double r;
    int idx;
} kvqo_ranked;

/* descending r, then ascending block index */
static int ranked_cmp(const void *a, const void *b)
{
    const kvqo_ranked *x = (const kvqo_ranked *)a, *y = (const kvqo_ranked *)b;
    if (x->r > y->r) return -1;
    if (x->r < y->r) return 1;
    return (x->idx > y->idx) - (x->idx < y->idx);
}

/* Block masses of a softmax over scores sc[0..T): P[b] = sum_{t in b} p_t. */
static void block_masses(const double *sc, int T, int block, double *P)
{
    int nb = (T + block - 1) / block;
    double mx = -INFINITY, L = 0.0;
    for (int b = 0; b < nb; b++) P[b] = 0.0;
    for (int t = 0; t < T; t++) mx = fmax(mx, sc[t]);
    for (int t = 0; t < T; t++) L += exp(sc[t] - mx);
    for (int t = 0; t < T; t++) P[t / block] += exp(sc[t] - mx) / L;
}

/* Key term of the bound for one head with the blocks flagged in `exact`
 * having exact keys (their score perturbation is zero):
 *   A = ln sum_b P_b e^{D_b},  E = sum_b P_b nu_b (e^{D_b + A} - 1),
 * D_b = 0 for exact blocks, Delta_b otherwise.  P are the masses of the
 * distribution the output is formed from. */
static double key_term(const double *P, const double *Dl, const double *nu, const char *exact, int nb)
{
    double s = 0.0, E = 0.0;
    for (int b = 0; b < nb; b++) s += P[b] * exp(exact[b] ? 0.0 : Dl[b]);
    double A = s > 0.0 ? log(s) : 0.0;
    for (int b = 0; b < nb; b++) E += P[b] * nu[b] * (exp((exact[b] ? 0.0 : Dl[b]) + A) - 1.0);
    return E;
}

/* Certified decode with the adaptive ladder.  Per (sequence, kv head), with
 * Phat_h(b) the block masses under the quantised scores of query head h,
 * Delta_h(b) = scale * ||q_r,h||_1 * eps_b and eta_b, nu_b the block's value
 * error and largest |value| (all as in kvqo_decode_certified):
 *  1. rank the blocks by r(b) = max_h Phat_h(b), descending, ties to the
 *     lower block index;
 *  2. K_cov = the fewest leading blocks whose estimated mass reaches tau_cov
 *     for every head of the group (0 if tau_cov <= 0);
 *  3. rung 1: K_key = the fewest leading blocks whose exact keys bring the
 *     predicted key term (key_term over Phat) of every head to key_tol or
 *     below; K* = min(ceil(max_frac * n_blocks), max(K_cov, K_key)); the
 *     first K* ranked blocks get their exact keys from tier 2;
 *  4. rung 2: blocks with max_h Phat_h(b) * eta_b > v_tol get their exact
 *     values from tier 2;
 *  5. attention with those keys/values exact and the rest dequantised (the
 *     mixed output);
 *  6. ranking-consistency check per head: order the key-promoted blocks by
 *     Phat_h; the check fails when a block placed lower has an exact mass
 *     above (1 + rank_tol) times that of a block placed higher;
 *  7. certified bound per head of the mixed output, from its own block masses
 *     P': key_term(P', Delta with zeros for exact-key blocks) plus
 *     sum over blocks with quantised values of P'(b) * eta_b.  It bounds
 *     ||o_r,exact - o_r,mixed||_inf (the distribution the output uses is the
 *     reference of the total-variation argument, as in the plain bound);
 *  8. rung 3: a head falls back to fp16 attention over its tier-2 rows when
 *     its ranking check fails or its bound exceeds cert_tol;
 *  9. rung 4: when more than layer_frac * B * Hq heads fall back, all do.
 * forced_flags ([B][Hkv][max_blocks], optional) replaces steps 1-4 by the
 * given key/value flags; forced_fallback ([B][Hq], optional) replaces the
 * decisions of steps 8-9 -- both for checking an implementation whose fp32
 * decisions legitimately differ on a near-tie.  Returns 0, -1 (bad table or
 * length), -2 (bad config) or -3 (a sequence has more than max_blocks). */
int kvqo_decode_ladder(const kvqo_config *c, const uint8_t *pool, const uint16_t *k_slots, const uint16_t *v_slots,
                       const uint16_t *q, const int32_t *block_table, int max_pages, const int32_t *ctx_lens, int B,
                       double scale, const kvqo_ladder *pol, const uint8_t *forced_flags,
                       const int32_t *forced_fallback, const kvqo_ladder_out *o)
{
    if (!kvqo_config_ok(c) || c->bound_block_tokens <= 0) return -2;
    if (!decode_args_ok(c, block_table, max_pages, ctx_lens, B)) return -1;
    int d = c->head_dim, hq = c->num_q_heads, hkv = c->num_kv_heads, g = hq / hkv;
    int block = c->bound_block_tokens, MB = o->max_blocks;
    for (int b = 0; b < B; b++)
        if ((ctx_lens[b] + block - 1) / block > MB) return -3;
    if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
    float s[KVQO_MAXD];
    kvqo_signs(c->rotation_seed, d, s);
    size_t nout = (size_t)B * hq * d;
    double *mixed = o->mixed ? o->mixed : (double *)calloc(nout + 1, sizeof(double));
    double *dense = o->dense ? o->dense : (double *)calloc(nout + 1, sizeof(double));
    int32_t *fall = (int32_t *)calloc((size_t)B * hq + 1, sizeof(int32_t));
    int32_t *stat = (int32_t *)calloc((size_t)B * hq + 1, sizeof(int32_t));
    for (size_t i = 0; i < nout; i++) mixed[i] = 0.0;

    for (int b = 0; b < B; b++) {
        int T = ctx_lens[b];
        int nb = (T + block - 1) / block;
        for (int kvh = 0; kvh < hkv; kvh++) {
            size_t n = (size_t)T * d + 1, bk = (size_t)b * hkv + kvh;
            double *Kq = (double *)malloc(sizeof(double) * n), *Vq = (double *)malloc(sizeof(double) * n);
            double *Ke = (double *)malloc(sizeof(double) * n), *Ve = (double *)malloc(sizeof(double) * n);
            double *eps = (double *)calloc((size_t)nb + 1, sizeof(double));
            double *eta = (double *)calloc((size_t)nb + 1, sizeof(double));
            double *nu = (double *)calloc((size_t)nb + 1, sizeof(double));
            double *Ph = (double *)calloc((size_t)g * nb + 1, sizeof(double));
            double *Pe = (double *)calloc((size_t)g * nb + 1, sizeof(double));
            double *Pm = (double *)calloc((size_t)nb + 1, sizeof(double));
            double *Dl = (double *)calloc((size_t)g * nb + 1, sizeof(double));
            double *scq = (double *)malloc(sizeof(double) * ((size_t)g * T + 1));
            double *sce = (double *)malloc(sizeof(double) * ((size_t)g * T + 1));
            double *sm = (double *)malloc(sizeof(double) * ((size_t)T + 1));
            double *cov = (double *)calloc((size_t)nb + 2, sizeof(double));
            double *run = (double *)calloc((size_t)g + 1, sizeof(double));
            kvqo_ranked *rk = (kvqo_ranked *)malloc(sizeof(kvqo_ranked) * ((size_t)nb + 1));
            char *kx = (char *)calloc((size_t)nb + 1, 1), *vx = (char *)calloc((size_t)nb + 1, 1);
            char *tmp = (char *)calloc((size_t)nb + 1, 1);
            double qr[16][KVQO_MAXD];

            /* quantised rows, exact rotated rows, block descriptors */
            for (int t = 0; t < T; t++) {
                int slot = slot_of(block_table, max_pages, b, t);
                size_t row = ((size_t)slot * hkv + kvh) * d;
                double xk[KVQO_MAXD], xv[KVQO_MAXD];
                kvqo_dequant_row(c, pool, slot, kvh, 0, Kq + (size_t)t * d);
                kvqo_dequant_row(c, pool, slot, kvh, 1, Vq + (size_t)t * d);
                for (int i = 0; i < d; i++) {
                    xk[i] = kvqo_h2f(k_slots[row + i]);
                    xv[i] = kvqo_h2f(v_slots[row + i]);
                }
                kvqo_rotate_f64(xk, s, d, c->rotate, Ke + (size_t)t * d);
                kvqo_rotate_f64(xv, s, d, c->rotate, Ve + (size_t)t * d);
            }
            for (int p = 0; p < (T + KVQO_PAGE_TOKENS - 1) / KVQO_PAGE_TOKENS; p++) {
                int pg = block_table[(size_t)b * max_pages + p];
                const float *desc = (const float *)(pool + kvqo_desc_offset(c) + ((size_t)pg * hkv + kvh) * 16);
                int blk = p * KVQO_PAGE_TOKENS / block;
                eps[blk] = fmax(eps[blk], (double)desc[0]);
                eta[blk] = fmax(eta[blk], (double)desc[1]);
                nu[blk] = fmax(nu[blk], (double)desc[2]);
            }
            /* per head: rotated query, scores, block masses, Delta */
            for (int hh = 0; hh < g; hh++) {
                int h = kvh * g + hh;
                double qx[KVQO_MAXD], qn = 0.0;
                for (int i = 0; i < d; i++) qx[i] = (double)kvqo_h2f(q[((size_t)b * hq + h) * d + i]);
                kvqo_rotate_f64(qx, s, d, c->rotate, qr[hh]);
                for (int i = 0; i < d; i++) qn += fabs(qr[hh][i]);
                for (int t = 0; t < T; t++) {
                    double dq = 0.0, de = 0.0;
                    for (int i = 0; i < d; i++) {
                        dq += qr[hh][i] * Kq[(size_t)t * d + i];
                        de += qr[hh][i] * Ke[(size_t)t * d + i];
                    }
                    scq[(size_t)hh * T + t] = scale * dq;
                    sce[(size_t)hh * T + t] = scale * de;
                }
                block_masses(scq + (size_t)hh * T, T, block, Ph + (size_t)hh * nb);
                block_masses(sce + (size_t)hh * T, T, block, Pe + (size_t)hh * nb);
                for (int bb = 0; bb < nb; bb++) Dl[(size_t)hh * nb + bb] = scale * qn * eps[bb];
            }
            /* 1. ranking */
            for (int bb = 0; bb < nb; bb++) {
                double r = 0.0;
                for (int hh = 0; hh < g; hh++) r = fmax(r, Ph[(size_t)hh * nb + bb]);
                rk[bb].r = r;
                rk[bb].idx = bb;
                if (o->rscore) o->rscore[bk * MB + bb] = r;
            }
            qsort(rk, (size_t)nb, sizeof(kvqo_ranked), ranked_cmp);
            /* 2. coverage of the first K ranked blocks, every head */
            for (int K = 0; K <= nb; K++) {
                if (K > 0)
                    for (int hh = 0; hh < g; hh++) run[hh] += Ph[(size_t)hh * nb + rk[K - 1].idx];
                double m = INFINITY;
                for (int hh = 0; hh < g; hh++) m = fmin(m, run[hh]);
                cov[K] = g > 0 ? m : 0.0;
                if (o->cov) o->cov[bk * (MB + 1) + K] = cov[K];
            }
            int k_cov = 0;
            if (pol->tau_cov > 0.0) {
                /* tau_cov >= 1 is all of the mass: every block (a rounded
                 * running sum can reach 1 before the last block joins) */
                k_cov = nb;
                for (int K = 0; K <= nb && pol->tau_cov < 1.0; K++)
                    if (cov[K] >= pol->tau_cov) {
                        k_cov = K;
                        break;
                    }
            }
            /* 3. rung 1: predicted key term with the first K ranked keys exact */
            int k_key = -1;
            for (int K = 0; K <= nb; K++) {
                memset(tmp, 0, (size_t)nb + 1);
                for (int r = 0; r < K; r++) tmp[rk[r].idx] = 1;
                double E = 0.0;
                for (int hh = 0; hh < g; hh++)
                    E = fmax(E, key_term(Ph + (size_t)hh * nb, Dl + (size_t)hh * nb, nu, tmp, nb));
                if (o->ekey) o->ekey[bk * (MB + 1) + K] = E;
                if (k_key < 0 && E <= pol->key_tol) k_key = K;
            }
            if (k_key < 0) k_key = nb;
            int k_cap = kvqo_promote_count(pol->max_frac, nb);
            int want = k_cov > k_key ? k_cov : k_key;
            int k_star = want < k_cap ? want : k_cap;
            /* 4. rung 2 and the flags */
            for (int r = 0; r < k_star; r++) kx[rk[r].idx] = 1;
            for (int bb = 0; bb < nb; bb++) {
                double w = 0.0;
                for (int hh = 0; hh < g; hh++) w = fmax(w, Ph[(size_t)hh * nb + bb] * eta[bb]);
                vx[bb] = w > pol->v_tol;
            }
            if (forced_flags) {
                k_star = 0;
                for (int bb = 0; bb < nb; bb++) {
                    uint8_t f = forced_flags[bk * MB + bb];
                    kx[bb] = f & 1;
                    vx[bb] = (f >> 1) & 1;
                    k_star += kx[bb];
                }
            }
            int gstat = 0;
            if (!forced_flags && k_star > k_cov) gstat |= KVQO_LADDER_EXPANDED;
            if (want > k_cap) gstat |= KVQO_LADDER_CAPPED;
            for (int bb = 0; bb < nb; bb++)
                if (vx[bb]) gstat |= KVQO_LADDER_VALUES;
            if (o->flags)
                for (int bb = 0; bb < MB; bb++) o->flags[bk * MB + bb] = bb < nb ? (uint8_t)(kx[bb] | (vx[bb] << 1)) : 0;
            if (o->k_star) o->k_star[bk] = k_star;
            if (o->k_cov) o->k_cov[bk] = k_cov;
            if (o->k_key) o->k_key[bk] = k_key;

            for (int hh = 0; hh < g; hh++) {
                int h = kvh * g + hh;
                const double *sq = scq + (size_t)hh * T, *se = sce + (size_t)hh * T;
                /* 5. mixed attention and exact attention (rotated domain) */
                double om[KVQO_MAXD], oe[KVQO_MAXD];
                for (int t = 0; t < T; t++) sm[t] = kx[t / block] ? se[t] : sq[t];
                double mm = -INFINITY, me = -INFINITY, lm = 0.0, le = 0.0;
                for (int i = 0; i < d; i++) om[i] = oe[i] = 0.0;
                for (int t = 0; t < T; t++) {
                    mm = fmax(mm, sm[t]);
                    me = fmax(me, se[t]);
                }
                for (int t = 0; t < T; t++) {
                    double pm = exp(sm[t] - mm), pe = exp(se[t] - me);
                    const double *vm = (vx[t / block] ? Ve : Vq) + (size_t)t * d, *ve = Ve + (size_t)t * d;
                    lm += pm;
                    le += pe;
                    for (int i = 0; i < d; i++) {
                        om[i] += pm * vm[i];
                        oe[i] += pe * ve[i];
                    }
                }
                double err = 0.0;
                for (int i = 0; i < d; i++) {
                    om[i] = T > 0 ? om[i] / lm : 0.0;
                    oe[i] = T > 0 ? oe[i] / le : 0.0;
                    err = fmax(err, fabs(oe[i] - om[i]));
                }
                kvqo_inv_rotate_f64(om, s, d, c->rotate, mixed + ((size_t)b * hq + h) * d);
                /* 6. ranking-consistency check over the key-promoted blocks */
                int fail_rank = 0;
                double margin = 0.0;
                int nS = 0;
                for (int bb = 0; bb < nb; bb++)
                    if (kx[bb]) {
                        rk[nS].r = Ph[(size_t)hh * nb + bb];
                        rk[nS].idx = bb;
                        nS++;
                    }
                qsort(rk, (size_t)nS, sizeof(kvqo_ranked), ranked_cmp);
                for (int i = 0; i < nS; i++)
                    for (int j = i + 1; j < nS; j++) {
                        double ei = Pe[(size_t)hh * nb + rk[i].idx], ej = Pe[(size_t)hh * nb + rk[j].idx];
                        if (!isinf(pol->rank_tol) && ej > (1.0 + pol->rank_tol) * ei) fail_rank = 1;
                        if (ei > 0.0) margin = fmax(margin, ej / ei - 1.0);
                        else if (ej > 0.0) margin = INFINITY;
                    }
                if (o->rank_margin) o->rank_margin[(size_t)b * hq + h] = margin;
                /* 7. certified bound of the mixed output */
                block_masses(sm, T, block, Pm);
                double bnd = key_term(Pm, Dl + (size_t)hh * nb, nu, kx, nb);
                for (int bb = 0; bb < nb; bb++)
                    if (!vx[bb]) bnd += Pm[bb] * eta[bb];
                int fail_bound = bnd > pol->cert_tol;
                int st = gstat | (fail_rank ? KVQO_LADDER_RANK_FAIL : 0) | (fail_bound ? KVQO_LADDER_BOUND_FAIL : 0);
                stat[(size_t)b * hq + h] = st;
                fall[(size_t)b * hq + h] = fail_rank || fail_bound;
                if (o->err) o->err[(size_t)b * hq + h] = err;
                if (o->bound) o->bound[(size_t)b * hq + h] = bnd;
            }
            free(Kq);
            free(Vq);
            free(Ke);
            free(Ve);
            free(eps);
            free(eta);
            free(nu);
            free(Ph);
            free(Pe);
            free(Pm);
            free(Dl);
            free(scq);
            free(sce);
            free(sm);
            free(cov);
            free(run);
            free(rk);
            free(kx);
            free(vx);
            free(tmp);
        }
    }
    /* 8-9. fallbacks: fp16 attention over the tier-2 rows */
    long long count = 0;
    for (size_t i = 0; i < (size_t)B * hq; i++) count += fall[i];
    int layer = (double)count > pol->layer_frac * (double)B * (double)hq;
    int rc = kvqo_decode_fp16(c, k_slots, v_slots, q, block_table, max_pages, ctx_lens, B, scale, NULL, dense);
    for (size_t i = 0; i < (size_t)B * hq && rc == 0; i++) {
        int fb;
        if (forced_fallback) {
            fb = forced_fallback[i] != 0;
            if (fb) stat[i] |= KVQO_LADDER_HEAD_DENSE;
        } else {
            fb = fall[i] || layer;
            if (fall[i]) stat[i] |= KVQO_LADDER_HEAD_DENSE;
            if (layer) stat[i] |= KVQO_LADDER_LAYER_DENSE;
        }
        if (o->status) o->status[i] = stat[i];
        for (int k = 0; k < d; k++) o->out[i * d + k] = fb ? dense[i * d + k] : mixed[i * d + k];
    }
    if (!o->mixed) free(mixed);
    if (!o->dense) free(dense);
    free(fall);
    free(stat);
    return rc;
}

/* ------------------------------------------------------------------------- */
/* Sink and recent windows at 16-bit precision ([OSCAR] 2.2b)                */
/* ------------------------------------------------------------------------- */

/* Decode where each sequence's first `sink` tokens and last `recent` tokens
 * attend with their fp16 rows and the tokens between with the quantised
 * cache: the page keeps the sink and recent tokens at full precision and the
 * middle history low-bit ([OSCAR] 2.2b, mixed-precision layout).  Window
 * rows come from a compact store win_k/win_v, fp16 [B][sink + recent][Hkv][d]:
 * row t for t < sink, row sink + t % recent for a recent token t (a ring
 * the caller keeps current).  Windows overlap when T < sink + recent; a token
 * is exact when it is in either.  Attention in fp64 in the rotated domain,
 * output inverse-rotated.  Returns 0, -1 (bad table or length), -2 (bad
 * config) or -3 (negative window sizes). */
int kvqo_decode_windows(const kvqo_config *c, const uint8_t *pool, const uint16_t *win_k, const uint16_t *win_v,
                        int sink, int recent, const uint16_t *q, const int32_t *block_table, int max_pages,
                        const int32_t *ctx_lens, int B, double scale, double *out)
{
    if (!kvqo_config_ok(c)) return -2;
    if (sink < 0 || recent < 0) return -3;
    if (!decode_args_ok(c, block_table, max_pages, ctx_lens, B)) return -1;
    int d = c->head_dim, hq = c->num_q_heads, hkv = c->num_kv_heads, g = hq / hkv;
    int W = sink + recent;
    if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
    float s[KVQO_MAXD];
    kvqo_signs(c->rotation_seed, d, s);
    for (int b = 0; b < B; b++) {
        int T = ctx_lens[b];
        for (int kvh = 0; kvh < hkv; kvh++) {
            double *K = (double *)malloc(sizeof(double) * ((size_t)T * d + 1));
            double *V = (double *)malloc(sizeof(double) * ((size_t)T * d + 1));
            for (int t = 0; t < T; t++) {
                int in_sink = t < sink, in_recent = recent > 0 && t >= T - recent;
                if (in_sink || in_recent) {
                    int row = in_sink ? t : sink + t % recent;
                    size_t off = (((size_t)b * W + row) * hkv + kvh) * d;
                    double xk[KVQO_MAXD], xv[KVQO_MAXD];
                    for (int i = 0; i < d; i++) {
                        xk[i] = kvqo_h2f(win_k[off + i]);
                        xv[i] = kvqo_h2f(win_v[off + i]);
                    }
                    kvqo_rotate_f64(xk, s, d, c->rotate, K + (size_t)t * d);
                    kvqo_rotate_f64(xv, s, d, c->rotate, V + (size_t)t * d);
                } else {
                    int slot = slot_of(block_table, max_pages, b, t);
                    kvqo_dequant_row(c, pool, slot, kvh, 0, K + (size_t)t * d);
                    kvqo_dequant_row(c, pool, slot, kvh, 1, V + (size_t)t * d);
                }
            }
            for (int hh = 0; hh < g; hh++) {
                int h = kvh * g + hh;
                double qx[KVQO_MAXD], qr[KVQO_MAXD], orot[KVQO_MAXD];
                for (int i = 0; i < d; i++) qx[i] = (double)kvqo_h2f(q[((size_t)b * hq + h) * d + i]);
                kvqo_rotate_f64(qx, s, d, c->rotate, qr);
                kvqo_attend(qr, K, V, T, d, scale, 1, orot);
                kvqo_inv_rotate_f64(orot, s, d, c->rotate, out + ((size_t)b * hq + h) * d);
            }
            free(K);
            free(V);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Array helpers for the tests                                               */
/* ------------------------------------------------------------------------- */

/* HQMQ on its own: encode rotated rows y[n][d] (fields [n][d/4], step [n],
 * mask [n], outliers [n][NO][4]) with the codebook S [NS][4]; and the
 * codeword index of single unit directions u[n][4]. */
void kvqo_hqmq_quantize_rows(const float *y, int n, int d, const float *S, uint32_t *field, uint16_t *step,
                             uint32_t *mask, uint16_t *outl)
{
    for (int r = 0; r < n; r++)
        hqmq_quantize_row(y + (size_t)r * d, d, S, field + (size_t)r * (d / 4), step + r, mask + r,
                          (uint16_t(*)[4])(outl + (size_t)r * KVQO_HQMQ_NO * 4));
}

void kvqo_nvfp4_quantize_rows(const float *y, int n, int d, int search, uint8_t *code, uint8_t *scale)
{
    for (int r = 0; r < n; r++) nvfp4_quantize_row(y + (size_t)r * d, d, search, code + (size_t)r * d, scale + (size_t)r * (d / 16));
}

void kvqo_e2m1_rn_n(const float *v, uint8_t *c, size_t n)
{
    for (size_t i = 0; i < n; i++) c[i] = kvqo_e2m1_rn(v[i]);
}

void kvqo_e4m3_rn_sat_n(const float *x, uint8_t *b, size_t n)
{
    for (size_t i = 0; i < n; i++) b[i] = kvqo_e4m3_rn_sat(x[i]);
}

void kvqo_hqmq_encode_dirs(const float *u, int n, const float *S, int32_t *idx)
{
    for (int i = 0; i < n; i++) idx[i] = hqmq_encode_dir(u + 4 * i, S);
}

void kvqo_f2h_rn_n(const float *x, uint16_t *h, size_t n)
{
    for (size_t i = 0; i < n; i++) h[i] = kvqo_f2h_rn(x[i]);
}

void kvqo_f2h_ru_n(const float *x, uint16_t *h, size_t n)
{
    for (size_t i = 0; i < n; i++) h[i] = kvqo_f2h_ru(x[i]);
}

void kvqo_h2f_n(const uint16_t *h, float *x, size_t n)
{
    for (size_t i = 0; i < n; i++) x[i] = kvqo_h2f(h[i]);
}

/* Quantise already-rotated rows y[n][d] on their own (no pool): codes
 * [n][d], scales/zeros [n][d/group] (int8: one scale per row); search = 1
 * applies ScaleSearch. */
void kvqo_quantize_rows(int fmt, int group, float clip, const float *y, int n, int d, int16_t *code,
                        uint16_t *scale_h, uint16_t *zero_h, float *err_max, float *abs_max, int search)
{
    int ng = (fmt == KVQO_INT8_SYM) ? 1 : d / group;
    for (int r = 0; r < n; r++)
        quantize_row(fmt, group, fmt == KVQO_INT8_SYM ? 1.0f : clip, search, y + (size_t)r * d, d,
                     code + (size_t)r * d, scale_h + (size_t)r * ng, zero_h + (size_t)r * ng, err_max + r, abs_max + r);
}
