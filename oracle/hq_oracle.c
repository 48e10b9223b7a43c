/*
 * hq_oracle.c -- plain, slow, fp64 CPU oracle for HyQuant hybrid-precision
 * attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file or the library built from it: only the test-suite, the
 * package smoke check and the CPU-baseline leg of the benchmark use it.  It
 * shares no code, header, table or helper with the CUDA library; the only
 * thing both sides have in common is the seeded input generator, which holds
 * none of the method's arithmetic.
 *
 * Sources (all web pages on HyQuant):
 *   [W]  "HyQuant: Hybrid-Precision Quantization for LLM Attention" (wiki
 *        summary) -- TL;DR; "What problem it solves"; "Key results".
 *   [B]  "How HyQuant uses hybrid-precision attention to cut decode compute"
 *        (blog) -- "What hybrid-precision attention changes"; "Why preserve
 *        selected positions?"; "What the authors tested"; "Memory and
 *        runtime costs".
 *   [A]  ACL Anthology author page -- the HyQuant abstract.
 * The pages state the policy (vertical-line columns plus a local window stay
 * in 16-bit, everything else is low-bit; the decode cache dequantizes inside
 * attention; prefill is a hybrid-precision operator) but not the quantizer,
 * the probe formula or the INT8 prefill granularity.  Those follow the
 * library's specification; every reading taken where the pages are silent is
 * listed next to the function that takes it.
 *
 * Conventions: tensors are row-major, head-major [B, H, T, D]; 16-bit
 * floating-point values arrive as raw bit patterns (uint16_t) and are widened
 * exactly to double here.  Query head h uses KV head h / (Hq / Hkv).
 * All floating-point arithmetic is IEEE double unless a function says
 * otherwise; OpenMP splits work over independent (batch, head, row) units
 * only, so every sum is taken in one fixed order.
 *
 * Parity pins: every function here is checked by the CPU test-suite against
 * values fixed by the pages or by mathematics (library routines, brute force,
 * closed forms, invariants).  No function is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* IEEE-754 16-bit formats, written from the format definitions.            */
/* ------------------------------------------------------------------------ */

/* bfloat16: the upper 16 bits of an IEEE binary32. Exact widening. */
static double bf16_to_f64(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. Exact widening. */
static double f16_to_f64(uint16_t h)
{
    int neg = h >> 15;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);                 /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(m | 0x400), e - 25);    /* (1024+m) * 2^(e-15-10) */
    return neg ? -v : v;
}

/* Round a double to the nearest binary16, ties to even (one rounding). */
static uint16_t f64_to_f16_rne(double x)
{
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    double a = fabs(x);
    if (isnan(x))
        return 0x7e00u;
    if (a >= 65520.0)                 /* halfway between 65504 and 2^16: even is inf */
        return (uint16_t)(sign | 0x7c00u);
    if (a < 0x1p-14) {                /* subnormal range, quantum 2^-24 */
        double r = nearbyint(a * 0x1p24);
        return (uint16_t)(sign | (uint16_t)r);   /* r == 1024 is the smallest normal */
    }
    int e;
    (void)frexp(a, &e);               /* a = f * 2^e, f in [0.5, 1) */
    double r = nearbyint(ldexp(a, 11 - e));      /* significand scaled to [1024, 2048] */
    int E = e - 1 + 15;
    uint32_t m = (uint32_t)r;
    if (m == 2048u) {
        m = 1024u;
        E += 1;
    }
    if (E >= 31)
        return (uint16_t)(sign | 0x7c00u);
    return (uint16_t)(sign | (uint16_t)(E << 10) | (uint16_t)(m - 1024u));
}

/* Exposed so the tests can pin the conversions against library routines. */
double hqo_bf16_to_f64(uint16_t b) { return bf16_to_f64(b); }
double hqo_f16_to_f64(uint16_t h) { return f16_to_f64(h); }
uint16_t hqo_f64_to_f16(double x) { return f64_to_f16_rne(x); }

/* ------------------------------------------------------------------------ */
/* P1-P2  Vertical-line-aware probe: column sums of softmax weights.        */
/* ------------------------------------------------------------------------ */
/*
 * [W] TL;DR and "What problem it solves": vertical-line tokens are key
 * columns that almost every query row attends to; finding them needs only a
 * light pattern signal.  [A]: "lightweight vertical-line-aware attention-
 * pattern signals".  Reading taken: the signal of column j is the sum, over
 * the P most recent queries of every query head that shares the KV head, of
 * that query's exact causal softmax weight on key j.  Probe row p sits at
 * absolute position L - P + p and sees keys 0 .. L - P + p.  Softmax scale is
 * `scale` (1/sqrt(D) by default).
 *
 * q_probe: bf16 [B, Hq, P, D];  k: bf16 [B, Hkv, L, D];
 * score:   double [B, Hkv, L]   (columns never seen are 0).
 */
int hqo_probe_scores(const uint16_t *q_probe, const uint16_t *k, int B, int Hq,
                     int Hkv, int P, int L, int D, double scale, double *score)
{
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || P <= 0 || P > L || D <= 0)
        return 1;
    const int G = Hq / Hkv;
    const long long nbh = (long long)B * Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (long long bh = 0; bh < nbh; ++bh) {
        const int b = (int)(bh / Hkv), kh = (int)(bh % Hkv);
        const uint16_t *kb = k + ((size_t)b * Hkv + kh) * (size_t)L * D;
        double *col = score + ((size_t)b * Hkv + kh) * (size_t)L;
        double *s = (double *)malloc(sizeof(double) * (size_t)L);
        double *qd = (double *)malloc(sizeof(double) * (size_t)D);
        for (int j = 0; j < L; ++j)
            col[j] = 0.0;
        for (int g = 0; g < G; ++g) {
            const int h = kh * G + g;
            for (int p = 0; p < P; ++p) {
                const uint16_t *qr = q_probe + (((size_t)b * Hq + h) * P + p) * (size_t)D;
                const int last = L - P + p;            /* causal: keys 0..last */
                for (int d = 0; d < D; ++d)
                    qd[d] = bf16_to_f64(qr[d]);
                double m = -INFINITY;
                for (int j = 0; j <= last; ++j) {
                    const uint16_t *kr = kb + (size_t)j * D;
                    double acc = 0.0;
                    for (int d = 0; d < D; ++d)
                        acc += qd[d] * bf16_to_f64(kr[d]);
                    s[j] = acc * scale;
                    if (s[j] > m)
                        m = s[j];
                }
                double z = 0.0;
                for (int j = 0; j <= last; ++j)
                    z += exp(s[j] - m);
                for (int j = 0; j <= last; ++j)
                    col[j] += exp(s[j] - m) / z;
            }
        }
        free(qd);
        free(s);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* P3  Top-k vertical columns outside the window.                           */
/* ------------------------------------------------------------------------ */
/*
 * [B] "Why preserve selected positions?": the top 5% of key positions plus a
 * 128-token local window.  Readings taken: k = floor(f * L) is passed in;
 * candidates are [0, L - W) so the vertical set and the window are disjoint;
 * order is (score descending, index ascending), so ties go to the lower
 * index; the k chosen indices are returned in ascending order.
 */
typedef struct {
    double s;
    int32_t j;
} hqo_cand;

static int cand_order(const void *pa, const void *pb)
{
    const hqo_cand *a = (const hqo_cand *)pa, *b = (const hqo_cand *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->j > b->j) - (a->j < b->j);
}

static int int_order(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

int hqo_topk(const double *score, int B, int Hkv, int L, int window, int kv, int32_t *idx)
{
    if (window < 0 || kv < 0 || kv > L - window)
        return 1;
    const int ncand = L - window;
    const long long nbh = (long long)B * Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (long long bh = 0; bh < nbh; ++bh) {
        const double *col = score + (size_t)bh * L;
        int32_t *out = idx + (size_t)bh * kv;
        hqo_cand *c = (hqo_cand *)malloc(sizeof(hqo_cand) * (size_t)(ncand > 0 ? ncand : 1));
        for (int j = 0; j < ncand; ++j) {
            c[j].s = col[j];
            c[j].j = j;
        }
        qsort(c, (size_t)ncand, sizeof *c, cand_order);
        for (int r = 0; r < kv; ++r)
            out[r] = c[r].j;
        qsort(out, (size_t)kv, sizeof *out, int_order);
        free(c);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Q1  Hybrid KV cache: quantize the low positions, keep the rest in bf16.  */
/* ------------------------------------------------------------------------ */
/*
 * [W] TL;DR: keep the critical set in high precision, quantize the rest hard,
 * with no smoothing.  [B] "What the authors tested": Key-4bit / Value-4bit.
 * [B] "Memory and runtime costs": +15% non-window cache at 5% retention
 * versus strict 4-bit, which holds when a vertical row is stored instead of
 * (not beside) its 4-bit copy -- so the low segment holds only the low
 * positions, compacted in ascending position order.
 *
 * Quantizer (readings taken; the pages give none): per token, per group of
 * `group` consecutive channels, asymmetric, `bits`-bit codes:
 *   mn, mx = min, max of the group (exact);
 *   s = f16_rne((mx - mn) / (2^bits - 1)),  z = f16_rne(mn + 0.0)
 *       (the quotient taken in double, then rounded once to binary16; the
 *       "+ 0.0" turns a -0 minimum into +0);
 *   c = clamp(rne((x - z) / s), 0, 2^bits - 1) with the fp16-rounded s, z,
 *       every step in double; if s == 0 every code is 0;
 *   dequantized x^ = s * c + z.
 * Packing: 4-bit codes two per byte, even channel in the low nibble; 8-bit
 * codes one per byte.  Scale and zero are stored interleaved per group:
 * sz[..., g, 0] = s, sz[..., g, 1] = z (binary16 bits).
 */
static void quant_group(const uint16_t *x, int n, int bits, uint8_t *codes,
                        uint16_t *s_out, uint16_t *z_out)
{
    const int qmax = (1 << bits) - 1;
    double mn = bf16_to_f64(x[0]), mx = mn;
    for (int i = 1; i < n; ++i) {
        double v = bf16_to_f64(x[i]);
        if (v < mn) mn = v;
        if (v > mx) mx = v;
    }
    uint16_t sb = f64_to_f16_rne((mx - mn) / (double)qmax);
    uint16_t zb = f64_to_f16_rne(mn + 0.0);
    double s = f16_to_f64(sb), z = f16_to_f64(zb);
    for (int i = 0; i < n; ++i) {
        int c = 0;
        if (s != 0.0) {
            double t = nearbyint((bf16_to_f64(x[i]) - z) / s);
            c = t < 0.0 ? 0 : (t > (double)qmax ? qmax : (int)t);
        }
        codes[i] = (uint8_t)c;
    }
    *s_out = sb;
    *z_out = zb;
}

/*
 * FP8 E4M3 codes (the "FN" variant of the OCP 8-bit floating-point formats):
 * 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0
 * holds subnormals m/8 * 2^-6; there is no infinity and only S.1111.111 is
 * NaN, so the largest finite magnitude is 1.75 * 2^8 = 448.  Written from
 * that definition.
 */
static double e4m3_to_f64(uint8_t c)
{
    const int e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    v = e == 0 ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
    return (c & 0x80) ? -v : v;
}

/* Round a double to E4M3, ties to the even code, magnitudes past the largest
 * finite one saturating to +-448 (never NaN).  The sign survives rounding to
 * zero (-0 is 0x80). */
static uint8_t f64_to_e4m3_rne_sat(double v)
{
    const uint8_t sign = signbit(v) ? 0x80 : 0x00;
    const double a = fabs(v);
    if (a >= 448.0)
        return sign | 0x7E;
    if (a < ldexp(1.0, -6))                        /* subnormal spacing 2^-9 */
        return sign | (uint8_t)nearbyint(a * 512.0);   /* 8 = the smallest normal */
    int e2;
    frexp(a, &e2);                                 /* a in [2^(e2-1), 2^e2) */
    int E = e2 - 1;
    double m = nearbyint(ldexp(a, 3 - E));         /* 8 .. 16 */
    if (m == 16.0) {
        m = 8.0;
        E += 1;
    }
    int code = ((E + 7) << 3) | ((int)m - 8);
    if (code > 0x7E)
        code = 0x7E;
    return sign | (uint8_t)code;
}

/* Exposed for the format pins. */
double hqo_e4m3_to_f64(uint8_t c) { return e4m3_to_f64(c); }
uint8_t hqo_f64_to_e4m3(double v) { return f64_to_e4m3_rne_sat(v); }

/*
 * FP8 low-bit format (fmt 1; a reading for the third precision point the
 * wiki summary's "Gaps" names for Blackwell -- the pages fix no FP8 recipe):
 * per token, per group of `group` channels, symmetric:
 *   amax = max |x| of the group (exact);
 *   s = f16_rne(amax / 448) (the quotient in double, rounded once);
 *   c = e4m3_rne_sat(x / s) (double quotient); all codes 0 if s == 0;
 *   z = +0 (stored, so the layout is that of the 8-bit integer format);
 *   dequantized x^ = s * e4m3(c).
 */
static void quant_group_fp8(const uint16_t *x, int n, uint8_t *codes, uint16_t *s_out,
                            uint16_t *z_out)
{
    double amax = 0.0;
    for (int i = 0; i < n; ++i) {
        const double a = fabs(bf16_to_f64(x[i]));
        if (a > amax)
            amax = a;
    }
    const uint16_t sb = f64_to_f16_rne(amax / 448.0);
    const double s = f16_to_f64(sb);
    for (int i = 0; i < n; ++i)
        codes[i] = s != 0.0 ? f64_to_e4m3_rne_sat(bf16_to_f64(x[i]) / s) : 0;
    *s_out = sb;
    *z_out = 0;
}

/* Quantize one row of D channels into packed codes + interleaved (s, z). */
static void quant_row(const uint16_t *x, int D, int bits, int group, int fmt, uint8_t *packed,
                      uint16_t *sz)
{
    uint8_t c[512];
    for (int g = 0; g < D / group; ++g) {
        if (fmt == 1)
            quant_group_fp8(x + g * group, group, c + g * group, &sz[2 * g], &sz[2 * g + 1]);
        else
            quant_group(x + g * group, group, bits, c + g * group, &sz[2 * g], &sz[2 * g + 1]);
    }
    if (bits == 8) {
        memcpy(packed, c, (size_t)D);
    } else {
        for (int i = 0; i < D / 2; ++i)
            packed[i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
    }
}

/* Exposed for the quantizer pins: one row of D bf16 values. */
int hqo_quant_row(const uint16_t *x, int D, int bits, int group, int fmt, uint8_t *packed,
                  uint16_t *sz)
{
    if ((bits != 4 && bits != 8) || group <= 0 || D % group || D > 512 || fmt < 0 || fmt > 1 ||
        (fmt == 1 && bits != 8))
        return 1;
    quant_row(x, D, bits, group, fmt, packed, sz);
    return 0;
}

/*
 * Partition [0, L) into low / vertical / window and write the hybrid cache:
 *   k_codes, v_codes: u8  [B, Hkv, n_lo, D*bits/8]
 *   k_sz, v_sz:       f16 [B, Hkv, n_lo, D/group, 2]
 *   k_hi, v_hi:       bf16 [B, Hkv, n_hi, D]  (vertical rows in ascending
 *                     index order, then the window: window position p in row
 *                     kv + p mod W)
 *   lo_pos:           i32 [B, Hkv, n_lo]  (nullable)
 * with n_lo = L - W - kv and n_hi = kv + W.
 * idx: [B, Hkv, kv] ascending, distinct, each in [0, L - W).
 * Window placement (reading; the pages do not fix a layout): the window is a
 * ring keyed by position, so that sliding it by one token during decode
 * rewrites one row and moves none (hqo_kv_append).  Attention does not
 * depend on the order of the rows.
 */
int hqo_pack_kv(const uint16_t *k, const uint16_t *v, const int32_t *idx, int B, int Hkv,
                int L, int D, int window, int kv, int bits, int group, int fmt, uint8_t *k_codes,
                uint8_t *v_codes, uint16_t *k_sz, uint16_t *v_sz, uint16_t *k_hi,
                uint16_t *v_hi, int32_t *lo_pos)
{
    if ((bits != 4 && bits != 8) || group <= 0 || D % group || D > 512 || window < 0 ||
        kv < 0 || kv > L - window || fmt < 0 || fmt > 1 || (fmt == 1 && bits != 8))
        return 1;
    const int n_lo = L - window - kv, n_hi = kv + window;
    const int row_bytes = D * bits / 8, ng = D / group;
    const long long nbh = (long long)B * Hkv;
    for (long long bh = 0; bh < nbh; ++bh) {
        const int32_t *id = idx + (size_t)bh * kv;
        for (int r = 0; r < kv; ++r)
            if (id[r] < 0 || id[r] >= L - window || (r > 0 && id[r] <= id[r - 1]))
                return 2;
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (long long bh = 0; bh < nbh; ++bh) {
        const int32_t *id = idx + (size_t)bh * kv;
        const uint16_t *kb = k + (size_t)bh * L * D, *vb = v + (size_t)bh * L * D;
        int lo = 0, vi = 0;
        for (int j = 0; j < L; ++j) {
            const uint16_t *kr = kb + (size_t)j * D, *vr = vb + (size_t)j * D;
            if (j >= L - window) {                       /* window row */
                size_t o = ((size_t)bh * n_hi + kv + j % window) * D;
                memcpy(k_hi + o, kr, sizeof(uint16_t) * D);
                memcpy(v_hi + o, vr, sizeof(uint16_t) * D);
            } else if (vi < kv && id[vi] == j) {         /* vertical row */
                size_t o = ((size_t)bh * n_hi + vi) * D;
                memcpy(k_hi + o, kr, sizeof(uint16_t) * D);
                memcpy(v_hi + o, vr, sizeof(uint16_t) * D);
                ++vi;
            } else {                                     /* low row */
                size_t r = (size_t)bh * n_lo + lo;
                quant_row(kr, D, bits, group, fmt, k_codes + r * row_bytes, k_sz + r * 2 * ng);
                quant_row(vr, D, bits, group, fmt, v_codes + r * row_bytes, v_sz + r * 2 * ng);
                if (lo_pos)
                    lo_pos[r] = j;
                ++lo;
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Decode cache maintenance: one new token.                                 */
/* ------------------------------------------------------------------------ */
/*
 * [W] TL;DR: in decode the prefill rule becomes a KV cache compression policy;
 * [B] "What hybrid-precision attention changes": most of the decode cache is
 * low-bit, the selected positions stay in higher precision.  The pages do not
 * say how the cache changes from one token to the next.  Readings taken:
 *   - the vertical set chosen at prefill stays fixed during decode;
 *   - the window is always the W most recent positions, so when token L (the
 *     new one) arrives, position L - W leaves the window and is quantized
 *     with the same row quantizer as the pack (quant_row); it becomes the last
 *     low row, which keeps the low rows in ascending position order because
 *     every earlier low position is below L - W;
 *   - the new token's bf16 K/V take the window row that position L - W held,
 *     row kv + L mod W (the ring placement of hqo_pack_kv);
 *   - W = 0: the new token itself is quantized into the low segment.
 * With these readings, the cache packed from L tokens and then given tokens
 * L .. L+t-1 one by one equals, field for field, the cache packed from L + t
 * tokens with the same vertical set.
 *
 * Cache arrays as in hqo_pack_kv, except that the low arrays hold lo_cap rows
 * per (b, kv head), of which the first n_lo are in use; n_lo = L - W - kv
 * must hold and n_lo < lo_cap.  k_new, v_new: bf16 [B, Hkv, D].  After the
 * call the low segment holds n_lo + 1 rows.
 */
int hqo_kv_append(const uint16_t *k_new, const uint16_t *v_new, int B, int Hkv, int D, int L,
                  int window, int kv, int bits, int group, int fmt, int n_lo, int lo_cap,
                  uint8_t *k_codes, uint8_t *v_codes, uint16_t *k_sz, uint16_t *v_sz,
                  uint16_t *k_hi, uint16_t *v_hi, int32_t *lo_pos)
{
    if ((bits != 4 && bits != 8) || group <= 0 || D % group || D > 512 || window < 0 ||
        kv < 0 || n_lo != L - window - kv || n_lo < 0 || n_lo >= lo_cap || fmt < 0 || fmt > 1 ||
        (fmt == 1 && bits != 8))
        return 1;
    const int row_bytes = D * bits / 8, ng = D / group, n_hi = kv + window;
    for (long long bh = 0; bh < (long long)B * Hkv; ++bh) {
        const uint16_t *kn = k_new + (size_t)bh * D, *vn = v_new + (size_t)bh * D;
        const size_t r = (size_t)bh * lo_cap + n_lo;          /* the new low row */
        if (window == 0) {
            quant_row(kn, D, bits, group, fmt, k_codes + r * row_bytes, k_sz + r * 2 * ng);
            quant_row(vn, D, bits, group, fmt, v_codes + r * row_bytes, v_sz + r * 2 * ng);
            if (lo_pos)
                lo_pos[r] = L;
            continue;
        }
        uint16_t *kh = k_hi + ((size_t)bh * n_hi + kv + L % window) * D;
        uint16_t *vh = v_hi + ((size_t)bh * n_hi + kv + L % window) * D;
        quant_row(kh, D, bits, group, fmt, k_codes + r * row_bytes, k_sz + r * 2 * ng);
        quant_row(vh, D, bits, group, fmt, v_codes + r * row_bytes, v_sz + r * 2 * ng);
        if (lo_pos)
            lo_pos[r] = L - window;
        memcpy(kh, kn, sizeof(uint16_t) * D);
        memcpy(vh, vn, sizeof(uint16_t) * D);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* D1-D2  Decode attention over the hybrid cache.                           */
/* ------------------------------------------------------------------------ */
/*
 * [W] TL;DR and "Key results": decode attends a low-bit cache whose
 * dequantization is fused into attention; the oracle states what that
 * computes: exact softmax attention of the single decode query over all L
 * cached positions, the low ones dequantized (x^ = s * c + z) and the
 * vertical / window ones taken from bf16.  No mask (the cache holds the
 * current token).  Attention does not depend on key order, so the compacted
 * order of the low segment does not matter.
 *
 * q: bf16 [B, Hq, D];  out: double [B, Hq, D];  lse: double [B, Hq] (nullable,
 * natural-log sum of exp of the scaled logits).
 */
static double dequant(const uint8_t *row, const uint16_t *sz, int bits, int group, int fmt, int d)
{
    const int g = d / group;
    if (fmt == 1)                                    /* FP8: s * e4m3(c) */
        return f16_to_f64(sz[2 * g]) * e4m3_to_f64(row[d]);
    int c = bits == 8 ? row[d] : ((row[d >> 1] >> ((d & 1) * 4)) & 0xf);
    return f16_to_f64(sz[2 * g]) * (double)c + f16_to_f64(sz[2 * g + 1]);
}

int hqo_decode_attn(const uint16_t *q, const uint8_t *k_codes, const uint8_t *v_codes,
                    const uint16_t *k_sz, const uint16_t *v_sz, const uint16_t *k_hi,
                    const uint16_t *v_hi, int B, int Hq, int Hkv, int D, int n_lo, int n_hi,
                    int bits, int group, int fmt, double scale, double *out, double *lse)
{
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || n_lo < 0 || n_hi < 0 ||
        n_lo + n_hi <= 0 || (bits != 4 && bits != 8) || group <= 0 || D % group || fmt < 0 ||
        fmt > 1 || (fmt == 1 && bits != 8))
        return 1;
    const int G = Hq / Hkv, row_bytes = D * bits / 8, ng = D / group;
    const long long nbh = (long long)B * Hq;
#pragma omp parallel for schedule(dynamic, 1)
    for (long long bhq = 0; bhq < nbh; ++bhq) {
        const int b = (int)(bhq / Hq), h = (int)(bhq % Hq);
        const size_t bh = (size_t)b * Hkv + h / G;
        const uint16_t *qr = q + (size_t)bhq * D;
        const int T = n_lo + n_hi;
        double *s = (double *)malloc(sizeof(double) * (size_t)T);
        double m = -INFINITY;
        for (int t = 0; t < T; ++t) {
            double acc = 0.0;
            if (t < n_lo) {
                const uint8_t *cr = k_codes + (bh * n_lo + t) * row_bytes;
                const uint16_t *sz = k_sz + (bh * n_lo + t) * 2 * ng;
                for (int d = 0; d < D; ++d)
                    acc += bf16_to_f64(qr[d]) * dequant(cr, sz, bits, group, fmt, d);
            } else {
                const uint16_t *kr = k_hi + (bh * n_hi + (t - n_lo)) * D;
                for (int d = 0; d < D; ++d)
                    acc += bf16_to_f64(qr[d]) * bf16_to_f64(kr[d]);
            }
            s[t] = acc * scale;
            if (s[t] > m) m = s[t];
        }
        double z = 0.0;
        for (int t = 0; t < T; ++t) {
            s[t] = exp(s[t] - m);
            z += s[t];
        }
        double *o = out + (size_t)bhq * D;
        for (int d = 0; d < D; ++d)
            o[d] = 0.0;
        for (int t = 0; t < T; ++t) {
            const double p = s[t] / z;
            if (t < n_lo) {
                const uint8_t *cr = v_codes + (bh * n_lo + t) * row_bytes;
                const uint16_t *sz = v_sz + (bh * n_lo + t) * 2 * ng;
                for (int d = 0; d < D; ++d)
                    o[d] += p * dequant(cr, sz, bits, group, fmt, d);
            } else {
                const uint16_t *vr = v_hi + (bh * n_hi + (t - n_lo)) * D;
                for (int d = 0; d < D; ++d)
                    o[d] += p * bf16_to_f64(vr[d]);
            }
        }
        if (lse)
            lse[bhq] = m + log(z);
        free(s);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* P4  Prefill pre-pass: symmetric INT8 codes for Q (per token) and for the  */
/*     remaining (non-vertical) keys (per block of 64 of them).              */
/* ------------------------------------------------------------------------ */
/*
 * [W] TL;DR / [A]: during prefill the vertical-line tokens and the window stay
 * in full precision and the remaining context is quantized ([B] "What
 * hybrid-precision attention changes": the rest of the context in low
 * precision).  Readings taken: Q gets one scale per (batch, head, query row).
 * K: the keys that are not vertical-line columns, taken in position order
 * (the "remaining" keys; window keys are among them, since every key is
 * outside the window of later queries), get one scale per block of `kblock`
 * consecutive such keys.  A vertical-line key is never quantized.
 * These are integer decisions, so they are taken in binary32, the precision of
 * the kernel that also takes them:
 *   amax = max |x| (exact);  s = fl32(amax / 127), s = 1 when amax == 0;
 *   c = clamp(rne(fl32(x / s)), -127, 127).
 * (A single rounded binary32 division, written with volatile to keep the
 * compiler from fusing or widening it.)
 */
static float q8_scale(const uint16_t *x, int n)
{
    float amax = 0.0f;
    for (int i = 0; i < n; ++i) {
        float a = fabsf((float)bf16_to_f64(x[i]));
        if (a > amax) amax = a;
    }
    if (amax == 0.0f)
        return 1.0f;
    volatile float s = amax / 127.0f;
    return s;
}

static int8_t q8_code(uint16_t xb, float s)
{
    volatile float t = (float)bf16_to_f64(xb) / s;
    float r = nearbyintf(t);
    if (r > 127.0f) r = 127.0f;
    if (r < -127.0f) r = -127.0f;
    return (int8_t)r;
}

/*
 * FP8 low part (fmt 1; a reading for the pages' FP8 "third precision point",
 * wiki summary "Gaps"): the same granularity, symmetric E4M3 codes,
 *   s = fl32(amax / 448), s = 1 when amax == 0;  c = e4m3_rne_sat(fl32(x / s)),
 * the binary32 quotient rounded once more, to E4M3 (nearest even,
 * saturating); the code's bits are stored in the 8-bit array.
 */
static float f8_scale(const uint16_t *x, int n)
{
    float amax = 0.0f;
    for (int i = 0; i < n; ++i) {
        float a = fabsf((float)bf16_to_f64(x[i]));
        if (a > amax) amax = a;
    }
    if (amax == 0.0f)
        return 1.0f;
    volatile float s = amax / 448.0f;
    return s;
}

static int8_t f8_code(uint16_t xb, float s)
{
    volatile float t = (float)bf16_to_f64(xb) / s;
    return (int8_t)f64_to_e4m3_rne_sat((double)t);
}

/* A low-part code as a number: the integer, or the E4M3 value. */
static double low_value(int8_t c, int fmt)
{
    return fmt == 1 ? e4m3_to_f64((uint8_t)c) : (double)c;
}

/*
 * q: bf16 [B, Hq, N, D] -> qi8 [B, Hq, N, D], sq [B, Hq, N].
 * k: bf16 [B, Hkv, N, D], idx [B, Hkv, kv] (ascending) ->
 *    ki8 [B, Hkv, N - kv, D] (the remaining keys, compacted in position order),
 *    sk  [B, Hkv, ceil((N - kv) / kblock)].
 */
int hqo_prefill_quant(const uint16_t *q, const uint16_t *k, const int32_t *idx, int B, int Hq,
                      int Hkv, int N, int D, int kv, int kblock, int fmt, int8_t *qi8, float *sq,
                      int8_t *ki8, float *sk)
{
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || D <= 0 || kblock <= 0 || kv < 0 || kv > N ||
        fmt < 0 || fmt > 1)
        return 1;
    const long long nq = (long long)B * Hq * N;
#pragma omp parallel for schedule(static)
    for (long long r = 0; r < nq; ++r) {
        const uint16_t *x = q + (size_t)r * D;
        float s = fmt == 1 ? f8_scale(x, D) : q8_scale(x, D);
        sq[r] = s;
        for (int d = 0; d < D; ++d)
            qi8[(size_t)r * D + d] = fmt == 1 ? f8_code(x[d], s) : q8_code(x[d], s);
    }
    const int nr = N - kv;                        /* remaining keys per (b, kv head) */
    const int nblk = (nr + kblock - 1) / kblock;
    const long long nbh = (long long)B * Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (long long bh = 0; bh < nbh; ++bh) {
        const int32_t *id = idx + (size_t)bh * kv;
        /* gather the remaining keys, in position order */
        uint16_t *rem = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)nr * D);
        int c = 0, vi = 0;
        for (int j = 0; j < N; ++j) {
            if (vi < kv && id[vi] == j) {
                ++vi;
                continue;
            }
            memcpy(rem + (size_t)c * D, k + ((size_t)bh * N + j) * D, sizeof(uint16_t) * D);
            ++c;
        }
        for (int blk = 0; blk < nblk; ++blk) {
            const int c0 = blk * kblock, n = (nr - c0 < kblock ? nr - c0 : kblock);
            const uint16_t *x = rem + (size_t)c0 * D;
            float s = fmt == 1 ? f8_scale(x, n * D) : q8_scale(x, n * D);
            sk[(size_t)bh * nblk + blk] = s;
            for (int e = 0; e < n * D; ++e)
                ki8[((size_t)bh * nr + c0) * D + e] = fmt == 1 ? f8_code(x[e], s) : q8_code(x[e], s);
        }
        free(rem);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* P5  Hybrid-precision prefill attention.                                  */
/* ------------------------------------------------------------------------ */
/*
 * [A] Prefill stage: a hybrid-precision attention operator that keeps the
 * vertical-line tokens and a local sliding window at full precision and
 * quantizes the rest.  [W] TL;DR: one rule for both phases.  Readings taken:
 * causal attention; for query i and key j <= i the pair is "high" when j is
 * in the window (j > i - W) or j is a vertical column, else "low".  A high
 * logit is q_i . k_j * scale from the bf16 values; a low logit is
 *   (sum_d qi8[i,d] * ki8[c,d]) * sq[i] * sk[c / kblock] * scale
 * with the dot product of the codes exact (integers, or E4M3 values for
 * fmt 1: products of 4-bit significands, summed in double without rounding
 * for D <= 512), where c = j - #(vertical columns < j) is
 * the key's rank among the remaining keys (see the pre-pass).  One exact softmax over all j <= i;
 * the output is sum_j p_ij v_j with v in bf16 and p unrounded.
 *
 * rows: the query rows to compute (nrows of them), or NULL for all N rows;
 * out: double [B, Hq, nrows, D].
 */
int hqo_prefill_attn(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                     const int32_t *idx, const int8_t *qi8, const float *sq, const int8_t *ki8,
                     const float *sk, int B, int Hq, int Hkv, int N, int D, int window, int kv,
                     int kblock, int fmt, double scale, const int32_t *rows, int nrows,
                     double *out)
{
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || N <= 0 || D <= 0 || window < 0 ||
        kv < 0 || kv > N || kblock <= 0 || fmt < 0 || fmt > 1)
        return 1;
    if (!rows)
        nrows = N;
    const int G = Hq / Hkv, nr = N - kv, nblk = (nr + kblock - 1) / kblock;
    const long long nunits = (long long)B * Hq * nrows;
#pragma omp parallel for schedule(dynamic, 4)
    for (long long u = 0; u < nunits; ++u) {
        const long long bhq = u / nrows;
        const int ri = (int)(u % nrows);
        const int b = (int)(bhq / Hq), h = (int)(bhq % Hq);
        const size_t bh = (size_t)b * Hkv + h / G;
        const int i = rows ? rows[ri] : ri;
        const int32_t *id = idx + bh * kv;
        const uint16_t *qr = q + ((size_t)bhq * N + i) * D;
        const int8_t *qc = qi8 + ((size_t)bhq * N + i) * D;
        double *s = (double *)malloc(sizeof(double) * (size_t)(i + 1));
        double m = -INFINITY;
        int vi = 0;
        for (int j = 0; j <= i; ++j) {
            while (vi < kv && id[vi] < j) ++vi;
            const int vert = (vi < kv && id[vi] == j);
            const int hi = (j > i - window) || vert;
            double logit;
            if (hi) {
                const uint16_t *kr = k + (bh * N + j) * D;
                double acc = 0.0;
                for (int d = 0; d < D; ++d)
                    acc += bf16_to_f64(qr[d]) * bf16_to_f64(kr[d]);
                logit = acc * scale;
            } else {
                const int c = j - vi;                  /* vi = #(vertical columns < j) */
                const int8_t *kc = ki8 + (bh * nr + c) * D;
                double acc = 0.0;                      /* exact for both formats */
                for (int d = 0; d < D; ++d)
                    acc += low_value(qc[d], fmt) * low_value(kc[d], fmt);
                logit = acc * (double)sq[(size_t)bhq * N + i] *
                        (double)sk[bh * nblk + c / kblock] * scale;
            }
            s[j] = logit;
            if (logit > m) m = logit;
        }
        double z = 0.0;
        for (int j = 0; j <= i; ++j) {
            s[j] = exp(s[j] - m);
            z += s[j];
        }
        double *o = out + ((size_t)bhq * nrows + ri) * D;
        for (int d = 0; d < D; ++d)
            o[d] = 0.0;
        for (int j = 0; j <= i; ++j) {
            const uint16_t *vr = v + (bh * N + j) * D;
            const double p = s[j] / z;
            for (int d = 0; d < D; ++d)
                o[d] += p * bf16_to_f64(vr[d]);
        }
        free(s);
    }
    return 0;
}

/* Threads the oracle's OpenMP loops use (for the CPU-baseline report). */
int hqo_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
