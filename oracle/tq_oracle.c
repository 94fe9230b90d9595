/*
 * tq_oracle.c -- plain fp64 CPU oracle for TQ4/4 KV-cache compression.
 *
 * TEST INFRASTRUCTURE ONLY: see tq_oracle.h.  Written for a reader who
 * checks it against the method by eye: every step is a direct loop over its
 * definition, with no blocking, fusion or reordering.  Speed is not a goal.
 *
 * Sources of each step:
 *   Key rotation by a normalised Walsh-Hadamard transform:
 *     "TurboQuant 在 AMD GPU 上把長上下文延遲壓下來", section 4;
 *     "UltraQuant：4-bit KV 快取加速長代理", section 「方法怎麼做，白話講」.
 *   Key look-up-table quantisation with a 16-entry table (Lloyd-Max or
 *   re-fitted on ~20 rotated vectors):
 *     "TurboQuant ...", section 2; "UltraQuant ...", 「方法怎麼做，白話講」.
 *   Value uniform quantisation:  "TurboQuant ...", section 2.
 *   The record layout, fp16 norm and group-32 scale/zero are the TQ4/4 cache
 *   format of this repository (its design document lists them as readings).
 */
#include "tq_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* scalar conversions (IEEE 754 binary16 / bfloat16 definitions)       */
/* ------------------------------------------------------------------ */

double orc_bf16_to_double(uint16_t bits)
{
    /* bfloat16 is the top half of an IEEE binary32 */
    uint32_t w = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

double orc_fp16_to_double(uint16_t bits)
{
    int sign = (bits >> 15) & 1;
    int expo = (bits >> 10) & 0x1f;
    int mant = bits & 0x3ff;
    double v;
    if (expo == 0)
        v = ldexp((double)mant, -24); /* subnormal: mant * 2^-24 */
    else if (expo == 31)
        v = mant ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + mant), expo - 25); /* (1024+mant) * 2^(e-15-10) */
    return sign ? -v : v;
}

uint16_t orc_fp16_from_double(double x, int mode)
{
    if (isnan(x))
        return 0x7e00;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    /* rounding of the magnitude: 0 nearest-even, -1 toward zero, +1 away from zero */
    int mag;
    if (mode == 0)
        mag = 0;
    else if ((mode < 0) == (sign != 0))
        mag = +1; /* toward -inf on a negative number grows the magnitude */
    else
        mag = -1;
    if (isinf(a))
        return sign | 0x7c00;
    if (a == 0.0)
        return sign;

    /* a lies in [2^E, 2^(E+1)); binary16 spacing there is 2^(E-10), and
     * below the normal range (E < -14) the spacing is fixed at 2^-24 */
    int e2;
    frexp(a, &e2);
    int E = e2 - 1;
    if (E < -14)
        E = -14;
    double ulp = ldexp(1.0, E - 10);
    double q = a / ulp; /* exact: scaling by a power of two */
    double fl = floor(q);
    double r;
    if (mag == 0) {
        double frac = q - fl;
        if (frac > 0.5 || (frac == 0.5 && fmod(fl, 2.0) != 0.0))
            r = fl + 1.0;
        else
            r = fl;
    } else if (mag < 0) {
        r = fl;
    } else {
        r = (q == fl) ? fl : fl + 1.0;
    }
    double val = r * ulp;
    if (val > 65504.0) /* beyond the largest finite binary16 */
        return (mag < 0) ? (uint16_t)(sign | 0x7bff) : (uint16_t)(sign | 0x7c00);
    /* r in [0, 2048]; the biased exponent field carries naturally when r == 2048,
     * and for the subnormal binade (E == -14, r < 1024) the formula gives r itself */
    uint32_t bits = (uint32_t)((E + 15) << 10) + (uint32_t)(r - 1024.0);
    return (uint16_t)(sign | bits);
}

float orc_fp32_from_double(double x) { return (float)x; /* C conversion: round to nearest */ }

/* ------------------------------------------------------------------ */
/* Lloyd-Max table for N(0,1)                                           */
/* ------------------------------------------------------------------ */

static double std_pdf(double x)
{
    if (isinf(x))
        return 0.0;
    return exp(-0.5 * x * x) / sqrt(2.0 * M_PI);
}

/* P(a < X < b) for X ~ N(0,1), written so that neither tail cancels */
static double std_mass(double a, double b)
{
    const double r2 = sqrt(2.0);
    if (a >= 0.0) /* both in the upper half: difference of upper tails */
        return 0.5 * (erfc(a / r2) - erfc(b / r2));
    if (b <= 0.0) /* both in the lower half: difference of lower tails */
        return 0.5 * (erfc(-b / r2) - erfc(-a / r2));
    return 1.0 - 0.5 * erfc(b / r2) - 0.5 * erfc(-a / r2);
}

int orc_lloyd_max_gaussian16(double c[16], double tol, int max_iter, int *iters_used)
{
    /* Lloyd's two conditions for a minimum-MSE scalar quantiser:
     *   each decision boundary is the midpoint of its two neighbouring levels,
     *   each level is the conditional mean of N(0,1) over its cell:
     *     c_j = (pdf(b_{j-1}) - pdf(b_j)) / (Phi(b_j) - Phi(b_{j-1})).
     * Iterate both from a uniform start until the levels stop moving. */
    double b[17];
    for (int j = 0; j < 16; j++)
        c[j] = (j - 7.5) * 0.33;
    int it;
    for (it = 0; it < max_iter; it++) {
        b[0] = -INFINITY;
        b[16] = INFINITY;
        for (int j = 1; j < 16; j++)
            b[j] = 0.5 * (c[j - 1] + c[j]);
        double change = 0.0;
        for (int j = 0; j < 16; j++) {
            double lo = b[j], hi = b[j + 1];
            double cj = (std_pdf(lo) - std_pdf(hi)) / std_mass(lo, hi);
            double dlt = fabs(cj - c[j]);
            if (dlt > change)
                change = dlt;
            c[j] = cj;
        }
        if (change < tol) {
            it++;
            break;
        }
    }
    if (iters_used)
        *iters_used = it;
    return (it >= max_iter) ? -1 : 0;
}

int orc_default_table(int d, uint16_t out[16])
{
    if (d <= 0)
        return -1;
    double c[16];
    if (orc_lloyd_max_gaussian16(c, 1e-15, 10000000, NULL) != 0)
        return -2;
    /* the rotated unit vector has coordinates of variance 1/d; the table is
     * stored as fp16 (round to nearest) */
    double sigma = 1.0 / sqrt((double)d);
    for (int j = 0; j < 16; j++)
        out[j] = orc_fp16_from_double(c[j] * sigma, 0);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Hadamard                                                             */
/* ------------------------------------------------------------------ */

static int popcount_u32(unsigned v)
{
    int n = 0;
    while (v) {
        n += (int)(v & 1u);
        v >>= 1;
    }
    return n;
}

static int is_pow2(int d) { return d > 0 && (d & (d - 1)) == 0; }

int orc_hadamard(int d, double *H)
{
    if (!is_pow2(d) || !H)
        return -1;
    double s = 1.0 / sqrt((double)d);
    for (int i = 0; i < d; i++)
        for (int j = 0; j < d; j++)
            H[(size_t)i * d + j] = (popcount_u32((unsigned)(i & j)) & 1) ? -s : s;
    return 0;
}

/* The dense normalised matrix of the most recent d, built once by orc_hadamard
 * (the oracle is single-threaded; rebuilding it for every vector only costs time). */
static const double *hadamard_cached(int d)
{
    static double *H = NULL;
    static int Hd = 0;
    if (Hd != d) {
        free(H);
        H = malloc(sizeof(double) * d * d);
        orc_hadamard(d, H);
        Hd = d;
    }
    return H;
}

/* y = H x with the dense matrix (deliberately not a fast transform) */
static void hadamard_apply(int d, const double *H, const double *x, double *y)
{
    for (int i = 0; i < d; i++) {
        double acc = 0.0;
        for (int j = 0; j < d; j++)
            acc += H[(size_t)i * d + j] * x[j];
        y[i] = acc;
    }
}

/* ------------------------------------------------------------------ */
/* keys                                                                 */
/* ------------------------------------------------------------------ */

static int nearest_centroid(double y, const uint16_t *table)
{
    int best = 0;
    double bd = fabs(y - orc_fp16_to_double(table[0]));
    for (int c = 1; c < 16; c++) {
        double dc = fabs(y - orc_fp16_to_double(table[c]));
        if (dc < bd) { /* strict: a tie keeps the lower index */
            bd = dc;
            best = c;
        }
    }
    return best;
}

int orc_encode_k(const uint16_t *k_bf16, int d, const uint16_t *table, uint8_t *idx,
                 uint16_t *norm16, double *y_out)
{
    if (!is_pow2(d) || !k_bf16 || !table || !idx || !norm16)
        return -1;
    double *k = malloc(sizeof(double) * d);
    double ss = 0.0;
    for (int i = 0; i < d; i++) {
        k[i] = orc_bf16_to_double(k_bf16[i]);
        ss += k[i] * k[i];
    }
    double n = sqrt(ss);
    *norm16 = orc_fp16_from_double(n, 0);
    /* y = H_d (k / n) with H_d = S / sqrt(d), S the +-1 Sylvester matrix.
     * The +-1 sums of bf16 values are exact in binary64, so S k is formed
     * first and the single scale 1/(n sqrt(d)) is applied last: a coordinate
     * that is exactly zero (or exactly on a midpoint) stays exact instead of
     * being decided by the rounding noise of a division done beforehand. */
    double denom = n * sqrt((double)d);
    const double *Hs = hadamard_cached(d); /* only its signs are used here */
    for (int i = 0; i < d; i++) {
        double acc = 0.0;
        for (int j = 0; j < d; j++)
            acc += (Hs[(size_t)i * d + j] < 0.0) ? -k[j] : k[j];
        double y = (n > 0.0) ? acc / denom : 0.0;
        idx[i] = (uint8_t)nearest_centroid(y, table);
        if (y_out)
            y_out[i] = y;
    }
    free(k);
    return 0;
}

int orc_decode_k(const uint8_t *idx, uint16_t norm16, int d, const uint16_t *table, double *k_hat)
{
    if (!is_pow2(d) || !idx || !table || !k_hat)
        return -1;
    double *c = malloc(sizeof(double) * d);
    const double *H = hadamard_cached(d);
    double n = orc_fp16_to_double(norm16);
    for (int i = 0; i < d; i++)
        c[i] = orc_fp16_to_double(table[idx[i] & 15]);
    /* H is symmetric and H*H = I, so H also undoes the rotation */
    hadamard_apply(d, H, c, k_hat);
    for (int i = 0; i < d; i++)
        k_hat[i] *= n;
    free(c);
    return 0;
}

/* The unrotated baseline ("TurboQuant 在 AMD GPU 上把長上下文延遲壓下來",
 * section 4: the rotation is there to spread the energy of outlier channels
 * evenly before the quantiser; without it the unit vector's own coordinates
 * go to the table).  Encode: y_i = k_i / n, idx_i = nearest centroid; decode:
 * k_hat = fp16(n) * C[idx]. */
int orc_encode_k_unrotated(const uint16_t *k_bf16, int d, const uint16_t *table, uint8_t *idx,
                           uint16_t *norm16, double *y_out)
{
    if (!is_pow2(d) || !k_bf16 || !table || !idx || !norm16)
        return -1;
    double ss = 0.0;
    for (int i = 0; i < d; i++) {
        double x = orc_bf16_to_double(k_bf16[i]);
        ss += x * x;
    }
    double n = sqrt(ss);
    *norm16 = orc_fp16_from_double(n, 0);
    for (int i = 0; i < d; i++) {
        double y = (n > 0.0) ? orc_bf16_to_double(k_bf16[i]) / n : 0.0;
        idx[i] = (uint8_t)nearest_centroid(y, table);
        if (y_out)
            y_out[i] = y;
    }
    return 0;
}

int orc_decode_k_unrotated(const uint8_t *idx, uint16_t norm16, int d, const uint16_t *table,
                           double *k_hat)
{
    if (!is_pow2(d) || !idx || !table || !k_hat)
        return -1;
    double n = orc_fp16_to_double(norm16);
    for (int i = 0; i < d; i++)
        k_hat[i] = n * orc_fp16_to_double(table[idx[i] & 15]);
    return 0;
}

/* ------------------------------------------------------------------ */
/* values                                                               */
/* ------------------------------------------------------------------ */

int orc_encode_v(const uint16_t *v_bf16, int d, uint8_t *q, uint16_t *scale16,
                 uint16_t *zero16, double *r_out)
{
    if (d <= 0 || d % ORC_VGROUP || !v_bf16 || !q || !scale16 || !zero16)
        return -1;
    for (int g = 0; g < d / ORC_VGROUP; g++) {
        const uint16_t *vg = v_bf16 + g * ORC_VGROUP;
        double mn = orc_bf16_to_double(vg[0]), mx = mn;
        for (int i = 1; i < ORC_VGROUP; i++) {
            double v = orc_bf16_to_double(vg[i]);
            if (v < mn)
                mn = v;
            if (v > mx)
                mx = v;
        }
        /* zero point rounded down and scale rounded up, so that every
         * (v - z)/s lands in [0, 15] */
        uint16_t z16 = orc_fp16_from_double(mn, -1);
        double z = orc_fp16_to_double(z16);
        uint16_t s16 = orc_fp16_from_double((mx - z) / 15.0, +1);
        double s = orc_fp16_to_double(s16);
        zero16[g] = z16;
        scale16[g] = s16;
        for (int i = 0; i < ORC_VGROUP; i++) {
            double v = orc_bf16_to_double(vg[i]);
            double r = (s > 0.0) ? (v - z) / s : 0.0;
            double qr = nearbyint(r); /* default rounding mode: ties to even */
            if (qr < 0.0)
                qr = 0.0;
            if (qr > 15.0)
                qr = 15.0;
            q[g * ORC_VGROUP + i] = (uint8_t)qr;
            if (r_out)
                r_out[g * ORC_VGROUP + i] = r;
        }
    }
    return 0;
}

int orc_decode_v(const uint8_t *q, const uint16_t *scale16, const uint16_t *zero16, int d,
                 double *v_hat)
{
    if (d <= 0 || d % ORC_VGROUP || !q || !scale16 || !zero16 || !v_hat)
        return -1;
    for (int i = 0; i < d; i++) {
        int g = i / ORC_VGROUP;
        v_hat[i] = (double)(q[i] & 15) * orc_fp16_to_double(scale16[g]) +
                   orc_fp16_to_double(zero16[g]);
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* record format of one (block, kv head) entry, 16 tokens               */
/*                                                                      */
/*   offset 0            key codes   [16 tokens][d/2 bytes]             */
/*   offset 8d           key norms   [16 tokens] fp16                   */
/*   offset 8d+32        value codes, 8d bytes (placement below)        */
/*   offset 16d+32       value scales, d bytes: fp16 per (token, group) */
/*   offset 17d+32       value zeros,  d bytes: same placement          */
/*   total 18d + 32 bytes (2336 at d=128, 1184 at d=64)                 */
/*                                                                      */
/* Code byte j of a token holds element 2j in its low nibble and        */
/* element 2j+1 in its high nibble.  Key byte j of token t sits at      */
/* t*(d/2) + j.  Multi-byte fields are little-endian.                   */
/*                                                                      */
/* The pages fix the contents of an entry but not the byte order; the   */
/* placement of the value fields is chosen so that a decode thread      */
/* finds its operands contiguous:                                       */
/*   value byte j of token t, with pair p = t/2, e = t%2, m = j/8,      */
/*   r = j%8, sits at (8p + r)*(d/8) + 4*(m/2) + 2e + (m%2);            */
/*   the scale (and zero) of token t, group G, with c = (t%8)/2 and     */
/*   u = 2*(t/8) + t%2, sits at 2*(4*(c*(d/32) + G) + u) within its     */
/*   area.                                                              */
/* ------------------------------------------------------------------ */

size_t orc_record_bytes(int d)
{
    return (size_t)ORC_BLOCK * (size_t)d / 2 * 2 + ORC_BLOCK * 2 + (size_t)2 * d;
}

static size_t off_knorm(int d) { return (size_t)ORC_BLOCK * d / 2; }
static size_t off_vcodes(int d) { return off_knorm(d) + ORC_BLOCK * 2; }
static size_t off_vscale(int d) { return off_vcodes(d) + (size_t)ORC_BLOCK * d / 2; }
static size_t off_vzero(int d) { return off_vscale(d) + (size_t)d; }

/* offset of value code byte j of token t within the value-code area: chunk
 * 8p + ((r + 2p) mod 8) of d/8 bytes (token pair p's chunks rotated by 2p),
 * byte 4 (m/2) + 2e + (m mod 2) of it */
static size_t vcode_pos(int d, int t, int j)
{
    int p = t / 2, e = t % 2, m = j / 8, r = j % 8;
    return (size_t)(8 * p + (r + 2 * p) % 8) * (d / 8) + 4 * (m / 2) + 2 * e + (m % 2);
}

/* offset of the scale (or zero) of token t, group G within its area */
static size_t group_pos(int d, int t, int G)
{
    int c = (t % 8) / 2, u = 2 * (t / 8) + t % 2;
    return (size_t)2 * (4 * (c * (d / ORC_VGROUP) + G) + u);
}

static void put_u16(uint8_t *p, uint16_t v)
{
    p[0] = (uint8_t)(v & 0xff);
    p[1] = (uint8_t)(v >> 8);
}

static uint16_t get_u16(const uint8_t *p) { return (uint16_t)(p[0] | (p[1] << 8)); }

int orc_pack_token(uint8_t *record, int d, int offset, const uint8_t *kidx, uint16_t knorm,
                   const uint8_t *vq, const uint16_t *vscale, const uint16_t *vzero)
{
    if (!record || offset < 0 || offset >= ORC_BLOCK || d <= 0 || d % ORC_VGROUP)
        return -1;
    uint8_t *kc = record + (size_t)offset * (d / 2);
    uint8_t *vc = record + off_vcodes(d);
    for (int j = 0; j < d / 2; j++) {
        kc[j] = (uint8_t)((kidx[2 * j] & 15) | ((kidx[2 * j + 1] & 15) << 4));
        vc[vcode_pos(d, offset, j)] = (uint8_t)((vq[2 * j] & 15) | ((vq[2 * j + 1] & 15) << 4));
    }
    put_u16(record + off_knorm(d) + 2 * offset, knorm);
    for (int g = 0; g < d / ORC_VGROUP; g++) {
        put_u16(record + off_vscale(d) + group_pos(d, offset, g), vscale[g]);
        put_u16(record + off_vzero(d) + group_pos(d, offset, g), vzero[g]);
    }
    return 0;
}

int orc_unpack_token(const uint8_t *record, int d, int offset, uint8_t *kidx, uint16_t *knorm,
                     uint8_t *vq, uint16_t *vscale, uint16_t *vzero)
{
    if (!record || offset < 0 || offset >= ORC_BLOCK || d <= 0 || d % ORC_VGROUP)
        return -1;
    const uint8_t *kc = record + (size_t)offset * (d / 2);
    const uint8_t *vc = record + off_vcodes(d);
    for (int j = 0; j < d / 2; j++) {
        uint8_t vb = vc[vcode_pos(d, offset, j)];
        kidx[2 * j] = kc[j] & 15;
        kidx[2 * j + 1] = kc[j] >> 4;
        vq[2 * j] = vb & 15;
        vq[2 * j + 1] = vb >> 4;
    }
    *knorm = get_u16(record + off_knorm(d) + 2 * offset);
    for (int g = 0; g < d / ORC_VGROUP; g++) {
        vscale[g] = get_u16(record + off_vscale(d) + group_pos(d, offset, g));
        vzero[g] = get_u16(record + off_vzero(d) + group_pos(d, offset, g));
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* paged cache                                                          */
/* ------------------------------------------------------------------ */

static const uint16_t *head_table(const uint16_t *tables, const uint16_t *deflt, int h)
{
    return tables ? tables + 16 * h : deflt;
}

int orc_quantize_append(const uint16_t *K, const uint16_t *V, int T, int Hkv, int d,
                        const int32_t *block_table, int num_seqs, int max_blocks,
                        const int32_t *slots, const uint16_t *tables, uint8_t *cache,
                        int num_blocks, double *ky, double *vr)
{
    return orc_quantize_append_ex(K, V, T, Hkv, d, block_table, num_seqs, max_blocks, slots, tables,
                                  cache, num_blocks, ky, vr, 1);
}

int orc_quantize_append_ex(const uint16_t *K, const uint16_t *V, int T, int Hkv, int d,
                           const int32_t *block_table, int num_seqs, int max_blocks,
                           const int32_t *slots, const uint16_t *tables, uint8_t *cache,
                           int num_blocks, double *ky, double *vr, int rotate)
{
    if (T < 0 || Hkv <= 0 || !is_pow2(d) || d % ORC_VGROUP || !slots || !cache)
        return -1;
    uint16_t deflt[16];
    if (!tables && orc_default_table(d, deflt) != 0)
        return -2;
    size_t rec = orc_record_bytes(d);
    uint8_t *kidx = malloc(d), *vq = malloc(d);
    uint16_t *vs = malloc(sizeof(uint16_t) * d / ORC_VGROUP);
    uint16_t *vz = malloc(sizeof(uint16_t) * d / ORC_VGROUP);
    int rc = 0;
    for (int t = 0; t < T; t++) {
        int32_t slot = slots[t];
        if (slot < 0)
            continue; /* padding token: nothing is written */
        int32_t phys;
        if (block_table) {
            int64_t cap = (int64_t)max_blocks * ORC_BLOCK;
            int64_t seq = slot / cap, pos = slot % cap;
            if (seq >= num_seqs) {
                rc = -3;
                continue;
            }
            int32_t blk = block_table[seq * max_blocks + pos / ORC_BLOCK];
            phys = blk * ORC_BLOCK + (int32_t)(pos % ORC_BLOCK);
        } else {
            phys = slot;
        }
        int32_t blk = phys / ORC_BLOCK, off = phys % ORC_BLOCK;
        if (phys < 0 || blk >= num_blocks) {
            rc = -3;
            continue;
        }
        for (int h = 0; h < Hkv; h++) {
            const uint16_t *k = K + ((size_t)t * Hkv + h) * d;
            const uint16_t *v = V + ((size_t)t * Hkv + h) * d;
            uint16_t kn;
            double *kyp = ky ? ky + ((size_t)t * Hkv + h) * d : NULL;
            double *vrp = vr ? vr + ((size_t)t * Hkv + h) * d : NULL;
            if (rotate)
                orc_encode_k(k, d, head_table(tables, deflt, h), kidx, &kn, kyp);
            else
                orc_encode_k_unrotated(k, d, head_table(tables, deflt, h), kidx, &kn, kyp);
            orc_encode_v(v, d, vq, vs, vz, vrp);
            uint8_t *record = cache + ((size_t)blk * Hkv + h) * rec;
            orc_pack_token(record, d, off, kidx, kn, vq, vs, vz);
        }
    }
    free(kidx);
    free(vq);
    free(vs);
    free(vz);
    return rc;
}

int orc_dequantize(const uint8_t *cache, int num_blocks, int Hkv, int d, const uint16_t *tables,
                   const int32_t *block_tables, int max_blocks, const int32_t *seq_lens, int B,
                   int max_len, double *Khat, double *Vhat)
{
    return orc_dequantize_ex(cache, num_blocks, Hkv, d, tables, block_tables, max_blocks, seq_lens,
                             B, max_len, Khat, Vhat, 1);
}

int orc_dequantize_ex(const uint8_t *cache, int num_blocks, int Hkv, int d, const uint16_t *tables,
                      const int32_t *block_tables, int max_blocks, const int32_t *seq_lens, int B,
                      int max_len, double *Khat, double *Vhat, int rotate)
{
    if (!cache || !block_tables || !seq_lens || !Khat || !Vhat || !is_pow2(d) ||
        d % ORC_VGROUP)
        return -1;
    uint16_t deflt[16];
    if (!tables && orc_default_table(d, deflt) != 0)
        return -2;
    size_t rec = orc_record_bytes(d);
    size_t total = (size_t)B * max_len * Hkv * d;
    memset(Khat, 0, sizeof(double) * total);
    memset(Vhat, 0, sizeof(double) * total);
    uint8_t *kidx = malloc(d), *vq = malloc(d);
    uint16_t *vs = malloc(sizeof(uint16_t) * d / ORC_VGROUP);
    uint16_t *vz = malloc(sizeof(uint16_t) * d / ORC_VGROUP);
    int rc = 0;
    for (int b = 0; b < B; b++) {
        int L = seq_lens[b];
        if (L > max_len || L > max_blocks * ORC_BLOCK) {
            rc = -3;
            L = 0;
        }
        for (int t = 0; t < L; t++) {
            int32_t blk = block_tables[(size_t)b * max_blocks + t / ORC_BLOCK];
            if (blk < 0 || blk >= num_blocks) {
                rc = -3;
                continue;
            }
            for (int h = 0; h < Hkv; h++) {
                const uint8_t *record = cache + ((size_t)blk * Hkv + h) * rec;
                uint16_t kn;
                orc_unpack_token(record, d, t % ORC_BLOCK, kidx, &kn, vq, vs, vz);
                size_t o = (((size_t)b * max_len + t) * Hkv + h) * d;
                if (rotate)
                    orc_decode_k(kidx, kn, d, head_table(tables, deflt, h), Khat + o);
                else
                    orc_decode_k_unrotated(kidx, kn, d, head_table(tables, deflt, h), Khat + o);
                orc_decode_v(vq, vs, vz, d, Vhat + o);
            }
        }
    }
    free(kidx);
    free(vq);
    free(vs);
    free(vz);
    return rc;
}

/* ------------------------------------------------------------------ */
/* attention                                                            */
/* ------------------------------------------------------------------ */

int orc_attention(const uint16_t *q, int B, int Hq, int Hkv, int d, const double *Khat,
                  const double *Vhat, int max_len, const int32_t *seq_lens, double scale,
                  double *out)
{
    if (!q || !Khat || !Vhat || !seq_lens || !out || Hkv <= 0 || Hq % Hkv)
        return -1;
    int G = Hq / Hkv;
    double *a = malloc(sizeof(double) * (max_len > 0 ? max_len : 1));
    double *qd = malloc(sizeof(double) * d);
    for (int b = 0; b < B; b++) {
        int L = seq_lens[b];
        if (L > max_len)
            L = max_len;
        for (int h = 0; h < Hq; h++) {
            int kv = h / G;
            double *o = out + ((size_t)b * Hq + h) * d;
            for (int i = 0; i < d; i++) {
                qd[i] = orc_bf16_to_double(q[((size_t)b * Hq + h) * d + i]);
                o[i] = 0.0;
            }
            if (L <= 0)
                continue;
            /* logits a_t = scale * <q, k_hat_t> */
            double amax = -INFINITY;
            for (int t = 0; t < L; t++) {
                const double *k = Khat + (((size_t)b * max_len + t) * Hkv + kv) * d;
                double acc = 0.0;
                for (int i = 0; i < d; i++)
                    acc += qd[i] * k[i];
                a[t] = scale * acc;
                if (a[t] > amax)
                    amax = a[t];
            }
            /* softmax with the maximum subtracted, then the weighted sum of v_hat */
            double denom = 0.0;
            for (int t = 0; t < L; t++) {
                a[t] = exp(a[t] - amax);
                denom += a[t];
            }
            for (int t = 0; t < L; t++) {
                const double *v = Vhat + (((size_t)b * max_len + t) * Hkv + kv) * d;
                double p = a[t] / denom;
                for (int i = 0; i < d; i++)
                    o[i] += p * v[i];
            }
        }
    }
    free(a);
    free(qd);
    return 0;
}

/* Chunked-prefill attention -- the prompt chunks of multi-turn serving, whose
 * reuse of a cached prefix is what the pages measure ("TurboQuant 在 AMD GPU 上把
 * 長上下文延遲壓下來", summary table, prefix-cache hit rate; "UltraQuant：4-bit
 * KV 快取加速長代理", 「它實際證明了什麼」, late-round TTFT from cache residency).
 * Sequence b's q_len = q_start[b+1] - q_start[b]
 * newest tokens are the chunk, already in the cache (seq_lens[b] tokens in
 * all), and chunk token i (position p = seq_lens[b] - q_len + i) attends to
 * the cached tokens [0, p] -- causal within the chunk.  q bf16 [T][Hq][d]
 * with T = q_start[B]; out fp64 [T][Hq][d]. */
int orc_prefill_attention(const uint16_t *q, const int32_t *q_start, int B, int Hq, int Hkv, int d,
                          const double *Khat, const double *Vhat, int max_len,
                          const int32_t *seq_lens, double scale, double *out)
{
    if (!q || !q_start || !Khat || !Vhat || !seq_lens || !out || Hkv <= 0 || Hq % Hkv)
        return -1;
    int G = Hq / Hkv;
    double *a = malloc(sizeof(double) * (max_len > 0 ? max_len : 1));
    double *qd = malloc(sizeof(double) * d);
    int rc = 0;
    for (int b = 0; b < B; b++) {
        int qlen = q_start[b + 1] - q_start[b];
        int L = seq_lens[b];
        for (int i = 0; i < qlen; i++) {
            int tok = q_start[b] + i;
            int n = L - qlen + i + 1; /* keys this query sees: positions 0 .. L - qlen + i */
            if (n > max_len || n < 1) {
                rc = -3;
                n = 0;
            }
            for (int h = 0; h < Hq; h++) {
                int kv = h / G;
                double *o = out + ((size_t)tok * Hq + h) * d;
                for (int e = 0; e < d; e++) {
                    qd[e] = orc_bf16_to_double(q[((size_t)tok * Hq + h) * d + e]);
                    o[e] = 0.0;
                }
                if (n <= 0)
                    continue;
                double amax = -INFINITY;
                for (int t = 0; t < n; t++) {
                    const double *k = Khat + (((size_t)b * max_len + t) * Hkv + kv) * d;
                    double acc = 0.0;
                    for (int e = 0; e < d; e++)
                        acc += qd[e] * k[e];
                    a[t] = scale * acc;
                    if (a[t] > amax)
                        amax = a[t];
                }
                double denom = 0.0;
                for (int t = 0; t < n; t++) {
                    a[t] = exp(a[t] - amax);
                    denom += a[t];
                }
                for (int t = 0; t < n; t++) {
                    const double *v = Vhat + (((size_t)b * max_len + t) * Hkv + kv) * d;
                    double pr = a[t] / denom;
                    for (int e = 0; e < d; e++)
                        o[e] += pr * v[e];
                }
            }
        }
    }
    free(a);
    free(qd);
    return rc;
}

/* ------------------------------------------------------------------ */
/* calibrated table                                                     */
/* ------------------------------------------------------------------ */

int orc_rotated_unit_samples(const uint16_t *k_bf16, int n_vec, int d, double *out)
{
    if (!k_bf16 || !out || !is_pow2(d) || n_vec < 0)
        return -1;
    uint16_t dummy_table[16] = {0};
    uint8_t *idx = malloc(d);
    for (int n = 0; n < n_vec; n++) {
        uint16_t n16;
        /* the same rotation as the key encoder; its codes are discarded */
        orc_encode_k(k_bf16 + (size_t)n * d, d, dummy_table, idx, &n16, out + (size_t)n * d);
    }
    free(idx);
    return 0;
}

static int cmp_double(const void *a, const void *b)
{
    double x = *(const double *)a, y = *(const double *)b;
    return (x > y) - (x < y);
}

int orc_kmeans_table(const double *samples, int n, const uint16_t *init, int max_iter, uint16_t out[16])
{
    if (!samples || !init || !out || n < 0 || max_iter < 0)
        return -1;
    double c[16];
    for (int j = 0; j < 16; j++)
        c[j] = orc_fp16_to_double(init[j]);
    int *assign = malloc(sizeof(int) * (n > 0 ? n : 1));
    for (int i = 0; i < n; i++)
        assign[i] = -1;
    int it;
    for (it = 0; it < max_iter; it++) {
        /* assignment step: nearest level, ties to the lower index */
        int changed = 0;
        for (int i = 0; i < n; i++) {
            int best = 0;
            double bd = fabs(samples[i] - c[0]);
            for (int j = 1; j < 16; j++) {
                double dj = fabs(samples[i] - c[j]);
                if (dj < bd) {
                    bd = dj;
                    best = j;
                }
            }
            if (best != assign[i]) {
                assign[i] = best;
                changed = 1;
            }
        }
        if (!changed)
            break;
        /* update step: each level moves to the mean of its cell */
        double sum[16] = {0};
        int cnt[16] = {0};
        for (int i = 0; i < n; i++) {
            sum[assign[i]] += samples[i];
            cnt[assign[i]]++;
        }
        for (int j = 0; j < 16; j++)
            if (cnt[j] > 0)
                c[j] = sum[j] / cnt[j];
    }
    qsort(c, 16, sizeof(double), cmp_double);
    for (int j = 0; j < 16; j++)
        out[j] = orc_fp16_from_double(c[j], 0);
    free(assign);
    return it;
}
