/*
 * rq_oracle.c -- plain, slow, fp64 CPU oracle for ResidualQuant decode
 * attention (INT4 anchor + INT2 residual KV cache).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * bench's CPU-baseline leg may load this library.  The product path (the
 * CUDA library under decode_attention_14_b200/) never links, includes or
 * calls it, and this file includes nothing from there.
 *
 * What it follows ("ResidualQuant: KV Cache Quantization for Looped
 * Transformers with 2-Bit Residuals", arXiv 2610.10381 abstract; the
 * ai4snews summary of it, paragraphs 1-4; the agihunt summary, "Confirmed"
 * bullets 2-3):
 *   - the final loop of a loop group is the shared anchor, stored at INT4;
 *   - every other loop is stored as a low-bit (INT2) residual against it;
 *   - least-squares scaling of the anchor before subtraction, with the
 *     coefficient stored in BF16 (ai4snews para. 2 counts these BF16
 *     coefficients in the storage budget);
 *   - an orthogonal rotation applied to the residuals only, never to the
 *     KV states (ai4snews para. 1);
 *   - grouped quantization, group size 16, with an FP8 scale and an FP8
 *     offset per group (ai4snews para. 2);
 *   - reconstruction from two reads: anchor + one residual (ai4snews
 *     para. 3).
 * Readings where the pages are silent:
 *   FP8 = OCP E4M3 (bias 7, max 448, no inf), round-to-nearest-even with
 *   saturation to +-448; "offset" = the group minimum; scale =
 *   (max-min)/(2^b-1) taken from the unrounded min/max; codes are computed
 *   against the rounded scale and min, ties to even, clamped to
 *   [0, 2^b-1]; a zero scale gives all-zero codes; the residual uses the
 *   stored (BF16-rounded) coefficient; the rotation is the Sylvester
 *   Hadamard matrix times a diagonal of seeded signs, divided by sqrt(d),
 *   with sign j = top bit of splitmix64(seed + j).
 *
 * Every function here is written from those definitions, step by step, in
 * fp64, with no blocking, fusion or reordering.  The rotation is applied as
 * an explicit O(d^2) matrix product (not a butterfly), in the factored form
 * of its definition: the +-1 matrix H diag(sigma) times the vector (an exact
 * signed sum for the cache's values), then the scalar 1/sqrt(d) once.
 *
 * Parity pins: see tests/test_oracle_pins.py (and tests/test_oracle_ablation.py
 * for orc_encode_ablation, the abstract's ablation variants: previous-loop
 * chained anchor, norm-ratio and no scaling).  Every function below is
 * pinned there against something other than itself.
 *
 * Logical record format (what this oracle produces and what the CUDA
 * library's export call returns):
 *   codes : d*b/8 bytes; element i sits in little-endian 32-bit word
 *           i/(32/b) at bit offset (i mod (32/b))*b  (equivalently byte
 *           i*b/8, bit (i*b)%8, LSB first).
 *   meta  : d/g groups x 2 bytes: [scale_e4m3, min_e4m3] per group.
 *   coef  : one BF16 (uint16 bits) per residual record.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <float.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_EXPORT __attribute__((visibility("default")))

/* Relative width of the window around a rounding boundary: elements whose
 * pre-rounding value lies within 1e-6 relative of a boundary are flagged and
 * left out of the bit-exact comparison of codes. */
static const double ORC_NEAR_REL = 1e-6;

/* ------------------------------------------------------------------ */
/* FP8 E4M3 (OCP): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits.   */
/* E=0: subnormal, value M * 2^-9.  E=1..15: 2^(E-7) * (1 + M/8).       */
/* E=15,M=7 (0x7F/0xFF) is NaN.  Largest finite = 448 (0x7E).           */
/* ------------------------------------------------------------------ */
ORC_EXPORT double orc_fp8_value(uint8_t code)
{
    int s = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* Round to the nearest E4M3 value, ties to the code with an even mantissa,
 * values at or beyond the largest finite magnitude saturate to +-448.
 * Plain table walk over the 127 non-negative finite values.
 * If near != NULL it is set to 1 when |v| lies within ORC_NEAR_REL
 * (relative) of the midpoint between two neighbouring E4M3 values. */
ORC_EXPORT uint8_t orc_fp8_round(double v, int *near)
{
    double a = fabs(v);
    uint8_t sign = (v < 0 || (v == 0 && signbit(v))) ? 0x80 : 0x00;
    int k, best = 0;
    if (near)
        *near = 0;
    if (isnan(v))
        return 0x7F;
    /* near-boundary flag: nearest midpoint among all neighbouring pairs */
    if (near) {
        for (k = 0; k < 126; k++) {
            double lo = orc_fp8_value((uint8_t)k), hi = orc_fp8_value((uint8_t)(k + 1));
            double mid = 0.5 * (lo + hi);
            double den = fmax(a, mid);
            if (fabs(a - mid) <= ORC_NEAR_REL * den)
                *near = 1;
        }
    }
    if (a >= 448.0)
        return (uint8_t)(sign | 0x7E);
    /* largest code whose value is <= a */
    for (k = 0; k <= 126; k++) {
        if (orc_fp8_value((uint8_t)k) <= a)
            best = k;
        else
            break;
    }
    if (orc_fp8_value((uint8_t)best) == a)
        return (uint8_t)(sign | best);
    {
        double lo = orc_fp8_value((uint8_t)best), hi = orc_fp8_value((uint8_t)(best + 1));
        double mid = 0.5 * (lo + hi);
        int pick;
        if (a < mid)
            pick = best;
        else if (a > mid)
            pick = best + 1;
        else
            pick = (best & 1) ? best + 1 : best;  /* tie: even mantissa LSB */
        return (uint8_t)(sign | pick);
    }
}

/* ------------------------------------------------------------------ */
/* BF16: the top 16 bits of an IEEE binary32; 8 significant bits.        */
/* ------------------------------------------------------------------ */
ORC_EXPORT double orc_bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round a double to the nearest BF16 value, ties to even, in ONE rounding
 * step (no detour through binary32).  Returns the BF16 bit pattern.
 * near: set when |v| is within ORC_NEAR_REL (relative) of a midpoint. */
ORC_EXPORT uint16_t orc_bf16_round(double v, int *near)
{
    double a = fabs(v), q, u, r, res, mid;
    int e;
    float f;
    uint32_t bits;
    if (near)
        *near = 0;
    if (isnan(v))
        return 0x7FC0;
    if (a == 0.0) {
        f = (float)v;
        memcpy(&bits, &f, 4);
        return (uint16_t)(bits >> 16);
    }
    frexp(a, &e);                 /* a = m * 2^e, m in [0.5, 1) */
    if (e - 1 >= -126)
        q = ldexp(1.0, e - 8);    /* spacing of 8-significant-bit values */
    else
        q = ldexp(1.0, -133);     /* BF16 subnormal spacing */
    u = a / q;                    /* exact: division by a power of two */
    r = nearbyint(u);             /* default mode: nearest, ties to even */
    res = r * q;
    mid = (floor(u) + 0.5) * q;
    if (near && fabs(a - mid) <= ORC_NEAR_REL * fmax(a, mid))
        *near = 1;
    if (res > 3.3895313892515355e38)
        res = INFINITY;
    f = (float)(v < 0 ? -res : res);  /* exact: res has <= 8 significant bits */
    memcpy(&bits, &f, 4);
    return (uint16_t)(bits >> 16);
}

/* ------------------------------------------------------------------ */
/* Rotation R = H_d * diag(sigma) / sqrt(d)                              */
/* H_d: Sylvester Hadamard, H_ij = (-1)^popcount(i & j).                 */
/* sigma_j = -1 if the top bit of splitmix64(seed + j) is set, else +1.  */
/* splitmix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number */
/* generators", OOPSLA 2014): add the golden gamma 0x9E3779B97F4A7C15,   */
/* then xor-shift-multiply mix with constants 0xBF58476D1CE4E5B9 and     */
/* 0x94D049BB133111EB (shifts 30, 27, 31).                               */
/* ------------------------------------------------------------------ */
ORC_EXPORT uint64_t orc_splitmix64(uint64_t x)
{
    uint64_t z = x + 0x9E3779B97F4A7C15ULL;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

ORC_EXPORT void orc_rotation_signs(uint64_t seed, int d, double *sigma)
{
    int j;
    for (j = 0; j < d; j++)
        sigma[j] = (orc_splitmix64(seed + (uint64_t)j) >> 63) ? -1.0 : 1.0;
}

static int popcount_int(unsigned x)
{
    int c = 0;
    while (x) {
        c += (int)(x & 1u);
        x >>= 1;
    }
    return c;
}

/* R = c * S with S = H_d diag(sigma) (entries +-1) and c = 1/sqrt(d) when
 * rotating; S = I and c = 1 otherwise.  d is a power of two (Sylvester), so
 * 1/sqrt(d) = 2^(-k/2) for d = 2^k: an exact power of two for even k, else
 * sqrt(1/2) (correctly rounded by IEEE sqrt) times an exact power of two --
 * the correctly rounded value either way. */
ORC_EXPORT double orc_rotation_scale(int d, int rotate)
{
    int k = 0;
    if (!rotate)
        return 1.0;
    while ((1 << k) < d)
        k++;
    return (k % 2) ? sqrt(0.5) * ldexp(1.0, -(k - 1) / 2) : ldexp(1.0, -k / 2);
}

/* S[i*d + j]: the +-1 matrix H_d diag(sigma), or the identity. */
ORC_EXPORT void orc_rotation_signs_matrix(uint64_t seed, int d, int rotate, double *S)
{
    int i, j;
    double *sigma = (double *)malloc(sizeof(double) * (size_t)d);
    orc_rotation_signs(seed, d, sigma);
    for (i = 0; i < d; i++)
        for (j = 0; j < d; j++) {
            if (!rotate)
                S[i * d + j] = (i == j) ? 1.0 : 0.0;
            else
                S[i * d + j] = ((popcount_int((unsigned)(i & j)) & 1) ? -1.0 : 1.0) * sigma[j];
        }
    free(sigma);
}

/* R[i*d + j] = c * S[i*d + j]; rotate == 0 gives the identity. */
ORC_EXPORT void orc_rotation_matrix(uint64_t seed, int d, int rotate, double *R)
{
    int i;
    double c = orc_rotation_scale(d, rotate);
    orc_rotation_signs_matrix(seed, d, rotate, R);
    for (i = 0; i < d * d; i++)
        R[i] *= c;
}

/* y = R v = c * (S v): the signed sum of S's +-1 entries times v first, then
 * one multiplication by c.  For the cache's values (sums of a bounded number
 * of binary digits) the signed sum is exact, so y carries a single rounding. */
static void rotate_vec(const double *S, double c, int d, const double *v, double *y)
{
    int i, j;
    for (i = 0; i < d; i++) {
        double acc = 0.0;
        for (j = 0; j < d; j++)
            acc += S[i * d + j] * v[j];
        y[i] = c * acc;
    }
}

/* x = R^T v = c * (S^T v): (R^T v)_i = sum_j R_ji v_j. */
static void rotate_back(const double *S, double c, int d, const double *v, double *x)
{
    int i, j;
    for (i = 0; i < d; i++) {
        double acc = 0.0;
        for (j = 0; j < d; j++)
            acc += S[j * d + i] * v[j];
        x[i] = c * acc;
    }
}

/* ------------------------------------------------------------------ */
/* Grouped asymmetric quantizer Q_{b,g} on one group of g values.        */
/*   mn = min, mx = max, sigma = (mx - mn) / (2^b - 1)                   */
/*   s8 = fp8(sigma), m8 = fp8(mn)                                        */
/*   s8 == 0 -> all codes 0; else c = clamp(rint((x - m8)/s8), 0, 2^b-1) */
/*   dequant: m8 + c * s8                                                */
/* Flags: meta_flag bit0 = scale near an FP8 boundary, bit1 = min near a  */
/* boundary; elem_flag[i] = 1 when x_i lies within ORC_NEAR_REL of a code */
/* boundary m8 + (k + 1/2) s8 (relative to max(|x|, |boundary|, s8)).    */
/* ------------------------------------------------------------------ */
ORC_EXPORT void orc_quantize_group(const double *x, int g, int bits,
                                   uint8_t *codes, uint8_t *s8_out, uint8_t *m8_out,
                                   uint8_t *elem_flag, uint8_t *meta_flag)
{
    int i, ns, nm, qmax = (1 << bits) - 1;
    double mn = x[0], mx = x[0], sig, s8, m8;
    uint8_t s8c, m8c;
    for (i = 1; i < g; i++) {
        if (x[i] < mn) mn = x[i];
        if (x[i] > mx) mx = x[i];
    }
    sig = (mx - mn) / (double)qmax;
    /* "+ 0.0" turns a -0 minimum into +0, so a zero minimum always encodes
     * as 0x00 whatever the sign of the zero that produced it. */
    s8c = orc_fp8_round(sig, &ns);
    m8c = orc_fp8_round(mn + 0.0, &nm);
    s8 = orc_fp8_value(s8c);
    m8 = orc_fp8_value(m8c);
    *s8_out = s8c;
    *m8_out = m8c;
    if (meta_flag)
        *meta_flag = (uint8_t)((ns ? 1 : 0) | (nm ? 2 : 0));
    for (i = 0; i < g; i++) {
        int c = 0, near = 0;
        if (s8 != 0.0) {
            double u = (x[i] - m8) / s8;
            double r = nearbyint(u);
            int kb;
            double beta;
            if (r < 0) r = 0;
            if (r > qmax) r = qmax;
            c = (int)r;
            /* nearest interior code boundary: u lies in [floor(u), floor(u)+1),
             * so the closest half-integer is floor(u) + 1/2; clamp it to the
             * boundaries that separate valid codes, k + 1/2 for k < qmax. */
            kb = (int)floor(u);
            if (kb < 0) kb = 0;
            if (kb > qmax - 1) kb = qmax - 1;
            beta = m8 + (kb + 0.5) * s8;
            if (fabs(x[i] - beta) <= ORC_NEAR_REL * fmax(fmax(fabs(x[i]), fabs(beta)), s8))
                near = 1;
        }
        codes[i] = (uint8_t)c;
        if (elem_flag)
            elem_flag[i] = (uint8_t)near;
    }
}

/* Pack one record's codes: element i -> byte (i*b)/8, bit (i*b)%8. */
ORC_EXPORT void orc_pack(const uint8_t *codes, int d, int bits, uint8_t *out)
{
    int i;
    memset(out, 0, (size_t)(d * bits / 8));
    for (i = 0; i < d; i++) {
        int bitpos = i * bits;
        out[bitpos / 8] |= (uint8_t)((codes[i] & ((1 << bits) - 1)) << (bitpos % 8));
    }
}

ORC_EXPORT void orc_unpack(const uint8_t *packed, int d, int bits, uint8_t *codes)
{
    int i;
    for (i = 0; i < d; i++) {
        int bitpos = i * bits;
        codes[i] = (uint8_t)((packed[bitpos / 8] >> (bitpos % 8)) & ((1 << bits) - 1));
    }
}

/* Dequantize one record (codes packed, meta = d/g pairs). */
ORC_EXPORT void orc_dequant(const uint8_t *packed, const uint8_t *meta, int d, int g, int bits,
                            double *out)
{
    int i;
    uint8_t *codes = (uint8_t *)malloc((size_t)d);
    orc_unpack(packed, d, bits, codes);
    for (i = 0; i < d; i++) {
        int grp = i / g;
        double s8 = orc_fp8_value(meta[2 * grp]);
        double m8 = orc_fp8_value(meta[2 * grp + 1]);
        out[i] = m8 + codes[i] * s8;
    }
    free(codes);
}

/* Quantize a whole record of d values with group size g. */
static void quantize_record(const double *x, int d, int g, int bits,
                            uint8_t *packed, uint8_t *meta,
                            uint8_t *elem_flag, uint8_t *meta_flag)
{
    int grp;
    uint8_t *codes = (uint8_t *)malloc((size_t)d);
    for (grp = 0; grp < d / g; grp++)
        orc_quantize_group(x + grp * g, g, bits, codes + grp * g,
                           &meta[2 * grp], &meta[2 * grp + 1],
                           elem_flag ? elem_flag + grp * g : NULL,
                           meta_flag ? meta_flag + grp : NULL);
    orc_pack(codes, d, bits, packed);
    free(codes);
}

/* ------------------------------------------------------------------ */
/* Encode one loop group for n token-heads.                             */
/*   x_bf16 : [L][n][d] BF16 bit patterns; loop L-1 is the anchor.      */
/* Outputs (logical format, see header):                                 */
/*   a_codes [n][d*ba/8], a_meta [n][2d/g]                              */
/*   r_codes [L-1][n][d*br/8], r_meta [L-1][n][2d/g], r_coef [L-1][n]  */
/* Flags (may be NULL):                                                  */
/*   a_eflag [n][d], a_mflag [n][d/g], r_eflag [L-1][n][d],             */
/*   r_mflag [L-1][n][d/g], r_cflag [L-1][n]                             */
/* Steps per token-head, in the order of the method:                     */
/*   1. anchor a_hat = Q_ba(x_anchor) (original basis, never rotated)    */
/*   2. for each other loop l: s = <x_l, a_hat>/<a_hat, a_hat> (0 when   */
/*      <a_hat, a_hat> = 0), s_hat = bf16(s), r = x_l - s_hat * a_hat,   */
/*      y = R r (explicit matrix product), y_hat = Q_br(y).              */
/* ------------------------------------------------------------------ */
ORC_EXPORT void orc_encode(int n, int L, int d, int g, int ba, int br, int rotate, uint64_t seed,
                           const uint16_t *x_bf16,
                           uint8_t *a_codes, uint8_t *a_meta,
                           uint8_t *r_codes, uint8_t *r_meta, uint16_t *r_coef,
                           uint8_t *a_eflag, uint8_t *a_mflag,
                           uint8_t *r_eflag, uint8_t *r_mflag, uint8_t *r_cflag)
{
    int t, l, i;
    int G = d / g;
    size_t ab = (size_t)(d * ba / 8), rb = (size_t)(d * br / 8);
    double *S = (double *)malloc(sizeof(double) * (size_t)d * d);
    double c = orc_rotation_scale(d, rotate);
    double *xa = (double *)malloc(sizeof(double) * (size_t)d);
    double *ahat = (double *)malloc(sizeof(double) * (size_t)d);
    double *xl = (double *)malloc(sizeof(double) * (size_t)d);
    double *r = (double *)malloc(sizeof(double) * (size_t)d);
    double *y = (double *)malloc(sizeof(double) * (size_t)d);
    orc_rotation_signs_matrix(seed, d, rotate, S);
    for (t = 0; t < n; t++) {
        const uint16_t *xa_bits = x_bf16 + ((size_t)(L - 1) * n + t) * d;
        for (i = 0; i < d; i++)
            xa[i] = orc_bf16_value(xa_bits[i]);
        quantize_record(xa, d, g, ba, a_codes + (size_t)t * ab, a_meta + (size_t)t * 2 * G,
                        a_eflag ? a_eflag + (size_t)t * d : NULL,
                        a_mflag ? a_mflag + (size_t)t * G : NULL);
        orc_dequant(a_codes + (size_t)t * ab, a_meta + (size_t)t * 2 * G, d, g, ba, ahat);
        for (l = 0; l < L - 1; l++) {
            const uint16_t *xl_bits = x_bf16 + ((size_t)l * n + t) * d;
            double num = 0.0, den = 0.0, s = 0.0, shat;
            int cnear = 0;
            uint16_t sbits;
            size_t rec = (size_t)l * n + t;
            for (i = 0; i < d; i++)
                xl[i] = orc_bf16_value(xl_bits[i]);
            for (i = 0; i < d; i++) {
                num += xl[i] * ahat[i];
                den += ahat[i] * ahat[i];
            }
            if (den != 0.0)
                s = num / den;
            sbits = orc_bf16_round(s, &cnear);
            shat = orc_bf16_value(sbits);
            r_coef[rec] = sbits;
            if (r_cflag)
                r_cflag[rec] = (uint8_t)cnear;
            for (i = 0; i < d; i++)
                r[i] = xl[i] - shat * ahat[i];
            rotate_vec(S, c, d, r, y);
            quantize_record(y, d, g, br, r_codes + rec * rb, r_meta + rec * 2 * G,
                            r_eflag ? r_eflag + rec * d : NULL,
                            r_mflag ? r_mflag + rec * G : NULL);
        }
    }
    free(S); free(xa); free(ahat); free(xl); free(r); free(y);
}

/* ------------------------------------------------------------------ */
/* Reconstruct all L loops of n token-heads from the logical records:   */
/*   anchor:      x_hat = a_hat                                          */
/*   other loop:  x_hat = s_hat * a_hat + R^T y_hat   (two reads)        */
/* out [L][n][d]                                                          */
/* ------------------------------------------------------------------ */
ORC_EXPORT void orc_reconstruct(int n, int L, int d, int g, int ba, int br, int rotate, uint64_t seed,
                                const uint8_t *a_codes, const uint8_t *a_meta,
                                const uint8_t *r_codes, const uint8_t *r_meta, const uint16_t *r_coef,
                                double *out)
{
    int t, l, i;
    int G = d / g;
    size_t ab = (size_t)(d * ba / 8), rb = (size_t)(d * br / 8);
    double *S = (double *)malloc(sizeof(double) * (size_t)d * d);
    double c = orc_rotation_scale(d, rotate);
    double *ahat = (double *)malloc(sizeof(double) * (size_t)d);
    double *yhat = (double *)malloc(sizeof(double) * (size_t)d);
    double *back = (double *)malloc(sizeof(double) * (size_t)d);
    orc_rotation_signs_matrix(seed, d, rotate, S);
    for (t = 0; t < n; t++) {
        orc_dequant(a_codes + (size_t)t * ab, a_meta + (size_t)t * 2 * G, d, g, ba, ahat);
        memcpy(out + ((size_t)(L - 1) * n + t) * d, ahat, sizeof(double) * (size_t)d);
        for (l = 0; l < L - 1; l++) {
            size_t rec = (size_t)l * n + t;
            double shat = orc_bf16_value(r_coef[rec]);
            double *o = out + rec * d;
            orc_dequant(r_codes + rec * rb, r_meta + rec * 2 * G, d, g, br, yhat);
            rotate_back(S, c, d, yhat, back);
            for (i = 0; i < d; i++)
                o[i] = shat * ahat[i] + back[i];
        }
    }
    free(S); free(ahat); free(yhat); free(back);
}

/* ------------------------------------------------------------------ */
/* Records of one loop group under the ablation modes, in the record     */
/* layout the CUDA library stores (the abstract's comparison of          */
/* reference choice and scaling method; see orc_encode_ablation below    */
/* for the same chain as reconstructions).                               */
/*   anchor_mode 0: the anchor record holds loop L-1; residual record j  */
/*                  holds loop j (j < L-1) against a_hat;                */
/*   anchor_mode 1: the anchor record holds loop 0; residual record j    */
/*                  holds loop j+1 against the reconstruction of loop j. */
/*   scale_mode 0 least squares <x, ref>/<ref, ref>, 1 norm ratio        */
/*   |x|/|ref| (both 0 when ref = 0), 2 none (s = 1).                    */
/* Outputs and flags as for orc_encode.  anchor_mode 0 with scale_mode 0 */
/* is orc_encode.                                                        */
/* ------------------------------------------------------------------ */
ORC_EXPORT void orc_encode_modes(int n, int L, int d, int g, int ba, int br, int rotate, uint64_t seed,
                                 int anchor_mode, int scale_mode, const uint16_t *x_bf16,
                                 uint8_t *a_codes, uint8_t *a_meta,
                                 uint8_t *r_codes, uint8_t *r_meta, uint16_t *r_coef,
                                 uint8_t *a_eflag, uint8_t *a_mflag,
                                 uint8_t *r_eflag, uint8_t *r_mflag, uint8_t *r_cflag)
{
    int t, j, i;
    int G = d / g;
    size_t ab = (size_t)(d * ba / 8), rb = (size_t)(d * br / 8);
    const int first = anchor_mode == 0 ? L - 1 : 0;   /* the loop in the anchor record */
    double *S = (double *)malloc(sizeof(double) * (size_t)d * d);
    double c = orc_rotation_scale(d, rotate);
    double *x = (double *)malloc(sizeof(double) * (size_t)d);
    double *ahat = (double *)malloc(sizeof(double) * (size_t)d);
    double *ref = (double *)malloc(sizeof(double) * (size_t)d);
    double *r = (double *)malloc(sizeof(double) * (size_t)d);
    double *y = (double *)malloc(sizeof(double) * (size_t)d);
    double *yhat = (double *)malloc(sizeof(double) * (size_t)d);
    double *back = (double *)malloc(sizeof(double) * (size_t)d);
    orc_rotation_signs_matrix(seed, d, rotate, S);
    for (t = 0; t < n; t++) {
        for (i = 0; i < d; i++)
            x[i] = orc_bf16_value(x_bf16[((size_t)first * n + t) * d + i]);
        quantize_record(x, d, g, ba, a_codes + (size_t)t * ab, a_meta + (size_t)t * 2 * G,
                        a_eflag ? a_eflag + (size_t)t * d : NULL,
                        a_mflag ? a_mflag + (size_t)t * G : NULL);
        orc_dequant(a_codes + (size_t)t * ab, a_meta + (size_t)t * 2 * G, d, g, ba, ahat);
        memcpy(ref, ahat, sizeof(double) * (size_t)d);
        for (j = 0; j < L - 1; j++) {
            const int loop = anchor_mode == 0 ? j : j + 1;
            double num = 0.0, den = 0.0, xx = 0.0, s = 0.0, shat;
            int cnear = 0;
            uint16_t sbits;
            size_t rec = (size_t)j * n + t;
            for (i = 0; i < d; i++)
                x[i] = orc_bf16_value(x_bf16[((size_t)loop * n + t) * d + i]);
            for (i = 0; i < d; i++) {
                num += x[i] * ref[i];
                den += ref[i] * ref[i];
                xx += x[i] * x[i];
            }
            if (scale_mode == 2)
                s = 1.0;
            else if (den != 0.0)
                s = scale_mode == 0 ? num / den : sqrt(xx) / sqrt(den);
            sbits = orc_bf16_round(s, &cnear);
            shat = orc_bf16_value(sbits);
            r_coef[rec] = sbits;
            if (r_cflag)
                r_cflag[rec] = (uint8_t)cnear;
            for (i = 0; i < d; i++)
                r[i] = x[i] - shat * ref[i];
            rotate_vec(S, c, d, r, y);
            quantize_record(y, d, g, br, r_codes + rec * rb, r_meta + rec * 2 * G,
                            r_eflag ? r_eflag + rec * d : NULL,
                            r_mflag ? r_mflag + rec * G : NULL);
            if (anchor_mode == 1) {
                /* the next loop's reference: this loop's reconstruction */
                orc_dequant(r_codes + rec * rb, r_meta + rec * 2 * G, d, g, br, yhat);
                rotate_back(S, c, d, yhat, back);
                for (i = 0; i < d; i++)
                    ref[i] = shat * ref[i] + back[i];
            }
        }
    }
    free(S); free(x); free(ahat); free(ref); free(r); free(y); free(yhat); free(back);
}

/* Reconstruction of all L loops from records laid out as orc_encode_modes
 * writes them: anchor_mode 0 as orc_reconstruct; anchor_mode 1: loop 0 =
 * a_hat, loop l = s_hat_{l-1} x_hat_{l-1} + R^T y_hat_{l-1} (record l-1).
 * out [L][n][d] in loop order. */
ORC_EXPORT void orc_reconstruct_modes(int n, int L, int d, int g, int ba, int br, int rotate, uint64_t seed,
                                      int anchor_mode, const uint8_t *a_codes, const uint8_t *a_meta,
                                      const uint8_t *r_codes, const uint8_t *r_meta, const uint16_t *r_coef,
                                      double *out)
{
    int t, l, i;
    int G = d / g;
    size_t ab = (size_t)(d * ba / 8), rb = (size_t)(d * br / 8);
    double *S, *yhat, *back, c;
    if (anchor_mode == 0) {
        orc_reconstruct(n, L, d, g, ba, br, rotate, seed, a_codes, a_meta, r_codes, r_meta, r_coef, out);
        return;
    }
    S = (double *)malloc(sizeof(double) * (size_t)d * d);
    c = orc_rotation_scale(d, rotate);
    yhat = (double *)malloc(sizeof(double) * (size_t)d);
    back = (double *)malloc(sizeof(double) * (size_t)d);
    orc_rotation_signs_matrix(seed, d, rotate, S);
    for (t = 0; t < n; t++) {
        orc_dequant(a_codes + (size_t)t * ab, a_meta + (size_t)t * 2 * G, d, g, ba, out + (size_t)t * d);
        for (l = 1; l < L; l++) {
            size_t rec = (size_t)(l - 1) * n + t;
            const double shat = orc_bf16_value(r_coef[rec]);
            const double *prev = out + ((size_t)(l - 1) * n + t) * d;
            double *o = out + ((size_t)l * n + t) * d;
            orc_dequant(r_codes + rec * rb, r_meta + rec * 2 * G, d, g, br, yhat);
            rotate_back(S, c, d, yhat, back);
            for (i = 0; i < d; i++)
                o[i] = shat * prev[i] + back[i];
        }
    }
    free(S); free(yhat); free(back);
}

/* ------------------------------------------------------------------ */
/* Ablation encoders (the arXiv abstract's comparison of reference      */
/* choice and scaling method): encode one loop group of n token-heads   */
/* and return the reconstruction, for reconstruction-error studies.     */
/*   anchor_mode 0: last-loop anchor, shared -- loop L-1 is quantized   */
/*                  at ba bits; every other loop l is a residual        */
/*                  against a_hat (the method; identical to orc_encode  */
/*                  followed by orc_reconstruct);                        */
/*   anchor_mode 1: previous-loop anchor, chained -- loop 0 is          */
/*                  quantized at ba bits; loop l >= 1 is a residual     */
/*                  against the reconstruction of loop l-1, so its      */
/*                  reconstruction reads l+1 records.                    */
/*   scale_mode  0: least squares  s = <x, ref>/<ref, ref> (0 if ref=0);*/
/*   scale_mode  1: norm ratio     s = |x| / |ref| (0 if ref=0);        */
/*   scale_mode  2: none           s = 1.                                */
/* In every mode s is stored as BF16, the residual x - s_hat ref is     */
/* rotated by R and quantized at br bits, and the reconstruction is     */
/* s_hat ref + R^T y_hat.                                                */
/*   x_bf16 [L][n][d]; xhat out [L][n][d]; coef out [L][n] (s_hat, 0 for */
/*   the anchor loop); reads out [L]: records read to rebuild each loop. */
/* Readings (the pages name the variants only): the previous-loop       */
/* anchor is the first loop of the group, so that every loop but one    */
/* has a reference; norm-ratio scaling keeps s >= 0.                     */
/* ------------------------------------------------------------------ */
ORC_EXPORT void orc_encode_ablation(int n, int L, int d, int g, int ba, int br, int rotate, uint64_t seed,
                                    int anchor_mode, int scale_mode, const uint16_t *x_bf16,
                                    double *xhat, double *coef, int *reads)
{
    int t, l, i;
    int G = d / g;
    double *S = (double *)malloc(sizeof(double) * (size_t)d * d);
    double c = orc_rotation_scale(d, rotate);
    double *x = (double *)malloc(sizeof(double) * (size_t)d);
    double *r = (double *)malloc(sizeof(double) * (size_t)d);
    double *y = (double *)malloc(sizeof(double) * (size_t)d);
    double *yhat = (double *)malloc(sizeof(double) * (size_t)d);
    double *back = (double *)malloc(sizeof(double) * (size_t)d);
    uint8_t *packed = (uint8_t *)malloc((size_t)d);
    uint8_t *meta = (uint8_t *)malloc((size_t)(2 * G));
    const int first = anchor_mode == 0 ? L - 1 : 0;   /* the anchor loop */
    orc_rotation_signs_matrix(seed, d, rotate, S);
    for (l = 0; l < L; l++)
        reads[l] = l == first ? 1 : (anchor_mode == 0 ? 2 : l + 1);
    for (t = 0; t < n; t++) {
        double *ahat = xhat + ((size_t)first * n + t) * d;
        for (i = 0; i < d; i++)
            x[i] = orc_bf16_value(x_bf16[((size_t)first * n + t) * d + i]);
        quantize_record(x, d, g, ba, packed, meta, NULL, NULL);
        orc_dequant(packed, meta, d, g, ba, ahat);
        coef[(size_t)first * n + t] = 0.0;
        for (l = 0; l < L; l++) {
            double num = 0.0, den = 0.0, xx = 0.0, s = 0.0, shat;
            const double *ref;
            double *o;
            if (l == first)
                continue;
            /* chained: loops 1, 2, ... in order, each against the one before */
            ref = anchor_mode == 0 ? ahat : xhat + ((size_t)(l - 1) * n + t) * d;
            o = xhat + ((size_t)l * n + t) * d;
            for (i = 0; i < d; i++)
                x[i] = orc_bf16_value(x_bf16[((size_t)l * n + t) * d + i]);
            for (i = 0; i < d; i++) {
                num += x[i] * ref[i];
                den += ref[i] * ref[i];
                xx += x[i] * x[i];
            }
            if (scale_mode == 2)
                s = 1.0;
            else if (den != 0.0)
                s = scale_mode == 0 ? num / den : sqrt(xx) / sqrt(den);
            shat = orc_bf16_value(orc_bf16_round(s, NULL));
            coef[(size_t)l * n + t] = shat;
            for (i = 0; i < d; i++)
                r[i] = x[i] - shat * ref[i];
            rotate_vec(S, c, d, r, y);
            quantize_record(y, d, g, br, packed, meta, NULL, NULL);
            orc_dequant(packed, meta, d, g, br, yhat);
            rotate_back(S, c, d, yhat, back);
            for (i = 0; i < d; i++)
                o[i] = shat * ref[i] + back[i];
        }
    }
    free(S); free(x); free(r); free(y); free(yhat); free(back); free(packed); free(meta);
}

/* ------------------------------------------------------------------ */
/* Direct softmax attention in fp64 (two passes: max, then weights).    */
/*   q   [B][Hq][d]                                                      */
/*   k,v [B][T][Hkv][d]  (all keys this query may see, in token order)   */
/*   out [B][Hq][d]                                                      */
/* query head h reads kv head h / (Hq/Hkv).  out = sum_t e^(z_t - zmax) */
/* v_t / sum_t e^(z_t - zmax), z_t = scale * <q, k_t>.  T == 0 -> zeros. */
/* threads > 1 splits the independent (b, h) units over OpenMP threads. */
/* ------------------------------------------------------------------ */
ORC_EXPORT void orc_attention(int B, int Hq, int Hkv, int d, int T, double scale,
                              const double *q, const double *k, const double *v,
                              double *out, int threads)
{
    int unit;
    int grp = Hq / Hkv;
#ifdef _OPENMP
    if (threads < 1) threads = 1;
#pragma omp parallel for num_threads(threads) schedule(dynamic)
#endif
    for (unit = 0; unit < B * Hq; unit++) {
        int b = unit / Hq, h = unit % Hq, hk = h / grp;
        const double *qq = q + ((size_t)b * Hq + h) * d;
        double *oo = out + ((size_t)b * Hq + h) * d;
        double *z = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
        double zmax = -INFINITY, den = 0.0;
        int t, i;
        for (i = 0; i < d; i++)
            oo[i] = 0.0;
        if (T > 0) {
            for (t = 0; t < T; t++) {
                const double *kk = k + (((size_t)b * T + t) * Hkv + hk) * d;
                double dot = 0.0;
                for (i = 0; i < d; i++)
                    dot += qq[i] * kk[i];
                z[t] = scale * dot;
                if (z[t] > zmax) zmax = z[t];
            }
            for (t = 0; t < T; t++)
                den += exp(z[t] - zmax);
            for (t = 0; t < T; t++) {
                const double *vv = v + (((size_t)b * T + t) * Hkv + hk) * d;
                double w = exp(z[t] - zmax) / den;
                for (i = 0; i < d; i++)
                    oo[i] += w * vv[i];
            }
        }
        free(z);
    }
}

/* Mean squared error between two arrays (helper for the MSE criterion). */
ORC_EXPORT double orc_mse(const double *a, const double *b, size_t n)
{
    size_t i;
    double acc = 0.0;
    for (i = 0; i < n; i++) {
        double e = a[i] - b[i];
        acc += e * e;
    }
    return n ? acc / (double)n : 0.0;
}
