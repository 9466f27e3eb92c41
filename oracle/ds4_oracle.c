/*
 * ds4_oracle.c -- CPU oracle for the ds4 routed-MoE expert FFN.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain reference that the
 * CUDA path is checked against.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline leg of bench.py may load or run it; the library never does.
 * It shares no code, header, table or constant generator with the CUDA path.
 *
 * What it follows (the pages publish no formula; the readings are this
 * project's, written down next to each function):
 *   - "antirez가 만든 DeepSeek V4 Flash 전용 로컬 추론 엔진 ds4" (jeff.news),
 *     2-bit quantization bullets: only the routed MoE experts are quantized,
 *     up/gate in IQ2_XXS, down in Q2_K; shared experts, projections and the
 *     routing stay at full precision.
 *   - "antirez/ds4 -- Metal용 DeepSeek V4 Flash 로컬 추론 엔진 완벽 가이드"
 *     (sigco.tistory.com), "왜 독자 엔진이 필요할까" (each input calls only some
 *     experts) and "설계 철학" (same quantization split).
 *   - the layer as the project states it: a full-precision router, softmax
 *     over the top-k experts, SwiGLU experts, gate-weighted sum plus an
 *     unquantized shared expert.
 *   - the 4-bit models the same pages name (q4, q4-imatrix), whose format
 *     they leave open: a Q4_K-style block of this project's own definition
 *     (see orc_dequant_q4k).
 *
 * Precision: floating point is fp64 except where a floating-point value
 * decides an integer (the router logits that pick the experts), which is
 * computed in the kernel's precision and order (binary32, canonical order,
 * see orc_router_logit).  Dequantized weights are the binary32 values the
 * block formats define.  Nothing here is blocked, fused or reordered beyond
 * what those definitions state.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fPIC -shared -o libds4oracle.so
 * (-ffp-contract=off: every a*b+c here is two roundings unless fma() is
 * written out, exactly as the readings state).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_QK 256                 /* weights per superblock, both formats */
#define ORC_Q2_BYTES 84            /* Q2_K-style block size */
#define ORC_IQ2_BYTES 66           /* IQ2_XXS-style block size */
#define ORC_Q4_BYTES 144           /* Q4_K-style block size (4-bit experts) */

/* ------------------------------------------------------------------------ */
/* IEEE binary16 and bfloat16, written from their definitions.               */
/* ------------------------------------------------------------------------ */

/* binary16 bits -> exact double.  1 sign, 5 exponent (bias 15), 10 fraction
 * bits; exponent 0 is subnormal (m * 2^-24), 31 is inf/nan. */
double orc_half_to_double(uint16_t h) {
    int s = (h >> 15) & 1, e = (h >> 10) & 0x1f, m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);
    return s ? -v : v;
}

/* Round a finite non-negative double to a binary floating-point format with
 * p significand bits and minimum normal exponent emin (value = r * 2^q with
 * r an integer < 2^p), round-half-to-even.  Returns the rounded value as a
 * double (exact: p <= 24). */
static double orc_round_format(double a, int p, int emin) {
    if (a == 0.0) return 0.0;
    int e;
    frexp(a, &e);                      /* a = f * 2^e, f in [0.5, 1) */
    int lg = e - 1;                    /* floor(log2 a) */
    if (lg < emin) lg = emin;          /* subnormal range: fixed quantum */
    int q = lg - (p - 1);              /* quantum exponent */
    double r = nearbyint(ldexp(a, -q));/* default mode: half to even */
    return ldexp(r, q);
}

/* double -> binary16 bits, round-half-to-even, overflow to inf. */
uint16_t orc_double_to_half(double v) {
    if (isnan(v)) return 0x7e00;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    double r = orc_round_format(a, 11, -14);
    if (r >= 65536.0) return sign | 0x7c00;       /* beyond max finite 65504 */
    if (r == 0.0) return sign;
    int e;
    frexp(r, &e);
    int lg = e - 1;
    if (lg < -14) {                               /* subnormal: r = m * 2^-24 */
        return sign | (uint16_t)ldexp(r, 24);
    }
    uint16_t m = (uint16_t)(ldexp(r, 10 - lg) - 1024.0);
    return sign | (uint16_t)((lg + 15) << 10) | m;
}

/* binary32 -> nearest bfloat16 (8 significand bits, binary32's exponent
 * range), half to even; returned as the binary32 value it represents. */
float orc_bf16_round(float v) {
    if (isnan(v)) return v;
    double a = fabs((double)v);
    double r = orc_round_format(a, 8, -126);
    if (r >= ldexp(1.0, 128)) r = INFINITY;
    float out = (float)r;
    return signbit(v) ? -out : out;
}

/* orc_bf16_round over an array. */
void orc_bf16_round_array(const float* v, int64_t n, float* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_round(v[i]);
}

static uint16_t rd16(const uint8_t* p) { return (uint16_t)(p[0] | (p[1] << 8)); }
static uint32_t rd32(const uint8_t* p) {
    return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
}

/* ------------------------------------------------------------------------ */
/* Q2_K-style superblock (84 bytes / 256 weights).                           */
/*   [0,16)  byte j: sc_j (low nibble) | m_j << 4, sub-block j = 16j..16j+15  */
/*   [16,80) code q_i of weight i at byte 16 + i/4, bits 2(i%4), 2(i%4)+1     */
/*   [80,82) d  (binary16, little endian)                                    */
/*   [82,84) dmin (binary16, little endian)                                  */
/* weight_i = (d*sc_j)*q_i - dmin*m_j, evaluated exactly and rounded once to */
/* binary32.                                                                 */
/* ------------------------------------------------------------------------ */
void orc_dequant_q2k(const uint8_t* blocks, int64_t n_blocks, float* out) {
    for (int64_t b = 0; b < n_blocks; ++b) {
        const uint8_t* p = blocks + b * ORC_Q2_BYTES;
        double d = orc_half_to_double(rd16(p + 80));
        double dmin = orc_half_to_double(rd16(p + 82));
        for (int i = 0; i < ORC_QK; ++i) {
            int j = i / 16;
            int sc = p[j] & 0xf, m = p[j] >> 4;
            int q = (p[16 + i / 4] >> (2 * (i % 4))) & 3;
            double v = d * sc * q - dmin * m;   /* exact in double */
            out[b * ORC_QK + i] = (float)v;     /* one rounding to binary32 */
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Q4_K-style superblock (144 bytes / 256 weights), the 4-bit routed-expert  */
/* variant.  The pages name 4-bit models (q4, q4-imatrix) but describe no    */
/* format; this reading carries the Q2_K-style structure over to 4-bit      */
/* codes and 32-weight sub-blocks:                                           */
/*   [0,2)    d    (binary16, little endian)                                 */
/*   [2,4)    dmin (binary16, little endian)                                 */
/*   [4,16)   sixteen 6-bit fields of the little-endian 96-bit integer of    */
/*            these bytes: field f at bits 6f..6f+5; f = j is sc_j, f = 8+j  */
/*            is m_j, sub-block j = weights 32j..32j+31                      */
/*   [16,144) code q_i of weight i at byte 16 + i/2, low nibble for even i   */
/* weight_i = (d*sc_j)*q_i - dmin*m_j, rounded once to binary32 (the double  */
/* difference is exact while the lowest set bits of the two products are    */
/* at most 32 binary places apart, as in every block a packer writes for    */
/* weights of one magnitude).                                                */
/* ------------------------------------------------------------------------ */
static int orc_q4_field(const uint8_t* p, int f) {
    /* bits 6f..6f+5 of bytes 4..15 read as one little-endian integer */
    int v = 0;
    for (int b = 0; b < 6; ++b) {
        int bit = 6 * f + b;
        v |= ((p[4 + bit / 8] >> (bit % 8)) & 1) << b;
    }
    return v;
}

void orc_dequant_q4k(const uint8_t* blocks, int64_t n_blocks, float* out) {
    for (int64_t b = 0; b < n_blocks; ++b) {
        const uint8_t* p = blocks + b * ORC_Q4_BYTES;
        double d = orc_half_to_double(rd16(p + 0));
        double dmin = orc_half_to_double(rd16(p + 2));
        for (int i = 0; i < ORC_QK; ++i) {
            int j = i / 32;
            int sc = orc_q4_field(p, j), m = orc_q4_field(p, 8 + j);
            int q = (p[16 + i / 2] >> (4 * (i % 2))) & 15;
            double v = d * sc * q - dmin * m;
            out[b * ORC_QK + i] = (float)v;     /* one rounding to binary32 */
        }
    }
}

/* ------------------------------------------------------------------------ */
/* IQ2_XXS-style superblock (66 bytes / 256 weights).                        */
/*   [0,2)  d (binary16, little endian)                                      */
/*   group g = 0..7 at offset 2 + 8g, covering weights 32g..32g+31:          */
/*     bytes 0..3: grid row a_c of chunk c (weights 32g+8c .. +7)            */
/*     bytes 4..7: uint32 S, bits 7c..7c+6 = sign field sigma_c, 28..31 = s_g */
/*   element i of a chunk is negative if bit i of sigma_c is set (i < 7);    */
/*   element 7 is negative if sigma_c has an odd number of set bits, so      */
/*   every chunk carries an even number of negatives.                        */
/* weight = (d*(2 s_g + 1)/8) * G[a_c][i] * (+-1), exact in binary32.        */
/* ------------------------------------------------------------------------ */
static int orc_popcount7(uint32_t v) {
    int c = 0;
    for (int i = 0; i < 7; ++i) c += (v >> i) & 1;
    return c;
}

void orc_dequant_iq2xxs(const uint8_t* blocks, int64_t n_blocks, const uint8_t* grid, float* out) {
    for (int64_t b = 0; b < n_blocks; ++b) {
        const uint8_t* p = blocks + b * ORC_IQ2_BYTES;
        double d = orc_half_to_double(rd16(p));
        for (int g = 0; g < 8; ++g) {
            const uint8_t* gp = p + 2 + 8 * g;
            uint32_t S = rd32(gp + 4);
            int s = (int)(S >> 28);
            double db = d * (2 * s + 1) / 8.0;
            for (int c = 0; c < 4; ++c) {
                int a = gp[c];
                uint32_t sigma = (S >> (7 * c)) & 0x7f;
                for (int i = 0; i < 8; ++i) {
                    int neg = (i < 7) ? (int)((sigma >> i) & 1) : (orc_popcount7(sigma) & 1);
                    double v = db * grid[a * 8 + i];
                    out[b * ORC_QK + 32 * g + 8 * c + i] = (float)(neg ? -v : v);
                }
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Packers (quantizers).  Decisions in double, round-half-to-even.          */
/* ------------------------------------------------------------------------ */
static double clampd(double v, double lo, double hi) { return v < lo ? lo : (v > hi ? hi : v); }

/* Q2_K-style packer, per superblock:
 *   per sub-block j: lo = min(0, min w), hi = max(0, max w),
 *                    scale_j = (hi - lo)/3, min_j = -lo
 *   d = half(max scale_j / 15), dmin = half(max min_j / 15)
 *   sc_j = clamp(rne(scale_j/d), 0, 15), m_j = clamp(rne(min_j/dmin), 0, 15)
 *   q_i  = clamp(rne((w_i + dmin*m_j)/(d*sc_j)), 0, 3)
 * (a zero divisor gives a zero field).  n must be a multiple of 256. */
int orc_pack_q2k(const float* w, int64_t n, uint8_t* out) {
    if (n % ORC_QK) return -1;
    for (int64_t b = 0; b < n / ORC_QK; ++b) {
        const float* x = w + b * ORC_QK;
        uint8_t* p = out + b * ORC_Q2_BYTES;
        double scale[16], mn[16], max_scale = 0.0, max_min = 0.0;
        for (int j = 0; j < 16; ++j) {
            double lo = 0.0, hi = 0.0;
            for (int i = 0; i < 16; ++i) {
                double v = x[16 * j + i];
                if (v < lo) lo = v;
                if (v > hi) hi = v;
            }
            scale[j] = (hi - lo) / 3.0;
            mn[j] = -lo;
            if (scale[j] > max_scale) max_scale = scale[j];
            if (mn[j] > max_min) max_min = mn[j];
        }
        uint16_t dh = orc_double_to_half(max_scale / 15.0);
        uint16_t mh = orc_double_to_half(max_min / 15.0);
        double d = orc_half_to_double(dh), dmin = orc_half_to_double(mh);
        memset(p, 0, ORC_Q2_BYTES);
        for (int j = 0; j < 16; ++j) {
            int sc = d > 0.0 ? (int)clampd(nearbyint(scale[j] / d), 0, 15) : 0;
            int m = dmin > 0.0 ? (int)clampd(nearbyint(mn[j] / dmin), 0, 15) : 0;
            p[j] = (uint8_t)(sc | (m << 4));
            double step = d * sc, off = dmin * m;
            for (int i = 0; i < 16; ++i) {
                int q = step > 0.0 ? (int)clampd(nearbyint((x[16 * j + i] + off) / step), 0, 3) : 0;
                int k = 16 * j + i;
                p[16 + k / 4] |= (uint8_t)(q << (2 * (k % 4)));
            }
        }
        p[80] = dh & 0xff; p[81] = dh >> 8;
        p[82] = mh & 0xff; p[83] = mh >> 8;
    }
    return 0;
}

/* Q4_K-style packer, per superblock (the Q2_K-style rule with 15 code steps
 * and 6-bit fields):
 *   per sub-block j (32 weights): lo = min(0, min w), hi = max(0, max w),
 *                                 scale_j = (hi - lo)/15, min_j = -lo
 *   d = half(max scale_j / 63), dmin = half(max min_j / 63)
 *   sc_j = clamp(rne(scale_j/d), 0, 63), m_j = clamp(rne(min_j/dmin), 0, 63)
 *   q_i  = clamp(rne((w_i + dmin*m_j)/(d*sc_j)), 0, 15)
 * (a zero divisor gives a zero field).  n must be a multiple of 256. */
static void orc_q4_set_field(uint8_t* p, int f, int v) {
    for (int b = 0; b < 6; ++b) {
        int bit = 6 * f + b;
        if ((v >> b) & 1) p[4 + bit / 8] |= (uint8_t)(1 << (bit % 8));
    }
}

int orc_pack_q4k(const float* w, int64_t n, uint8_t* out) {
    if (n % ORC_QK) return -1;
    for (int64_t b = 0; b < n / ORC_QK; ++b) {
        const float* x = w + b * ORC_QK;
        uint8_t* p = out + b * ORC_Q4_BYTES;
        double scale[8], mn[8], max_scale = 0.0, max_min = 0.0;
        for (int j = 0; j < 8; ++j) {
            double lo = 0.0, hi = 0.0;
            for (int i = 0; i < 32; ++i) {
                double v = x[32 * j + i];
                if (v < lo) lo = v;
                if (v > hi) hi = v;
            }
            scale[j] = (hi - lo) / 15.0;
            mn[j] = -lo;
            if (scale[j] > max_scale) max_scale = scale[j];
            if (mn[j] > max_min) max_min = mn[j];
        }
        uint16_t dh = orc_double_to_half(max_scale / 63.0);
        uint16_t mh = orc_double_to_half(max_min / 63.0);
        double d = orc_half_to_double(dh), dmin = orc_half_to_double(mh);
        memset(p, 0, ORC_Q4_BYTES);
        for (int j = 0; j < 8; ++j) {
            int sc = d > 0.0 ? (int)clampd(nearbyint(scale[j] / d), 0, 63) : 0;
            int m = dmin > 0.0 ? (int)clampd(nearbyint(mn[j] / dmin), 0, 63) : 0;
            orc_q4_set_field(p, j, sc);
            orc_q4_set_field(p, 8 + j, m);
            double step = d * sc, off = dmin * m;
            for (int i = 0; i < 32; ++i) {
                int q = step > 0.0 ? (int)clampd(nearbyint((x[32 * j + i] + off) / step), 0, 15) : 0;
                int k = 32 * j + i;
                p[16 + k / 2] |= (uint8_t)(q << (4 * (k % 2)));
            }
        }
        p[0] = dh & 0xff; p[1] = dh >> 8;
        p[2] = mh & 0xff; p[3] = mh >> 8;
    }
    return 0;
}

/* IQ2_XXS-style packer, per superblock:
 *   d = half(max|w| / (43 * 31/8)); d == 0 -> all-zero block
 *   per group: s_g = clamp(rne(4*max|w_g|/(43 d) - 0.5), 0, 15), db = d(2s_g+1)/8
 *   per chunk: negative flags neg_i = (w_i < 0); if their count is odd, the
 *     element of smallest |w_i| (lowest i on ties) is flipped; targets
 *     t_i = |w_i| for unflipped elements, -|w_i| for the flipped one;
 *     a = argmin_a sum_i (db*G[a][i] - t_i)^2, ties to the lowest a;
 *     sigma = neg_0..neg_6.
 * n must be a multiple of 256. */
int orc_pack_iq2xxs(const float* w, int64_t n, const uint8_t* grid, uint8_t* out) {
    if (n % ORC_QK) return -1;
    for (int64_t b = 0; b < n / ORC_QK; ++b) {
        const float* x = w + b * ORC_QK;
        uint8_t* p = out + b * ORC_IQ2_BYTES;
        memset(p, 0, ORC_IQ2_BYTES);
        double amax = 0.0;
        for (int i = 0; i < ORC_QK; ++i) {
            double a = fabs((double)x[i]);
            if (a > amax) amax = a;
        }
        uint16_t dh = orc_double_to_half(amax / (43.0 * 31.0 / 8.0));
        double d = orc_half_to_double(dh);
        if (d == 0.0) continue;
        p[0] = dh & 0xff; p[1] = dh >> 8;
        for (int g = 0; g < 8; ++g) {
            const float* xg = x + 32 * g;
            double gmax = 0.0;
            for (int i = 0; i < 32; ++i) {
                double a = fabs((double)xg[i]);
                if (a > gmax) gmax = a;
            }
            int s = (int)clampd(nearbyint(4.0 * gmax / (43.0 * d) - 0.5), 0, 15);
            double db = d * (2 * s + 1) / 8.0;
            uint32_t S = (uint32_t)s << 28;
            for (int c = 0; c < 4; ++c) {
                const float* xc = xg + 8 * c;
                int neg[8], cnt = 0;
                for (int i = 0; i < 8; ++i) { neg[i] = xc[i] < 0.0f; cnt += neg[i]; }
                int flip = -1;
                if (cnt & 1) {
                    double best = INFINITY;
                    for (int i = 0; i < 8; ++i) {
                        double a = fabs((double)xc[i]);
                        if (a < best) { best = a; flip = i; }
                    }
                    neg[flip] = !neg[flip];
                }
                double t[8];
                for (int i = 0; i < 8; ++i) {
                    double a = fabs((double)xc[i]);
                    t[i] = (i == flip) ? -a : a;
                }
                int best_a = 0;
                double best_err = INFINITY;
                for (int a = 0; a < 256; ++a) {
                    double err = 0.0;
                    for (int i = 0; i < 8; ++i) {
                        double diff = db * grid[a * 8 + i] - t[i];
                        err = err + diff * diff;
                    }
                    if (err < best_err) { best_err = err; best_a = a; }
                }
                uint32_t sigma = 0;
                for (int i = 0; i < 7; ++i) sigma |= (uint32_t)neg[i] << i;
                p[2 + 8 * g + c] = (uint8_t)best_a;
                S |= sigma << (7 * c);
            }
            uint8_t* sp = p + 2 + 8 * g + 4;
            sp[0] = S & 0xff; sp[1] = (S >> 8) & 0xff; sp[2] = (S >> 16) & 0xff; sp[3] = S >> 24;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Router.                                                                   */
/* ------------------------------------------------------------------------ */

/* Canonical binary32 router logit (the order both sides follow, so that the
 * selected experts are the same bits everywhere).  H must be a multiple of
 * 128.  Thirty-two partial sums p_L; p_L accumulates, for i = 0, 1, ... and
 * r = 0..3, fma(x[128 i + 4 L + r], w[same], p_L) in that order.  Then
 * p_L <- p_L + p_{L xor m} for m = 16, 8, 4, 2, 1; the logit is p_0 (plus
 * the bias, one binary32 add, when a bias is given). */
float orc_router_logit(const float* x, const float* w, int32_t H, const float* bias) {
    float p[32], q[32];
    for (int L = 0; L < 32; ++L) p[L] = 0.0f;
    for (int i = 0; i < H / 128; ++i)
        for (int L = 0; L < 32; ++L)
            for (int r = 0; r < 4; ++r) {
                int idx = 128 * i + 4 * L + r;
                p[L] = fmaf(x[idx], w[idx], p[L]);
            }
    for (int m = 16; m >= 1; m >>= 1) {
        for (int L = 0; L < 32; ++L) q[L] = p[L] + p[L ^ m];
        memcpy(p, q, sizeof(p));
    }
    return bias ? p[0] + *bias : p[0];
}

/* logits[t][e] for n tokens of x [n][H] and router rows W [E][H]. */
void orc_router_logits(const float* x, const float* W, const float* b, int64_t n, int32_t E, int32_t H,
                       float* logits) {
    for (int64_t t = 0; t < n; ++t)
        for (int e = 0; e < E; ++e)
            logits[t * E + e] = orc_router_logit(x + t * H, W + (int64_t)e * H, H, b ? b + e : NULL);
}

/* Plain fp64 dot products (diagnostics: distance of the canonical logit from
 * the exact one, and the top-k margin). */
void orc_router_logits_f64(const float* x, const float* W, const float* b, int64_t n, int32_t E, int32_t H,
                           double* logits) {
    for (int64_t t = 0; t < n; ++t)
        for (int e = 0; e < E; ++e) {
            double s = 0.0;
            for (int h = 0; h < H; ++h) s += (double)x[t * H + h] * (double)W[(int64_t)e * H + h];
            logits[t * E + e] = s + (b ? (double)b[e] : 0.0);
        }
}

/* Top-k by (logit descending, expert index ascending), one pick at a time;
 * then the softmax over the k selected logits:
 *   w_j = exp(l_j - l_max) / sum_{i in S} exp(l_i - l_max)
 * (equal to the full softmax renormalized over the selected experts). */
void orc_topk_softmax(const float* logits, int64_t n, int32_t E, int32_t k, int32_t* ids, double* w) {
    char* taken = (char*)malloc((size_t)E);
    for (int64_t t = 0; t < n; ++t) {
        const float* l = logits + t * E;
        memset(taken, 0, (size_t)E);
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e;   /* strict: lower index wins ties */
            }
            taken[best] = 1;
            ids[t * k + j] = best;
        }
        double lmax = l[ids[t * k]], den = 0.0;
        for (int j = 0; j < k; ++j) den += exp((double)l[ids[t * k + j]] - lmax);
        for (int j = 0; j < k; ++j) w[t * k + j] = exp((double)l[ids[t * k + j]] - lmax) / den;
    }
    free(taken);
}

/* ------------------------------------------------------------------------ */
/* The layer.                                                                */
/* ------------------------------------------------------------------------ */
typedef struct {
    int32_t H, I, E, k;
    const float* W_r;               /* [E][H] router rows */
    const float* b_r;               /* [E] or NULL */
    const uint8_t* grid;            /* [256][8] IQ2 grid magnitudes */
    const uint8_t* const* gate;     /* E pointers: IQ2 blocks of W_gate [I][H] (row-major, flat) */
    const uint8_t* const* up;       /* E pointers: IQ2 blocks of W_up [I][H] */
    const uint8_t* const* down;     /* E pointers: Q2 blocks of W_down [H][I] */
    const uint16_t* sh_gate;        /* bf16 bits [I][H] or NULL: no shared expert */
    const uint16_t* sh_up;          /* bf16 bits [I][H] */
    const uint16_t* sh_down;        /* bf16 bits [H][I] */
    int32_t expert_bits;            /* 2: gate/up IQ2_XXS-style, down Q2_K-style;
                                       4: all three Q4_K-style (the 4-bit variant) */
} orc_layer;

static double bf16_bits_to_double(uint16_t v) {
    uint32_t u = (uint32_t)v << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* y = W h, W [rows][cols] as float, h and y double. */
static void matvec_f(const float* W, int64_t rows, int64_t cols, const double* h, double* y) {
    for (int64_t r = 0; r < rows; ++r) {
        double s = 0.0;
        for (int64_t c = 0; c < cols; ++c) s += (double)W[r * cols + c] * h[c];
        y[r] = s;
    }
}

static void matvec_bf16(const uint16_t* W, int64_t rows, int64_t cols, const double* h, double* y) {
    for (int64_t r = 0; r < rows; ++r) {
        double s = 0.0;
        for (int64_t c = 0; c < cols; ++c) s += bf16_bits_to_double(W[r * cols + c]) * h[c];
        y[r] = s;
    }
}

/* Forward of the layer on n tokens x [n][H].
 *
 * For each token: logits (canonical binary32, orc_router_logit), the top-k
 * experts and their softmax weights (orc_topk_softmax), for each selected
 * expert e:  g = W_gate_e x, u = W_up_e x, h = silu(g) * u, y_e = W_down_e h;
 * shared: y_s = W_down_s (silu(W_gate_s x) * (W_up_s x));
 * out = y_s + sum_{j=0}^{k-1} w_j y_{ids_j}.
 *
 * mode 0 (decode reading): x as given, dequantized weights exact, all in fp64.
 * mode 1 (bf16 tensor-core reading): x, the dequantized routed weights and
 * both intermediates h (routed and shared) are rounded to bfloat16 where the
 * tensor-core path rounds them; sums stay fp64.  The router always sees x as
 * given.
 *
 * Experts are dequantized once each (in first-use order) and applied to all
 * the (token, slot) pairs that chose them.  ids/w may be NULL.
 * Returns 0, or -1 on a bad argument / missing expert pointer. */
int orc_moe_forward(const orc_layer* L, const float* x, int64_t n, int32_t mode, double* out, int32_t* ids_out,
                    double* w_out) {
    const int64_t H = L->H, I = L->I;
    const int32_t E = L->E, k = L->k;
    if (H % 256 || k < 1 || k > E || n < 0) return -1;
    if (L->expert_bits != 2 && L->expert_bits != 4) return -1;
    if (n == 0) return 0;
    float* logits = (float*)malloc(sizeof(float) * (size_t)(n * E));
    int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)(n * k));
    double* w = (double*)malloc(sizeof(double) * (size_t)(n * k));
    double* xin = (double*)malloc(sizeof(double) * (size_t)(n * H));
    double* yslot = (double*)calloc((size_t)(n * k * H), sizeof(double));
    float* Wg = (float*)malloc(sizeof(float) * (size_t)(I * H));
    float* Wu = (float*)malloc(sizeof(float) * (size_t)(I * H));
    float* Wd = (float*)malloc(sizeof(float) * (size_t)(H * I));
    double *g = (double*)malloc(sizeof(double) * (size_t)I), *u = (double*)malloc(sizeof(double) * (size_t)I);
    double* h = (double*)malloc(sizeof(double) * (size_t)I);
    double* y = (double*)malloc(sizeof(double) * (size_t)H);
    int rc = 0;

    orc_router_logits(x, L->W_r, L->b_r, n, E, (int32_t)H, logits);
    orc_topk_softmax(logits, n, E, k, ids, w);
    for (int64_t i = 0; i < n * H; ++i) xin[i] = mode == 1 ? (double)orc_bf16_round(x[i]) : (double)x[i];

    for (int32_t e = 0; e < E && rc == 0; ++e) {
        int used = 0;
        for (int64_t s = 0; s < n * k; ++s) used |= ids[s] == e;
        if (!used) continue;
        if (!L->gate[e] || !L->up[e] || !L->down[e]) { rc = -1; break; }
        if (L->expert_bits == 4) {
            orc_dequant_q4k(L->gate[e], I * H / ORC_QK, Wg);
            orc_dequant_q4k(L->up[e], I * H / ORC_QK, Wu);
            orc_dequant_q4k(L->down[e], H * I / ORC_QK, Wd);
        } else {
            orc_dequant_iq2xxs(L->gate[e], I * H / ORC_QK, L->grid, Wg);
            orc_dequant_iq2xxs(L->up[e], I * H / ORC_QK, L->grid, Wu);
            orc_dequant_q2k(L->down[e], H * I / ORC_QK, Wd);
        }
        if (mode == 1)
            for (int64_t i = 0; i < I * H; ++i) {
                Wg[i] = orc_bf16_round(Wg[i]);
                Wu[i] = orc_bf16_round(Wu[i]);
                Wd[i] = orc_bf16_round(Wd[i]);
            }
        for (int64_t s = 0; s < n * k; ++s) {
            if (ids[s] != e) continue;
            const double* xt = xin + (s / k) * H;
            matvec_f(Wg, I, H, xt, g);
            matvec_f(Wu, I, H, xt, u);
            for (int64_t i = 0; i < I; ++i) {
                h[i] = silu(g[i]) * u[i];
                if (mode == 1) h[i] = (double)orc_bf16_round((float)h[i]);
            }
            matvec_f(Wd, H, I, h, yslot + s * H);
        }
    }
    for (int64_t t = 0; t < n && rc == 0; ++t) {
        const double* xt = xin + t * H;
        double* o = out + t * H;
        for (int64_t r = 0; r < H; ++r) o[r] = 0.0;
        if (L->sh_gate) {
            matvec_bf16(L->sh_gate, I, H, xt, g);
            matvec_bf16(L->sh_up, I, H, xt, u);
            for (int64_t i = 0; i < I; ++i) {
                h[i] = silu(g[i]) * u[i];
                if (mode == 1) h[i] = (double)orc_bf16_round((float)h[i]);
            }
            matvec_bf16(L->sh_down, H, I, h, y);
            for (int64_t r = 0; r < H; ++r) o[r] = y[r];
        }
        for (int32_t j = 0; j < k; ++j) {
            const double* ys = yslot + (t * k + j) * H;
            for (int64_t r = 0; r < H; ++r) o[r] += w[t * k + j] * ys[r];
        }
    }
    if (ids_out) memcpy(ids_out, ids, sizeof(int32_t) * (size_t)(n * k));
    if (w_out) memcpy(w_out, w, sizeof(double) * (size_t)(n * k));
    free(logits); free(ids); free(w); free(xin); free(yslot);
    free(Wg); free(Wu); free(Wd); free(g); free(u); free(h); free(y);
    return rc;
}
