/*
 * spot_oracle.c -- plain, slow, fp64 CPU oracle for the SpotAttention
 * decode-time hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  The product path
 * (the CUDA library under block_sparse_long_spot_b200/) never calls it and
 * shares no code, header, table or helper with it.
 *
 * Source: "SpotAttention: Plug-In Block-Sparse Routing for Pretrained
 * Long-Context Transformers" (arXiv HTML).  Each function names the section
 * or equation it follows.  Everything is computed in fp64 with plain loops,
 * in the order the definitions state; the only library primitives are exp(),
 * log(), frexp()/ldexp(), isfinite() and qsort().
 *
 * Readings taken where the paper is silent:
 *  - one selector key per (block, KV head); the index heads of a KV head are
 *    the G query heads of its GQA group, mixing weight w[b,h] (NULL -> 1/G);
 *  - the score of a block is s = (1/tau) * sum_h w_h * ReLU(q_h . k);
 *  - "reaches p" means cumulative mass >= p; equal scores rank lower block
 *    index first; p >= 1 takes the whole residual, p <= 0 an empty nucleus;
 *  - the K_min floor is counted on |S| (reserved blocks included) and is
 *    clamped to the number of blocks;
 *  - a block that is not complete (seq_len not a multiple of the block size)
 *    has no selector key and joins the recency set;
 *  - attention scale sigma is an argument (1/sqrt(D) in every workload);
 *    positions >= seq_len are not attended;
 *  - INT4 keys: symmetric, scale = fp16_rne(amax/7) per group of 32,
 *    code = clamp(rne(x/scale), -8, 7), two's complement nibbles, even
 *    element in the low nibble; a scale above the fp16 range saturates to
 *    65504;
 *  - FP4 keys: OCP Microscaling v1.0 MXFP4 -- E2M1 elements, one E8M0 scale
 *    per 32, X = floor(log2 amax) - 2 clamped to [-127, 127], elements
 *    rounded to nearest even on the E2M1 grid with saturation at 6; the sign
 *    bit is set only for x < 0; same nibble order as INT4;
 *  - FP8 keys: OCP FP8 E4M3 (bias 7, no infinities, S.1111.111 is NaN), one
 *    byte per element and no scale (8 bits = 0.5x bf16, App. G Tab. 9),
 *    round to nearest even, saturating at +-448;
 *  - INT8 keys: symmetric, one binary16 scale per key = fp16_rne(amax/127)
 *    (saturating at 65504), code = clamp(rne(x/scale), -128, 127);
 *  - non-finite inputs: OCP MX v1.0 gives a block that holds a NaN or an
 *    infinity the NaN shared scale.  The same rule is taken for every scaled
 *    format: a scale group (32 elements for INT4 / MXFP4, the whole key for
 *    INT8) holding NaN or +-inf stores the NaN scale (E8M0 0xFF, binary16
 *    0x7E00) and all-zero codes, so it reads back as NaN; FP8 stores a NaN or
 *    +-inf element as the E4M3 NaN 0x7F.  The selector score's ReLU maps an
 *    undefined (NaN) dot product to 0.
 *
 * Parity status: every function here is pinned by tests/test_oracle_pins.py
 * (hand-worked examples, brute force, closed forms, library special cases).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_FMT_BF16 = 0, ORC_FMT_INT4 = 1, ORC_FMT_MXFP4 = 2, ORC_FMT_FP8 = 3, ORC_FMT_INT8 = 4 };
enum { ORC_MODE_TOPP = 0, ORC_MODE_TOPK = 1 };

/* ------------------------------------------------------------------ */
/* Exact decoders of the storage formats.                              */
/* ------------------------------------------------------------------ */

/* bf16 is the top half of an IEEE binary32. */
static double bf16_to_f64(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
static double f16_to_f64(uint16_t bits) {
    int sign = bits >> 15;
    int e = (bits >> 10) & 0x1f;
    int m = bits & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);                 /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(m + 1024), e - 25);     /* (1 + m/1024) 2^(e-15) */
    return sign ? -v : v;
}

/* fp64 -> binary16, round to nearest even, finite overflow saturates to
 * the largest finite half (65504).  Only used for non-negative scales. */
static uint16_t f64_to_f16_sat(double x) {
    if (!(x > 0.0)) return 0;                      /* zero (and NaN -> 0) */
    if (x >= 65504.0) return 0x7bff;
    int ex;
    (void)frexp(x, &ex);                           /* x = f 2^ex, f in [.5,1) */
    int e = ex - 1;                                /* x in [2^e, 2^(e+1)) */
    if (e < -14) e = -14;                          /* subnormal range: ulp 2^-24 */
    double ulp = ldexp(1.0, e - 10);
    double q = x / ulp;                            /* exact (power-of-2 divide) */
    double r = floor(q);
    double frac = q - r;
    if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
    double y = r * ulp;                            /* rounded value, exact */
    if (y >= 65504.0) return 0x7bff;
    /* Re-encode y exactly. */
    if (y < ldexp(1.0, -14)) return (uint16_t)(y / ldexp(1.0, -24));
    (void)frexp(y, &ex);
    e = ex - 1;
    int mant = (int)(y / ldexp(1.0, e - 10)) - 1024;
    return (uint16_t)(((e + 15) << 10) | mant);
}

/* OCP MX v1.0 E2M1 element: sign, 2 exponent bits (bias 1), 1 mantissa bit.
 * Magnitudes by code 0..7: 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
static double e2m1_to_f64(unsigned code) {
    unsigned e = (code >> 1) & 3, m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, (int)e - 1);
    return (code & 8) ? -mag : mag;
}

/* OCP MX v1.0 E8M0 scale: 2^(E-127); E = 255 is NaN. */
static double e8m0_to_f64(uint8_t e) {
    return e == 255 ? NAN : ldexp(1.0, (int)e - 127);
}

/* OCP FP8 E4M3: sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent
 * 0 is subnormal (m 2^-9); S.1111.111 is NaN (no infinities). */
static double e4m3_to_f64(uint8_t code) {
    int e = (code >> 3) & 15, m = code & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) mag = ldexp((double)m, -9);
    else mag = ldexp(1.0 + m / 8.0, e - 7);
    return (code & 0x80) ? -mag : mag;
}

/* fp64 -> E4M3, round to nearest even, magnitudes beyond 448 saturate to
 * 448 (the largest finite E4M3); NaN and +-inf become the NaN 0x7F. */
static uint8_t f64_to_e4m3_sat(double x) {
    if (!isfinite(x)) return 0x7F;
    uint8_t sign = (x < 0.0) ? 0x80 : 0x00;
    double a = fabs(x);
    if (a >= 448.0) return sign | 0x7E;
    int ex;
    (void)frexp(a, &ex);                   /* a = f 2^ex, f in [.5, 1) */
    int e = ex - 1;                        /* a in [2^e, 2^(e+1)) */
    if (a == 0.0 || e < -6) e = -6;        /* subnormal range: ulp 2^-9 */
    double ulp = ldexp(1.0, e - 3);
    double q = a / ulp;                    /* exact */
    double r = floor(q);
    double frac = q - r;
    if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
    double y = r * ulp;                    /* rounded magnitude, exact */
    if (y >= 448.0) return sign | 0x7E;
    if (y < ldexp(1.0, -6)) return sign | (uint8_t)(y / ldexp(1.0, -9));
    (void)frexp(y, &ex);
    e = ex - 1;
    int mant = (int)(y / ldexp(1.0, e - 3)) - 8;
    return sign | (uint8_t)(((e + 7) << 3) | mant);
}

/* Dequantise `rows` selector keys of `ds` elements each into fp64.
 * bf16:  data = uint16 [rows][ds], scales unused.
 * INT4:  data = uint8 [rows][ds/2], scales = binary16 [rows][ds/32].
 * MXFP4: data = uint8 [rows][ds/2], scales = E8M0 [rows][ds/32].
 * FP8:   data = uint8 E4M3 [rows][ds], scales unused.
 * INT8:  data = int8 [rows][ds], scales = binary16 [rows][1].
 * Returns 0, or -1 for an unknown format. */
int oracle_dequant_selector(int fmt, int64_t rows, int ds, const void* data,
                            const void* scales, double* out) {
    for (int64_t r = 0; r < rows; ++r) {
        for (int i = 0; i < ds; ++i) {
            double v;
            if (fmt == ORC_FMT_BF16) {
                v = bf16_to_f64(((const uint16_t*)data)[r * ds + i]);
            } else if (fmt == ORC_FMT_FP8) {
                v = e4m3_to_f64(((const uint8_t*)data)[r * ds + i]);
            } else if (fmt == ORC_FMT_INT8) {
                v = (double)((const int8_t*)data)[r * ds + i] * f16_to_f64(((const uint16_t*)scales)[r]);
            } else if (fmt == ORC_FMT_INT4 || fmt == ORC_FMT_MXFP4) {
                uint8_t byte = ((const uint8_t*)data)[r * (ds / 2) + i / 2];
                unsigned nib = (i % 2 == 0) ? (byte & 0xf) : (byte >> 4);
                if (fmt == ORC_FMT_INT4) {
                    int q = (nib >= 8) ? (int)nib - 16 : (int)nib;
                    double s = f16_to_f64(((const uint16_t*)scales)[r * (ds / 32) + i / 32]);
                    v = (double)q * s;
                } else {
                    double s = e8m0_to_f64(((const uint8_t*)scales)[r * (ds / 32) + i / 32]);
                    v = e2m1_to_f64(nib) * s;
                }
            } else {
                return -1;
            }
            out[r * ds + i] = v;
        }
    }
    return 0;
}

/* binary16 quiet NaN: the scale of an INT4 group or INT8 key that holds a
 * NaN or an infinity. */
#define F16_NAN_BITS ((uint16_t)0x7E00)

/* Round |a| to the E2M1 grid, nearest, ties to the even code, saturating
 * at 6.  Returns the 3-bit magnitude code. */
static unsigned e2m1_rne_code(double a) {
    static const double grid[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    if (a >= 6.0) return 7;
    for (unsigned c = 0; c < 7; ++c) {
        if (a <= grid[c + 1]) {
            double mid = 0.5 * (grid[c] + grid[c + 1]);
            if (a < mid) return c;
            if (a > mid) return c + 1;
            return (c % 2 == 0) ? c : c + 1;
        }
    }
    return 7;
}

/* Quantise bf16 selector keys (the append step of the selector K-cache,
 * SpotAttention §5.3 and App. G: group-32 INT4 / FP4 microscale, INT8, FP8).
 * Layouts as in oracle_dequant_selector.  bf16 is a plain copy. */
int oracle_quantize_selector(int fmt, int64_t rows, int ds, const uint16_t* keys,
                             void* data, void* scales) {
    if (ds % 32 != 0) return -1;
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t* row = keys + r * ds;
        if (fmt == ORC_FMT_BF16) {
            memcpy((uint16_t*)data + r * ds, row, (size_t)ds * sizeof(uint16_t));
            continue;
        }
        if (fmt == ORC_FMT_FP8) {
            for (int i = 0; i < ds; ++i)
                ((uint8_t*)data)[r * ds + i] = f64_to_e4m3_sat(bf16_to_f64(row[i]));
            continue;
        }
        if (fmt == ORC_FMT_INT8) {
            double amax = 0.0;
            int finite = 1;
            for (int i = 0; i < ds; ++i) {
                double x = fabs(bf16_to_f64(row[i]));
                if (!isfinite(x)) finite = 0;
                else if (x > amax) amax = x;
            }
            if (!finite) {                         /* NaN scale, zero codes */
                ((uint16_t*)scales)[r] = F16_NAN_BITS;
                memset((int8_t*)data + r * ds, 0, (size_t)ds);
                continue;
            }
            uint16_t sbits = f64_to_f16_sat(amax / 127.0);
            ((uint16_t*)scales)[r] = sbits;
            double sc = f16_to_f64(sbits);
            for (int i = 0; i < ds; ++i) {
                int q = 0;
                if (sc > 0.0) {
                    double t = nearbyint(bf16_to_f64(row[i]) / sc);    /* ties to even */
                    if (t > 127.0) t = 127.0;
                    if (t < -128.0) t = -128.0;
                    q = (int)t;
                }
                ((int8_t*)data)[r * ds + i] = (int8_t)q;
            }
            continue;
        }
        uint8_t* out = (uint8_t*)data + r * (ds / 2);
        memset(out, 0, (size_t)ds / 2);
        for (int g = 0; g < ds / 32; ++g) {
            double amax = 0.0;
            int finite = 1;
            for (int i = 0; i < 32; ++i) {
                double x = fabs(bf16_to_f64(row[g * 32 + i]));
                if (!isfinite(x)) finite = 0;
                else if (x > amax) amax = x;
            }
            if (!finite) {                         /* NaN scale; the codes stay 0 */
                if (fmt == ORC_FMT_INT4)
                    ((uint16_t*)scales)[r * (ds / 32) + g] = F16_NAN_BITS;
                else if (fmt == ORC_FMT_MXFP4)
                    ((uint8_t*)scales)[r * (ds / 32) + g] = 0xFF;
                else
                    return -1;
                continue;
            }
            if (fmt == ORC_FMT_INT4) {
                uint16_t sbits = f64_to_f16_sat(amax / 7.0);
                ((uint16_t*)scales)[r * (ds / 32) + g] = sbits;
                double s = f16_to_f64(sbits);
                for (int i = 0; i < 32; ++i) {
                    double x = bf16_to_f64(row[g * 32 + i]);
                    int q = 0;
                    if (s > 0.0) {
                        double t = nearbyint(x / s);       /* ties to even */
                        if (t > 7.0) t = 7.0;
                        if (t < -8.0) t = -8.0;
                        q = (int)t;
                    }
                    unsigned nib = (unsigned)q & 0xf;
                    int idx = g * 32 + i;
                    out[idx / 2] |= (uint8_t)((idx % 2 == 0) ? nib : (nib << 4));
                }
            } else if (fmt == ORC_FMT_MXFP4) {
                int X;
                if (amax == 0.0) {
                    X = -127;
                } else {
                    int ex;
                    (void)frexp(amax, &ex);       /* amax = f 2^ex, f in [.5,1) */
                    X = (ex - 1) - 2;             /* floor(log2 amax) - emax(E2M1) */
                    if (X < -127) X = -127;
                    if (X > 127) X = 127;
                }
                ((uint8_t*)scales)[r * (ds / 32) + g] = (uint8_t)(X + 127);
                for (int i = 0; i < 32; ++i) {
                    double x = bf16_to_f64(row[g * 32 + i]);
                    double v = ldexp(x, -X);
                    unsigned code = e2m1_rne_code(fabs(v)) | (x < 0.0 ? 8u : 0u);
                    int idx = g * 32 + i;
                    out[idx / 2] |= (uint8_t)((idx % 2 == 0) ? code : (code << 4));
                }
            } else {
                return -1;
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Shapes shared by the functions below.                               */
/* ------------------------------------------------------------------ */

typedef struct {
    int32_t batch, num_q_heads, num_kv_heads, head_dim, block_size, sel_dim;
    int32_t sel_fmt, num_pages, max_blocks;
} orc_shape_t;

typedef struct {
    int32_t mode;          /* ORC_MODE_TOPP (Eq. 8) or ORC_MODE_TOPK (Eq. 6) */
    int32_t sink_blocks, recency_blocks, kmin_blocks, topk_blocks;
    double temperature;
    int32_t quantize_queries;  /* 1: selector queries quantised like the keys */
} orc_params_t;

static int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

/* Selector queries of KV head g's G query heads for sequence b, as fp64
 * [G][ds].  With quantize_queries (SpotAttention §5.3 and App. G Tab. 9: the
 * selector's queries and key cache are quantised together, at inference)
 * each query row goes through the same quantiser as a key row of the
 * selector format and is read back exactly; otherwise the bf16 values are
 * widened.  Returns 0, or -1 for an unknown format. */
static int unit_queries(const orc_shape_t* sh, const orc_params_t* pr, int b, int g,
                        const uint16_t* q_sel, double* qv) {
    int G = sh->num_q_heads / sh->num_kv_heads;
    int ds = sh->sel_dim;
    const uint16_t* q0 = q_sel + ((int64_t)b * sh->num_q_heads + (int64_t)g * G) * ds;
    if (!pr->quantize_queries || sh->sel_fmt == ORC_FMT_BF16) {
        for (int64_t i = 0; i < (int64_t)G * ds; ++i) qv[i] = bf16_to_f64(q0[i]);
        return 0;
    }
    /* room for the largest row of codes (ds bytes) and scales (ds/32 x 2 bytes) */
    uint8_t* codes = (uint8_t*)malloc((size_t)G * ds);
    uint16_t* scales = (uint16_t*)malloc((size_t)G * (ds / 32 + 1) * sizeof(uint16_t));
    int rc = (codes && scales) ? 0 : -2;
    if (rc == 0) rc = oracle_quantize_selector(sh->sel_fmt, G, ds, q0, codes, scales);
    if (rc == 0) rc = oracle_dequant_selector(sh->sel_fmt, G, ds, codes, scales, qv);
    free(codes);
    free(scales);
    return rc;
}

/* Selector score for every complete block of sequence b, KV head g
 * (SpotAttention §2.1: s = sum_h w_h ReLU(q^I_h . k^I); block score = max
 * over the block's keys, §2.3, which is the single key here; temperature
 * from App. A Tab. 3).  qv = the unit's queries from unit_queries;
 * keys_f64 = dequantised selector pool [num_pages][Hkv][ds].  Writes n_full
 * scores into out. */
static void unit_scores(const orc_shape_t* sh, const orc_params_t* pr, int b, int g,
                        const double* qv, const float* w, const double* keys_f64,
                        const int32_t* page_table, int64_t n_full, double* out) {
    int G = sh->num_q_heads / sh->num_kv_heads;
    int ds = sh->sel_dim;
    for (int64_t j = 0; j < n_full; ++j) {
        int32_t page = page_table[(int64_t)b * sh->max_blocks + j];
        const double* k = keys_f64 + ((int64_t)page * sh->num_kv_heads + g) * ds;
        double s = 0.0;
        for (int i = 0; i < G; ++i) {
            int h = g * G + i;
            const double* q = qv + (int64_t)i * ds;
            double dot = 0.0;
            for (int d = 0; d < ds; ++d) dot += q[d] * k[d];
            double wh = w ? (double)w[(int64_t)b * sh->num_q_heads + h] : 1.0 / G;
            s += wh * (dot > 0.0 ? dot : 0.0);
        }
        out[j] = s / pr->temperature;
    }
}

/* Public form of unit_scores over all (b, g): scores[b][g][j] for
 * j < floor(seq_len/bs); entries beyond are left untouched. */
int oracle_block_scores(const orc_shape_t* sh, const orc_params_t* pr, const uint16_t* q_sel,
                        const float* w, const void* sel_data, const void* sel_scales,
                        const int32_t* page_table, const int32_t* seq_lens, double* scores) {
    int64_t rows = (int64_t)sh->num_pages * sh->num_kv_heads;
    double* keys = (double*)malloc((size_t)(rows * sh->sel_dim) * sizeof(double));
    if (!keys) return -2;
    if (oracle_dequant_selector(sh->sel_fmt, rows, sh->sel_dim, sel_data, sel_scales, keys)) {
        free(keys);
        return -1;
    }
    int G = sh->num_q_heads / sh->num_kv_heads;
    double* qv = (double*)malloc((size_t)G * sh->sel_dim * sizeof(double));
    int rc = qv ? 0 : -2;
    for (int b = 0; b < sh->batch && rc == 0; ++b)
        for (int g = 0; g < sh->num_kv_heads && rc == 0; ++g) {
            rc = unit_queries(sh, pr, b, g, q_sel, qv);
            if (rc == 0)
                unit_scores(sh, pr, b, g, qv, w, keys, page_table, seq_lens[b] / sh->block_size,
                            scores + ((int64_t)b * sh->num_kv_heads + g) * sh->max_blocks);
        }
    free(qv);
    free(keys);
    return rc;
}

/* Ranking of residual blocks: score descending, lower block index first. */
typedef struct { double s; int32_t j; } ranked_t;
static int rank_cmp(const void* a, const void* b) {
    const ranked_t* x = (const ranked_t*)a;
    const ranked_t* y = (const ranked_t*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->j < y->j) ? -1 : (x->j > y->j);
}

/* Block selection for one (sequence, KV head) from its block scores
 * (SpotAttention §2.3).
 *   nb       = number of blocks, n_full = blocks that have a score;
 *   TOPP:    S = S_sink U S_rec U S_nuc, S_nuc the smallest prefix of the
 *            residual blocks ranked by the residual softmax (Eq. 7) whose
 *            cumulative mass reaches p; |S| >= K_min extends along the same
 *            ranking (Eq. 8);
 *   TOPK:    S = the topk_blocks best blocks (Eq. 6), still after the
 *            reserved sink / recency blocks.
 * Writes the selected block ids ascending into sel (capacity nb) and returns
 * their count.  nuc_mass (may be NULL) receives the residual-softmax mass of
 * the chosen residual blocks. */
int oracle_select_from_scores(const double* scores, int32_t nb, int32_t n_full,
                              const orc_params_t* pr, double p, int32_t* sel, double* nuc_mass) {
    if (nb <= 0) { if (nuc_mass) *nuc_mass = 0.0; return 0; }
    int32_t sink = pr->sink_blocks < nb ? pr->sink_blocks : nb;
    if (sink < 0) sink = 0;
    int32_t rec = pr->recency_blocks > 0 ? pr->recency_blocks : 0;
    if (rec < nb - n_full) rec = nb - n_full;          /* incomplete block has no key */
    if (rec > nb) rec = nb;
    char* keep = (char*)calloc((size_t)nb, 1);
    ranked_t* res = (ranked_t*)malloc((size_t)nb * sizeof(ranked_t));
    int32_t n_res = 0, n_reserved = 0;
    for (int32_t j = 0; j < nb; ++j) {
        if (j < sink || j >= nb - rec) { keep[j] = 1; ++n_reserved; }
        else { res[n_res].s = scores[j]; res[n_res].j = j; ++n_res; }
    }
    int32_t n_take = 0;
    double taken_mass = 0.0;
    if (n_res > 0) {
        /* Residual softmax, Eq. 7. */
        double m = res[0].s;
        for (int32_t k = 1; k < n_res; ++k) if (res[k].s > m) m = res[k].s;
        double Z = 0.0;
        for (int32_t k = 0; k < n_res; ++k) Z += exp(res[k].s - m);
        qsort(res, (size_t)n_res, sizeof(ranked_t), rank_cmp);
        if (pr->mode == ORC_MODE_TOPK) {
            n_take = pr->topk_blocks;
        } else {
            if (p >= 1.0) {
                n_take = n_res;
            } else if (p <= 0.0) {
                n_take = 0;                           /* the empty prefix reaches p */
            } else {
                double cum = 0.0;
                n_take = n_res;                       /* never reached: take all */
                for (int32_t k = 0; k < n_res; ++k) {
                    cum += exp(res[k].s - m) / Z;
                    if (cum >= p) { n_take = k + 1; break; }
                }
            }
            int32_t floor_res = pr->kmin_blocks - n_reserved;   /* |S| >= K_min */
            if (n_take < floor_res) n_take = floor_res;
        }
        if (n_take > n_res) n_take = n_res;
        if (n_take < 0) n_take = 0;
        for (int32_t k = 0; k < n_take; ++k) {
            keep[res[k].j] = 1;
            taken_mass += exp(res[k].s - m) / Z;
        }
    }
    int32_t cnt = 0;
    for (int32_t j = 0; j < nb; ++j) if (keep[j]) sel[cnt++] = j;
    if (nuc_mass) *nuc_mass = taken_mass;
    free(keep);
    free(res);
    return cnt;
}

/* Exact softmax attention of the G query heads of KV head g over the tokens
 * of the selected blocks (SpotAttention §2.3: the layer attends only to keys
 * in the selected blocks; §3: decode only).  Selected block j covers
 * positions [j*sb, (j+1)*sb); position t sits in pool page
 * page_table[b][t / ps] (row stride pt_stride), row t % ps of that page
 * (pool layout [pages][Hkv][ps][D]).  Positions >= seq_len are not attended.
 * out[h][D] and lse[h] (natural log of the softmax denominator, -inf when no
 * token is attended, out = 0 then). */
static void attend_blocks(int Hq, int Hkv, int D, int ps, int64_t pt_stride, int sb, int b,
                          int g, const uint16_t* q, const uint16_t* k_pool,
                          const uint16_t* v_pool, const int32_t* page_table, int32_t seq_len,
                          const int32_t* sel, int32_t cnt, double sm_scale, double* out,
                          double* lse) {
    int G = Hq / Hkv;
    int64_t ntok_max = (int64_t)cnt * sb;
    double* logit = (double*)malloc((size_t)(ntok_max > 0 ? ntok_max : 1) * sizeof(double));
    int64_t* row = (int64_t*)malloc((size_t)(ntok_max > 0 ? ntok_max : 1) * sizeof(int64_t));
    for (int i = 0; i < G; ++i) {
        int h = g * G + i;
        const uint16_t* qh = q + ((int64_t)b * Hq + h) * D;
        int64_t n = 0;
        for (int32_t c = 0; c < cnt; ++c) {
            int32_t j = sel[c];
            for (int t = 0; t < sb; ++t) {
                int64_t pos = (int64_t)j * sb + t;
                if (pos >= seq_len) break;
                int32_t page = page_table[(int64_t)b * pt_stride + pos / ps];
                int64_t r = (((int64_t)page * Hkv + g) * ps + pos % ps) * D;
                double dot = 0.0;
                for (int d = 0; d < D; ++d) dot += bf16_to_f64(qh[d]) * bf16_to_f64(k_pool[r + d]);
                logit[n] = sm_scale * dot;
                row[n] = r;
                ++n;
            }
        }
        double* o = out + (int64_t)i * D;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        if (n == 0) { lse[i] = -INFINITY; continue; }
        double m = logit[0];
        for (int64_t k = 1; k < n; ++k) if (logit[k] > m) m = logit[k];
        double z = 0.0;
        for (int64_t k = 0; k < n; ++k) z += exp(logit[k] - m);
        for (int64_t k = 0; k < n; ++k) {
            double pk = exp(logit[k] - m) / z;
            for (int d = 0; d < D; ++d) o[d] += pk * bf16_to_f64(v_pool[row[k] + d]);
        }
        lse[i] = m + log(z);
    }
    free(logit);
    free(row);
}

/* The per-(block, KV head) selector's attention: selection blocks are the
 * pool pages (sb = ps = block_size), page table row stride max_blocks. */
static void unit_attention(const orc_shape_t* sh, int b, int g, const uint16_t* q,
                           const uint16_t* k_pool, const uint16_t* v_pool,
                           const int32_t* page_table, int32_t seq_len, const int32_t* sel,
                           int32_t cnt, double sm_scale, double* out, double* lse) {
    attend_blocks(sh->num_q_heads, sh->num_kv_heads, sh->head_dim, sh->block_size,
                  sh->max_blocks, sh->block_size, b, g, q, k_pool, v_pool, page_table, seq_len,
                  sel, cnt, sm_scale, out, lse);
}

/* Attention over given selections, for every (b, g):
 * sel_idx[b][g][max_blocks], sel_cnt[b][g]; out[b][h][D], lse[b][h]. */
int oracle_sparse_attention(const orc_shape_t* sh, const uint16_t* q, const uint16_t* k_pool,
                            const uint16_t* v_pool, const int32_t* page_table,
                            const int32_t* seq_lens, const int32_t* sel_idx,
                            const int32_t* sel_cnt, double sm_scale, double* out, double* lse) {
    int G = sh->num_q_heads / sh->num_kv_heads;
    int units = sh->batch * sh->num_kv_heads;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int u = 0; u < units; ++u) {
        int b = u / sh->num_kv_heads, g = u % sh->num_kv_heads;
        unit_attention(sh, b, g, q, k_pool, v_pool, page_table, seq_lens[b],
                       sel_idx + (int64_t)u * sh->max_blocks, sel_cnt[u], sm_scale,
                       out + ((int64_t)b * sh->num_q_heads + g * G) * sh->head_dim,
                       lse + (int64_t)b * sh->num_q_heads + g * G);
    }
    return 0;
}

/* The whole decode step for a list of units (b, g) -- scoring, residual
 * softmax, dual top-p (or static top-K), sparse attention -- as
 * SpotAttention §2.1 and §2.3 define it.  units[n_units] holds b*Hkv+g;
 * NULL means every unit.  Outputs are indexed as in the full problem:
 * sel_idx[b][g][max_blocks], sel_cnt[b][g], nuc_mass[b][g] (may be NULL),
 * out[b][h][D], lse[b][h].  Units run in parallel when built with OpenMP. */
int oracle_decode_step(const orc_shape_t* sh, const orc_params_t* pr, const uint16_t* q_sel,
                       const float* w, const void* sel_data, const void* sel_scales,
                       const uint16_t* q, const uint16_t* k_pool, const uint16_t* v_pool,
                       const int32_t* page_table, const int32_t* seq_lens, const float* top_p,
                       double sm_scale, const int32_t* units, int32_t n_units,
                       int32_t* sel_idx, int32_t* sel_cnt, double* nuc_mass, double* out,
                       double* lse) {
    int G = sh->num_q_heads / sh->num_kv_heads;
    int64_t rows = (int64_t)sh->num_pages * sh->num_kv_heads;
    double* keys = (double*)malloc((size_t)(rows * sh->sel_dim) * sizeof(double));
    if (!keys) return -2;
    if (oracle_dequant_selector(sh->sel_fmt, rows, sh->sel_dim, sel_data, sel_scales, keys)) {
        free(keys);
        return -1;
    }
    int total = units ? n_units : sh->batch * sh->num_kv_heads;
    int err = 0;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int k = 0; k < total; ++k) {
        int u = units ? units[k] : k;
        int b = u / sh->num_kv_heads, g = u % sh->num_kv_heads;
        int32_t L = seq_lens[b];
        int64_t nb = ceil_div64(L, sh->block_size), n_full = L / sh->block_size;
        double* s = (double*)malloc((size_t)(nb > 0 ? nb : 1) * sizeof(double));
        double* qv = (double*)malloc((size_t)G * sh->sel_dim * sizeof(double));
        if (!s || !qv || unit_queries(sh, pr, b, g, q_sel, qv) != 0) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = -2;
            free(s);
            free(qv);
            continue;
        }
        unit_scores(sh, pr, b, g, qv, w, keys, page_table, n_full, s);
        free(qv);
        int32_t* sel = sel_idx + (int64_t)u * sh->max_blocks;
        double mass = 0.0;
        int32_t cnt = oracle_select_from_scores(s, (int32_t)nb, (int32_t)n_full, pr,
                                                (double)top_p[b], sel, &mass);
        sel_cnt[u] = cnt;
        if (nuc_mass) nuc_mass[u] = mass;
        unit_attention(sh, b, g, q, k_pool, v_pool, page_table, L, sel, cnt, sm_scale,
                       out + ((int64_t)b * sh->num_q_heads + g * G) * sh->head_dim,
                       lse + (int64_t)b * sh->num_q_heads + g * G);
        free(s);
    }
    free(keys);
    return err;
}

/* ------------------------------------------------------------------ */
/* Sparse prefill (§2.3 applied to a chunk of queries).                */
/* ------------------------------------------------------------------ */

/* Sequence b holds seq_lens[b] tokens in the cache; its last q_lens[b] are
 * the chunk's queries, packed as rows q_off(b) .. q_off(b) + q_lens[b] - 1
 * of q / q_sel / w / out / lse (q_off = running sum of q_lens).  A query
 * tile is the set of chunk queries whose positions fall in one KV block m;
 * tiles are numbered sequence by sequence, m ascending.  Tile (b, m) selects
 * for each KV head exactly as a decode query at L_eff = 1 + the tile's last
 * position would (Eq. 6-8, sink / recency / K_min, the incomplete block
 * kept), from the block scores s[j] = max over the tile's queries of the
 * query's score (1/tau) sum_h w_h ReLU(q^I_h . k_j) -- the paper's
 * per-block maximum taken over the query block as well (§2.1: one score per
 * query-block x key-block tile).  Every query then attends, causally (key
 * positions <= its own), to the tokens of its tile's selected blocks. */

static int64_t prefill_tiles_of(int32_t seq_len, int32_t q_len, int bs) {
    if (q_len <= 0) return 0;
    int32_t q_start = seq_len - q_len;
    return (int64_t)((seq_len - 1) / bs) - (q_start / bs) + 1;
}

/* Number of query tiles of the whole batch (the rows of sel_idx / sel_cnt). */
int64_t oracle_prefill_num_tiles(const orc_shape_t* sh, const int32_t* seq_lens,
                                 const int32_t* q_lens) {
    int64_t t = 0;
    for (int b = 0; b < sh->batch; ++b) t += prefill_tiles_of(seq_lens[b], q_lens[b], sh->block_size);
    return t;
}

/* Locate tile `tile`: sequence, first / last query position, first row. */
static void prefill_tile(const orc_shape_t* sh, const int32_t* seq_lens, const int32_t* q_lens,
                         int64_t tile, int* b_out, int32_t* p_lo, int32_t* p_hi, int64_t* row0) {
    int bs = sh->block_size;
    int64_t t = tile, off = 0;
    for (int b = 0; b < sh->batch; ++b) {
        int64_t n = prefill_tiles_of(seq_lens[b], q_lens[b], bs);
        if (t < n) {
            int32_t q_start = seq_lens[b] - q_lens[b];
            int32_t m = q_start / bs + (int32_t)t;
            *b_out = b;
            *p_lo = m * bs > q_start ? m * bs : q_start;
            *p_hi = m * bs + bs - 1 < seq_lens[b] - 1 ? m * bs + bs - 1 : seq_lens[b] - 1;
            *row0 = off + (*p_lo - q_start);
            return;
        }
        t -= n;
        off += q_lens[b] > 0 ? q_lens[b] : 0;
    }
    *b_out = -1;
}

/* Scores of tile `tile` for KV head g: s[j], j < floor(L_eff / bs). */
static int prefill_tile_scores(const orc_shape_t* sh, const orc_params_t* pr,
                               const uint16_t* q_sel, const float* w, const double* keys_f64,
                               const int32_t* page_table, int b, int32_t p_lo, int32_t p_hi,
                               int64_t row0, int g, double* s) {
    int G = sh->num_q_heads / sh->num_kv_heads, ds = sh->sel_dim;
    int64_t n_full = (int64_t)(p_hi + 1) / sh->block_size;
    double* qv = (double*)malloc((size_t)G * ds * sizeof(double));
    double* tmp = (double*)malloc((size_t)(n_full > 0 ? n_full : 1) * sizeof(double));
    if (!qv || !tmp) { free(qv); free(tmp); return -2; }
    for (int64_t j = 0; j < n_full; ++j) s[j] = -INFINITY;
    /* the query rows are laid out like a batch of rows: row r plays "b = r" */
    orc_shape_t rs = *sh;
    rs.max_blocks = sh->max_blocks;
    for (int32_t pos = p_lo; pos <= p_hi; ++pos) {
        int64_t r = row0 + (pos - p_lo);
        if (unit_queries(&rs, pr, (int)r, g, q_sel, qv)) { free(qv); free(tmp); return -1; }
        for (int64_t j = 0; j < n_full; ++j) {
            int32_t page = page_table[(int64_t)b * sh->max_blocks + j];
            const double* k = keys_f64 + ((int64_t)page * sh->num_kv_heads + g) * ds;
            double sc = 0.0;
            for (int i = 0; i < G; ++i) {
                int h = g * G + i;
                const double* qq = qv + (int64_t)i * ds;
                double dot = 0.0;
                for (int d = 0; d < ds; ++d) dot += qq[d] * k[d];
                double wh = w ? (double)w[r * sh->num_q_heads + h] : 1.0 / G;
                sc += wh * (dot > 0.0 ? dot : 0.0);
            }
            sc /= pr->temperature;
            if (sc > s[j]) s[j] = sc;
        }
    }
    free(qv);
    free(tmp);
    return 0;
}

/* Block scores of the tiles `tiles[n_tiles]` (NULL: all):
 * scores[tile][g][max_blocks] (entries past a tile's complete blocks
 * untouched). */
int oracle_prefill_scores(const orc_shape_t* sh, const orc_params_t* pr, const uint16_t* q_sel,
                          const float* w, const void* sel_data, const void* sel_scales,
                          const int32_t* page_table, const int32_t* seq_lens,
                          const int32_t* q_lens, const int32_t* tiles, int32_t n_tiles,
                          double* scores) {
    int64_t rows = (int64_t)sh->num_pages * sh->num_kv_heads;
    double* keys = (double*)malloc((size_t)(rows * sh->sel_dim) * sizeof(double));
    if (!keys) return -2;
    if (oracle_dequant_selector(sh->sel_fmt, rows, sh->sel_dim, sel_data, sel_scales, keys)) {
        free(keys);
        return -1;
    }
    int64_t nt = tiles ? n_tiles : oracle_prefill_num_tiles(sh, seq_lens, q_lens);
    int err = 0;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int64_t k = 0; k < nt * sh->num_kv_heads; ++k) {
        int64_t t = tiles ? tiles[k / sh->num_kv_heads] : k / sh->num_kv_heads;
        int g = (int)(k % sh->num_kv_heads);
        int b;
        int32_t p_lo, p_hi;
        int64_t row0;
        prefill_tile(sh, seq_lens, q_lens, t, &b, &p_lo, &p_hi, &row0);
        if (prefill_tile_scores(sh, pr, q_sel, w, keys, page_table, b, p_lo, p_hi, row0, g,
                                scores + (t * sh->num_kv_heads + g) * sh->max_blocks)) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = -2;
        }
    }
    free(keys);
    return err;
}

/* The whole sparse-prefill step for tiles `tiles[n_tiles]` (NULL: all):
 * selection per (tile, KV head) into sel_idx[tile][g][max_blocks] /
 * sel_cnt[tile][g], and out[row][h][D] / lse[row][h] of the tiles' query
 * rows (rows of other tiles untouched). */
int oracle_prefill_step(const orc_shape_t* sh, const orc_params_t* pr, const uint16_t* q_sel,
                        const float* w, const void* sel_data, const void* sel_scales,
                        const uint16_t* q, const uint16_t* k_pool, const uint16_t* v_pool,
                        const int32_t* page_table, const int32_t* seq_lens,
                        const int32_t* q_lens, const float* top_p, double sm_scale,
                        const int32_t* tiles, int32_t n_tiles, int32_t* sel_idx,
                        int32_t* sel_cnt, double* out, double* lse) {
    int G = sh->num_q_heads / sh->num_kv_heads;
    int64_t rows = (int64_t)sh->num_pages * sh->num_kv_heads;
    double* keys = (double*)malloc((size_t)(rows * sh->sel_dim) * sizeof(double));
    if (!keys) return -2;
    if (oracle_dequant_selector(sh->sel_fmt, rows, sh->sel_dim, sel_data, sel_scales, keys)) {
        free(keys);
        return -1;
    }
    int64_t total = tiles ? n_tiles : oracle_prefill_num_tiles(sh, seq_lens, q_lens);
    int err = 0;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int64_t k = 0; k < total * sh->num_kv_heads; ++k) {
        int64_t t = tiles ? tiles[k / sh->num_kv_heads] : k / sh->num_kv_heads;
        int g = (int)(k % sh->num_kv_heads);
        int b;
        int32_t p_lo, p_hi;
        int64_t row0;
        prefill_tile(sh, seq_lens, q_lens, t, &b, &p_lo, &p_hi, &row0);
        int32_t L_eff = p_hi + 1;
        int64_t nb = ceil_div64(L_eff, sh->block_size), n_full = L_eff / sh->block_size;
        double* s = (double*)malloc((size_t)(nb > 0 ? nb : 1) * sizeof(double));
        if (!s || prefill_tile_scores(sh, pr, q_sel, w, keys, page_table, b, p_lo, p_hi, row0,
                                      g, s)) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = -2;
            free(s);
            continue;
        }
        int32_t* sel = sel_idx + (t * sh->num_kv_heads + g) * sh->max_blocks;
        double mass = 0.0;
        int32_t cnt = oracle_select_from_scores(s, (int32_t)nb, (int32_t)n_full, pr,
                                                (double)top_p[b], sel, &mass);
        sel_cnt[t * sh->num_kv_heads + g] = cnt;
        for (int32_t pos = p_lo; pos <= p_hi; ++pos) {
            int64_t r = row0 + (pos - p_lo);
            attend_blocks(sh->num_q_heads, sh->num_kv_heads, sh->head_dim, sh->block_size,
                          sh->max_blocks, sh->block_size, 0, g,
                          q + r * sh->num_q_heads * sh->head_dim, k_pool, v_pool,
                          page_table + (int64_t)b * sh->max_blocks, pos + 1, sel, cnt, sm_scale,
                          out + (r * sh->num_q_heads + g * G) * sh->head_dim,
                          lse + r * sh->num_q_heads + g * G);
        }
        (void)n_full;
        free(s);
    }
    free(keys);
    return err;
}

/* ------------------------------------------------------------------ */
/* Token-level, layer-shared selector (SpotAttention §2.1, §2.3 and    */
/* App. A Tab. 3 as written).                                          */
/* ------------------------------------------------------------------ */

typedef struct {
    int32_t batch, num_q_heads, num_kv_heads, head_dim;
    int32_t page_size;       /* tokens per pool page (KV and selector pools) */
    int32_t idx_heads;       /* H_idx */
    int32_t idx_dim;         /* d_idx */
    int32_t sel_block;       /* tokens per selection block; divides page_size */
    int32_t num_pages;
    int32_t max_pages;       /* page-table row stride */
    int32_t max_blocks;      /* selection row stride (sel_idx, scores) */
    int32_t sel_fmt;         /* ORC_FMT_*: each (token, head) key row of d_idx elements is
                                stored like a selector key row (oracle_dequant_selector) */
} orc_tok_shape_t;

/* Exact values of key row `row` (= (page * page_size + slot) * H_idx + h) of
 * a per-token selector pool stored in sh->sel_fmt. */
static int tok_key_row(const orc_tok_shape_t* sh, const void* data, const void* scales,
                       int64_t row, double* out) {
    int di = sh->idx_dim;
    switch (sh->sel_fmt) {
        case ORC_FMT_BF16:
            return oracle_dequant_selector(ORC_FMT_BF16, 1, di,
                                           (const uint16_t*)data + row * di, NULL, out);
        case ORC_FMT_FP8:
            return oracle_dequant_selector(ORC_FMT_FP8, 1, di,
                                           (const uint8_t*)data + row * di, NULL, out);
        case ORC_FMT_INT8:
            return oracle_dequant_selector(ORC_FMT_INT8, 1, di, (const int8_t*)data + row * di,
                                           (const uint16_t*)scales + row, out);
        case ORC_FMT_INT4:
            return oracle_dequant_selector(ORC_FMT_INT4, 1, di,
                                           (const uint8_t*)data + row * (di / 2),
                                           (const uint16_t*)scales + row * (di / 32), out);
        case ORC_FMT_MXFP4:
            return oracle_dequant_selector(ORC_FMT_MXFP4, 1, di,
                                           (const uint8_t*)data + row * (di / 2),
                                           (const uint8_t*)scales + row * (di / 32), out);
    }
    return -1;
}

/* The index-head queries of sequence b as fp64 [H_idx][d_idx].  With
 * quantize_queries (SpotAttention §5.3 and App. G Tab. 9 quantise the
 * selector's queries together with its key cache) each head's query row
 * goes through the same quantiser as a key row of the format and is read
 * back exactly; otherwise the bf16 values are widened. */
static int tok_queries(const orc_tok_shape_t* sh, const orc_params_t* pr, int b,
                       const uint16_t* q_idx, double* qv) {
    int Hi = sh->idx_heads, di = sh->idx_dim;
    const uint16_t* q0 = q_idx + (int64_t)b * Hi * di;
    if (!pr->quantize_queries || sh->sel_fmt == ORC_FMT_BF16) {
        for (int64_t i = 0; i < (int64_t)Hi * di; ++i) qv[i] = bf16_to_f64(q0[i]);
        return 0;
    }
    uint8_t* codes = (uint8_t*)malloc((size_t)Hi * di);
    uint16_t* scales = (uint16_t*)malloc((size_t)Hi * (di / 32 + 1) * sizeof(uint16_t));
    int rc = (codes && scales) ? 0 : -2;
    if (rc == 0) rc = oracle_quantize_selector(sh->sel_fmt, Hi, di, q0, codes, scales);
    if (rc == 0) rc = oracle_dequant_selector(sh->sel_fmt, Hi, di, codes, scales, qv);
    free(codes);
    free(scales);
    return rc;
}

/* Score of every complete selection block of sequence b (§2.1 and §2.3):
 * the token score s[t] = (1/tau) sum_h w_h ReLU(q^I_h . k^I_{h,t}) with one
 * key per index head and token, and the block score is the maximum of its
 * tokens' scores.  Token t's keys sit in sel_tok[page][t % ps][h][d_idx]
 * with page = page_table[b][t / ps].  w (NULL -> 1/H_idx) is [B][H_idx];
 * the queries are those of tok_queries.  Writes n_full =
 * floor(seq_len / sel_block) scores into out. */
static int tok_unit_scores(const orc_tok_shape_t* sh, const orc_params_t* pr, int b,
                           const uint16_t* q_idx, const float* w, const void* sel_tok,
                           const void* sel_scales, const int32_t* page_table, int32_t seq_len,
                           double* out) {
    int Hi = sh->idx_heads, di = sh->idx_dim, sb = sh->sel_block, ps = sh->page_size;
    int64_t n_full = seq_len / sb;
    double* k = (double*)malloc((size_t)di * sizeof(double));
    double* qv = (double*)malloc((size_t)Hi * di * sizeof(double));
    if (!k || !qv || tok_queries(sh, pr, b, q_idx, qv) != 0) {
        free(k);
        free(qv);
        return -2;
    }
    for (int64_t j = 0; j < n_full; ++j) {
        double best = -INFINITY;
        for (int64_t t = j * sb; t < (j + 1) * sb; ++t) {
            int32_t page = page_table[(int64_t)b * sh->max_pages + t / ps];
            double s = 0.0;
            for (int h = 0; h < Hi; ++h) {
                const double* q = qv + (int64_t)h * di;
                if (tok_key_row(sh, sel_tok, sel_scales,
                                ((int64_t)page * ps + t % ps) * Hi + h, k)) {
                    free(k);
                    free(qv);
                    return -1;
                }
                double dot = 0.0;
                for (int d = 0; d < di; ++d) dot += q[d] * k[d];
                double wh = w ? (double)w[(int64_t)b * Hi + h] : 1.0 / Hi;
                s += wh * (dot > 0.0 ? dot : 0.0);
            }
            s /= pr->temperature;
            if (s > best) best = s;
        }
        out[j] = best;
    }
    free(k);
    free(qv);
    return 0;
}

/* Block scores [B][max_blocks] of the token-level selector; entries past
 * each sequence's complete blocks are left untouched. */
int oracle_tok_block_scores(const orc_tok_shape_t* sh, const orc_params_t* pr,
                            const uint16_t* q_idx, const float* w, const void* sel_tok,
                            const void* sel_scales, const int32_t* page_table,
                            const int32_t* seq_lens, double* scores) {
    if (sh->sel_block <= 0 || sh->page_size % sh->sel_block != 0) return -1;
    for (int b = 0; b < sh->batch; ++b)
        if (tok_unit_scores(sh, pr, b, q_idx, w, sel_tok, sel_scales, page_table, seq_lens[b],
                            scores + (int64_t)b * sh->max_blocks))
            return -1;
    return 0;
}

/* The decode step of the token-level selector for sequences seqs[n_seqs]
 * (NULL: all): block scores, one selection per sequence shared by every
 * head (§2.3, Eq. 6-8, blocks of sel_block tokens), and exact attention of
 * every query head over the selected blocks' tokens.  Outputs indexed as
 * in the full problem: sel_idx[b][max_blocks], sel_cnt[b], nuc_mass[b] (may
 * be NULL), out[b][h][D], lse[b][h]. */
int oracle_tok_decode_step(const orc_tok_shape_t* sh, const orc_params_t* pr,
                           const uint16_t* q_idx, const float* w, const void* sel_tok,
                           const void* sel_scales, const uint16_t* q, const uint16_t* k_pool, const uint16_t* v_pool,
                           const int32_t* page_table, const int32_t* seq_lens,
                           const float* top_p, double sm_scale, const int32_t* seqs,
                           int32_t n_seqs, int32_t* sel_idx, int32_t* sel_cnt, double* nuc_mass,
                           double* out, double* lse) {
    if (sh->sel_block <= 0 || sh->page_size % sh->sel_block != 0) return -1;
    int G = sh->num_q_heads / sh->num_kv_heads;
    int total = seqs ? n_seqs : sh->batch;
    int err = 0;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int k = 0; k < total; ++k) {
        int b = seqs ? seqs[k] : k;
        int32_t L = seq_lens[b];
        int64_t nb = ceil_div64(L, sh->sel_block), n_full = L / sh->sel_block;
        double* s = (double*)malloc((size_t)(nb > 0 ? nb : 1) * sizeof(double));
        if (!s) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = -2;
            continue;
        }
        if (tok_unit_scores(sh, pr, b, q_idx, w, sel_tok, sel_scales, page_table, L, s)) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = -1;
            free(s);
            continue;
        }
        int32_t* sel = sel_idx + (int64_t)b * sh->max_blocks;
        double mass = 0.0;
        int32_t cnt = oracle_select_from_scores(s, (int32_t)nb, (int32_t)n_full, pr,
                                                (double)top_p[b], sel, &mass);
        sel_cnt[b] = cnt;
        if (nuc_mass) nuc_mass[b] = mass;
        free(s);
    }
    /* attention of every (sequence, KV head) over the shared selection */
    int units = total * sh->num_kv_heads;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int u = 0; u < units; ++u) {
        int k = u / sh->num_kv_heads, g = u % sh->num_kv_heads;
        int b = seqs ? seqs[k] : k;
        attend_blocks(sh->num_q_heads, sh->num_kv_heads, sh->head_dim, sh->page_size,
                      sh->max_pages, sh->sel_block, b, g, q, k_pool, v_pool, page_table,
                      seq_lens[b], sel_idx + (int64_t)b * sh->max_blocks, sel_cnt[b], sm_scale,
                      out + ((int64_t)b * sh->num_q_heads + g * G) * sh->head_dim,
                      lse + (int64_t)b * sh->num_q_heads + g * G);
    }
    return err;
}

/* Threads the OpenMP runtime will use (1 without OpenMP). */
int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Sets the number of OpenMP threads later calls use (n >= 1); returns the
 * count in effect.  Lets one process time the oracle on every host core and
 * on one. */
int oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n >= 1) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}
