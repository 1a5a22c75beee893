/*
 * oracle.c -- plain, slow, CPU reference for the FP8 in-context-learning (ICL)
 * attention layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark load this file's library.  The CUDA library
 * never calls it, links it or shares a header, helper or constant with it.
 *
 * Sources (web pages, cited by title and section):
 *   [QS]  "Fuse shared-length query scaling during inference"
 *         (structured-data-models PR #1168), sections "Problem identified"
 *         and "Solution".
 *   [FP8] "[FP8 3/4] Integrate FP8 attention and caching into TabICLv2"
 *         (structured-data-models PR #879), opening section and usage example.
 *   [KT]  "[FP8 4/5]" KumoTabular page (structured-data-models PR #880),
 *         opening section.
 * The pages name LogScale, GatedLogScale, the FP8 attention and the cached
 * prediction, but print no formula.  The formulas used here are the layer's
 * fixed definitions: q' = q * (c_h * ln n); gated q'' = q' * (1 + tanh g);
 * per-head scale s = amax / 448 from context rows only; e4m3 with
 * round-to-nearest-even and saturation; P quantised to e4m3 before P.V.
 *
 * Every function below is pinned by tests under tests/ against something other
 * than itself (library casts, closed forms, brute force, invariants).  Nothing
 * here is "parity unpinned".
 *
 * Arithmetic conventions.  fp16 and e4m3 values travel as their bit patterns
 * (uint16_t / uint8_t) and are encoded/decoded here from the format
 * definitions, never by a compiler cast.  Build with -ffp-contract=off so that
 * every float expression rounds where it is written.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* IEEE binary16                                                              */
/* ------------------------------------------------------------------------- */

/* Decode binary16 bits: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
double orc_f16_decode(uint16_t h) {
    int s = h >> 15, e = (h >> 10) & 31, f = h & 1023;
    double v;
    if (e == 31) v = f ? NAN : INFINITY;
    else if (e == 0) v = ldexp((double)f, -24);           /* subnormal: f * 2^-24 */
    else v = ldexp((double)(1024 + f), e - 15 - 10);      /* normal: 1.f * 2^(e-15) */
    return s ? -v : v;
}

/* Round a double to the nearest binary16, ties to even; overflow -> inf. */
uint16_t orc_f16_encode(double y) {
    if (isnan(y)) return 0x7E00;
    uint16_t sign = signbit(y) ? 0x8000 : 0;
    double a = fabs(y);
    if (a >= 65520.0) return sign | 0x7C00;   /* 65520 = midpoint 65504..65536 */
    int e;                                     /* binade exponent: a in [2^e, 2^(e+1)) */
    if (a < 0x1p-14) e = -14;                  /* subnormals share the 2^-14 spacing */
    else { int E; frexp(a, &E); e = E - 1; }
    double step = ldexp(1.0, e - 10);          /* spacing of representable values */
    double k = nearbyint(a / step);            /* a/step is exact; RNE on the integer */
    double v = k * step;
    if (v >= 65536.0) return sign | 0x7C00;
    if (v == 0.0) return sign;
    if (v < 0x1p-14) return sign | (uint16_t)(v / 0x1p-24);
    int E; frexp(v, &E); int ev = E - 1;
    uint16_t frac = (uint16_t)(v / ldexp(1.0, ev - 10)) - 1024;
    return sign | (uint16_t)((ev + 15) << 10) | frac;
}

/* ------------------------------------------------------------------------- */
/* OCP FP8 E4M3 ("fn": no infinities, 0x7F/0xFF are NaN, max finite 448)      */
/* ------------------------------------------------------------------------- */

double orc_e4m3_decode(uint8_t c) {
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    double v = (e == 0) ? ldexp((double)m, -9)            /* subnormal: m * 2^-9 */
                        : ldexp((double)(8 + m), e - 7 - 3); /* 1.m * 2^(e-7) */
    return s ? -v : v;
}

/* Round to the nearest e4m3 value, ties to even, saturating every finite or
 * infinite magnitude at or beyond the largest finite value to +-448; NaN maps
 * to 0x7F.  The sign of a result that rounds to zero is kept. */
uint8_t orc_e4m3_encode(double y) {
    if (isnan(y)) return 0x7F;
    uint8_t sign = signbit(y) ? 0x80 : 0;
    double a = fabs(y);
    if (a >= 448.0) return sign | 0x7E;
    if (a <= 0x1p-10) return sign;             /* at or below half of 2^-9: ties to even 0 */
    int e;                                     /* binade: a in [2^e, 2^(e+1)) */
    if (a < 0x1p-6) e = -6;                    /* subnormals share the 2^-6 spacing */
    else { int E; frexp(a, &E); e = E - 1; }
    double step = ldexp(1.0, e - 3);           /* 3 mantissa bits */
    double k = nearbyint(a / step);
    double v = k * step;                       /* < 448 always: a < 448 and step 32 at the top */
    if (v == 0.0) return sign;
    if (v < 0x1p-6) return sign | (uint8_t)(v / 0x1p-9);
    int E; frexp(v, &E); int ev = E - 1;
    uint8_t mant = (uint8_t)(v / ldexp(1.0, ev - 3)) - 8;
    return sign | (uint8_t)((ev + 7) << 3) | mant;
}

/* Array helpers for the tests. */
void orc_f16_encode_array(const double* y, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_f16_encode(y[i]);
}
void orc_f16_decode_array(const uint16_t* h, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_f16_decode(h[i]);
}
void orc_e4m3_encode_array(const double* y, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(y[i]);
}
void orc_e4m3_decode_array(const uint8_t* c, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_decode(c[i]);
}

/* Decode tables, filled once from the decode functions above (memoisation
 * only: every entry is orc_*_decode of its index). */
static double g_e4m3[256];
static float g_e4m3_f[256];
static double g_f16[65536];
static int g_tables_ready = 0;

static void init_tables(void) {
    if (g_tables_ready) return;
    for (int c = 0; c < 256; ++c) { g_e4m3[c] = orc_e4m3_decode((uint8_t)c); g_e4m3_f[c] = (float)g_e4m3[c]; }
    for (int h = 0; h < 65536; ++h) g_f16[h] = orc_f16_decode((uint16_t)h);
    g_tables_ready = 1;
}
#define F16(h) (g_f16[(uint16_t)(h)])

/* ------------------------------------------------------------------------- */
/* Step 1: LogScale / GatedLogScale ([QS] "Problem identified", "Solution")   */
/* ------------------------------------------------------------------------- */

/* [QS] "Solution": the shared integer key length is prepared in float32.  The
 * eager path clamps the logarithm's argument ("clamped log scaling", [QS]
 * sequence diagram); read here as ln(max(n, 1)). */
float orc_log_length(int64_t n) {
    if (n < 1) n = 1;
    return logf((float)n);
}

/* q layout [B][rows][H][d] fp16 bits; c_h [H] fp32; gate [B][rows][H] fp16
 * bits or NULL.  The unfused eager chain, one rounding per eager op:
 *   lam = ln(n) (fp32)        t_h = c_h * lam (fp32)    s_h = fp16(t_h)
 *   q1  = fp16(q * s_h)
 *   gated: u = fp16(tanh g)   w = fp16(1 + u)           q2 = fp16(q1 * w)
 * tanh of an fp16 input is rounded once to fp16 (computed in double first). */
void orc_qscale(const uint16_t* q, int B, int64_t rows, int H, int d, int64_t n,
                const float* c_h, const uint16_t* gate, uint16_t* out) {
    float lam = orc_log_length(n);
    init_tables();
    #pragma omp parallel for schedule(static)
    for (int64_t br = 0; br < (int64_t)B * rows; ++br) {
        for (int h = 0; h < H; ++h) {
            float t = c_h[h] * lam;
            uint16_t s16 = orc_f16_encode((double)t);
            float s = (float)orc_f16_decode(s16);
            float w = 1.0f;
            if (gate) {
                double g = F16(gate[br * H + h]);
                uint16_t u16 = orc_f16_encode(tanh(g));
                float one_plus_u = 1.0f + (float)orc_f16_decode(u16);
                w = (float)orc_f16_decode(orc_f16_encode((double)one_plus_u));
            }
            const uint16_t* qi = q + (br * H + h) * d;
            uint16_t* oi = out + (br * H + h) * d;
            for (int e = 0; e < d; ++e) {
                float prod = (float)F16(qi[e]) * s;
                uint16_t q1 = orc_f16_encode((double)prod);
                if (gate) {
                    float prod2 = (float)F16(q1) * w;
                    q1 = orc_f16_encode((double)prod2);
                }
                oi[e] = q1;
            }
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Step 2: context-derived per-head scales and e4m3 quantisation              */
/* ([FP8] opening section: "Context-derived Q scales make cached prediction   */
/*  independent of query-batch partitioning"; K and V scales likewise come    */
/*  from the context rows, which are all that K and V hold.)                  */
/* ------------------------------------------------------------------------- */

/* x layout [B][rows][H][d] fp16 bits.  scale[b*H+h] = amax / 448 over context
 * rows [0, n_ctx) of (b, h), fp32 IEEE division; amax == 0 gives scale 1. */
void orc_context_scales(const uint16_t* x, int B, int64_t rows, int64_t n_ctx,
                        int H, int d, float* scale) {
    init_tables();
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            float amax = 0.0f;
            for (int64_t r = 0; r < n_ctx; ++r) {
                const uint16_t* xi = x + (((int64_t)b * rows + r) * H + h) * d;
                for (int e = 0; e < d; ++e) {
                    float a = (float)fabs(F16(xi[e]));
                    if (a > amax) amax = a;
                }
            }
            scale[b * H + h] = (amax > 0.0f) ? amax / 448.0f : 1.0f;
        }
}

/* x8[b][h][r][e] = e4m3(fp32(x[b][r][h][e]) / scale[b*H+h]) for r < rows.
 * Rows past the context (the query rows of Q) saturate at +-448. */
void orc_quantize(const uint16_t* x, int B, int64_t rows, int H, int d,
                  const float* scale, uint8_t* x8) {
    init_tables();
    #pragma omp parallel for schedule(static)
    for (int64_t br = 0; br < (int64_t)B * rows; ++br) {
        int64_t b = br / rows, r = br % rows;
        for (int h = 0; h < H; ++h) {
            float s = scale[b * H + h];
            const uint16_t* xi = x + (br * H + h) * d;
            uint8_t* oi = x8 + (((b * H + h) * rows) + r) * d;
            for (int e = 0; e < d; ++e) {
                float y = (float)F16(xi[e]) / s;
                oi[e] = orc_e4m3_encode((double)y);
            }
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Steps 3 and 4: FP8 flash attention and split-KV cached prediction          */
/* ------------------------------------------------------------------------- */

/* Nearest rounding midpoints around the e4m3 code c (for a value p > 0 that
 * encodes to c): returns in *lo_mid / *hi_mid the decision boundaries and in
 * *lo_alt / *hi_alt the values a value just across them would encode to. */
static void e4m3_neighbours(uint8_t c, double* lo_mid, double* lo_alt,
                            double* hi_mid, double* hi_alt) {
    double v = orc_e4m3_decode(c);
    double below = (c & 0x7F) == 0 ? 0.0 : orc_e4m3_decode((uint8_t)(c - 1));
    double above = (c & 0x7F) >= 0x7E ? v : orc_e4m3_decode((uint8_t)(c + 1));
    *lo_mid = (v + below) / 2; *lo_alt = below;
    *hi_mid = (v + above) / 2; *hi_alt = above;
}

/*
 * One (b, h, query row) of the FP8 online-softmax attention over keys
 * [j_begin, j_end), in KV tiles of bc keys aligned to j_begin.  Two
 * arithmetics, selected by `arith`:
 *
 * ORC_ARITH_DEFINITION (the oracle proper) -- the layer's definition written
 * out in double ([FP8] opening section: logits of the e4m3 Q and K with the
 * per-head scales, online softmax over key tiles, P quantised to e4m3 before
 * P.V; the softmax scale is SDPA's default 1/sqrt(d)):
 *   z_j  = sum_e dec(q8[e]) * dec(k8_j[e])    exact: every product is a multiple
 *                                             of 2^-18 below 2^18, so 64 of them
 *                                             add up within double's 53 bits
 *   x_j  = z_j * (s_q * s_k / sqrt(d))        natural-log units
 *   per tile: m' = max(m, max_j x_j),  P_j = exp(x_j - m'),  P8_j = e4m3(P_j)
 *   when m' > m:  l and acc are multiplied by alpha = exp(m - m')
 *   l += sum_j dec(P8_j);   acc += sum_j dec(P8_j) * dec(v8_j)
 *
 * ORC_ARITH_FP32 (a diagnostic only) -- the same steps in the single-precision
 * sequence a tensor-core kernel takes, in base-2 units:
 *   z_j  = fp32 sum, e ascending;   c2 = fp32(fp32(s_q*s_k) * fp32(log2(e)/sqrt(d)))
 *   m2 = fp32(m * c2);  t_j = fma(z_j, c2, -m2);  p_j = fp32(2^t_j);  P8_j = e4m3(p_j)
 *   alpha = 2^(fp32(m2_old - m2_new)).
 * It shows how far an fp32 implementation's e4m3 codes move from the
 * definition's; no test gates the CUDA path against it.
 *
 * In both, the running maximum is reported in base-2 units (m2 = m * log2 e
 * for the definition), and with quant_p == 0 the e4m3 rounding of P is
 * skipped: the plain softmax.
 *
 * Ambiguity allowance.  An implementation that forms the logits in fp32 (a
 * tensor core accumulates z in fp32; m2 and t are rounded to fp32) moves each
 * probability by a small relative error, and where the definition's
 * probability lies that close to an e4m3 rounding midpoint either neighbouring
 * code is what such an implementation may produce.  For key j the radius is
 *   r_j = delta0 + kappa * (|m2| + |t_j|)      (base-2 units: m2 the running
 *                                                maximum, t_j = x_j log2 e - m2)
 * -- a fixed part for the 2^x evaluation and a part proportional to the size
 * of the fp32 numbers the logit passes through.  A key whose probability p
 * lies within relative distance r_j of a midpoint is "ambiguous": amb0
 * accumulates |dw|, the weight change its other code would make, and amb1[e]
 * |dw| * |dec(v8_j[e])|, with the same rescaling as l/acc.
 */
enum { ORC_ARITH_DEFINITION = 0, ORC_ARITH_FP32 = 1 };
enum { KV_TILE_ORACLE = 128 };  /* the layer's online-softmax key tile */

typedef struct {
    double m2;     /* running max in log2 units; -inf if no key */
    double l, amb0;
    double* acc;   /* [d] */
    double* amb1;  /* [d] */
} orc_partial;

static void partial_scale(orc_partial* st, int d, double alpha) {
    st->l *= alpha; st->amb0 *= alpha;
    for (int e = 0; e < d; ++e) { st->acc[e] *= alpha; st->amb1[e] *= alpha; }
}

/* Adds key j with probability p (>= 0) to the running sums: its e4m3 weight
 * (or p itself when quant_p == 0) and its ambiguity contribution. */
static void partial_add_key(orc_partial* st, double p, const uint8_t* vj, int d,
                            int quant_p, double radius) {
    double w = p, dw = 0.0;
    if (quant_p) {
        uint8_t c = orc_e4m3_encode(p);
        w = orc_e4m3_decode(c);
        if (p > 0.0 && radius > 0.0) {
            double lo_mid, lo_alt, hi_mid, hi_alt;
            e4m3_neighbours(c, &lo_mid, &lo_alt, &hi_mid, &hi_alt);
            if (fabs(p - lo_mid) <= radius * p) dw = fabs(w - lo_alt);
            if (fabs(p - hi_mid) <= radius * p) dw = fabs(hi_alt - w);
        }
    }
    if (w == 0.0 && dw == 0.0) return;
    st->l += w; st->amb0 += dw;
    for (int e = 0; e < d; ++e) {
        double ve = g_e4m3[vj[e]];
        st->acc[e] += w * ve;
        st->amb1[e] += dw * fabs(ve);
    }
}

static void partial_reset(orc_partial* st, int d) {
    st->m2 = -INFINITY; st->l = 0; st->amb0 = 0;
    for (int e = 0; e < d; ++e) { st->acc[e] = 0; st->amb1[e] = 0; }
}

static const double kLog2e = 1.4426950408889634074;

static void attend_range_definition(const uint8_t* q8row, const uint8_t* k8, const uint8_t* v8,
                                    int64_t j_begin, int64_t j_end, int d, double scale,
                                    int64_t bc, int quant_p, double delta0, double kappa,
                                    orc_partial* st, double* xbuf) {
    double m = -INFINITY;                     /* running max of x (natural-log units) */
    partial_reset(st, d);
    for (int64_t j0 = j_begin; j0 < j_end; j0 += bc) {
        int64_t j1 = j0 + bc < j_end ? j0 + bc : j_end;
        double mt = m;
        for (int64_t j = j0; j < j1; ++j) {
            const uint8_t* kj = k8 + j * d;
            double z = 0.0;
            for (int e = 0; e < d; ++e) z += g_e4m3[q8row[e]] * g_e4m3[kj[e]];
            xbuf[j - j0] = z * scale;
            if (xbuf[j - j0] > mt) mt = xbuf[j - j0];
        }
        if (mt > m) {
            partial_scale(st, d, m == -INFINITY ? 0.0 : exp(m - mt));
            m = mt;
        }
        for (int64_t j = j0; j < j1; ++j) {
            double r = delta0 + kappa * (fabs(m) + (m - xbuf[j - j0])) * kLog2e;
            partial_add_key(st, exp(xbuf[j - j0] - m), v8 + j * d, d, quant_p, r);
        }
    }
    st->m2 = m * kLog2e;
}

static void attend_range_f32(const uint8_t* q8row, const uint8_t* k8, const uint8_t* v8,
                             int64_t j_begin, int64_t j_end, int d, float c2,
                             int64_t bc, int quant_p, double delta0, double kappa,
                             orc_partial* st, double* xbuf) {
    float m = -INFINITY;                      /* running max of z (raw units) */
    float m2 = -INFINITY;
    partial_reset(st, d);
    for (int64_t j0 = j_begin; j0 < j_end; j0 += bc) {
        int64_t j1 = j0 + bc < j_end ? j0 + bc : j_end;
        float mt = m;
        for (int64_t j = j0; j < j1; ++j) {
            const uint8_t* kj = k8 + j * d;
            float z = 0.0f;   /* each product of two e4m3 values is exact in fp32 */
            for (int e = 0; e < d; ++e) z += g_e4m3_f[q8row[e]] * g_e4m3_f[kj[e]];
            xbuf[j - j0] = z;
            if (z > mt) mt = z;
        }
        float m2_new = mt * c2;
        if (mt > m) {
            partial_scale(st, d, m == -INFINITY ? 0.0 : exp2((double)(m2 - m2_new)));
            m = mt; m2 = m2_new;
        }
        for (int64_t j = j0; j < j1; ++j) {
            float t = fmaf((float)xbuf[j - j0], c2, -m2);
            double r = delta0 + kappa * (fabs((double)m2) + fabs((double)t));
            partial_add_key(st, (double)(float)exp2((double)t), v8 + j * d, d, quant_p, r);
        }
    }
    st->m2 = m2;
}

static float softmax_c2(float s_q, float s_k, int d) {
    float sqk = s_q * s_k;
    float k2 = (float)(kLog2e / sqrt((double)d)); /* log2(e)/sqrt(d) */
    return sqk * k2;
}

/*
 * FP8 attention of selected query rows of every (b, h) to the context keys.
 *   q8  [B][H][T][d]   k8, v8 [B][H][N][d]   scales s_q/s_k/s_v [B*H]
 *   rows[n_rows]       which of the T rows to compute (row indices in [0,T))
 *   bc                 KV tile length (the online-softmax block)
 *   split              0: one pass over all N keys ([FP8] "one model call");
 *                      >0: cached prediction ([FP8] "model.predict(queries)"
 *                      after fit) -- keys cut into chunks of `split` keys,
 *                      each processed from a fresh state, then combined in
 *                      chunk order:  M = max m_s;  w_s = exp(m_s - M);
 *                      L = sum w_s l_s;  ACC = sum w_s acc_s  (in base-2 units
 *                      and fp32 exponent differences under ORC_ARITH_FP32).
 *   arith              ORC_ARITH_DEFINITION or ORC_ARITH_FP32 (see above)
 *   out16 [B][n_rows][H][d]   fp16 bits of ACC * s_v / L
 *   out   [B][n_rows][H][d]   the same value before fp16 rounding (double)
 *   delta0, kappa      radius of the ambiguity allowance (see above); 0, 0: none
 *   allow [B][n_rows][H][d]   ambiguity allowance (may be NULL): an upper bound
 *                      on |O' - O| when any subset of the ambiguous keys takes
 *                      its other code:  s_v * (amb1[e] + amb0 * vmax_e) / (L - amb0)
 *                      (infinite if amb0 >= L), vmax_e the largest |dec(v8[.][e])|
 *                      of the head.  Flipping a set S changes the numerator by
 *                      sum_S dw_j (v_j - O) and L by sum_S dw_j, and
 *                      |v_j - O| <= |v_j| + vmax_e, L' >= L - amb0.
 */
void orc_attention(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8,
                   const float* s_q, const float* s_k, const float* s_v,
                   int B, int H, int64_t T, int64_t N, int d,
                   const int64_t* rows, int64_t n_rows, int64_t bc, int64_t split,
                   int quant_p, int arith, double delta0, double kappa,
                   uint16_t* out16, double* out, double* allow) {
    int64_t n_chunks = (split > 0) ? (N + split - 1) / split : 1;
    int64_t chunk = (split > 0) ? split : N;
    init_tables();
    double* vmax = (double*)calloc((size_t)B * H * d, sizeof(double));
    for (int64_t bh = 0; bh < (int64_t)B * H; ++bh)
        for (int64_t j = 0; j < N; ++j)
            for (int e = 0; e < d; ++e) {
                double a = fabs(g_e4m3[v8[(bh * N + j) * d + e]]);
                if (a > vmax[bh * d + e]) vmax[bh * d + e] = a;
            }
    #pragma omp parallel
    {
        double* xbuf = (double*)malloc(sizeof(double) * (size_t)bc);
        double* tmp = (double*)malloc(sizeof(double) * (size_t)(4 * d));
        orc_partial st; st.acc = tmp; st.amb1 = tmp + d;
        double* ACC = tmp + 2 * d; double* A1 = tmp + 3 * d;
        #pragma omp for schedule(dynamic, 1)
        for (int64_t task = 0; task < (int64_t)B * H * n_rows; ++task) {
            int64_t bh = task / n_rows, ri = task % n_rows;
            int64_t b = bh / H, h = bh % H, i = rows[ri];
            const uint8_t* qrow = q8 + (bh * T + i) * d;
            const uint8_t* kb = k8 + bh * N * d;
            const uint8_t* vb = v8 + bh * N * d;
            /* softmax scale of the definition: s_q * s_k / sqrt(d), in double */
            double scale = (double)s_q[bh] * (double)s_k[bh] / sqrt((double)d);
            float c2 = softmax_c2(s_q[bh], s_k[bh], d);
            double M = -INFINITY;             /* natural-log units (definition) or base 2 */
            double L = 0, A0 = 0;
            for (int e = 0; e < d; ++e) { ACC[e] = 0; A1[e] = 0; }
            /* chunk maxima first, then the fixed-order combine */
            for (int64_t s = 0; s < n_chunks; ++s) {
                int64_t jb = s * chunk, je = jb + chunk < N ? jb + chunk : N;
                double ms;
                if (arith == ORC_ARITH_FP32) {
                    attend_range_f32(qrow, kb, vb, jb, je, d, c2, bc, quant_p, delta0, kappa, &st, xbuf);
                    ms = st.m2;
                } else {
                    attend_range_definition(qrow, kb, vb, jb, je, d, scale, bc, quant_p, delta0, kappa,
                                            &st, xbuf);
                    ms = st.m2 / kLog2e;      /* back to natural-log units */
                }
                if (st.m2 == -INFINITY) continue;
                if (ms > M) {
                    double a = (M == -INFINITY) ? 0.0
                             : (arith == ORC_ARITH_FP32) ? exp2((double)(float)(M - ms)) : exp(M - ms);
                    L *= a; A0 *= a;
                    for (int e = 0; e < d; ++e) { ACC[e] *= a; A1[e] *= a; }
                    M = ms;
                }
                double w = (arith == ORC_ARITH_FP32) ? exp2((double)(float)(ms - M)) : exp(ms - M);
                L += w * st.l; A0 += w * st.amb0;
                for (int e = 0; e < d; ++e) { ACC[e] += w * st.acc[e]; A1[e] += w * st.amb1[e]; }
            }
            int64_t o = ((b * n_rows + ri) * H + h) * d;
            for (int e = 0; e < d; ++e) {
                double val = ACC[e] * (double)s_v[bh] / L;
                if (out) out[o + e] = val;
                if (out16) out16[o + e] = orc_f16_encode(val);
                if (allow) allow[o + e] = A0 == 0.0 ? 0.0
                                        : (A0 >= L ? INFINITY
                                                   : (double)s_v[bh] * (A1[e] + A0 * vmax[bh * d + e]) / (L - A0));
            }
        }
        free(xbuf); free(tmp);
    }
    free(vmax);
}

/*
 * The per-chunk partial states of cached prediction (definition arithmetic):
 * for chunks [c0, c1) of `split` keys, the state each chunk ends with --
 * m (running maximum, natural-log units), l and acc[d] -- from a slice of the
 * keys: k8s / v8s [B][H][n_slice][d] hold keys [c0 split, c0 split + n_slice)
 * of the N.  Outputs [c1 - c0][B][H][n_rows] (m, l) and [...][d] (acc); a chunk
 * with no keys gives m = -inf, l = 0, acc = 0.  Combining every chunk's state in
 * chunk order (M = max m, w = exp(m - M), L = sum w l, ACC = sum w acc,
 * O = ACC s_v / L) is orc_attention with the same split.
 */
void orc_attention_partials(const uint8_t* q8, const uint8_t* k8s, const uint8_t* v8s,
                            const float* s_q, const float* s_k,
                            int B, int H, int64_t T, int64_t N, int64_t n_slice, int d,
                            const int64_t* rows, int64_t n_rows, int64_t split, int64_t c0, int64_t c1,
                            double* m_out, double* l_out, double* acc_out) {
    init_tables();
    int64_t nc = c1 - c0;
    #pragma omp parallel
    {
        double* xbuf = (double*)malloc(sizeof(double) * (size_t)KV_TILE_ORACLE);
        double* tmp = (double*)malloc(sizeof(double) * (size_t)(2 * d));
        orc_partial st; st.acc = tmp; st.amb1 = tmp + d;
        #pragma omp for schedule(dynamic, 1)
        for (int64_t task = 0; task < (int64_t)B * H * n_rows * nc; ++task) {
            int64_t c = task % nc, rest = task / nc;
            int64_t ri = rest % n_rows, bh = rest / n_rows;
            const uint8_t* qrow = q8 + (bh * T + rows[ri]) * d;
            const uint8_t* kb = k8s + bh * n_slice * d;
            const uint8_t* vb = v8s + bh * n_slice * d;
            int64_t jb = (c0 + c) * split, je = jb + split < N ? jb + split : N;
            double scale = (double)s_q[bh] * (double)s_k[bh] / sqrt((double)d);
            int64_t o = (c * B * H + bh) * n_rows + ri;
            if (je <= jb) {
                m_out[o] = -INFINITY; l_out[o] = 0.0;
                for (int e = 0; e < d; ++e) acc_out[o * d + e] = 0.0;
                continue;
            }
            /* keys [jb, je) are slice keys [jb - c0 split, je - c0 split); tiles are
             * aligned to the chunk start either way */
            int64_t off = c0 * split;
            attend_range_definition(qrow, kb, vb, jb - off, je - off, d, scale, KV_TILE_ORACLE, 1,
                                    0.0, 0.0, &st, xbuf);
            m_out[o] = st.m2 / kLog2e;
            l_out[o] = st.l;
            for (int e = 0; e < d; ++e) acc_out[o * d + e] = st.acc[e];
        }
        free(xbuf); free(tmp);
    }
}

/*
 * Exact attention, for reporting the quantisation error only: double
 * precision, no FP8 anywhere, full-row softmax with scale 1/sqrt(d).
 *   q [B][T][H][d] fp16 bits (already LogScale'd), k, v [B][N][H][d] fp16 bits
 *   out [B][n_rows][H][d] double
 */
void orc_attention_exact(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                         int B, int H, int64_t T, int64_t N, int d,
                         const int64_t* rows, int64_t n_rows, double* out) {
    double inv_sqrt_d = 1.0 / sqrt((double)d);
    init_tables();
    #pragma omp parallel
    {
        double* x = (double*)malloc(sizeof(double) * (size_t)N);
        double* qd = (double*)malloc(sizeof(double) * (size_t)d);
        #pragma omp for schedule(dynamic, 1)
        for (int64_t task = 0; task < (int64_t)B * H * n_rows; ++task) {
            int64_t bh = task / n_rows, ri = task % n_rows;
            int64_t b = bh / H, h = bh % H, i = rows[ri];
            for (int e = 0; e < d; ++e) qd[e] = F16(q[((b * T + i) * H + h) * d + e]);
            double mx = -INFINITY;
            for (int64_t j = 0; j < N; ++j) {
                const uint16_t* kj = k + ((b * N + j) * H + h) * d;
                double z = 0;
                for (int e = 0; e < d; ++e) z += qd[e] * F16(kj[e]);
                x[j] = z * inv_sqrt_d;
                if (x[j] > mx) mx = x[j];
            }
            double l = 0;
            for (int64_t j = 0; j < N; ++j) { x[j] = exp(x[j] - mx); l += x[j]; }
            double* o = out + ((b * n_rows + ri) * H + h) * d;
            for (int e = 0; e < d; ++e) o[e] = 0;
            for (int64_t j = 0; j < N; ++j) {
                const uint16_t* vj = v + ((b * N + j) * H + h) * d;
                for (int e = 0; e < d; ++e) o[e] += x[j] * F16(vj[e]);
            }
            for (int e = 0; e < d; ++e) o[e] /= l;
        }
        free(x); free(qd);
    }
}

/* Threads the OpenMP runtime will use (for the CPU-baseline report), and a
 * setter for single-thread timings. */
#ifdef _OPENMP
#include <omp.h>
int orc_num_threads(void) { return omp_get_max_threads(); }
void orc_set_num_threads(int n) { omp_set_num_threads(n > 0 ? n : 1); }
#else
int orc_num_threads(void) { return 1; }
void orc_set_num_threads(int n) { (void)n; }
#endif
