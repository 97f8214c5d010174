/*
 * CPU oracle for decode attention over the DepthWeave-KV compressed cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or calls this
 * file; only the tests, the graft smoke check and the bench's CPU baseline do.  It shares
 * no code, header, table or helper with the CUDA path.
 *
 * Source of the method: "DepthWeave-KV: Token-Adaptive Cross-Layer Residual Factorization
 * for Long-Context KV Cache Compression" (arXiv 2607.06523), cited below as [DW].
 *
 *   [DW] §3 Method, Eq. (1):  X^_{l,h,t} = A_{l,h,t} B_{m,h} + g_{l,h,t} R_{l,h,t},  Z in {K, V}
 *   [DW] §3 Method, Eq. (3):  e_{l,h} = ||Attn(Q,K,V) - Attn(Q,K^,V^)||_2 / (||Attn(Q,K,V)||_2 + eps)
 *
 * Readings taken where [DW] is silent (each one is listed in the design notes):
 *   - g = 1 by default (no trained gates exist); a given gate g folds into the stored
 *     residual scale, fp16_rn(g * scale).  The basis is stored transposed, d x r_max with
 *     columns as basis vectors, so A B becomes sum_{j<r_t} B[:, j] c_t[j].
 *   - The router's rank r_t truncates the coefficient vector; the residual keeps a fixed
 *     number s of channels: R = scale_t * sum_i code_{t,i} e_{idx_{t,i}}.
 *   - Attention is standard scaled dot-product attention with tau = 1/sqrt(d) unless the
 *     caller passes another scale.
 *   - The probe compares the output with the residual against the output without it.
 *   - Encoding: project x on the basis, keep r_t coefficients rounded to bf16, take the
 *     residual against the *stored* coefficients, keep the s largest |residual| channels
 *     (ties -> lower channel), quantise symmetrically with one fp16 scale per token.
 *   - The 8-bit coefficient variant: blocks of 16 coefficients, one fp16 scale a block
 *     (max |c| / 127), codes rounded to nearest even; the residual is taken against the
 *     dequantised coefficients.  Decode then reads the coefficients as exact fp64 values.
 *
 * Precision: everything of decode and probe runs in fp64 from the stored values, which
 * convert exactly (bf16, fp16, integer codes).  Encode runs in fp32 with a fully stated
 * operation order so that it is reproducible bit for bit.  Build with
 * -ffp-contract=off and without fast-math.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------------------ */
/* Number formats (IEEE 754 binary16, and bfloat16 = the top 16 bits of binary32).        */
/* ------------------------------------------------------------------------------------ */

static float u32_as_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f32_as_u32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

double oracle_bf16_to_f64(uint16_t h) { return (double)u32_as_f32((uint32_t)h << 16); }

double oracle_fp16_to_f64(uint16_t h) {
    int sign = (h >> 15) & 1, e = (h >> 10) & 0x1f, m = h & 0x3ff;
    double v;
    if (e == 0)       v = ldexp((double)m, -24);                 /* zero / subnormal   */
    else if (e == 31) v = m ? NAN : INFINITY;                     /* inf / nan          */
    else              v = ldexp((double)(m | 0x400), e - 25);     /* normal: 1.m * 2^(e-15) */
    return sign ? -v : v;
}

/* float -> bfloat16, round to nearest, ties to even. */
uint16_t oracle_f32_to_bf16_rn(float x) {
    uint32_t u = f32_as_u32(x);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu))   /* nan: keep it a nan */
        return (uint16_t)((u >> 16) | 0x40);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/* float -> binary16, round to nearest, ties to even, with subnormals and overflow to inf.
 * Written from the format's definition: the exact value is scaled to an integer
 * significand at the target exponent and rounded once. */
uint16_t oracle_f32_to_fp16_rn(float x) {
    uint32_t u = f32_as_u32(x);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    double a = fabs((double)x);
    if (isnan(x)) return (uint16_t)(sign | 0x7e00u);
    if (isinf(x) || a >= 65520.0) return (uint16_t)(sign | 0x7c00u); /* >= max + half ulp */
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);                    /* a = f * 2^e, f in [0.5, 1) -> unbiased exponent e-1 */
    int ue = e - 1;
    if (ue < -14) ue = -14;          /* subnormal range: fixed quantum 2^-24 */
    double q = ldexp(a, 10 - ue);    /* significand in units of the target ulp (exact) */
    double r = nearbyint(q);         /* default rounding mode: ties to even */
    uint32_t mant = (uint32_t)r;
    if (mant >= 2048u) { mant >>= 1; ue += 1; }     /* rounding carried into next binade */
    if (ue > 15) return (uint16_t)(sign | 0x7c00u);
    if (mant < 1024u) return (uint16_t)(sign | mant); /* subnormal (ue == -14) */
    return (uint16_t)(sign | ((uint32_t)(ue + 15) << 10) | (mant & 0x3ffu));
}

/* ------------------------------------------------------------------------------------ */
/* [DW] §3 Eq. (1), g = 1: reconstruct one stored vector.                                  */
/*   basis : bf16 [d][r_max], column j is basis vector j                                  */
/*   coeff : bf16 [r_max], only the first r_t entries are part of the token               */
/*   idx, codes : s residual channels and their integer codes; scale : fp16 bits          */
/* ------------------------------------------------------------------------------------ */
/* coeff_f (nullable): the coefficients as exact fp64 values instead of bf16 bits (the 8-bit */
/* blockwise form, dequantised: code x scale).                                             */
static void oracle_reconstruct_any(int d, int r_max, const uint16_t* basis, int r_t, const uint16_t* coeff,
                                   const double* coeff_f, int s, const uint8_t* idx, const int8_t* codes,
                                   uint16_t scale, int with_residual, double* out) {
    for (int i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int j = 0; j < r_t; ++j)
            acc += oracle_bf16_to_f64(basis[(size_t)i * r_max + j]) *
                   (coeff_f ? coeff_f[j] : oracle_bf16_to_f64(coeff[j]));
        out[i] = acc;
    }
    if (with_residual) {
        double sc = oracle_fp16_to_f64(scale);
        for (int k = 0; k < s; ++k) out[idx[k]] += sc * (double)codes[k];
    }
}

void oracle_reconstruct(int d, int r_max, const uint16_t* basis, int r_t, const uint16_t* coeff,
                        int s, const uint8_t* idx, const int8_t* codes, uint16_t scale,
                        int with_residual, double* out) {
    oracle_reconstruct_any(d, r_max, basis, r_t, coeff, NULL, s, idx, codes, scale, with_residual, out);
}

/* ------------------------------------------------------------------------------------ */
/* Decode attention for one (sequence, layer, kv-head) and its gq query heads.            */
/*   o = sum_t softmax_t(tau * q . K^_t) V^_t      ([DW] §3: attention over the            */
/*   reconstructed cache; the reconstruction is never stored).                            */
/* Token arrays are token-ordered: rank[T]; ck/cv [T][r_max] bf16; ik/iv [T][s] u8;       */
/* qk/qv [T][s] i8 codes; sk/sv [T] fp16.  q: bf16 [gq][d].  out: [gq][d].                 */
/* nres (nullable): token t keeps only its first nres[t] <= s residual entries ([DW] §3     */
/* Eq. (2): the router's level is the number of retained residual channels).               */
/* p_out (nullable): softmax weights [gq][T].  Returns 0, or -1 on allocation failure.    */
/* ckf / cvf (nullable): the coefficients as fp64 values [T][r_max], used instead of ck /   */
/* cv (the 8-bit blockwise coefficients of [DW] §3, dequantised exactly).                  */
/* T == 0 gives a zero output (attention over an empty cache).                            */
/* ------------------------------------------------------------------------------------ */
int oracle_decode_head(int d, int r_max, int T, int gq, int s,
                       const uint16_t* bk, const uint16_t* bv, const int32_t* rank,
                       const uint16_t* ck, const uint8_t* ik, const int8_t* qk, const uint16_t* sk,
                       const uint16_t* cv, const uint8_t* iv, const int8_t* qv, const uint16_t* sv,
                       const uint16_t* q, double tau, int with_residual,
                       double* out, double* p_out, const int32_t* nres, const double* ckf, const double* cvf) {
    for (int h = 0; h < gq * d; ++h) out[h] = 0.0;
    if (T <= 0) return 0;
    double* score = (double*)malloc(sizeof(double) * (size_t)T * gq);
    double* x = (double*)malloc(sizeof(double) * (size_t)d);
    double* qd = (double*)malloc(sizeof(double) * (size_t)gq * d);
    if (!score || !x || !qd) { free(score); free(x); free(qd); return -1; }
    for (int h = 0; h < gq * d; ++h) qd[h] = oracle_bf16_to_f64(q[h]);

    /* scores: tau * q . K^_t */
    for (int t = 0; t < T; ++t) {
        oracle_reconstruct_any(d, r_max, bk, rank[t], ck + (size_t)t * r_max, ckf ? ckf + (size_t)t * r_max : NULL,
                               nres ? nres[t] : s, ik + (size_t)t * s, qk + (size_t)t * s, sk[t], with_residual, x);
        for (int h = 0; h < gq; ++h) {
            double dot = 0.0;
            for (int i = 0; i < d; ++i) dot += qd[(size_t)h * d + i] * x[i];
            score[(size_t)t * gq + h] = tau * dot;
        }
    }
    /* softmax over t, per head, with the maximum subtracted */
    for (int h = 0; h < gq; ++h) {
        double mx = -INFINITY, sum = 0.0;
        for (int t = 0; t < T; ++t) if (score[(size_t)t * gq + h] > mx) mx = score[(size_t)t * gq + h];
        for (int t = 0; t < T; ++t) {
            double e = exp(score[(size_t)t * gq + h] - mx);
            score[(size_t)t * gq + h] = e;
            sum += e;
        }
        for (int t = 0; t < T; ++t) score[(size_t)t * gq + h] /= sum;
    }
    /* o = sum_t p_t V^_t */
    for (int t = 0; t < T; ++t) {
        oracle_reconstruct_any(d, r_max, bv, rank[t], cv + (size_t)t * r_max, cvf ? cvf + (size_t)t * r_max : NULL,
                               nres ? nres[t] : s, iv + (size_t)t * s, qv + (size_t)t * s, sv[t], with_residual, x);
        for (int h = 0; h < gq; ++h) {
            double p = score[(size_t)t * gq + h];
            for (int i = 0; i < d; ++i) out[(size_t)h * d + i] += p * x[i];
        }
    }
    if (p_out)
        for (int h = 0; h < gq; ++h)
            for (int t = 0; t < T; ++t) p_out[(size_t)h * T + t] = score[(size_t)t * gq + h];
    free(score); free(x); free(qd);
    return 0;
}

/* ------------------------------------------------------------------------------------ */
/* Probe, [DW] §3 Eq. (3), with the two caches read as "with residual" (the reference)     */
/* and "without residual":  e = ||o_full - o_nores||_2 / (||o_full||_2 + eps), the norm    */
/* running over the gq x d outputs of the kv-head.  o_full / o_nores are optional outputs. */
/* ------------------------------------------------------------------------------------ */
int oracle_probe_head(int d, int r_max, int T, int gq, int s,
                      const uint16_t* bk, const uint16_t* bv, const int32_t* rank,
                      const uint16_t* ck, const uint8_t* ik, const int8_t* qk, const uint16_t* sk,
                      const uint16_t* cv, const uint8_t* iv, const int8_t* qv, const uint16_t* sv,
                      const uint16_t* q, double tau, double eps,
                      double* err, double* o_full, double* o_nores, const int32_t* nres,
                      const double* ckf, const double* cvf) {
    double* a = (double*)malloc(sizeof(double) * (size_t)gq * d);
    double* b = (double*)malloc(sizeof(double) * (size_t)gq * d);
    if (!a || !b) { free(a); free(b); return -1; }
    int rc = oracle_decode_head(d, r_max, T, gq, s, bk, bv, rank, ck, ik, qk, sk, cv, iv, qv, sv,
                                q, tau, 1, a, NULL, nres, ckf, cvf);
    if (rc == 0)
        rc = oracle_decode_head(d, r_max, T, gq, s, bk, bv, rank, ck, ik, qk, sk, cv, iv, qv, sv,
                                q, tau, 0, b, NULL, nres, ckf, cvf);
    if (rc == 0) {
        double num = 0.0, den = 0.0;
        for (int k = 0; k < gq * d; ++k) { num += (a[k] - b[k]) * (a[k] - b[k]); den += a[k] * a[k]; }
        *err = sqrt(num) / (sqrt(den) + eps);
        if (o_full)  memcpy(o_full, a, sizeof(double) * (size_t)gq * d);
        if (o_nores) memcpy(o_nores, b, sizeof(double) * (size_t)gq * d);
    }
    free(a); free(b);
    return rc;
}

/* Many independent (sequence, layer, kv-head) decode problems, run in parallel over the
 * problems (the arithmetic of each problem is exactly oracle_decode_head).  Used to time
 * the oracle on the host's cores.  Pointer arrays have one entry per problem. */
int oracle_decode_many(int n, int d, int r_max, int gq, int s, const int32_t* T,
                       const uint16_t* const* bk, const uint16_t* const* bv,
                       const int32_t* const* rank,
                       const uint16_t* const* ck, const uint8_t* const* ik, const int8_t* const* qk,
                       const uint16_t* const* sk,
                       const uint16_t* const* cv, const uint8_t* const* iv, const int8_t* const* qv,
                       const uint16_t* const* sv,
                       const uint16_t* const* q, double tau, double* const* out, int nthreads,
                       const int32_t* const* nres, const double* const* ckf, const double* const* cvf) {
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(| : bad)
    for (int k = 0; k < n; ++k)
        bad |= (oracle_decode_head(d, r_max, T[k], gq, s, bk[k], bv[k], rank[k], ck[k], ik[k], qk[k],
                                   sk[k], cv[k], iv[k], qv[k], sv[k], q[k], tau, 1, out[k], NULL,
                                   nres ? nres[k] : NULL, ckf ? ckf[k] : NULL, cvf ? cvf[k] : NULL) != 0);
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------------------ */
/* Encode one dense vector ([DW] §3: "projecting the original cache vector onto the        */
/* current basis", a quantised sparse residual kept at the routed rank).                  */
/*   x     : bf16 [d];  basis : bf16 [d][r_max];  r_t <= r_max;  0 <= s <= d;  bits 8 or 4 */
/* Outputs: coeff bf16 [r_max] (zeros beyond r_t), c32 fp32 [r_max] (nullable, the         */
/* unrounded projection, zeros beyond r_t), idx [s] ascending, codes [s], scale fp16 bits,  */
/* resid fp32 [d] (nullable, the residual before selection).                               */
/*                                                                                          */
/* Arithmetic, fp32, in this exact order:                                                  */
/*   1. c_j  = fma chain over i = 0..d-1 of B[i][j] * x_i, starting from +0     (j < r_t)  */
/*   2. cb_j = bf16_rn(c_j)                                                                */
/*   3. r_i  = x_i - a_i,  a_i = fma chain over j = 0..r_t-1 of B[i][j] * cb_j from +0     */
/*   4. the s channels with the largest |r_i|, ties to the lower channel, ascending        */
/*   5. scale = fp16_rn(max_sel |r_i| / qmax)   (IEEE fp32 division), qmax = 127 or 7      */
/*   6. code_i = clamp(rint(r_i / float(scale)), -qmax, qmax); all zero if scale == 0     */
/* ------------------------------------------------------------------------------------ */
typedef struct { float mag; int ch; } oracle_rank_item;

static int oracle_cmp_mag_desc(const void* pa, const void* pb) {
    const oracle_rank_item* a = (const oracle_rank_item*)pa;
    const oracle_rank_item* b = (const oracle_rank_item*)pb;
    if (a->mag > b->mag) return -1;
    if (a->mag < b->mag) return 1;
    return (a->ch > b->ch) - (a->ch < b->ch);
}
static int oracle_cmp_int(const void* pa, const void* pb) {
    int a = *(const int*)pa, b = *(const int*)pb;
    return (a > b) - (a < b);
}

/* Steps 4-6 on a given residual r fp32 [d]: the s channels with the largest |r_i| (ties to the
 * lower channel) in ascending channel order, the fp16 scale and the codes. */
int oracle_quantize_residual(int d, int s, int bits, const float* r, uint8_t* idx, int8_t* codes,
                             uint16_t* scale) {
    if (d <= 0 || d > 256 || s < 0 || s > d || (bits != 8 && bits != 4)) return -1;
    oracle_rank_item items[256];
    int sel[256];
    /* 4: top-s by magnitude, ties to the lower channel, then ascending channel order */
    for (int i = 0; i < d; ++i) { items[i].mag = fabsf(r[i]); items[i].ch = i; }
    qsort(items, (size_t)d, sizeof(items[0]), oracle_cmp_mag_desc);
    for (int k = 0; k < s; ++k) sel[k] = items[k].ch;
    qsort(sel, (size_t)s, sizeof(int), oracle_cmp_int);
    /* 5-6: symmetric quantisation with one fp16 scale */
    const float qmax = (bits == 8) ? 127.0f : 7.0f;
    float amax = 0.0f;
    for (int k = 0; k < s; ++k) if (fabsf(r[sel[k]]) > amax) amax = fabsf(r[sel[k]]);
    uint16_t sh = oracle_f32_to_fp16_rn(amax / qmax);
    float sf = (float)oracle_fp16_to_f64(sh);
    *scale = sh;
    for (int k = 0; k < s; ++k) {
        idx[k] = (uint8_t)sel[k];
        float c = 0.0f;
        if (sf != 0.0f) {
            c = rintf(r[sel[k]] / sf);
            if (c > qmax) c = qmax;
            if (c < -qmax) c = -qmax;
        }
        codes[k] = (int8_t)c;
    }
    return 0;
}

/* Steps 2-6 on a given fp32 projection c (c[j] for j < r_t): what an encoder stores once it
 * has its coefficients, whatever arithmetic produced them.  Arguments as oracle_encode_vector,
 * with c32 the input. */
int oracle_encode_from_coeffs(int d, int r_max, const uint16_t* basis, const uint16_t* x, const float* c32,
                              int r_t, int s, int bits, uint16_t* coeff, uint8_t* idx, int8_t* codes,
                              uint16_t* scale, float* resid) {
    if (d <= 0 || d > 256 || r_t < 0 || r_t > r_max || s < 0 || s > d || (bits != 8 && bits != 4))
        return -1;
    float xf[256], cb[256], r[256];
    for (int i = 0; i < d; ++i) xf[i] = (float)oracle_bf16_to_f64(x[i]);
    for (int j = 0; j < r_max; ++j) coeff[j] = 0;
    /* 2: bf16 rounding of the coefficients kept */
    for (int j = 0; j < r_t; ++j) {
        coeff[j] = oracle_f32_to_bf16_rn(c32[j]);
        cb[j] = (float)oracle_bf16_to_f64(coeff[j]);
    }
    /* 3: residual against the stored coefficients */
    for (int i = 0; i < d; ++i) {
        float a = 0.0f;
        for (int j = 0; j < r_t; ++j)
            a = fmaf((float)oracle_bf16_to_f64(basis[(size_t)i * r_max + j]), cb[j], a);
        r[i] = xf[i] - a;
        if (resid) resid[i] = r[i];
    }
    oracle_quantize_residual(d, s, bits, r, idx, codes, scale);
    return 0;
}

/* The residual gate g of [DW] §3 Eq. (1) (X^ = A B + g R) folded into the dequantisation:   */
/* the token's stored residual scale becomes fp16_rn(g * float(scale)), an fp32 product;      */
/* the codes stay those of step 6.                                                           */
uint16_t oracle_gate_scale(uint16_t scale, float g) {
    return oracle_f32_to_fp16_rn(g * (float)oracle_fp16_to_f64(scale));
}

void oracle_gate_scales(int64_t n, const uint16_t* scale, const float* g, uint16_t* out) {
    for (int64_t k = 0; k < n; ++k) out[k] = oracle_gate_scale(scale[k], g[k]);
}

/* ------------------------------------------------------------------------------------ */
/* The 8-bit blockwise coefficient form ([DW] §3 Method, the shared-bases paragraph: the    */
/* coefficient vector is kept as 8-bit codes, a block at a time).  Reading: blocks of 16    */
/* coefficients j < r_t (r_t a multiple of 16), each with one fp16 scale, in the residual   */
/* codec's symmetric form:                                                                   */
/*   s_b = fp16_rn(max_{j in b} |c_j| / 127)   (IEEE fp32 division)                        */
/*   q_j = clamp(rint(c_j / float(s_b)), -127, 127); all zero if s_b == 0                  */
/*   c^_j = q_j * float(s_b)                    (fp32, exact)                              */
/* q, sc (nullable), cbar: [r_max], [r_max / 16], [r_max], zero past r_t.                  */
/* ------------------------------------------------------------------------------------ */
int oracle_quantize_coeffs8(int r_t, int r_max, const float* c, int8_t* q, uint16_t* sc, float* cbar) {
    if (r_t < 0 || r_t > r_max || r_t % 16 || r_max % 16) return -1;
    for (int j = 0; j < r_max; ++j) { if (q) q[j] = 0; cbar[j] = 0.0f; }
    for (int b = 0; b < r_max / 16; ++b) if (sc) sc[b] = 0;
    for (int b = 0; b < r_t / 16; ++b) {
        float amax = 0.0f;
        for (int j = 16 * b; j < 16 * b + 16; ++j) if (fabsf(c[j]) > amax) amax = fabsf(c[j]);
        const uint16_t sh = oracle_f32_to_fp16_rn(amax / 127.0f);
        const float sf = (float)oracle_fp16_to_f64(sh);
        if (sc) sc[b] = sh;
        for (int j = 16 * b; j < 16 * b + 16; ++j) {
            float v = 0.0f;
            if (sf != 0.0f) {
                v = rintf(c[j] / sf);
                if (v > 127.0f) v = 127.0f;
                if (v < -127.0f) v = -127.0f;
            }
            if (q) q[j] = (int8_t)v;
            cbar[j] = v * sf;
        }
    }
    return 0;
}

/* Encode one vector with 8-bit blockwise coefficients: step 1 of oracle_encode_vector (or   */
/* the given fp32 projections c_in [r_max], only [:r_t] read, for an encoder that computed  */
/* them in another order), the coefficients in the 8-bit form above, the residual against   */
/* their dequantised values c^, then steps 4-6.  Outputs: ccodes int8 [r_max], cscales fp16  */
/* [r_max / 16], c32 (nullable) the projections, idx / codes / scale as oracle_encode_vector. */
int oracle_encode_vector8(int d, int r_max, const uint16_t* basis, const uint16_t* x, const float* c_in, int r_t,
                          int s, int bits, int8_t* ccodes, uint16_t* cscales, float* c32, uint8_t* idx,
                          int8_t* codes, uint16_t* scale) {
    if (d <= 0 || d > 256 || r_max > 256 || r_t < 0 || r_t > r_max || r_t % 16 || s < 0 || s > d ||
        (bits != 8 && bits != 4))
        return -1;
    float xf[256], c[256], cbar[256], r[256];
    for (int i = 0; i < d; ++i) xf[i] = (float)oracle_bf16_to_f64(x[i]);
    for (int j = 0; j < r_max; ++j) c[j] = 0.0f;
    for (int j = 0; j < r_t; ++j) {
        if (c_in) { c[j] = c_in[j]; continue; }
        float acc = 0.0f;
        for (int i = 0; i < d; ++i)
            acc = fmaf((float)oracle_bf16_to_f64(basis[(size_t)i * r_max + j]), xf[i], acc);
        c[j] = acc;
    }
    if (c32) for (int j = 0; j < r_max; ++j) c32[j] = c[j];
    if (oracle_quantize_coeffs8(r_t, r_max, c, ccodes, cscales, cbar)) return -1;
    for (int i = 0; i < d; ++i) {
        float a = 0.0f;
        for (int j = 0; j < r_t; ++j)
            a = fmaf((float)oracle_bf16_to_f64(basis[(size_t)i * r_max + j]), cbar[j], a);
        r[i] = xf[i] - a;
    }
    return oracle_quantize_residual(d, s, bits, r, idx, codes, scale);
}

/* Many vectors sharing one basis (token-ordered): x [n][d], rank [n]; c_in (nullable)       */
/* [n][r_max]; nres (nullable) per-vector residual counts <= s (the arrays' stride stays s).  */
int oracle_encode_many8(int n, int d, int r_max, const uint16_t* basis, const uint16_t* x, const float* c_in,
                        const int32_t* rank, int s, int bits, int8_t* ccodes, uint16_t* cscales, float* c32,
                        uint8_t* idx, int8_t* codes, uint16_t* scale, int nthreads, const int32_t* nres) {
    if (r_max % 16) return -1;
    int bad = 0;
#pragma omp parallel for schedule(static) num_threads(nthreads) reduction(| : bad)
    for (int k = 0; k < n; ++k)
        bad |= (oracle_encode_vector8(d, r_max, basis, x + (size_t)k * d, c_in ? c_in + (size_t)k * r_max : NULL,
                                      rank[k], nres ? nres[k] : s, bits, ccodes + (size_t)k * r_max,
                                      cscales + (size_t)k * (r_max / 16), c32 ? c32 + (size_t)k * r_max : NULL,
                                      idx + (size_t)k * s, codes + (size_t)k * s, scale + k) != 0);
    return bad ? -1 : 0;
}

int oracle_encode_vector(int d, int r_max, const uint16_t* basis, const uint16_t* x, int r_t,
                         int s, int bits, uint16_t* coeff, float* c32, uint8_t* idx, int8_t* codes,
                         uint16_t* scale, float* resid) {
    if (d <= 0 || d > 256 || r_t < 0 || r_t > r_max || s < 0 || s > d || (bits != 8 && bits != 4))
        return -1;
    float xf[256], c[256];
    for (int i = 0; i < d; ++i) xf[i] = (float)oracle_bf16_to_f64(x[i]);
    /* 1: projection, an fma chain over i = 0..d-1 from +0 */
    for (int j = 0; j < r_max; ++j) c[j] = 0.0f;
    for (int j = 0; j < r_t; ++j) {
        float acc = 0.0f;
        for (int i = 0; i < d; ++i)
            acc = fmaf((float)oracle_bf16_to_f64(basis[(size_t)i * r_max + j]), xf[i], acc);
        c[j] = acc;
    }
    if (c32) for (int j = 0; j < r_max; ++j) c32[j] = c[j];
    /* 2-6 */
    return oracle_encode_from_coeffs(d, r_max, basis, x, c, r_t, s, bits, coeff, idx, codes, scale, resid);
}

/* Steps 2-6 for many vectors that share one basis, from given projections c32 [n][r_max]. */
int oracle_encode_many_from_coeffs(int n, int d, int r_max, const uint16_t* basis, const uint16_t* x,
                                   const float* c32, const int32_t* rank, int s, int bits, uint16_t* coeff,
                                   uint8_t* idx, int8_t* codes, uint16_t* scale, int nthreads,
                                   const int32_t* nres) {
    int bad = 0;
#pragma omp parallel for schedule(static) num_threads(nthreads) reduction(| : bad)
    for (int k = 0; k < n; ++k)
        bad |= (oracle_encode_from_coeffs(d, r_max, basis, x + (size_t)k * d, c32 + (size_t)k * r_max, rank[k],
                                          nres ? nres[k] : s,
                                          bits, coeff + (size_t)k * r_max, idx + (size_t)k * s, codes + (size_t)k * s,
                                          scale + k, NULL) != 0);
    return bad ? -1 : 0;
}

/* Encode many vectors that share one basis (token-ordered): x [n][d], rank [n]. */
int oracle_encode_many(int n, int d, int r_max, const uint16_t* basis, const uint16_t* x,
                       const int32_t* rank, int s, int bits, uint16_t* coeff, float* c32,
                       uint8_t* idx, int8_t* codes, uint16_t* scale, int nthreads, const int32_t* nres) {
    int bad = 0;
#pragma omp parallel for schedule(static) num_threads(nthreads) reduction(| : bad)
    for (int k = 0; k < n; ++k)
        bad |= (oracle_encode_vector(d, r_max, basis, x + (size_t)k * d, rank[k], nres ? nres[k] : s, bits,
                                     coeff + (size_t)k * r_max, c32 ? c32 + (size_t)k * r_max : NULL,
                                     idx + (size_t)k * s, codes + (size_t)k * s, scale + k, NULL) != 0);
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------------------ */
/* Re-tiering a stored vector ([DW] §3, Eq. (2)-(3) paragraphs: the probe feedback lowers   */
/* the router threshold, so tokens move to another rank tier).  The dense vector is not     */
/* kept, so the token is re-encoded from its reconstruction (Eq. (1), g = 1), rounded to    */
/* bf16 like any input vector, at the new rank:                                            */
/*   a_i  = fma chain over j = 0..r_old-1 of B[i][j] * cb_j from +0      (fp32)            */
/*   xh_i = bf16_rn(a_i + scale * code_i) for the stored residual channels, bf16_rn(a_i)    */
/*          for the others (scale * code is exact in fp32; one rounding in the add)         */
/* then the six encode steps of oracle_encode_vector on xh at rank r_new with s_new        */
/* residual channels (a tier of the residual-count routing reading keeps its own count;     */
/* otherwise s_new = s), on basis_new (nullable: the same basis).  A basis update (the     */
/* shared bases' moving average, [DW] §3) moves a token with basis_new the updated basis    */
/* and r_new = r_old.                                                                       */
/* Inputs: the stored coeff (bf16 [r_max], entries >= r_old ignored), idx / codes [s],      */
/* scale (fp16 bits).  Outputs as oracle_encode_vector (idx / codes [s_new]); xh_out        */
/* (nullable) bf16 bits [d].                                                                */
/* ------------------------------------------------------------------------------------ */
int oracle_reencode_vector(int d, int r_max, const uint16_t* basis, int r_old, const uint16_t* coeff_old,
                           int s, const uint8_t* idx_old, const int8_t* codes_old, uint16_t scale_old,
                           int r_new, int s_new, int bits, uint16_t* coeff, uint8_t* idx, int8_t* codes,
                           uint16_t* scale, uint16_t* xh_out, const uint16_t* basis_new) {
    if (d <= 0 || d > 256 || r_old < 0 || r_old > r_max || r_new < 0 || r_new > r_max || s < 0 || s > d ||
        s_new < 0 || s_new > d)
        return -1;
    float a[256];
    uint16_t xh[256];
    for (int i = 0; i < d; ++i) {
        float acc = 0.0f;
        for (int j = 0; j < r_old; ++j)
            acc = fmaf((float)oracle_bf16_to_f64(basis[(size_t)i * r_max + j]), (float)oracle_bf16_to_f64(coeff_old[j]),
                       acc);
        a[i] = acc;
    }
    const float sf = (float)oracle_fp16_to_f64(scale_old);
    for (int k = 0; k < s; ++k) {
        if (idx_old[k] >= d) return -1;
        a[idx_old[k]] = a[idx_old[k]] + sf * (float)codes_old[k];
    }
    for (int i = 0; i < d; ++i) {
        xh[i] = oracle_f32_to_bf16_rn(a[i]);
        if (xh_out) xh_out[i] = xh[i];
    }
    return oracle_encode_vector(d, r_max, basis_new ? basis_new : basis, xh, r_new, s_new, bits, coeff, NULL, idx,
                                codes, scale, NULL);
}

/* The same re-encode for the 8-bit blockwise coefficient form: the stored coefficients are */
/* cb_j = code_j * scale_{j/16} (exact in fp32: 8 x 11 significant bits), the reconstruction */
/* chain and its bf16 rounding are those of oracle_reencode_vector, and xh is encoded by     */
/* oracle_encode_vector8 (its own projection) at rank r_new with s_new residual channels.    */
/* Inputs: ccodes_old int8 [r_max] and cscales_old fp16 bits [r_max / 16] (entries of j >=  */
/* r_old ignored), the residual as oracle_reencode_vector.  Outputs: ccodes [r_max],        */
/* cscales [r_max / 16], idx / codes [s_new], scale; xh_out (nullable) bf16 bits [d].       */
int oracle_reencode_vector8(int d, int r_max, const uint16_t* basis, int r_old, const int8_t* ccodes_old,
                            const uint16_t* cscales_old, int s, const uint8_t* idx_old, const int8_t* codes_old,
                            uint16_t scale_old, int r_new, int s_new, int bits, int8_t* ccodes, uint16_t* cscales,
                            uint8_t* idx, int8_t* codes, uint16_t* scale, uint16_t* xh_out,
                            const uint16_t* basis_new) {
    if (d <= 0 || d > 256 || r_max > 256 || r_max % 16 || r_old < 0 || r_old > r_max || r_old % 16 || r_new < 0 ||
        r_new > r_max || s < 0 || s > d || s_new < 0 || s_new > d)
        return -1;
    float cb[256], a[256];
    uint16_t xh[256];
    for (int j = 0; j < r_old; ++j)
        cb[j] = (float)ccodes_old[j] * (float)oracle_fp16_to_f64(cscales_old[j / 16]);
    for (int i = 0; i < d; ++i) {
        float acc = 0.0f;
        for (int j = 0; j < r_old; ++j)
            acc = fmaf((float)oracle_bf16_to_f64(basis[(size_t)i * r_max + j]), cb[j], acc);
        a[i] = acc;
    }
    const float sf = (float)oracle_fp16_to_f64(scale_old);
    for (int k = 0; k < s; ++k) {
        if (idx_old[k] >= d) return -1;
        a[idx_old[k]] = a[idx_old[k]] + sf * (float)codes_old[k];
    }
    for (int i = 0; i < d; ++i) {
        xh[i] = oracle_f32_to_bf16_rn(a[i]);
        if (xh_out) xh_out[i] = xh[i];
    }
    return oracle_encode_vector8(d, r_max, basis_new ? basis_new : basis, xh, NULL, r_new, s_new, bits, ccodes,
                                 cscales, NULL, idx, codes, scale);
}

/* Element-wise format conversions over arrays (used to pin the converters). */
void oracle_f32_to_bf16_rn_many(int64_t n, const float* x, uint16_t* out) {
    for (int64_t k = 0; k < n; ++k) out[k] = oracle_f32_to_bf16_rn(x[k]);
}
void oracle_f32_to_fp16_rn_many(int64_t n, const float* x, uint16_t* out) {
    for (int64_t k = 0; k < n; ++k) out[k] = oracle_f32_to_fp16_rn(x[k]);
}
void oracle_fp16_to_f64_many(int64_t n, const uint16_t* x, double* out) {
    for (int64_t k = 0; k < n; ++k) out[k] = oracle_fp16_to_f64(x[k]);
}
void oracle_bf16_to_f64_many(int64_t n, const uint16_t* x, double* out) {
    for (int64_t k = 0; k < n; ++k) out[k] = oracle_bf16_to_f64(x[k]);
}
