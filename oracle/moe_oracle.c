/*
 * moe_oracle.c -- plain, slow, fp64 CPU oracle for the routed MoE expert FFN.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file: only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark do.  It shares no code, header, table or helper with the
 * CUDA library; the two meet only at the seeded input bytes.
 *
 * What it computes (rocketrecap.com "FlyDSL kernels in JAX" summary, paragraph 2
 * and timestamp 5:56: routed MoE = gather -> group GEMM (w1/w3) -> SwiGLU ->
 * group GEMM (w2) -> scatter, replacing the masked dense GEMM path; timestamp
 * 8:14: top-2 routing, Mixtral 8x7B; glossary entries "SwiGLU" and "Group GEMM"):
 *
 *   out[t] = bf16( sum_{j<k} w[t,j] * Y(e[t,j], t) )
 *   Y(e,t) = W2_e . q_h( bf16( silu(W1_e x_t) * (W3_e x_t) ) )
 *
 * with every product and sum in fp64 over the same dequantised operand values
 * the GPU consumes (e4m3 code value x fp32 scale, or bf16 value).  The pages
 * are silent on the numeric details; the readings taken here are:
 *   - top-k: larger logit first, equal logits -> lower expert index, NaN ranks
 *     as -inf (below every other value, ties among them again by index);
 *   - routing weights: softmax over the k selected logits only;
 *   - stable counting sort of assignments a = t*k + j by expert;
 *   - FP8 mode: x quantised per token (sx = fp32(absmax/448), sx = 1 for an
 *     all-zero row, xq = e4m3_rn_satfinite(fp32(x / sx)));
 *     h rounded to bf16, then quantised to e4m3 in blocks of 32 consecutive
 *     d_ff elements with a power-of-two (UE8M0) scale 2^ceil(log2(absmax/448)),
 *     clamped to [2^-127, 2^127], scale 1 for an all-zero block;
 *   - BF16 mode: h rounded to bf16 and used as is;
 *   - MXFP4 mode (MX-scaled FP4 expert weights, the kinachrichten.com page
 *     "PyTorch erhaelt FlyDSL-Backend", its list of kernel benchmarks: MXFP4
 *     scaled GEMM, E8M0 scales per 32 values): every weight is an OCP e2m1
 *     code times the power of two 2^(s - 127) that its block of 32
 *     consecutive K elements (along d_model for w1/w3, along d_ff for w2)
 *     shares; x and h are quantised as in FP8 mode;
 *   - the combine is an fp64 sum, rounded once to bf16.
 *
 * The last section holds the backward pass (custom VJP) of the BF16 layer on
 * fp64 inputs: the gradients of <dy, out> with respect to x, w1, w3, w2 and
 * the router logits (timestamp 10:07 names it as the next step).
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC -fno-fast-math -ffp-contract=off moe_oracle.c
 *        -o liboracle.so -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_BF16 0
#define ORACLE_FP8 1
#define ORACLE_MXFP4 2

/* ------------------------------------------------------------------------ */
/* Number formats, written from their definitions.                          */
/* ------------------------------------------------------------------------ */

/* OCP FP8 E4M3 ("fn" variant): 1 sign, 4 exponent bits (bias 7), 3 mantissa
 * bits; no infinities; S.1111.111 is NaN; largest finite magnitude 448. */
double oracle_e4m3_to_double(uint8_t code) {
    int sign = (code >> 7) & 1;
    int ex = (code >> 3) & 0xF;
    int man = code & 7;
    double mag;
    if (ex == 0xF && man == 7) return NAN;
    if (ex == 0)
        mag = ldexp((double)man / 8.0, -6);           /* subnormal: 0.man * 2^-6 */
    else
        mag = ldexp(1.0 + (double)man / 8.0, ex - 7); /* normal: 1.man * 2^(ex-7) */
    return sign ? -mag : mag;
}

/* OCP e2m1 (the MX FP4 element): 1 sign, 2 exponent bits (bias 1), 1 mantissa
 * bit, no infinities or NaN; exponent field 0 is subnormal (0.m * 2^0).  Only
 * the low 4 bits of `code` are read.  Magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
double oracle_e2m1_to_double(uint8_t code) {
    int sign = (code >> 3) & 1;
    int ex = (code >> 1) & 3;
    int man = code & 1;
    double mag = (ex == 0) ? (double)man * 0.5 : ldexp(1.0 + (double)man * 0.5, ex - 1);
    return sign ? -mag : mag;
}

/* UE8M0 (the MX block scale): an unsigned 8-bit biased exponent, value
 * 2^(e - 127); e = 255 is NaN. */
double oracle_ue8m0_to_double(uint8_t e) { return e == 255 ? NAN : ldexp(1.0, (int)e - 127); }

/* Values of the 256 codes, filled once when the library is loaded. */
static double e4m3_value[256];
__attribute__((constructor)) static void e4m3_table_init(void) {
    for (int c = 0; c < 256; ++c) e4m3_value[c] = oracle_e4m3_to_double((uint8_t)c);
}

/* Round a float to the nearest e4m3 value, ties to even mantissa, and clamp
 * out-of-range magnitudes to +-448 (satfinite).  NaN maps to the NaN code.
 * The non-negative finite codes 0x00..0x7E increase with their value, so the
 * two neighbours of |v| are found by bisection over the code range. */
uint8_t oracle_e4m3_from_float(float v) {
    double x = (double)v;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs(x);
    if (isnan(x)) return 0x7F;
    if (a >= 448.0) return sign | 0x7E;
    int lo = 0, hi = 0x7E; /* invariant: value(lo) <= a < value(hi) */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (e4m3_value[mid] <= a) lo = mid;
        else hi = mid;
    }
    double dlo = a - e4m3_value[lo], dhi = e4m3_value[hi] - a;
    int best;
    if (dlo < dhi) best = lo;
    else if (dhi < dlo) best = hi;
    else best = (lo % 2 == 0) ? lo : hi; /* tie: even mantissa = even code */
    return sign | (uint8_t)best;
}

/* bf16 = the upper 16 bits of an IEEE binary32.  Rounding from a double goes
 * straight to the 8-bit significand, nearest, ties to even. */
double oracle_bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

uint16_t oracle_bf16_from_double(double v) {
    if (isnan(v)) return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return sign;
    if (isinf(a)) return sign | 0x7F80;
    int e;
    frexp(a, &e);                 /* a = m * 2^e, m in [0.5, 1) */
    int ulp_exp = e - 8;          /* 8 significant bits: ulp = 2^(e-8) */
    if (ulp_exp < -133) ulp_exp = -133; /* bf16 subnormal spacing 2^-133 */
    double q = ldexp(a, -ulp_exp); /* exact: scaling by a power of two */
    double fl = floor(q);
    double rem = q - fl;
    double r;
    if (rem > 0.5) r = fl + 1.0;
    else if (rem < 0.5) r = fl;
    else r = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
    double rounded = ldexp(r, ulp_exp);
    if (rounded > 3.3895313892515355e38) return sign | 0x7F80; /* overflow -> inf */
    float f = (float)rounded; /* exactly representable in binary32 */
    uint32_t u;
    memcpy(&u, &f, 4);
    return sign | (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------------ */
/* R0: per-token activation quantisation (FP8 mode).                        */
/* ------------------------------------------------------------------------ */

/* sx[t] = fp32(absmax_t / 448) (IEEE single division), 1 for an all-zero row;
 * xq[t,i] = e4m3_rn_satfinite(fp32(x[t,i] / sx[t])).  The division is done in
 * binary32 because its result decides an integer code on both sides. */
void oracle_quant_x(const uint16_t* x, int T, int H, uint8_t* xq, float* sx) {
    for (int t = 0; t < T; ++t) {
        float amax = 0.0f;
        for (int i = 0; i < H; ++i) {
            float v = (float)oracle_bf16_to_double(x[(size_t)t * H + i]);
            if (fabsf(v) > amax) amax = fabsf(v);
        }
        volatile float s = (amax == 0.0f) ? 1.0f : amax / 448.0f;
        sx[t] = s;
        for (int i = 0; i < H; ++i) {
            volatile float v = (float)oracle_bf16_to_double(x[(size_t)t * H + i]);
            volatile float q = v / s;
            xq[(size_t)t * H + i] = oracle_e4m3_from_float(q);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* MX block quantisation of the intermediate h (FP8 mode).                  */
/* ------------------------------------------------------------------------ */

/* Power-of-two exponent e = ceil(log2(amax / 448)) clamped to [-127, 127];
 * 0 (scale 1) for amax == 0.  frexp gives amax/448 = m * 2^x with m in
 * [0.5, 1); the smallest power of two >= m * 2^x is 2^(x-1) when m == 0.5
 * and 2^x otherwise. */
int oracle_mx_exponent(double amax) {
    if (amax == 0.0) return 0;
    int x;
    double m = frexp(amax / 448.0, &x);
    int e = (m == 0.5) ? x - 1 : x;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

/* Quantise n bf16 values (given as doubles) that form one block: returns the
 * scale exponent, writes e4m3 codes. */
int oracle_mx_quant_block(const double* hb, int n, uint8_t* codes) {
    double amax = 0.0;
    for (int i = 0; i < n; ++i)
        if (fabs(hb[i]) > amax) amax = fabs(hb[i]);
    int e = oracle_mx_exponent(amax);
    for (int i = 0; i < n; ++i) {
        /* hb is a bf16 value and the divisor a power of two in [2^-127, 2^127]:
         * the quotient is exact in binary32 */
        float q = (float)ldexp(hb[i], -e);
        codes[i] = oracle_e4m3_from_float(q);
    }
    return e;
}

/* ------------------------------------------------------------------------ */
/* R1/R2: routing.                                                          */
/* ------------------------------------------------------------------------ */

/* Ranking key: NaN behaves as -inf. */
static double rank_value(float l) { return isnan(l) ? -INFINITY : (double)l; }

/* Is (va, ia) ranked before (vb, ib)?  Larger value first, lower index on a tie. */
static int ranks_before(double va, int ia, double vb, int ib) {
    if (va > vb) return 1;
    if (va < vb) return 0;
    return ia < ib;
}

/* Top-k of one token's E logits by selection: k passes, each taking the best
 * not-yet-chosen expert.  Weights = softmax over the chosen logits, fp64:
 * w_j = exp(l_j - l_max) / sum_i exp(l_i - l_max).  Limits for non-finite
 * logits: if the largest chosen logit is +inf the weight is shared equally by
 * the +inf entries; if it is -inf (all chosen are -inf/NaN) it is shared
 * equally by all k. */
static void topk_one(const float* l, int E, int k, int32_t* ids, double* w) {
    char chosen[64];
    memset(chosen, 0, sizeof(chosen));
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (chosen[e]) continue;
            if (best < 0 || ranks_before(rank_value(l[e]), e, rank_value(l[best]), best)) best = e;
        }
        chosen[best] = 1;
        ids[j] = best;
    }
    double lmax = rank_value(l[ids[0]]);
    if (isinf(lmax)) {
        int n = 0;
        for (int j = 0; j < k; ++j) n += (rank_value(l[ids[j]]) == lmax);
        for (int j = 0; j < k; ++j) w[j] = (rank_value(l[ids[j]]) == lmax) ? 1.0 / n : 0.0;
        return;
    }
    double den = 0.0;
    for (int j = 0; j < k; ++j) den += exp(rank_value(l[ids[j]]) - lmax);
    for (int j = 0; j < k; ++j) w[j] = exp(rank_value(l[ids[j]]) - lmax) / den;
}

/* Route T tokens.  Outputs: ids/w [T,k]; counts [E]; offsets [E+1] (exclusive
 * scan of counts); perm [T*k]: sorted position -> assignment a = t*k + j,
 * assignments grouped by expert, ascending a inside a group; inv_perm: the
 * inverse.  Any output pointer may be NULL except ids and w. */
int oracle_route(const float* logits, int T, int E, int k, int32_t* ids, double* w,
                 int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv_perm) {
    if (T < 0 || E < 1 || E > 64 || k < 1 || k > E) return -1;
    for (int t = 0; t < T; ++t) topk_one(logits + (size_t)t * E, E, k, ids + (size_t)t * k, w + (size_t)t * k);
    int32_t cnt[64], off[65];
    memset(cnt, 0, sizeof(cnt));
    for (long a = 0; a < (long)T * k; ++a) cnt[ids[a]]++;
    off[0] = 0;
    for (int e = 0; e < E; ++e) off[e + 1] = off[e] + cnt[e];
    if (counts) memcpy(counts, cnt, sizeof(int32_t) * E);
    if (offsets) memcpy(offsets, off, sizeof(int32_t) * (E + 1));
    if (perm || inv_perm) {
        int32_t fill[64];
        memcpy(fill, off, sizeof(int32_t) * E);
        for (long a = 0; a < (long)T * k; ++a) {
            int32_t p = fill[ids[a]]++;
            if (perm) perm[p] = (int32_t)a;
            if (inv_perm) inv_perm[a] = p;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* S1/S2: the expert FFN of one token for one expert.                       */
/* ------------------------------------------------------------------------ */

typedef struct {
    const uint16_t* x;   /* [T,H] bf16 */
    const void* w1;      /* [E,F,H] bf16 or e4m3; MXFP4: [E,F,H/2] packed e2m1 */
    const void* w3;      /* [E,F,H] */
    const void* s1;      /* FP8: fp32 [E,F] per output channel; MXFP4: uint8 [E,F,H/32] block exponents */
    const void* s3;
    const void* w2;      /* [E,H,F]; MXFP4: [E,H,F/2] */
    const void* s2;      /* FP8: fp32 [E,H]; MXFP4: uint8 [E,H,F/32] */
    int T, H, F, E, k, dtype;
    double e4m3_table[256];
    const uint8_t* xq;   /* [T,H] (FP8, MXFP4) */
    const float* sx;     /* [T] */
} ffn_ctx;

/* Element (row, col) of expert e's matrix [rows, cols] (cols = K).  MXFP4:
 * two e2m1 codes per byte, the even column in the low 4 bits; the block
 * exponent of (row, col / 32). */
static double weight_value(const ffn_ctx* c, const void* w, const void* s, int e, int row, int col,
                           int rows, int cols) {
    size_t r = (size_t)e * rows + row;
    if (c->dtype == ORACLE_BF16) return oracle_bf16_to_double(((const uint16_t*)w)[r * cols + col]);
    if (c->dtype == ORACLE_FP8) return c->e4m3_table[((const uint8_t*)w)[r * cols + col]] * (double)((const float*)s)[r];
    uint8_t byte = ((const uint8_t*)w)[r * (cols / 2) + col / 2];
    uint8_t code = (col & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15);
    return oracle_e2m1_to_double(code) * oracle_ue8m0_to_double(((const uint8_t*)s)[r * (cols / 32) + col / 32]);
}

static double x_value(const ffn_ctx* c, int t, int i) {
    size_t idx = (size_t)t * c->H + i;
    if (c->dtype == ORACLE_BF16) return oracle_bf16_to_double(c->x[idx]);
    return c->e4m3_table[c->xq[idx]] * (double)c->sx[t];
}

/* y[H] = Y(e, t) in fp64.  h_out (optional, [F]) receives the dequantised
 * intermediate that enters the second GEMM; h_exact (optional, [F]) the exact
 * value silu(g) * u before any rounding. */
static void expert_ffn(const ffn_ctx* c, int e, int t, double* y, double* h_out, double* h_exact) {
    int H = c->H, F = c->F;
    double* hq = (double*)malloc(sizeof(double) * F);
    for (int n = 0; n < F; ++n) {
        double g = 0.0, u = 0.0;
        for (int i = 0; i < H; ++i) {
            double xv = x_value(c, t, i);
            g += weight_value(c, c->w1, c->s1, e, n, i, F, H) * xv;
            u += weight_value(c, c->w3, c->s3, e, n, i, F, H) * xv;
        }
        double silu = g / (1.0 + exp(-g));
        if (h_exact) h_exact[n] = silu * u;
        hq[n] = oracle_bf16_to_double(oracle_bf16_from_double(silu * u));
    }
    if (c->dtype != ORACLE_BF16) {
        uint8_t codes[32];
        for (int b = 0; b < F; b += 32) {
            int n = (F - b < 32) ? F - b : 32;
            int ex = oracle_mx_quant_block(hq + b, n, codes);
            for (int i = 0; i < n; ++i) hq[b + i] = ldexp(c->e4m3_table[codes[i]], ex);
        }
    }
    if (h_out) memcpy(h_out, hq, sizeof(double) * F);
    for (int o = 0; o < H; ++o) {
        double acc = 0.0;
        for (int n = 0; n < F; ++n) acc += weight_value(c, c->w2, c->s2, e, o, n, H, F) * hq[n];
        y[o] = acc;
    }
    free(hq);
}

static int ctx_init(ffn_ctx* c, const uint16_t* x, const void* w1, const void* w3, const void* s1,
                    const void* s3, const void* w2, const void* s2, int T, int H, int F, int E, int k,
                    int dtype) {
    if (T < 0 || H < 1 || F < 1 || E < 1 || E > 64 || k < 1 || k > E) return -1;
    if (dtype != ORACLE_BF16 && dtype != ORACLE_FP8 && dtype != ORACLE_MXFP4) return -1;
    if (dtype != ORACLE_BF16 && (!s1 || !s3 || !s2)) return -1;
    if (dtype == ORACLE_MXFP4 && (H % 32 || F % 32)) return -1;
    c->x = x; c->w1 = w1; c->w3 = w3; c->s1 = s1; c->s3 = s3; c->w2 = w2; c->s2 = s2;
    c->T = T; c->H = H; c->F = F; c->E = E; c->k = k; c->dtype = dtype;
    for (int i = 0; i < 256; ++i) c->e4m3_table[i] = oracle_e4m3_to_double((uint8_t)i);
    c->xq = NULL; c->sx = NULL;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* The whole layer, two formulations.                                       */
/* ------------------------------------------------------------------------ */

/* mode 0 = routed (route, group the assignments by expert, per-expert FFN on
 * the gathered rows, weighted scatter-add back to token order);
 * mode 1 = masked dense (every expert on every token, multiplied by a mask
 * that holds the routing weight for the chosen experts and 0 elsewhere).
 * out: bf16 [T,H]; out64 (optional): the fp64 sum before rounding;
 * h_sorted (optional, routed mode): [T*k, F] dequantised intermediate in
 * sorted order.  Returns 0, or -1 on a bad argument. */
int oracle_moe_ffn(int mode, const uint16_t* x, const float* logits, const void* w1, const void* w3,
                   const void* s1, const void* s3, const void* w2, const void* s2, int T, int H, int F,
                   int E, int k, int dtype, uint16_t* out, double* out64, double* h_sorted, int nthreads) {
    ffn_ctx c;
    if (ctx_init(&c, x, w1, w3, s1, s3, w2, s2, T, H, F, E, k, dtype)) return -1;
    if (mode != 0 && mode != 1) return -1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
    long A = (long)T * k;
    int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (A ? A : 1));
    double* w = (double*)malloc(sizeof(double) * (A ? A : 1));
    int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (A ? A : 1));
    int32_t offsets[65];
    uint8_t* xq = NULL;
    float* sx = NULL;
    if (dtype != ORACLE_BF16) {
        xq = (uint8_t*)malloc((size_t)T * H + 1);
        sx = (float*)malloc(sizeof(float) * (T ? T : 1));
        oracle_quant_x(x, T, H, xq, sx);
        c.xq = xq; c.sx = sx;
    }
    oracle_route(logits, T, E, k, ids, w, NULL, offsets, perm, NULL);
    double* acc = (double*)calloc((size_t)T * H + 1, sizeof(double));

    if (mode == 0) {
        /* per expert: gathered rows perm[offsets[e] .. offsets[e+1]) */
        double* ybuf = (double*)malloc(sizeof(double) * (size_t)H * (A ? A : 1));
        #pragma omp parallel for schedule(dynamic, 1)
        for (long p = 0; p < A; ++p) {
            int32_t a = perm[p];
            int e = ids[a];
            expert_ffn(&c, e, (int)(a / k), ybuf + (size_t)p * H, h_sorted ? h_sorted + (size_t)p * F : NULL, NULL);
        }
        /* scatter-add in sorted order (deterministic) */
        for (long p = 0; p < A; ++p) {
            int32_t a = perm[p];
            int t = (int)(a / k);
            for (int o = 0; o < H; ++o) acc[(size_t)t * H + o] += w[a] * ybuf[(size_t)p * H + o];
        }
        free(ybuf);
    } else {
        #pragma omp parallel for schedule(dynamic, 1)
        for (int t = 0; t < T; ++t) {
            double* y = (double*)malloc(sizeof(double) * H);
            for (int e = 0; e < E; ++e) {
                double mask = 0.0;
                for (int j = 0; j < k; ++j)
                    if (ids[(size_t)t * k + j] == e) mask = w[(size_t)t * k + j];
                expert_ffn(&c, e, t, y, NULL, NULL);
                for (int o = 0; o < H; ++o) acc[(size_t)t * H + o] += mask * y[o];
            }
            free(y);
        }
    }
    for (size_t i = 0; i < (size_t)T * H; ++i) {
        out[i] = oracle_bf16_from_double(acc[i]);
        if (out64) out64[i] = acc[i];
    }
    free(acc); free(ids); free(w); free(perm); free(xq); free(sx);
    (void)offsets;
    return 0;
}

/* Output rows for a list of tokens only (each token's result depends on its
 * own activations and logits alone), per-token routed form.  out: [ntok,H]
 * bf16; out64 optional [ntok,H].  Optional per-assignment intermediates, row
 * i*k + j for the j-th expert of the i-th listed token: h_deq [ntok*k, F] (the
 * dequantised values entering the second GEMM) and h_exact [ntok*k, F] (silu(g)*u
 * before rounding).  Used for sampled checks at full size and for the CPU
 * timing sample. */
int oracle_moe_ffn_tokens(const uint16_t* x, const float* logits, const void* w1, const void* w3,
                          const void* s1, const void* s3, const void* w2, const void* s2, int T, int H,
                          int F, int E, int k, int dtype, const int32_t* tokens, int ntok, uint16_t* out,
                          double* out64, double* h_deq, double* h_exact, int nthreads) {
    ffn_ctx c;
    if (ctx_init(&c, x, w1, w3, s1, s3, w2, s2, T, H, F, E, k, dtype)) return -1;
    for (int i = 0; i < ntok; ++i)
        if (tokens[i] < 0 || tokens[i] >= T) return -1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
    long work = (long)ntok * k;
    int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (work ? work : 1));
    double* w = (double*)malloc(sizeof(double) * (work ? work : 1));
    uint8_t* xq = NULL;
    float* sx = NULL;
    if (dtype != ORACLE_BF16) {
        /* quantise only the sampled rows, indexed by their own token id */
        xq = (uint8_t*)calloc((size_t)T * H + 1, 1);
        sx = (float*)calloc((size_t)(T ? T : 1), sizeof(float));
        for (int i = 0; i < ntok; ++i) {
            int t = tokens[i];
            oracle_quant_x(x + (size_t)t * H, 1, H, xq + (size_t)t * H, sx + t);
        }
        c.xq = xq; c.sx = sx;
    }
    for (int i = 0; i < ntok; ++i)
        oracle_route(logits + (size_t)tokens[i] * E, 1, E, k, ids + (size_t)i * k, w + (size_t)i * k, NULL,
                     NULL, NULL, NULL);
    double* ybuf = (double*)malloc(sizeof(double) * (size_t)H * (work ? work : 1));
    #pragma omp parallel for schedule(dynamic, 1)
    for (long q = 0; q < work; ++q)
        expert_ffn(&c, ids[q], tokens[q / k], ybuf + (size_t)q * H, h_deq ? h_deq + (size_t)q * F : NULL,
                   h_exact ? h_exact + (size_t)q * F : NULL);
    for (int i = 0; i < ntok; ++i) {
        for (int o = 0; o < H; ++o) {
            double acc = 0.0;
            /* combine in expert order, as the routed form does */
            for (int pass = 0; pass < E; ++pass)
                for (int j = 0; j < k; ++j)
                    if (ids[(size_t)i * k + j] == pass) acc += w[(size_t)i * k + j] * ybuf[((size_t)i * k + j) * H + o];
            out[(size_t)i * H + o] = oracle_bf16_from_double(acc);
            if (out64) out64[(size_t)i * H + o] = acc;
        }
    }
    free(ybuf); free(ids); free(w); free(xq); free(sx);
    return 0;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Backward (custom VJP) of the BF16 layer, fp64.                           */
/* ------------------------------------------------------------------------ */
/*
 * The pages list a custom VJP for training as the next step of the routed
 * kernel (rocketrecap.com "FlyDSL kernels in JAX", timestamp 10:07) and do not
 * define it; what is computed here is the gradient of the BF16 layer above
 * with respect to x, w1, w3, w2 and the router logits, for an upstream
 * gradient dy = dL/dout.  For each assignment a = (t, j) of token t to expert
 * e with routing weight w_a:
 *
 *   g = W1_e x_t,  u = W3_e x_t,  h = silu(g) * u   (rounded to bf16 with
 *       ORACLE_ROUND_H, as the forward rounds it; the rounding passes
 *       gradients through unchanged),  o = W2_e h
 *   dw_a = <dy_t, o>,   dO = w_a dy_t,   dh = W2_e^T dO
 *   du = dh * silu(g),  dg = dh * u * silu'(g),  silu'(g) = s(g) (1 + g (1 - s(g)))
 *       with s the logistic function
 *   dx_t  += W1_e^T dg + W3_e^T du
 *   dW1_e += dg x_t^T,  dW3_e += du x_t^T,  dW2_e += dO h^T
 *
 * Router: w = softmax over the k chosen logits, so for the chosen experts
 * dlogit[t, e_j] = w_j (dw_j - sum_i w_i dw_i), and 0 for the others (the
 * choice itself is piecewise constant in the logits).
 *
 * Inputs are fp64 so that finite differences can perturb them.  The choice of
 * experts follows the forward's ranking rule (larger logit first, lower index
 * on a tie, NaN as -inf); gradients are defined for finite logits.
 *
 * `round` flags: ORACLE_ROUND_H rounds h to bf16 (the forward's rounding);
 * ORACLE_ROUND_INTER also rounds to bf16 the values a bf16 implementation
 * stores between its backward steps -- dg and du, and the products w_a dy_t
 * that enter dW2 (dh uses w_a dy_t unrounded).  All else is exact.
 *
 * Optional error scales (`abs` outputs): each gradient entry's sum of the
 * absolute values of its terms -- |W1|^T |dg| + |W3|^T |du| for dx, |dg| |x|^T
 * for dW1, |du| |x|^T for dW3, |w_a dy| |h|^T for dW2, and for the router
 * w_j (s_j + sum_i w_i s_i) with s_a = sum_f |dh_f / w_a| |h_f| -- the scale
 * against which a perturbation of the individual terms is measured.
 */
#define ORACLE_ROUND_H 1
#define ORACLE_ROUND_INTER 2

typedef struct {
    const double *x, *w1, *w3, *w2;  /* [T,H], [E,F,H], [E,F,H], [E,H,F] */
    int T, H, F, E, k, round_h, round_inter;
} bctx;

static double bf16r(double v) { return oracle_bf16_to_double(oracle_bf16_from_double(v)); }

static double ranked64(double l) { return isnan(l) ? -INFINITY : l; }

/* top-k and the softmax over the chosen logits of one token (fp64 logits) */
static void topk64(const double* l, int E, int k, int32_t* ids, double* w) {
    char chosen[64];
    memset(chosen, 0, sizeof(chosen));
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (chosen[e]) continue;
            if (best < 0 || ranks_before(ranked64(l[e]), e, ranked64(l[best]), best)) best = e;
        }
        chosen[best] = 1;
        ids[j] = best;
    }
    double lmax = ranked64(l[ids[0]]);
    if (isinf(lmax)) {
        int n = 0;
        for (int j = 0; j < k; ++j) n += (ranked64(l[ids[j]]) == lmax);
        for (int j = 0; j < k; ++j) w[j] = (ranked64(l[ids[j]]) == lmax) ? 1.0 / n : 0.0;
        return;
    }
    double den = 0.0;
    for (int j = 0; j < k; ++j) den += exp(ranked64(l[ids[j]]) - lmax);
    for (int j = 0; j < k; ++j) w[j] = exp(ranked64(l[ids[j]]) - lmax) / den;
}

static int bctx_init(bctx* c, const double* x, const double* w1, const double* w3, const double* w2, int T,
                     int H, int F, int E, int k, int round) {
    if (T < 0 || H < 1 || F < 1 || E < 1 || E > 64 || k < 1 || k > E) return -1;
    c->x = x; c->w1 = w1; c->w3 = w3; c->w2 = w2;
    c->T = T; c->H = H; c->F = F; c->E = E; c->k = k;
    c->round_h = (round & ORACLE_ROUND_H) != 0;
    c->round_inter = (round & ORACLE_ROUND_INTER) != 0;
    return 0;
}

/* g, u, h [F] and o [H] of token t through expert e */
static void fwd_assign(const bctx* c, int e, int t, double* g, double* u, double* h, double* o) {
    int H = c->H, F = c->F;
    const double* xt = c->x + (size_t)t * H;
    for (int n = 0; n < F; ++n) {
        const double* r1 = c->w1 + ((size_t)e * F + n) * H;
        const double* r3 = c->w3 + ((size_t)e * F + n) * H;
        double gv = 0.0, uv = 0.0;
        for (int i = 0; i < H; ++i) {
            gv += r1[i] * xt[i];
            uv += r3[i] * xt[i];
        }
        double hv = gv / (1.0 + exp(-gv)) * uv;
        if (c->round_h) hv = bf16r(hv);
        g[n] = gv; u[n] = uv; h[n] = hv;
    }
    for (int m = 0; m < H; ++m) {
        const double* r2 = c->w2 + ((size_t)e * H + m) * F;
        double acc = 0.0;
        for (int n = 0; n < F; ++n) acc += r2[n] * h[n];
        o[m] = acc;
    }
}

/* dg, du [F] from dh and the forward values (rounded to bf16 with round_inter) */
static void swiglu_bwd(int F, const double* g, const double* u, const double* dh, double* dg, double* du,
                       int round_inter) {
    for (int n = 0; n < F; ++n) {
        double s = 1.0 / (1.0 + exp(-g[n]));
        du[n] = dh[n] * (g[n] / (1.0 + exp(-g[n])));
        dg[n] = dh[n] * u[n] * (s * (1.0 + g[n] * (1.0 - s)));
        if (round_inter) {
            du[n] = bf16r(du[n]);
            dg[n] = bf16r(dg[n]);
        }
    }
}

/* y [T,H] (fp64, not rounded) of the layer on fp64 inputs; the combine adds
 * each token's expert outputs in ascending expert order, as the routed form */
int oracle_moe_ffn64(const double* x, const double* logits, const double* w1, const double* w3, const double* w2,
                     int T, int H, int F, int E, int k, int round, double* y, int nthreads) {
    bctx c;
    if (bctx_init(&c, x, w1, w3, w2, T, H, F, E, k, round)) return -1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
    #pragma omp parallel for schedule(dynamic, 1)
    for (int t = 0; t < T; ++t) {
        int32_t ids[64];
        double w[64];
        double *g = malloc(sizeof(double) * F), *u = malloc(sizeof(double) * F), *h = malloc(sizeof(double) * F);
        double** o = malloc(sizeof(double*) * k);
        topk64(logits + (size_t)t * E, E, k, ids, w);
        for (int j = 0; j < k; ++j) {
            o[j] = malloc(sizeof(double) * H);
            fwd_assign(&c, ids[j], t, g, u, h, o[j]);
        }
        for (int m = 0; m < H; ++m) {
            double acc = 0.0;
            for (int e = 0; e < E; ++e)
                for (int j = 0; j < k; ++j)
                    if (ids[j] == e) acc += w[j] * o[j][m];
            y[(size_t)t * H + m] = acc;
        }
        for (int j = 0; j < k; ++j) free(o[j]);
        free(o); free(g); free(u); free(h);
    }
    return 0;
}

/* Full gradients: dx [T,H], dw1/dw3 [E,F,H], dw2 [E,H,F], dlogits [T,E]; dwa
 * (optional) [T*k] the gradients of the routing weights; the error scales
 * (optional, all or none) in arrays of the same shapes.  Experts run in
 * parallel; inside one, assignments in ascending order. */
int oracle_moe_ffn_bwd64(const double* x, const double* logits, const double* w1, const double* w3,
                         const double* w2, const double* dy, int T, int H, int F, int E, int k, int round,
                         double* dx, double* dw1, double* dw3, double* dw2, double* dlogits, double* dwa_out,
                         double* dx_abs, double* dw1_abs, double* dw3_abs, double* dw2_abs, double* dl_abs,
                         int nthreads) {
    bctx c;
    if (bctx_init(&c, x, w1, w3, w2, T, H, F, E, k, round)) return -1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
    long A = (long)T * k;
    int32_t* ids = malloc(sizeof(int32_t) * (A ? A : 1));
    double* w = malloc(sizeof(double) * (A ? A : 1));
    double* dwa = calloc(A ? A : 1, sizeof(double));
    double* dxa = calloc((size_t)(A ? A : 1) * H, sizeof(double));
    const int want_abs = dx_abs != NULL;
    double* dwabs = calloc(A ? A : 1, sizeof(double));
    double* dxabs = want_abs ? calloc((size_t)(A ? A : 1) * H, sizeof(double)) : NULL;
    for (int t = 0; t < T; ++t) topk64(logits + (size_t)t * E, E, k, ids + (size_t)t * k, w + (size_t)t * k);
    memset(dw1, 0, sizeof(double) * (size_t)E * F * H);
    memset(dw3, 0, sizeof(double) * (size_t)E * F * H);
    memset(dw2, 0, sizeof(double) * (size_t)E * H * F);
    if (want_abs) {
        memset(dw1_abs, 0, sizeof(double) * (size_t)E * F * H);
        memset(dw3_abs, 0, sizeof(double) * (size_t)E * F * H);
        memset(dw2_abs, 0, sizeof(double) * (size_t)E * H * F);
    }
    #pragma omp parallel for schedule(dynamic, 1)
    for (int e = 0; e < E; ++e) {
        double *g = malloc(sizeof(double) * F), *u = malloc(sizeof(double) * F), *h = malloc(sizeof(double) * F);
        double *dh = malloc(sizeof(double) * F), *dg = malloc(sizeof(double) * F), *du = malloc(sizeof(double) * F);
        double *o = malloc(sizeof(double) * H), *dO = malloc(sizeof(double) * H);
        for (long a = 0; a < A; ++a) {
            if (ids[a] != e) continue;
            int t = (int)(a / k);
            const double* dyt = dy + (size_t)t * H;
            const double* xt = x + (size_t)t * H;
            fwd_assign(&c, e, t, g, u, h, o);
            double s = 0.0;
            for (int m = 0; m < H; ++m) s += dyt[m] * o[m];
            dwa[a] = s;
            for (int m = 0; m < H; ++m) dO[m] = w[a] * dyt[m];
            for (int n = 0; n < F; ++n) {
                double acc = 0.0;
                for (int m = 0; m < H; ++m) acc += w2[((size_t)e * H + m) * F + n] * dO[m];
                dh[n] = acc;
            }
            swiglu_bwd(F, g, u, dh, dg, du, c.round_inter);
            double* dxr = dxa + (size_t)a * H;
            for (int i = 0; i < H; ++i) {
                double acc = 0.0;
                for (int n = 0; n < F; ++n)
                    acc += w1[((size_t)e * F + n) * H + i] * dg[n] + w3[((size_t)e * F + n) * H + i] * du[n];
                dxr[i] = acc;
            }
            for (int n = 0; n < F; ++n) {
                double* r1 = dw1 + ((size_t)e * F + n) * H;
                double* r3 = dw3 + ((size_t)e * F + n) * H;
                for (int i = 0; i < H; ++i) {
                    r1[i] += dg[n] * xt[i];
                    r3[i] += du[n] * xt[i];
                }
            }
            for (int m = 0; m < H; ++m) {
                double* r2 = dw2 + ((size_t)e * H + m) * F;
                const double dom = c.round_inter ? bf16r(dO[m]) : dO[m];
                for (int n = 0; n < F; ++n) r2[n] += dom * h[n];
            }
            if (want_abs) {
                double sa = 0.0;
                for (int n = 0; n < F; ++n) sa += fabs(dh[n]) * fabs(h[n]);
                dwabs[a] = (w[a] > 0.0) ? sa / w[a] : 0.0;
                double* xr = dxabs + (size_t)a * H;
                for (int i = 0; i < H; ++i) {
                    double acc = 0.0;
                    for (int n = 0; n < F; ++n)
                        acc += fabs(w1[((size_t)e * F + n) * H + i] * dg[n]) +
                               fabs(w3[((size_t)e * F + n) * H + i] * du[n]);
                    xr[i] = acc;
                }
                for (int n = 0; n < F; ++n) {
                    double* r1 = dw1_abs + ((size_t)e * F + n) * H;
                    double* r3 = dw3_abs + ((size_t)e * F + n) * H;
                    for (int i = 0; i < H; ++i) {
                        r1[i] += fabs(dg[n] * xt[i]);
                        r3[i] += fabs(du[n] * xt[i]);
                    }
                }
                for (int m = 0; m < H; ++m) {
                    double* r2 = dw2_abs + ((size_t)e * H + m) * F;
                    const double dom = fabs(c.round_inter ? bf16r(dO[m]) : dO[m]);
                    for (int n = 0; n < F; ++n) r2[n] += dom * fabs(h[n]);
                }
            }
        }
        free(g); free(u); free(h); free(dh); free(dg); free(du); free(o); free(dO);
    }
    for (int t = 0; t < T; ++t) {
        for (int i = 0; i < H; ++i) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j) acc += dxa[((size_t)t * k + j) * H + i];
            dx[(size_t)t * H + i] = acc;
        }
        double sw = 0.0;
        for (int j = 0; j < k; ++j) sw += w[(size_t)t * k + j] * dwa[(size_t)t * k + j];
        for (int e = 0; e < E; ++e) dlogits[(size_t)t * E + e] = 0.0;
        for (int j = 0; j < k; ++j) {
            size_t a = (size_t)t * k + j;
            dlogits[(size_t)t * E + ids[a]] = w[a] * (dwa[a] - sw);
        }
        if (want_abs) {
            for (int i = 0; i < H; ++i) {
                double acc = 0.0;
                for (int j = 0; j < k; ++j) acc += dxabs[((size_t)t * k + j) * H + i];
                dx_abs[(size_t)t * H + i] = acc;
            }
            double swa = 0.0;
            for (int j = 0; j < k; ++j) swa += w[(size_t)t * k + j] * dwabs[(size_t)t * k + j];
            for (int e = 0; e < E; ++e) dl_abs[(size_t)t * E + e] = 0.0;
            for (int j = 0; j < k; ++j) {
                size_t a = (size_t)t * k + j;
                dl_abs[(size_t)t * E + ids[a]] = w[a] * (dwabs[a] + swa);
            }
        }
    }
    if (dwa_out) memcpy(dwa_out, dwa, sizeof(double) * A);
    free(ids); free(w); free(dwa); free(dxa); free(dwabs); free(dxabs);
    return 0;
}

/* Sampled gradients, for sizes where the full form takes too long: dx and
 * dlogits of the listed tokens ([ntok,H], [ntok,E]); for each listed pair
 * (e, n) of feats [nfeat,2], row n of dW1_e and of dW3_e and column n of
 * dW2_e ([nfeat,H] each).  Same arithmetic and order as the full form; the
 * error scales (optional, all or none) in arrays of the same shapes. */
int oracle_moe_ffn_bwd64_sampled(const double* x, const double* logits, const double* w1, const double* w3,
                                 const double* w2, const double* dy, int T, int H, int F, int E, int k,
                                 int round, const int32_t* tokens, int ntok, double* dx_s, double* dl_s,
                                 const int32_t* feats, int nfeat, double* dw1_s, double* dw3_s, double* dw2_s,
                                 double* dx_abs, double* dl_abs, double* dw1_abs, double* dw3_abs, double* dw2_abs,
                                 int nthreads) {
    bctx c;
    if (bctx_init(&c, x, w1, w3, w2, T, H, F, E, k, round)) return -1;
    for (int i = 0; i < ntok; ++i)
        if (tokens[i] < 0 || tokens[i] >= T) return -1;
    for (int i = 0; i < nfeat; ++i)
        if (feats[2 * i] < 0 || feats[2 * i] >= E || feats[2 * i + 1] < 0 || feats[2 * i + 1] >= F) return -1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
    long A = (long)T * k;
    int32_t* ids = malloc(sizeof(int32_t) * (A ? A : 1));
    double* w = malloc(sizeof(double) * (A ? A : 1));
    for (int t = 0; t < T; ++t) topk64(logits + (size_t)t * E, E, k, ids + (size_t)t * k, w + (size_t)t * k);
    #pragma omp parallel for schedule(dynamic, 1)
    for (int q = 0; q < ntok; ++q) {
        int t = tokens[q];
        const double* dyt = dy + (size_t)t * H;
        double *g = malloc(sizeof(double) * F), *u = malloc(sizeof(double) * F), *h = malloc(sizeof(double) * F);
        double *dh = malloc(sizeof(double) * F), *dg = malloc(sizeof(double) * F), *du = malloc(sizeof(double) * F);
        double *o = malloc(sizeof(double) * H), *dO = malloc(sizeof(double) * H);
        double* dxa = calloc((size_t)k * H, sizeof(double));
        double* dxab = calloc((size_t)k * H, sizeof(double));
        double dwa[64], dwab[64];
        for (int j = 0; j < k; ++j) {
            size_t a = (size_t)t * k + j;
            int e = ids[a];
            fwd_assign(&c, e, t, g, u, h, o);
            double s = 0.0;
            for (int m = 0; m < H; ++m) s += dyt[m] * o[m];
            dwa[j] = s;
            for (int m = 0; m < H; ++m) dO[m] = w[a] * dyt[m];
            for (int n = 0; n < F; ++n) {
                double acc = 0.0;
                for (int m = 0; m < H; ++m) acc += w2[((size_t)e * H + m) * F + n] * dO[m];
                dh[n] = acc;
            }
            swiglu_bwd(F, g, u, dh, dg, du, c.round_inter);
            for (int i = 0; i < H; ++i) {
                double acc = 0.0;
                for (int n = 0; n < F; ++n)
                    acc += w1[((size_t)e * F + n) * H + i] * dg[n] + w3[((size_t)e * F + n) * H + i] * du[n];
                dxa[(size_t)j * H + i] = acc;
            }
            if (dx_abs) {
                double sa = 0.0;
                for (int n = 0; n < F; ++n) sa += fabs(dh[n]) * fabs(h[n]);
                dwab[j] = (w[a] > 0.0) ? sa / w[a] : 0.0;
                for (int i = 0; i < H; ++i) {
                    double acc = 0.0;
                    for (int n = 0; n < F; ++n)
                        acc += fabs(w1[((size_t)e * F + n) * H + i] * dg[n]) +
                               fabs(w3[((size_t)e * F + n) * H + i] * du[n]);
                    dxab[(size_t)j * H + i] = acc;
                }
            }
        }
        for (int i = 0; i < H; ++i) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j) acc += dxa[(size_t)j * H + i];
            dx_s[(size_t)q * H + i] = acc;
        }
        double sw = 0.0;
        for (int j = 0; j < k; ++j) sw += w[(size_t)t * k + j] * dwa[j];
        for (int e = 0; e < E; ++e) dl_s[(size_t)q * E + e] = 0.0;
        for (int j = 0; j < k; ++j) {
            size_t a = (size_t)t * k + j;
            dl_s[(size_t)q * E + ids[a]] = w[a] * (dwa[j] - sw);
        }
        if (dx_abs) {
            for (int i = 0; i < H; ++i) {
                double acc = 0.0;
                for (int j = 0; j < k; ++j) acc += dxab[(size_t)j * H + i];
                dx_abs[(size_t)q * H + i] = acc;
            }
            double swa = 0.0;
            for (int j = 0; j < k; ++j) swa += w[(size_t)t * k + j] * dwab[j];
            for (int e = 0; e < E; ++e) dl_abs[(size_t)q * E + e] = 0.0;
            for (int j = 0; j < k; ++j) {
                size_t a = (size_t)t * k + j;
                dl_abs[(size_t)q * E + ids[a]] = w[a] * (dwab[j] + swa);
            }
        }
        free(g); free(u); free(h); free(dh); free(dg); free(du); free(o); free(dO); free(dxa); free(dxab);
    }
    #pragma omp parallel for schedule(dynamic, 1)
    for (int q = 0; q < nfeat; ++q) {
        int e = feats[2 * q], n = feats[2 * q + 1];
        double* r1 = dw1_s + (size_t)q * H;
        double* r3 = dw3_s + (size_t)q * H;
        double* c2 = dw2_s + (size_t)q * H;
        for (int i = 0; i < H; ++i) r1[i] = r3[i] = c2[i] = 0.0;
        double* a1 = dw1_abs ? dw1_abs + (size_t)q * H : NULL;
        double* a3 = dw1_abs ? dw3_abs + (size_t)q * H : NULL;
        double* a2 = dw1_abs ? dw2_abs + (size_t)q * H : NULL;
        if (a1)
            for (int i = 0; i < H; ++i) a1[i] = a3[i] = a2[i] = 0.0;
        const double* w1r = w1 + ((size_t)e * F + n) * H;
        const double* w3r = w3 + ((size_t)e * F + n) * H;
        for (long a = 0; a < A; ++a) {
            if (ids[a] != e) continue;
            int t = (int)(a / k);
            const double* xt = x + (size_t)t * H;
            const double* dyt = dy + (size_t)t * H;
            double gv = 0.0, uv = 0.0;
            for (int i = 0; i < H; ++i) {
                gv += w1r[i] * xt[i];
                uv += w3r[i] * xt[i];
            }
            double hv = gv / (1.0 + exp(-gv)) * uv;
            if (c.round_h) hv = bf16r(hv);
            double dhv = 0.0;
            for (int m = 0; m < H; ++m) dhv += w2[((size_t)e * H + m) * F + n] * (w[a] * dyt[m]);
            double dgv, duv;
            swiglu_bwd(1, &gv, &uv, &dhv, &dgv, &duv, c.round_inter);
            for (int i = 0; i < H; ++i) {
                r1[i] += dgv * xt[i];
                r3[i] += duv * xt[i];
            }
            for (int m = 0; m < H; ++m) c2[m] += (c.round_inter ? bf16r(w[a] * dyt[m]) : w[a] * dyt[m]) * hv;
            if (a1) {
                for (int i = 0; i < H; ++i) {
                    a1[i] += fabs(dgv * xt[i]);
                    a3[i] += fabs(duv * xt[i]);
                }
                for (int m = 0; m < H; ++m)
                    a2[m] += fabs((c.round_inter ? bf16r(w[a] * dyt[m]) : w[a] * dyt[m]) * hv);
            }
        }
    }
    free(ids); free(w);
    return 0;
}
