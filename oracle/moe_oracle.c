/*
 * moe_oracle.c -- plain, slow CPU oracle of the FP8 x FP4 MoE expert layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline / reference leg load this library.  It shares no
 * code, header, table or helper with the CUDA library, and the CUDA library
 * never calls it.
 *
 * What it computes (the "Mega MoE" expert layer on one GPU, restated):
 *   route each token's k slots to experts; for every routed row (t, j, e)
 *     C1   = dequant(x[t]) . dequant(L1[e])^T        (fp32 accumulation)
 *     h    = silu(C1[0:I]) * C1[I:2I]                (SwiGLU, gate first)
 *     hq   = requantise h to FP8 E4M3 + UE8M0 per 32 (same rule as x)
 *     Y    = dequant(hq) . dequant(L2[e])^T          (fp32 accumulation)
 *   out[t] = bf16_rne( sum_j w[t,j] * Y(t,j) ),  j ascending, fp32 sum.
 * Sources: "Mega moe fusion with symmetric memory" (Procedure step 5, phases
 * 1-5; Key design points: FP8 activations, FP4 weights, fp32 accumulator);
 * MATE "Mega MoE" API (recipe=(1,1,32), swiglu default, bf16 output);
 * DeepGEMM PR #416 review thread (test body: gate = first chunk of L1's
 * output, activation applied to gate; per-token FP8 cast with UE8M0, gran 32).
 *
 * SiTU (the second activation of MATE's "Mega MoE" page, section Activations;
 * formula in the DeepGEMM PR #416 test body):
 *     h = sigmoid(g) * (beta * tanh(g / beta)) * (beta_lin * tanh(u / beta_lin))
 * with beta > 0 required and beta_lin optional; without beta_lin the up factor
 * is u itself (the beta_lin -> infinity limit) -- a reading, the pages only
 * say the coefficient is optional.
 *
 * Readings where the pages are silent or disagree (all listed in the design
 * notes): SwiGLU is silu(gate)*up (one page writes "gate x silu(up)"; the
 * review thread's test applies the nonlinearity to the gate chunk); the top-k
 * weight is applied at the combine, after GEMM2; a group whose amax is 0 gets
 * scale byte 127 and +-0 codes; the code's sign bit is the sign bit of the
 * scaled value; within an expert routed rows are in ascending t*k+j order;
 * out-of-range expert ids are dropped and counted.
 *
 * NVFP4 variant (the "NVFP4 Mega MoE Kernel -- Mojo Rewrite" README, sections
 * Key operations and NVFP4 specifics): activations, weights and the
 * intermediate h are all FP4 E2M1 with one UE4M3 scale per 16 consecutive K
 * elements.  The pages give no scale rule; the reading taken here mirrors the
 * MX one: s = the smallest UE4M3 value with 6 * s >= amax (so no code
 * saturates; amax = 0 gives s = 1), code = round-to-nearest-even onto the
 * E2M1 grid of the fp32 quotient v / s.  No per-tensor scale (none is named).
 *
 * Floating-point formats (OCP Microscaling Formats v1.0, the format the pages
 * name as FP8 E4M3 / FP4 E2M1 / UE8M0; UE4M3 = the E4M3 bit fields with the
 * sign bit 0): decoded from their bit fields.
 *
 * Every function is written for a reader checking it against the definition,
 * not for speed: no blocking, no SIMD, no reordering of the sums.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* ------------------------------------------------------------------ */
/* Format decoders                                                     */
/* ------------------------------------------------------------------ */

/* FP8 E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa bits; exponent field 0 is
 * subnormal (m/8 * 2^-6); S.1111.111 is NaN; there is no infinity. */
double oracle_e4m3_value(uint32_t code)
{
    code &= 0xFFu;
    int s = (int)(code >> 7);
    int e = (int)((code >> 3) & 0xFu);
    int m = (int)(code & 7u);
    double mag;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, -6);
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* FP4 E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; exponent field 0 is
 * subnormal (m/2 * 2^0).  Magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
double oracle_e2m1_value(uint32_t code)
{
    code &= 0xFu;
    int s = (int)(code >> 3);
    int e = (int)((code >> 1) & 3u);
    int m = (int)(code & 1u);
    double mag;
    if (e == 0)
        mag = 0.5 * (double)m;
    else
        mag = ldexp(1.0 + (double)m / 2.0, e - 1);
    return s ? -mag : mag;
}

/* UE8M0 scale byte b: 2^(b-127); 0xFF is NaN. */
double oracle_ue8m0_value(uint32_t b)
{
    b &= 0xFFu;
    if (b == 0xFFu)
        return NAN;
    return ldexp(1.0, (int)b - 127);
}

/* UE4M3: an E4M3 code with sign bit 0 (0x7F is NaN) */
double oracle_ue4m3_value(uint32_t b)
{
    return oracle_e4m3_value(b & 0x7Fu);
}

/* ------------------------------------------------------------------ */
/* Quantisation rule (per row, per 32 consecutive elements along K)    */
/* ------------------------------------------------------------------ */

/* Smallest integer e with amax <= qmax * 2^e, i.e. e = ceil(log2(amax/qmax)),
 * decided by exact comparisons (qmax * 2^e is exact in double).  amax == 0
 * gives e = 0.  The result is clamped so that the scale byte e + 127 stays in
 * [0, 254]. */
int oracle_scale_exponent(double amax, double qmax)
{
    int e;
    if (!(amax > 0.0))
        return 0;
    frexp(amax / qmax, &e); /* a first guess, corrected below */
    while (amax > qmax * ldexp(1.0, e))
        e++;
    while (amax <= qmax * ldexp(1.0, e - 1))
        e--;
    if (e < -127)
        e = -127;
    if (e > 127)
        e = 127;
    return e;
}

/* Round |v| <= 448 to the nearest E4M3 value, ties to the even code. */
uint32_t oracle_round_e4m3(double v)
{
    uint32_t sign = signbit(v) ? 0x80u : 0u;
    double a = fabs(v);
    uint32_t mag;
    if (a < ldexp(1.0, -6)) {
        /* subnormal binade: grid step 2^-9; n = 8 is the smallest normal */
        mag = (uint32_t)rint(a * 512.0);
    } else {
        int E;
        frexp(a, &E);            /* a in [2^(E-1), 2^E) */
        int ex = E - 1;          /* a in [2^ex, 2^(ex+1)) */
        double n = rint(ldexp(a, 3 - ex)); /* in [8, 16]; 16 carries into the exponent */
        mag = (uint32_t)((ex + 7) * 8) + (uint32_t)(n - 8.0);
    }
    return sign | mag;
}

/* Round |v| <= 6 to the nearest E2M1 value, ties to the even code. */
uint32_t oracle_round_e2m1(double v)
{
    uint32_t sign = signbit(v) ? 0x8u : 0u;
    double a = fabs(v);
    uint32_t mag;
    if (a < 1.0) {
        mag = (uint32_t)rint(a * 2.0);   /* 0, 0.5, 1.0 */
    } else {
        int E;
        frexp(a, &E);
        int ex = E - 1;                  /* 0, 1 or 2 */
        double n = rint(ldexp(a, 1 - ex)); /* in [2, 4] */
        mag = (uint32_t)((ex + 1) * 2) + (uint32_t)(n - 2.0);
    }
    return sign | mag;
}

/* Quantise one group of 32 values with format maximum qmax.  Writes the
 * scale byte and returns e; the caller rounds v * 2^-e per element. */
static int group_scale(const double *v, int n, double qmax, uint8_t *sf)
{
    double amax = 0.0;
    for (int i = 0; i < n; i++)
        if (fabs(v[i]) > amax)
            amax = fabs(v[i]);
    int e = oracle_scale_exponent(amax, qmax);
    *sf = (uint8_t)(e + 127);
    return e;
}

/* FP8 E4M3 + UE8M0 per 32 along each row.  src: [rows, cols] fp32,
 * codes: [rows, cols] u8, sf: [rows, cols/32] u8.  cols % 32 == 0. */
void oracle_quantize_e4m3(const float *src, int64_t rows, int64_t cols,
                          uint8_t *codes, uint8_t *sf)
{
    double v[32];
    for (int64_t r = 0; r < rows; r++)
        for (int64_t g = 0; g < cols / 32; g++) {
            for (int i = 0; i < 32; i++)
                v[i] = (double)src[r * cols + g * 32 + i];
            int e = group_scale(v, 32, 448.0, &sf[r * (cols / 32) + g]);
            for (int i = 0; i < 32; i++)
                codes[r * cols + g * 32 + i] = (uint8_t)oracle_round_e4m3(ldexp(v[i], -e));
        }
}

/* FP4 E2M1 + UE8M0 per 32 along each row.  src: [rows, cols] fp32,
 * packed: [rows, cols/2] u8 with element 2c in the low nibble of byte c,
 * sf: [rows, cols/32] u8.  cols % 32 == 0. */
void oracle_quantize_e2m1(const float *src, int64_t rows, int64_t cols,
                          uint8_t *packed, uint8_t *sf)
{
    double v[32];
    for (int64_t r = 0; r < rows; r++)
        for (int64_t g = 0; g < cols / 32; g++) {
            for (int i = 0; i < 32; i++)
                v[i] = (double)src[r * cols + g * 32 + i];
            int e = group_scale(v, 32, 6.0, &sf[r * (cols / 32) + g]);
            for (int i = 0; i < 32; i += 2) {
                uint32_t lo = oracle_round_e2m1(ldexp(v[i], -e));
                uint32_t hi = oracle_round_e2m1(ldexp(v[i + 1], -e));
                packed[r * (cols / 2) + (g * 32 + i) / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
}

/* fp32 -> bf16 bits, round to nearest even (NaN -> canonical quiet NaN). */
/* NVFP4 scale code of a 16-element group: the smallest UE4M3 value s with
 * 6 * s >= amax (6 * s is exact in double), scanning the codebook upward;
 * amax = 0 gives 1.0 (code 0x38); above 6 * 448 the largest finite code. */
uint32_t oracle_nvfp4_scale(double amax)
{
    if (!(amax > 0.0))
        return 0x38u;
    for (uint32_t c = 1; c < 0x7Fu; c++)
        if (6.0 * oracle_e4m3_value(c) >= amax)
            return c;
    return 0x7Eu;
}

/* FP4 E2M1 codes (two per byte, even column in the low nibble) and one UE4M3
 * scale byte per 16 consecutive columns; cols % 16 == 0. */
void oracle_quantize_nvfp4(const float *src, int64_t rows, int64_t cols,
                           uint8_t *q, uint8_t *sf)
{
    for (int64_t r = 0; r < rows; r++)
        for (int64_t g = 0; g < cols / 16; g++) {
            const float *v = src + r * cols + g * 16;
            double amax = 0.0;
            for (int i = 0; i < 16; i++)
                if (fabs((double)v[i]) > amax)
                    amax = fabs((double)v[i]);
            uint32_t c = oracle_nvfp4_scale(amax);
            float s = (float)oracle_e4m3_value(c);
            sf[r * (cols / 16) + g] = (uint8_t)c;
            for (int i = 0; i < 16; i += 2) {
                uint32_t lo = oracle_round_e2m1((double)(v[i] / s));
                uint32_t hi = oracle_round_e2m1((double)(v[i + 1] / s));
                q[(r * cols + g * 16 + i) / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
}

uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu))
        return 0x7FC0;
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------ */
/* Routing: per-expert histogram, exclusive scan, stable permutation   */
/* ------------------------------------------------------------------ */

/* topk_idx: [T, k] int64.  count: [E], offset: [E+1], perm: [T*k] (first
 * sum(count) entries valid; perm[r] = t*k+j), inv: [T*k] (inv[t*k+j] = r or -1
 * for an out-of-range id).  Routed rows of one expert are in ascending t*k+j
 * order (a stable counting sort).  Returns the number of dropped slots. */
int oracle_route(const int64_t *topk_idx, int T, int k, int E,
                 int32_t *count, int32_t *offset, int32_t *perm, int32_t *inv)
{
    int64_t n = (int64_t)T * k;
    int dropped = 0;
    int32_t *fill = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E > 0 ? E : 1));
    for (int e = 0; e < E; e++)
        count[e] = 0;
    for (int64_t s = 0; s < n; s++) {
        int64_t e = topk_idx[s];
        if (e < 0 || e >= E)
            dropped++;
        else
            count[e]++;
    }
    offset[0] = 0;
    for (int e = 0; e < E; e++)
        offset[e + 1] = offset[e] + count[e];
    for (int e = 0; e < E; e++)
        fill[e] = offset[e];
    for (int64_t s = 0; s < n; s++) {
        int64_t e = topk_idx[s];
        if (e < 0 || e >= E) {
            inv[s] = -1;
            continue;
        }
        int32_t r = fill[e]++;
        perm[r] = (int32_t)s;
        inv[s] = r;
    }
    free(fill);
    return dropped;
}

/* ------------------------------------------------------------------ */
/* The layer, one token at a time                                      */
/* ------------------------------------------------------------------ */

typedef struct {
    /* inputs */
    const uint8_t *x, *x_sf;          /* [T, H], [T, H/32] */
    const int64_t *topk_idx;          /* [T, k] */
    const float *topk_w;              /* [T, k] */
    const uint8_t *const *l1;         /* per expert [2I, H/2] (NULL if absent) */
    const uint8_t *const *l1_sf;      /* per expert [2I, H/32] */
    const uint8_t *const *l2;         /* per expert [H, I/2] */
    const uint8_t *const *l2_sf;      /* per expert [H, I/32] */
    int T, E, k, H, I;
    const int32_t *tokens;            /* which tokens to evaluate (NULL: all) */
    int ntok;
    int use_double;                   /* 0: fp32 accumulation (the method); 1: double */
    int activation;                   /* 0: SwiGLU, 1: SiTU */
    double beta, linear_beta;         /* SiTU coefficients; linear_beta <= 0: absent */
    int nv;                           /* 0: FP8 x FP4, UE8M0 / 32; 1: NVFP4 (FP4, UE4M3 / 16) */
    int gs;                           /* scale group: 32 or 16 */
    /* outputs, indexed by position p in the token list */
    uint16_t *out_bf16;               /* [ntok, H] */
    float *out_f32;                   /* [ntok, H]       (nullable) */
    float *h_pre;                     /* [ntok, k, I]    (nullable) SwiGLU before requant */
    uint8_t *h_q;                     /* [ntok, k, I] (NVFP4: [ntok, k, I/2]) (nullable) */
    uint8_t *h_sf;                    /* [ntok, k, I/gs] (nullable) */
    float *y;                         /* [ntok, k, H]    (nullable) GEMM2 output */
    /* decode tables, each filled once from the bit-field decoders above */
    double e4m3[256], e2m1[16], ue8m0[256], ue4m3[256];
    /* work distribution */
    int next;
    int missing_expert;
} job_t;

/* element (row, col) of a packed FP4 matrix with `cols` columns and one
 * scale byte per J->gs columns */
static double dq_w(const job_t *J, const uint8_t *w, const uint8_t *sf, int64_t row,
                   int cols, int col)
{
    uint8_t byte = w[row * (cols / 2) + col / 2];
    uint32_t nib = (col % 2 == 0) ? (byte & 0xFu) : (byte >> 4);
    uint8_t sb = sf[row * (cols / J->gs) + col / J->gs];
    return J->e2m1[nib] * (J->nv ? J->ue4m3[sb] : J->ue8m0[sb]);
}

static double dq_x(const job_t *J, int t, int kk)
{
    if (J->nv)  /* packed FP4 [T, H/2] with UE4M3 per 16 */
        return dq_w(J, J->x, J->x_sf, t, J->H, kk);
    return J->e4m3[J->x[(int64_t)t * J->H + kk]] *
           J->ue8m0[J->x_sf[(int64_t)t * (J->H / 32) + kk / 32]];
}

static void token_forward(job_t *J, int p, double *xd, double *c1, double *h,
                          double *hd, double *yrow, double *acc, float *c1f,
                          float *hf, float *yf, float *accf)
{
    const int H = J->H, I = J->I, k = J->k;
    const int t = J->tokens ? J->tokens[p] : p;
    uint8_t hq[32];
    const int gs = J->gs;

    for (int kk = 0; kk < H; kk++)
        xd[kk] = dq_x(J, t, kk);
    for (int c = 0; c < H; c++) {
        acc[c] = 0.0;
        accf[c] = 0.0f;
    }

    for (int j = 0; j < k; j++) {
        int64_t e = J->topk_idx[(int64_t)t * k + j];
        if (e < 0 || e >= J->E)
            continue; /* dropped slot: contributes nothing */
        const uint8_t *w1 = J->l1[e], *s1 = J->l1_sf[e], *w2 = J->l2[e], *s2 = J->l2_sf[e];
        if (!w1 || !s1 || !w2 || !s2) {
            __atomic_store_n(&J->missing_expert, 1, __ATOMIC_RELAXED);
            continue;
        }
        /* GEMM1: C1[n] = sum_kk xd[kk] * wd[n, kk], ascending kk */
        for (int n = 0; n < 2 * I; n++) {
            if (J->use_double) {
                double s = 0.0;
                for (int kk = 0; kk < H; kk++)
                    s += xd[kk] * dq_w(J, w1, s1, n, H, kk);
                c1[n] = s;
            } else {
                float s = 0.0f;
                for (int kk = 0; kk < H; kk++)
                    s += (float)xd[kk] * (float)dq_w(J, w1, s1, n, H, kk);
                c1f[n] = s;
            }
        }
        /* activation of gate = C1[i] and up = C1[I+i]:
         *   SwiGLU: h = silu(gate) * up
         *   SiTU:   h = sigmoid(gate) * (beta*tanh(gate/beta)) * (beta_lin*tanh(up/beta_lin)) */
        for (int i = 0; i < I; i++) {
            if (J->use_double) {
                double g = c1[i], u = c1[I + i];
                if (J->activation == 0) {
                    h[i] = g / (1.0 + exp(-g)) * u;
                } else {
                    double up = J->linear_beta > 0 ? J->linear_beta * tanh(u / J->linear_beta) : u;
                    h[i] = (1.0 / (1.0 + exp(-g))) * (J->beta * tanh(g / J->beta)) * up;
                }
            } else {
                float g = c1f[i], u = c1f[I + i];
                if (J->activation == 0) {
                    hf[i] = g / (1.0f + expf(-g)) * u;
                } else {
                    float bt = (float)J->beta, lb = (float)J->linear_beta;
                    float up = lb > 0 ? lb * tanhf(u / lb) : u;
                    hf[i] = (1.0f / (1.0f + expf(-g))) * (bt * tanhf(g / bt)) * up;
                }
                h[i] = (double)hf[i];
            }
        }
        if (J->h_pre)
            for (int i = 0; i < I; i++)
                J->h_pre[((int64_t)p * k + j) * I + i] = (float)h[i];
        /* requantise h (FP8 E4M3 + UE8M0 per 32, or NVFP4), then dequantise */
        for (int g = 0; g < I / gs; g++) {
            uint8_t sfb;
            if (!J->nv) {
                int ex = group_scale(&h[g * 32], 32, 448.0, &sfb);
                for (int i = 0; i < 32; i++) {
                    hq[i] = (uint8_t)oracle_round_e4m3(ldexp(h[g * 32 + i], -ex));
                    hd[g * 32 + i] = J->e4m3[hq[i]] * J->ue8m0[sfb];
                    if (J->h_q)
                        J->h_q[((int64_t)p * k + j) * I + g * 32 + i] = hq[i];
                }
            } else {
                double amax = 0.0;
                for (int i = 0; i < 16; i++)
                    if (fabs(h[g * 16 + i]) > amax)
                        amax = fabs(h[g * 16 + i]);
                sfb = (uint8_t)oracle_nvfp4_scale(amax);
                for (int i = 0; i < 16; i++) {
                    /* the fp32 quotient (fp32 mode); the double one in double mode */
                    double qv = J->use_double ? h[g * 16 + i] / J->ue4m3[sfb]
                                              : (double)((float)h[g * 16 + i] / (float)J->ue4m3[sfb]);
                    hq[i] = (uint8_t)oracle_round_e2m1(qv);
                    hd[g * 16 + i] = J->e2m1[hq[i]] * J->ue4m3[sfb];
                }
                if (J->h_q)
                    for (int i = 0; i < 16; i += 2)
                        J->h_q[((int64_t)p * k + j) * (I / 2) + (g * 16 + i) / 2] =
                            (uint8_t)(hq[i] | (hq[i + 1] << 4));
            }
            if (J->h_sf)
                J->h_sf[((int64_t)p * k + j) * (I / gs) + g] = sfb;
        }
        /* GEMM2: Y[c] = sum_i hd[i] * w2d[c, i], ascending i */
        for (int c = 0; c < H; c++) {
            if (J->use_double) {
                double s = 0.0;
                for (int i = 0; i < I; i++)
                    s += hd[i] * dq_w(J, w2, s2, c, I, i);
                yrow[c] = s;
            } else {
                float s = 0.0f;
                for (int i = 0; i < I; i++)
                    s += (float)hd[i] * (float)dq_w(J, w2, s2, c, I, i);
                yf[c] = s;
                yrow[c] = (double)s;
            }
        }
        if (J->y)
            for (int c = 0; c < H; c++)
                J->y[((int64_t)p * k + j) * H + c] = (float)yrow[c];
        /* combine: out += w[t, j] * Y, slots in ascending j */
        float wt = J->topk_w[(int64_t)t * k + j];
        for (int c = 0; c < H; c++) {
            if (J->use_double)
                acc[c] += (double)wt * yrow[c];
            else
                accf[c] += wt * yf[c];
        }
    }
    for (int c = 0; c < H; c++) {
        float o = J->use_double ? (float)acc[c] : accf[c];
        J->out_bf16[(int64_t)p * H + c] = oracle_f32_to_bf16(o);
        if (J->out_f32)
            J->out_f32[(int64_t)p * H + c] = o;
    }
}

static void *worker(void *arg)
{
    job_t *J = (job_t *)arg;
    const int H = J->H, I = J->I;
    double *xd = (double *)malloc(sizeof(double) * (size_t)H);
    double *c1 = (double *)malloc(sizeof(double) * (size_t)(2 * I));
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
    double *hd = (double *)malloc(sizeof(double) * (size_t)I);
    double *yrow = (double *)malloc(sizeof(double) * (size_t)H);
    double *acc = (double *)malloc(sizeof(double) * (size_t)H);
    float *c1f = (float *)malloc(sizeof(float) * (size_t)(2 * I));
    float *hf = (float *)malloc(sizeof(float) * (size_t)I);
    float *yf = (float *)malloc(sizeof(float) * (size_t)H);
    float *accf = (float *)malloc(sizeof(float) * (size_t)H);
    for (;;) {
        int p = __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED);
        if (p >= J->ntok)
            break;
        token_forward(J, p, xd, c1, h, hd, yrow, acc, c1f, hf, yf, accf);
    }
    free(xd); free(c1); free(h); free(hd); free(yrow); free(acc);
    free(c1f); free(hf); free(yf); free(accf);
    return NULL;
}

int oracle_num_threads(int requested)
{
    if (requested > 0)
        return requested;
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

/* Evaluates the layer for `ntok` tokens (tokens == NULL: tokens 0..ntok-1).
 * Expert weight pointers are per expert (length E arrays); an expert that a
 * listed token uses must be present.  Returns 0, or -1 if a needed expert was
 * missing, or -2 on a bad argument.  Each token is evaluated by one thread in
 * a fixed order, so the result does not depend on the thread count.
 * nvfp4 = 0: x is FP8 [T, H] with UE8M0 per 32 ([T, H/32]), weight scales
 * UE8M0 per 32.  nvfp4 = 1: x is packed FP4 [T, H/2] with UE4M3 per 16
 * ([T, H/16]), weight scales UE4M3 per 16, and h is requantised to NVFP4. */
int oracle_moe_forward_fmt(const uint8_t *x, const uint8_t *x_sf,
                           const int64_t *topk_idx, const float *topk_w,
                           const uint8_t *const *l1, const uint8_t *const *l1_sf,
                           const uint8_t *const *l2, const uint8_t *const *l2_sf,
                           int T, int E, int k, int H, int I,
                           const int32_t *tokens, int ntok, int use_double, int nthreads,
                           int activation, double beta, double linear_beta, int nvfp4,
                           uint16_t *out_bf16, float *out_f32, float *h_pre,
                           uint8_t *h_q, uint8_t *h_sf, float *y)
{
    if (H % 32 || I % 32 || H <= 0 || I <= 0 || k <= 0 || E <= 0 || T < 0 || ntok < 0)
        return -2;
    if (nvfp4 != 0 && nvfp4 != 1)
        return -2;
    if (activation != 0 && !(activation == 1 && beta > 0 && isfinite(beta) && isfinite(linear_beta)))
        return -2;
    if (tokens)
        for (int p = 0; p < ntok; p++)
            if (tokens[p] < 0 || tokens[p] >= T)
                return -2;
    job_t J;
    memset(&J, 0, sizeof(J));
    J.x = x; J.x_sf = x_sf; J.topk_idx = topk_idx; J.topk_w = topk_w;
    J.l1 = l1; J.l1_sf = l1_sf; J.l2 = l2; J.l2_sf = l2_sf;
    J.T = T; J.E = E; J.k = k; J.H = H; J.I = I;
    J.tokens = tokens; J.ntok = ntok; J.use_double = use_double;
    J.activation = activation; J.beta = beta; J.linear_beta = linear_beta;
    J.nv = nvfp4; J.gs = nvfp4 ? 16 : 32;
    J.out_bf16 = out_bf16; J.out_f32 = out_f32; J.h_pre = h_pre;
    J.h_q = h_q; J.h_sf = h_sf; J.y = y;
    for (int c = 0; c < 256; c++) {
        J.e4m3[c] = oracle_e4m3_value((uint32_t)c);
        J.ue8m0[c] = oracle_ue8m0_value((uint32_t)c);
        J.ue4m3[c] = oracle_ue4m3_value((uint32_t)c);
    }
    for (int c = 0; c < 16; c++)
        J.e2m1[c] = oracle_e2m1_value((uint32_t)c);
    int nt = oracle_num_threads(nthreads);
    if (nt > ntok)
        nt = ntok > 0 ? ntok : 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nt);
    for (int i = 0; i < nt; i++)
        pthread_create(&th[i], NULL, worker, &J);
    for (int i = 0; i < nt; i++)
        pthread_join(th[i], NULL);
    free(th);
    return J.missing_expert ? -1 : 0;
}

/* The FP8 x FP4 layer with a chosen activation (see oracle_moe_forward_fmt). */
int oracle_moe_forward_act(const uint8_t *x, const uint8_t *x_sf,
                           const int64_t *topk_idx, const float *topk_w,
                           const uint8_t *const *l1, const uint8_t *const *l1_sf,
                           const uint8_t *const *l2, const uint8_t *const *l2_sf,
                           int T, int E, int k, int H, int I,
                           const int32_t *tokens, int ntok, int use_double, int nthreads,
                           int activation, double beta, double linear_beta,
                           uint16_t *out_bf16, float *out_f32, float *h_pre,
                           uint8_t *h_q, uint8_t *h_sf, float *y)
{
    return oracle_moe_forward_fmt(x, x_sf, topk_idx, topk_w, l1, l1_sf, l2, l2_sf, T, E, k, H, I,
                                  tokens, ntok, use_double, nthreads, activation, beta, linear_beta, 0,
                                  out_bf16, out_f32, h_pre, h_q, h_sf, y);
}

/* The layer with SwiGLU (see oracle_moe_forward_act). */
int oracle_moe_forward(const uint8_t *x, const uint8_t *x_sf,
                       const int64_t *topk_idx, const float *topk_w,
                       const uint8_t *const *l1, const uint8_t *const *l1_sf,
                       const uint8_t *const *l2, const uint8_t *const *l2_sf,
                       int T, int E, int k, int H, int I,
                       const int32_t *tokens, int ntok, int use_double, int nthreads,
                       uint16_t *out_bf16, float *out_f32, float *h_pre,
                       uint8_t *h_q, uint8_t *h_sf, float *y)
{
    return oracle_moe_forward_act(x, x_sf, topk_idx, topk_w, l1, l1_sf, l2, l2_sf, T, E, k, H, I,
                                  tokens, ntok, use_double, nthreads, 0, 1.0, 0.0,
                                  out_bf16, out_f32, h_pre, h_q, h_sf, y);
}

/* ------------------------------------------------------------------ */
/* BF16 shared expert                                                  */
/* ------------------------------------------------------------------ */

/* The optional dense expert of DeepGEMM PR #416 (its BF16 shared-expert test
 * body defines it), run on every token beside the routed experts and written
 * to its own output.  With bf16 values x [T, SH], L1 [2 SI, SH] (gate rows
 * 0..SI-1, up rows SI..2 SI-1) and L2 [SH, SI]:
 *   gate, up = bf16_rne(x . L1^T)          (the linear layer's bf16 output)
 *   h        = bf16_rne(act(gate, up))     (SwiGLU or SiTU, as above)
 *   y        = bf16_rne(h . L2^T)
 * The dot products are exact sums in double, ascending k (the test body
 * leaves the accumulation to its bf16 linear layer; any order of a sum of
 * bf16 products rounds to the same bf16 value except near ties). */

static double bf16_value(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static double bf16_round(double v)
{
    return bf16_value(oracle_f32_to_bf16((float)v));
}

typedef struct {
    const uint16_t *x, *l1, *l2;
    int SH, SI, activation;
    double beta, linear_beta;
    const int32_t *tokens;
    int ntok;
    uint16_t *y;   /* [ntok, SH] */
    uint16_t *h;   /* [ntok, SI] or NULL */
    int next;
} shared_job_t;

static void shared_token(shared_job_t *J, int p, double *xd, double *hd)
{
    const int SH = J->SH, SI = J->SI;
    const int t = J->tokens ? J->tokens[p] : p;
    for (int kk = 0; kk < SH; kk++)
        xd[kk] = bf16_value(J->x[(int64_t)t * SH + kk]);
    for (int i = 0; i < SI; i++) {
        double g = 0.0, u = 0.0;
        for (int kk = 0; kk < SH; kk++) {
            g += xd[kk] * bf16_value(J->l1[(int64_t)i * SH + kk]);
            u += xd[kk] * bf16_value(J->l1[(int64_t)(SI + i) * SH + kk]);
        }
        g = bf16_round(g);
        u = bf16_round(u);
        double a;
        if (J->activation == 0) {
            a = g / (1.0 + exp(-g)) * u;
        } else {
            double up = J->linear_beta > 0 ? J->linear_beta * tanh(u / J->linear_beta) : u;
            a = (1.0 / (1.0 + exp(-g))) * (J->beta * tanh(g / J->beta)) * up;
        }
        hd[i] = bf16_round(a);
        if (J->h)
            J->h[(int64_t)p * SI + i] = oracle_f32_to_bf16((float)hd[i]);
    }
    for (int c = 0; c < SH; c++) {
        double s = 0.0;
        for (int i = 0; i < SI; i++)
            s += hd[i] * bf16_value(J->l2[(int64_t)c * SI + i]);
        J->y[(int64_t)p * SH + c] = oracle_f32_to_bf16((float)s);
    }
}

static void *shared_worker(void *arg)
{
    shared_job_t *J = (shared_job_t *)arg;
    double *xd = (double *)malloc(sizeof(double) * (size_t)J->SH);
    double *hd = (double *)malloc(sizeof(double) * (size_t)J->SI);
    for (;;) {
        int p = __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED);
        if (p >= J->ntok)
            break;
        shared_token(J, p, xd, hd);
    }
    free(xd);
    free(hd);
    return NULL;
}

/* The shared expert for `ntok` tokens (tokens == NULL: 0..ntok-1); all arrays
 * bf16 bit patterns.  activation 0: SwiGLU, 1: SiTU(beta, linear_beta; 0 =
 * none).  y: [ntok, SH]; h: [ntok, SI] (the rounded intermediate) or NULL.
 * Returns 0, or -2 on a bad argument.  One thread per token. */
int oracle_shared_forward(const uint16_t *x, const uint16_t *l1, const uint16_t *l2, int T, int SH, int SI,
                          const int32_t *tokens, int ntok, int nthreads, int activation, double beta,
                          double linear_beta, uint16_t *y, uint16_t *h)
{
    if (!x || !l1 || !l2 || !y || T < 0 || SH <= 0 || SI <= 0 || ntok < 0)
        return -2;
    if (activation == 1 && !(beta > 0))
        return -2;
    for (int p = 0; p < ntok; p++)
        if (tokens && (tokens[p] < 0 || tokens[p] >= T))
            return -2;
    shared_job_t J = {x, l1, l2, SH, SI, activation, beta, linear_beta, tokens, ntok, y, h, 0};
    int n = oracle_num_threads(nthreads);
    if (n > ntok)
        n = ntok > 0 ? ntok : 1;
    pthread_t th[256];
    if (n > 256)
        n = 256;
    for (int i = 0; i < n; i++)
        pthread_create(&th[i], NULL, shared_worker, &J);
    for (int i = 0; i < n; i++)
        pthread_join(th[i], NULL);
    return 0;
}
