/*
 * stepq_oracle.c -- CPU oracle of the quantized gated Delta-rule decode step (STEPQuant).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call
 * this file; only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark do.  It shares no code with the CUDA path.
 *
 * It is deliberately plain and slow: loops in the order the method states its
 * steps, all arithmetic in double precision, values that the method stores
 * (codes, row and column scales, the output y) rounded to their storage types.
 *
 * Sources (web pages on STEPQuant, arXiv 2609.38169), cited by title + section:
 *   [SUM]  hyper.ai paper summary "STEPQuant ..." -- sections "Method", "Key Contributions"
 *   [EXP]  "Paper Explained: STEPQuant -- When and Where Quantization Errors Matter
 *          in Delta-Rule Recurrent States" -- sections "The mechanism: rewriting state
 *          with the delta rule", "The intuition: errors get carried forward"
 *   [BLOG] ONTLE blog post on STEPQuant (blog.ontle.kr) -- paragraphs on the state pool,
 *          lifetime-aware bit allocation, dual-axis fitting and the fused kernel
 *
 * Readings taken where the pages are silent (the pages lost every equation):
 *   - step order: fade with the retention gate, then predict from the faded state,
 *     then write the difference, then read out from the updated state, then
 *     quantize for storage ([EXP] mechanism; [SUM] Method para 1);
 *   - dual-axis fit without clipping: c_j = sqrt(max_i |S_ij|),
 *     r_i = max_j (|S_ij| / c_j) / qmax, qmax = 2^(b-1) - 1 ([SUM] Method para 4,
 *     impact weights dropped);
 *   - symmetric uniform levels, nearest level with ties to even ([SUM] Method para 1, 4);
 *   - storage: codes as offset binary u = Q + 2^(b-1) in a little-endian bit
 *     stream of b-bit fields; element order is panel-major (16-column panels,
 *     each panel row-major); a head block is [codes | r fp32[d_k] | c fp32[d_v]];
 *     the pool is slot-major with heads in order inside a slot.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_PANEL 16

/* ------------------------------------------------------------------------- */
/* Sizes and layout                                                           */
/* ------------------------------------------------------------------------- */

int oracle_qmax(int bits) { return (1 << (bits - 1)) - 1; }

long oracle_codes_bytes(int bits, int dk, int dv) { return (long)dk * dv * bits / 8; }

long oracle_block_bytes(int bits, int dk, int dv)
{
    if (bits == 16) return 2L * dk * dv;               /* FP16 pivot head: the state, no scales */
    return oracle_codes_bytes(bits, dk, dv) + 4L * dk + 4L * dv;
}

/* ------------------------------------------------------------------------- */
/* FP16 pivot heads ([SUM] Method para 2: the highest-risk units are kept in   */
/* FP16 as sparse pivots)                                                      */
/* ------------------------------------------------------------------------- */
/* A head of width 16 stores its state as IEEE binary16 values, row-major, element (i, j)
 * at byte 2 (i d_v + j), little-endian, with no scales.  Reading: the step fades, writes
 * and reads out as for every head; the updated state is rounded to fp32 (the fp32 store
 * that precedes the fit of a quantized head) and then to binary16, nearest, ties to even. */

/* Nearest binary16 value of x (ties to even), as its bit pattern.  binary16: 1 sign bit,
 * 5 exponent bits (bias 15), 10 fraction bits; subnormals are multiples of 2^-24; the
 * largest finite value is 65504 and everything from 65520 (the halfway point to 2^16) up
 * rounds to infinity. */
uint16_t oracle_fp16_from_double(double x)
{
    if (isnan(x)) return 0x7E00;
    const uint16_t sign = signbit(x) ? 0x8000 : 0;
    const double a = fabs(x);
    if (a >= 65520.0) return sign | 0x7C00;
    if (a < 0x1p-14) {
        /* subnormal range: an integer multiple of 2^-24 (1024 of them is the smallest normal) */
        return sign | (uint16_t)nearbyint(a * 0x1p24);
    }
    int e;
    frexp(a, &e);
    e -= 1;                                           /* a in [2^e, 2^(e+1)), -14 <= e <= 15 */
    double m = nearbyint(ldexp(a, 10 - e));           /* 1024 .. 2048: 11 significant bits */
    if (m == 2048.0) {
        m = 1024.0;
        e += 1;
    }
    return sign | (uint16_t)((e + 15) << 10) | (uint16_t)(m - 1024.0);
}

double oracle_fp16_to_double(uint16_t h)
{
    const int e = (h >> 10) & 31, f = h & 1023;
    double v;
    if (e == 0) v = ldexp((double)f, -24);
    else if (e == 31) v = f ? NAN : INFINITY;
    else v = ldexp((double)(1024 + f), e - 25);
    return (h & 0x8000) ? -v : v;
}

void oracle_fp16_encode(long n, const double *x, uint16_t *out)
{
    for (long e = 0; e < n; e++) out[e] = oracle_fp16_from_double(x[e]);
}

void oracle_fp16_decode(long n, const uint16_t *in, double *out)
{
    for (long e = 0; e < n; e++) out[e] = oracle_fp16_to_double(in[e]);
}

static void read_pivot(const uint8_t *blk, long ne, double *S)
{
    for (long e = 0; e < ne; e++)
        S[e] = oracle_fp16_to_double((uint16_t)(blk[2 * e] | (blk[2 * e + 1] << 8)));
}

static void write_pivot(uint8_t *blk, long ne, const double *S)
{
    for (long e = 0; e < ne; e++) {
        const uint16_t h = oracle_fp16_from_double((double)(float)S[e]);
        blk[2 * e] = (uint8_t)(h & 0xFF);
        blk[2 * e + 1] = (uint8_t)(h >> 8);
    }
}

/* Position of element (i, j) in the code stream: panel-major, row-major inside a panel. */
static long stream_index(int i, int j, int dk)
{
    return (long)(j / ORACLE_PANEL) * dk * ORACLE_PANEL + (long)i * ORACLE_PANEL + (j % ORACLE_PANEL);
}

/* Write codes Q[dk*dv] (row-major, each in [-qmax, qmax]) as a bit stream; one bit at a time. */
void oracle_pack_codes(int bits, int dk, int dv, const int32_t *Q, uint8_t *out)
{
    long nbytes = oracle_codes_bytes(bits, dk, dv);
    memset(out, 0, (size_t)nbytes);
    for (int i = 0; i < dk; i++)
        for (int j = 0; j < dv; j++) {
            long n = stream_index(i, j, dk);
            uint32_t u = (uint32_t)(Q[(long)i * dv + j] + (1 << (bits - 1)));
            for (int b = 0; b < bits; b++) {
                long bit = n * bits + b;
                if ((u >> b) & 1u)
                    out[bit / 8] |= (uint8_t)(1u << (bit % 8));
            }
        }
}

/* Inverse of oracle_pack_codes. */
void oracle_unpack_codes(int bits, int dk, int dv, const uint8_t *in, int32_t *Q)
{
    for (int i = 0; i < dk; i++)
        for (int j = 0; j < dv; j++) {
            long n = stream_index(i, j, dk);
            uint32_t u = 0;
            for (int b = 0; b < bits; b++) {
                long bit = n * bits + b;
                u |= (uint32_t)((in[bit / 8] >> (bit % 8)) & 1u) << b;
            }
            Q[(long)i * dv + j] = (int32_t)u - (1 << (bits - 1));
        }
}

/* ------------------------------------------------------------------------- */
/* Per-key-row widths ([BLOG]: the allocation unit of Kimi's KDA is a single key */
/* row)                                                                        */
/* ------------------------------------------------------------------------- */
/* A head whose key rows carry their own widths rb[i] in {4, 6, 8}.  Readings (the pages
 * give no layout): the rows are stored grouped by width -- 8-bit rows, then 4-bit, then
 * 6-bit, each group in ascending key-row order -- so each width's segments stay aligned;
 * a panel (16 value columns) holds one segment of 16 codes per stored row (the row's
 * width, a little-endian bit stream of offset-binary fields), padded to a multiple of 16
 * bytes; the head block is the 8 panels, then r[d_k] in stored-row order, then c[d_v].
 * With every rb[i] = b this is exactly the uniform layout above. */

/* Stored position -> key row. */
void oracle_rows_order(int dk, const int32_t *rb, int32_t *order)
{
    const int widths[3] = {8, 4, 6};
    int p = 0;
    for (int w = 0; w < 3; w++)
        for (int i = 0; i < dk; i++)
            if (rb[i] == widths[w]) order[p++] = i;
}

long oracle_rows_panel_bytes(int dk, const int32_t *rb)
{
    long sum = 0;
    for (int i = 0; i < dk; i++) sum += 2L * rb[i];              /* 16 codes of rb[i] bits */
    return (sum + 15) / 16 * 16;
}

long oracle_rows_block_bytes(int dk, int dv, const int32_t *rb)
{
    return (long)(dv / ORACLE_PANEL) * oracle_rows_panel_bytes(dk, rb) + 4L * dk + 4L * dv;
}

/* Codes Q[dk*dv] (key-row-major) of a per-row head into its code region; one bit at a time. */
void oracle_rows_pack(int dk, int dv, const int32_t *rb, const int32_t *Q, uint8_t *out)
{
    int32_t *order = (int32_t *)malloc((size_t)dk * sizeof(int32_t));
    oracle_rows_order(dk, rb, order);
    const long panel = oracle_rows_panel_bytes(dk, rb);
    memset(out, 0, (size_t)((dv / ORACLE_PANEL) * panel));
    for (int pj = 0; pj < dv / ORACLE_PANEL; pj++) {
        long seg = pj * panel;                                   /* byte offset of the segment */
        for (int p = 0; p < dk; p++) {
            const int i = order[p], b = rb[i];
            for (int jj = 0; jj < ORACLE_PANEL; jj++) {
                uint32_t u = (uint32_t)(Q[(long)i * dv + pj * ORACLE_PANEL + jj] + (1 << (b - 1)));
                for (int t = 0; t < b; t++) {
                    long bit = seg * 8 + (long)jj * b + t;
                    if ((u >> t) & 1u) out[bit / 8] |= (uint8_t)(1u << (bit % 8));
                }
            }
            seg += 2L * b;
        }
    }
    free(order);
}

void oracle_rows_unpack(int dk, int dv, const int32_t *rb, const uint8_t *in, int32_t *Q)
{
    int32_t *order = (int32_t *)malloc((size_t)dk * sizeof(int32_t));
    oracle_rows_order(dk, rb, order);
    const long panel = oracle_rows_panel_bytes(dk, rb);
    for (int pj = 0; pj < dv / ORACLE_PANEL; pj++) {
        long seg = pj * panel;
        for (int p = 0; p < dk; p++) {
            const int i = order[p], b = rb[i];
            for (int jj = 0; jj < ORACLE_PANEL; jj++) {
                uint32_t u = 0;
                for (int t = 0; t < b; t++) {
                    long bit = seg * 8 + (long)jj * b + t;
                    u |= (uint32_t)((in[bit / 8] >> (bit % 8)) & 1u) << t;
                }
                Q[(long)i * dv + pj * ORACLE_PANEL + jj] = (int32_t)u - (1 << (b - 1));
            }
            seg += 2L * b;
        }
    }
    free(order);
}

/* ------------------------------------------------------------------------- */
/* Quantization: dual-axis fit + nearest level ([SUM] Method para 4)          */
/* ------------------------------------------------------------------------- */

/* Fit the scales of an fp32 state and quantize it.  Returns the number of codes
 * that would have fallen outside [-qmax, qmax] (0 for a clip-free fit). */
int oracle_quantize(int bits, int dk, int dv, const float *S32, int32_t *Q, float *r, float *c)
{
    const int qmax = oracle_qmax(bits);
    int clipped = 0;
    /* column scales: c_j = sqrt(max_i |S_ij|) */
    for (int j = 0; j < dv; j++) {
        double M = 0.0;
        for (int i = 0; i < dk; i++) {
            double a = fabs((double)S32[(long)i * dv + j]);
            if (a > M) M = a;
        }
        c[j] = (float)sqrt(M);
    }
    /* row factors: r_i = max_j (|S_ij| / c_j) / qmax, over columns with c_j > 0 */
    for (int i = 0; i < dk; i++) {
        double m = 0.0;
        for (int j = 0; j < dv; j++) {
            if (c[j] > 0.0f) {
                double t = fabs((double)S32[(long)i * dv + j]) / (double)c[j];
                if (t > m) m = t;
            }
        }
        r[i] = (float)(m / (double)qmax);
    }
    /* codes: nearest level, ties to even; rows or columns with zero scale get 0 */
    for (int i = 0; i < dk; i++)
        for (int j = 0; j < dv; j++) {
            double scale = (double)r[i] * (double)c[j];
            double x = scale > 0.0 ? (double)S32[(long)i * dv + j] / scale : 0.0;
            double qv = nearbyint(x);
            if (qv > qmax) { qv = qmax; clipped++; }
            if (qv < -qmax) { qv = -qmax; clipped++; }
            Q[(long)i * dv + j] = (int32_t)qv;
        }
    return clipped;
}

/* The clip-free fit with each key row's own width: c_j = sqrt(max_i |S_ij|),
 * r_i = max_j (|S_ij| / c_j) / qmax(rb[i]), codes at the row's levels. */
int oracle_rows_quantize(int dk, int dv, const int32_t *rb, const float *S32, int32_t *Q, float *r, float *c)
{
    int clipped = 0;
    for (int j = 0; j < dv; j++) {
        double M = 0.0;
        for (int i = 0; i < dk; i++) {
            double a = fabs((double)S32[(long)i * dv + j]);
            if (a > M) M = a;
        }
        c[j] = (float)sqrt(M);
    }
    for (int i = 0; i < dk; i++) {
        const int qmax = oracle_qmax(rb[i]);
        double m = 0.0;
        for (int j = 0; j < dv; j++)
            if (c[j] > 0.0f) {
                double t = fabs((double)S32[(long)i * dv + j]) / (double)c[j];
                if (t > m) m = t;
            }
        r[i] = (float)(m / (double)qmax);
        for (int j = 0; j < dv; j++) {
            double scale = (double)r[i] * (double)c[j];
            double x = scale > 0.0 ? (double)S32[(long)i * dv + j] / scale : 0.0;
            double qv = nearbyint(x);
            if (qv > qmax) { qv = qmax; clipped++; }
            if (qv < -qmax) { qv = -qmax; clipped++; }
            Q[(long)i * dv + j] = (int32_t)qv;
        }
    }
    return clipped;
}

/* S_hat_ij = Q_ij * r_i * c_j (exact in double: <= 8-bit int times two fp32 values). */
void oracle_dequantize(int dk, int dv, const int32_t *Q, const float *r, const float *c, double *S)
{
    for (int i = 0; i < dk; i++)
        for (int j = 0; j < dv; j++)
            S[(long)i * dv + j] = (double)Q[(long)i * dv + j] * (double)r[i] * (double)c[j];
}

/* ------------------------------------------------------------------------- */
/* Key-row-aware dual-axis fit with row-impact scores ([SUM] Method para 4;    */
/* [BLOG] offline vs per-step work)                                           */
/* ------------------------------------------------------------------------- */
/* Readings (the formulas did not survive): the row factor weighs the row's current
 * magnitude against its impact with square-root scaling (a wider range for larger rows,
 * finer resolution for higher-impact rows); the column scales are then fitted by the
 * impact-weighted least-squares error, starting from the clip-free column scales of
 * those rows; every entry goes to the nearest level.  One refit: from (c0, Q0) to
 * c1 = the weighted least-squares scale of the codes Q0, then Q = the nearest levels
 * under c1 (clipped to +-qmax).  Each half step can only lower the weighted error. */

/* Row-impact weights normalized to mean 1: w_i = fp32(omega_i / mean(omega)), in double. */
void oracle_impact_normalize(int dk, const float *omega, float *w)
{
    double sum = 0.0;
    for (int i = 0; i < dk; i++) sum += (double)omega[i];
    for (int i = 0; i < dk; i++) w[i] = (float)((double)omega[i] / (sum / dk));
}

/* Fit and quantize an fp32 state with normalized row-impact weights w (all > 0):
 *   m_i  = max_j |S_ij|;   r_i = fp32(sqrt(m_i / w_i))
 *   c0_j = fp32(max_{i: r_i > 0} (|S_ij| / r_i) / qmax)
 *   Q0   = nearest level of S / (r c0)
 *   c1_j = fp32(sum_i w_i r_i Q0_ij S_ij / sum_i w_i r_i^2 Q0_ij^2), or c0_j when either
 *          sum is not positive
 *   Q    = nearest level of S / (r c1), clipped to [-qmax, qmax]
 * Returns the number of codes the final clip moved. */
int oracle_quantize_impact(int bits, int dk, int dv, const float *S32, const float *w, int32_t *Q, float *r, float *c)
{
    const int qmax = oracle_qmax(bits);
    int clipped = 0;
    for (int i = 0; i < dk; i++) {
        double m = 0.0;
        for (int j = 0; j < dv; j++) {
            double a = fabs((double)S32[(long)i * dv + j]);
            if (a > m) m = a;
        }
        r[i] = (float)sqrt(m / (double)w[i]);
    }
    for (int j = 0; j < dv; j++) {
        double mx = 0.0;
        for (int i = 0; i < dk; i++)
            if (r[i] > 0.0f) {
                double t = fabs((double)S32[(long)i * dv + j]) / (double)r[i];
                if (t > mx) mx = t;
            }
        const float c0 = (float)(mx / (double)qmax);
        double num = 0.0, den = 0.0;
        for (int i = 0; i < dk; i++) {
            double scale = (double)r[i] * (double)c0;
            double q0 = scale > 0.0 ? nearbyint((double)S32[(long)i * dv + j] / scale) : 0.0;
            if (q0 > qmax) q0 = qmax;
            if (q0 < -qmax) q0 = -qmax;
            num += (double)w[i] * (double)r[i] * q0 * (double)S32[(long)i * dv + j];
            den += (double)w[i] * (double)r[i] * (double)r[i] * q0 * q0;
        }
        c[j] = (num > 0.0 && den > 0.0) ? (float)(num / den) : c0;
        for (int i = 0; i < dk; i++) {
            double scale = (double)r[i] * (double)c[j];
            double qv = scale > 0.0 ? nearbyint((double)S32[(long)i * dv + j] / scale) : 0.0;
            if (qv > qmax) { qv = qmax; clipped++; }
            if (qv < -qmax) { qv = -qmax; clipped++; }
            Q[(long)i * dv + j] = (int32_t)qv;
        }
    }
    return clipped;
}

/* ------------------------------------------------------------------------- */
/* Gated Delta-rule step ([EXP] mechanism)                                    */
/* ------------------------------------------------------------------------- */

/* One unquantized step on a double state S[dk*dv], in place:
 *   fade      S'_ij = alpha_i * S_ij                (GDN: all alpha_i equal; KDA: one per key channel)
 *   predict   u_j   = sum_i S'_ij k_i               (what the key currently retrieves)
 *   write     d_j   = beta * (v_j - u_j);  S_ij = S'_ij + k_i d_j
 *   read      y_j   = sum_i S_ij q_i                (from the updated state)
 * y may be NULL. */
void oracle_delta_step(int dk, int dv, double *S, const float *q, const float *k, const float *v,
                       const float *alpha, float beta, double *y)
{
    double *u = (double *)calloc((size_t)dv, sizeof(double));
    for (int i = 0; i < dk; i++)
        for (int j = 0; j < dv; j++)
            S[(long)i * dv + j] = (double)alpha[i] * S[(long)i * dv + j];
    for (int j = 0; j < dv; j++) {
        double s = 0.0;
        for (int i = 0; i < dk; i++)
            s += S[(long)i * dv + j] * (double)k[i];
        u[j] = s;
    }
    for (int j = 0; j < dv; j++) {
        double d = (double)beta * ((double)v[j] - u[j]);
        for (int i = 0; i < dk; i++)
            S[(long)i * dv + j] += (double)k[i] * d;
    }
    if (y)
        for (int j = 0; j < dv; j++) {
            double s = 0.0;
            for (int i = 0; i < dk; i++)
                s += S[(long)i * dv + j] * (double)q[i];
            y[j] = s;
        }
    free(u);
}

/* One quantized decode step of one state ([SUM] Method para 1 and 4; [BLOG] per-step refit):
 * dequantize -> delta step -> readout -> round the state to fp32 -> fit -> quantize.
 * S_pre (optional, [dk*dv]) receives the updated state before quantization (double).
 * Returns the clip count of the fit (0 expected). */
static int step_state_fit(int dk, int dv, int bits, const int32_t *Q_in, const float *r_in, const float *c_in,
                          const float *q, const float *k, const float *v, const float *alpha, float beta,
                          int32_t *Q_out, float *r_out, float *c_out, float *y_out, double *S_pre,
                          const float *impact);

int oracle_step_state(int dk, int dv, int bits, const int32_t *Q_in, const float *r_in, const float *c_in,
                      const float *q, const float *k, const float *v, const float *alpha, float beta,
                      int32_t *Q_out, float *r_out, float *c_out, float *y_out, double *S_pre)
{
    return step_state_fit(dk, dv, bits, Q_in, r_in, c_in, q, k, v, alpha, beta, Q_out, r_out, c_out, y_out,
                          S_pre, NULL);
}

/* The same step with the impact-weighted fit (normalized weights w[dk]); returns the number
 * of codes its final clip moved (legitimate for this fit). */
int oracle_step_state_impact(int dk, int dv, int bits, const int32_t *Q_in, const float *r_in, const float *c_in,
                             const float *q, const float *k, const float *v, const float *alpha, float beta,
                             const float *w, int32_t *Q_out, float *r_out, float *c_out, float *y_out)
{
    return step_state_fit(dk, dv, bits, Q_in, r_in, c_in, q, k, v, alpha, beta, Q_out, r_out, c_out, y_out,
                          NULL, w);
}

/* The same step for a head with per-key-row widths rb[dk]: the clip-free fit at each row's
 * levels.  Returns the clip count (0 when the fit holds). */
int oracle_step_state_rows(int dk, int dv, const int32_t *rb, const int32_t *Q_in, const float *r_in,
                           const float *c_in, const float *q, const float *k, const float *v, const float *alpha,
                           float beta, int32_t *Q_out, float *r_out, float *c_out, float *y_out)
{
    long ne = (long)dk * dv;
    double *S = (double *)malloc((size_t)ne * sizeof(double));
    double *y = (double *)malloc((size_t)dv * sizeof(double));
    float *S32 = (float *)malloc((size_t)ne * sizeof(float));
    oracle_dequantize(dk, dv, Q_in, r_in, c_in, S);
    oracle_delta_step(dk, dv, S, q, k, v, alpha, beta, y);
    for (int j = 0; j < dv; j++) y_out[j] = (float)y[j];
    for (long e = 0; e < ne; e++) S32[e] = (float)S[e];
    int clipped = oracle_rows_quantize(dk, dv, rb, S32, Q_out, r_out, c_out);
    free(S); free(y); free(S32);
    return clipped;
}

static int step_state_fit(int dk, int dv, int bits, const int32_t *Q_in, const float *r_in, const float *c_in,
                          const float *q, const float *k, const float *v, const float *alpha, float beta,
                          int32_t *Q_out, float *r_out, float *c_out, float *y_out, double *S_pre,
                          const float *impact)
{
    long ne = (long)dk * dv;
    double *S = (double *)malloc((size_t)ne * sizeof(double));
    double *y = (double *)malloc((size_t)dv * sizeof(double));
    float *S32 = (float *)malloc((size_t)ne * sizeof(float));
    oracle_dequantize(dk, dv, Q_in, r_in, c_in, S);
    oracle_delta_step(dk, dv, S, q, k, v, alpha, beta, y);
    for (int j = 0; j < dv; j++) y_out[j] = (float)y[j];
    if (S_pre) memcpy(S_pre, S, (size_t)ne * sizeof(double));
    for (long e = 0; e < ne; e++) S32[e] = (float)S[e];
    int clipped = impact ? oracle_quantize_impact(bits, dk, dv, S32, impact, Q_out, r_out, c_out)
                         : oracle_quantize(bits, dk, dv, S32, Q_out, r_out, c_out);
    free(S); free(y); free(S32);
    return clipped;
}

/* ------------------------------------------------------------------------- */
/* Pool-level drivers (slot-major pool of packed head blocks)                 */
/* ------------------------------------------------------------------------- */

/* Byte offset of each head block inside a slot, and the slot stride.  A head of width 0
 * has per-key-row widths row_bits[h * dk .. h * dk + dk) (row_bits may be NULL otherwise). */
long oracle_head_offsets(int H, const int32_t *head_bits, int dk, int dv, long *offsets, const int32_t *row_bits)
{
    long off = 0;
    for (int h = 0; h < H; h++) {
        offsets[h] = off;
        off += head_bits[h] ? oracle_block_bytes(head_bits[h], dk, dv)
                            : oracle_rows_block_bytes(dk, dv, row_bits + (long)h * dk);
    }
    return off;
}

/* Read one head block into codes + scales (r by key row).  rb: the per-row widths of a
 * head of width 0, else NULL. */
static void read_block(const uint8_t *blk, int bits, const int32_t *rb, int dk, int dv, int32_t *Q, float *r,
                       float *c)
{
    if (rb) {
        const long cb = (long)(dv / ORACLE_PANEL) * oracle_rows_panel_bytes(dk, rb);
        int32_t *order = (int32_t *)malloc((size_t)dk * sizeof(int32_t));
        oracle_rows_order(dk, rb, order);
        oracle_rows_unpack(dk, dv, rb, blk, Q);
        for (int p = 0; p < dk; p++) memcpy(&r[order[p]], blk + cb + 4L * p, 4);
        memcpy(c, blk + cb + 4L * dk, 4L * dv);
        free(order);
        return;
    }
    long cb = oracle_codes_bytes(bits, dk, dv);
    oracle_unpack_codes(bits, dk, dv, blk, Q);
    memcpy(r, blk + cb, 4L * dk);
    memcpy(c, blk + cb + 4L * dk, 4L * dv);
}

static void write_block(uint8_t *blk, int bits, const int32_t *rb, int dk, int dv, const int32_t *Q, const float *r,
                        const float *c)
{
    if (rb) {
        const long cb = (long)(dv / ORACLE_PANEL) * oracle_rows_panel_bytes(dk, rb);
        int32_t *order = (int32_t *)malloc((size_t)dk * sizeof(int32_t));
        oracle_rows_order(dk, rb, order);
        oracle_rows_pack(dk, dv, rb, Q, blk);
        for (int p = 0; p < dk; p++) memcpy(blk + cb + 4L * p, &r[order[p]], 4);
        memcpy(blk + cb + 4L * dk, c, 4L * dv);
        free(order);
        return;
    }
    long cb = oracle_codes_bytes(bits, dk, dv);
    oracle_pack_codes(bits, dk, dv, Q, blk);
    memcpy(blk + cb, r, 4L * dk);
    memcpy(blk + cb + 4L * dk, c, 4L * dv);
}

/* One decode step for n requests over all H value heads of a pool.
 *   pool      [num_slots * slot_stride] bytes, updated in place
 *   slot_ids  [n]
 *   q, k      [n, Hk, dk]; v [n, H, dv]; beta [n, H]
 *   alpha     gate_mode 0 (GDN): [n, H];  gate_mode 1 (KDA): [n, H, dk]
 *   y         [n, H, dv] (fp32 out)
 *   impact    NULL (clip-free fit) or [H, dk] normalized row-impact weights (impact fit of
 *             the uniform-width heads)
 *   row_bits  [H, dk] per-key-row widths of the heads of width 0 (NULL if there are none)
 * Value head h reads key head h / (H / Hk).  Returns the clip count of the clip-free fit
 * (0 when it holds), or -1 for an out-of-range slot id (that request is skipped). */
long oracle_decode_step(int H, int Hk, int dk, int dv, int gate_mode, const int32_t *head_bits,
                        int num_slots, uint8_t *pool, const int32_t *slot_ids, int n,
                        const float *q, const float *k, const float *v, const float *alpha,
                        const float *beta, float *y, int nthreads, const float *impact,
                        const int32_t *row_bits)
{
    long *offsets = (long *)malloc((size_t)H * sizeof(long));
    long stride = oracle_head_offsets(H, head_bits, dk, dv, offsets, row_bits);
    long clipped = 0;
    int bad = 0;
    int group = H / Hk;
    long items = (long)n * H;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(+ : clipped) reduction(| : bad)
    for (long it = 0; it < items; it++) {
        int b = (int)(it / H), h = (int)(it % H);
        int slot = slot_ids[b];
        if (slot < 0 || slot >= num_slots) { bad |= 1; continue; }
        int bits = head_bits[h];
        int g = h / group;
        long ne = (long)dk * dv;
        if (bits == 16) {
            double *S = (double *)malloc((size_t)ne * sizeof(double));
            double *yd = (double *)malloc((size_t)dv * sizeof(double));
            float *alp = (float *)malloc(4L * dk);
            uint8_t *pblk = pool + (long)slot * stride + offsets[h];
            for (int i = 0; i < dk; i++)
                alp[i] = gate_mode == 0 ? alpha[(long)b * H + h] : alpha[((long)b * H + h) * dk + i];
            read_pivot(pblk, ne, S);
            oracle_delta_step(dk, dv, S, q + ((long)b * Hk + g) * dk, k + ((long)b * Hk + g) * dk,
                              v + ((long)b * H + h) * dv, alp, beta[(long)b * H + h], yd);
            for (int j = 0; j < dv; j++) y[((long)b * H + h) * dv + j] = (float)yd[j];
            write_pivot(pblk, ne, S);
            free(S); free(yd); free(alp);
            continue;
        }
        int32_t *Q = (int32_t *)malloc((size_t)ne * sizeof(int32_t));
        int32_t *Q2 = (int32_t *)malloc((size_t)ne * sizeof(int32_t));
        float *r = (float *)malloc(4L * dk), *c = (float *)malloc(4L * dv);
        float *r2 = (float *)malloc(4L * dk), *c2 = (float *)malloc(4L * dv);
        float *al = (float *)malloc(4L * dk);
        uint8_t *blk = pool + (long)slot * stride + offsets[h];
        const int32_t *rb = bits ? NULL : row_bits + (long)h * dk;
        read_block(blk, bits, rb, dk, dv, Q, r, c);
        for (int i = 0; i < dk; i++)
            al[i] = gate_mode == 0 ? alpha[(long)b * H + h] : alpha[((long)b * H + h) * dk + i];
        if (rb)
            clipped += oracle_step_state_rows(dk, dv, rb, Q, r, c, q + ((long)b * Hk + g) * dk,
                                              k + ((long)b * Hk + g) * dk, v + ((long)b * H + h) * dv, al,
                                              beta[(long)b * H + h], Q2, r2, c2, y + ((long)b * H + h) * dv);
        else if (impact)
            (void)oracle_step_state_impact(dk, dv, bits, Q, r, c, q + ((long)b * Hk + g) * dk,
                                           k + ((long)b * Hk + g) * dk, v + ((long)b * H + h) * dv, al,
                                           beta[(long)b * H + h], impact + (long)h * dk, Q2, r2, c2,
                                           y + ((long)b * H + h) * dv);
        else
            clipped += oracle_step_state(dk, dv, bits, Q, r, c,
                                         q + ((long)b * Hk + g) * dk, k + ((long)b * Hk + g) * dk,
                                         v + ((long)b * H + h) * dv, al, beta[(long)b * H + h],
                                         Q2, r2, c2, y + ((long)b * H + h) * dv, NULL);
        write_block(blk, bits, rb, dk, dv, Q2, r2, c2);
        free(Q); free(Q2); free(r); free(c); free(r2); free(c2); free(al);
    }
    free(offsets);
    return bad ? -1 : clipped;
}

/* Quantize fp32 states S [n, H, dk, dv] into the slots slot_ids[n] of a pool (impact,
 * row_bits: as for oracle_decode_step). */
long oracle_pool_load(int H, int dk, int dv, const int32_t *head_bits, int num_slots, uint8_t *pool,
                      const int32_t *slot_ids, int n, const float *S, int nthreads, const float *impact,
                      const int32_t *row_bits)
{
    long *offsets = (long *)malloc((size_t)H * sizeof(long));
    long stride = oracle_head_offsets(H, head_bits, dk, dv, offsets, row_bits);
    long clipped = 0;
    int bad = 0;
    long items = (long)n * H;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(+ : clipped) reduction(| : bad)
    for (long it = 0; it < items; it++) {
        int b = (int)(it / H), h = (int)(it % H);
        int slot = slot_ids[b];
        if (slot < 0 || slot >= num_slots) { bad |= 1; continue; }
        long ne = (long)dk * dv;
        if (head_bits[h] == 16) {
            double *Sd = (double *)malloc((size_t)ne * sizeof(double));
            for (long e = 0; e < ne; e++) Sd[e] = (double)S[it * ne + e];
            write_pivot(pool + (long)slot * stride + offsets[h], ne, Sd);
            free(Sd);
            continue;
        }
        int32_t *Q = (int32_t *)malloc((size_t)ne * sizeof(int32_t));
        float *r = (float *)malloc(4L * dk), *c = (float *)malloc(4L * dv);
        const int32_t *rb = head_bits[h] ? NULL : row_bits + (long)h * dk;
        if (rb)
            clipped += oracle_rows_quantize(dk, dv, rb, S + it * ne, Q, r, c);
        else if (impact)
            (void)oracle_quantize_impact(head_bits[h], dk, dv, S + it * ne, impact + (long)h * dk, Q, r, c);
        else
            clipped += oracle_quantize(head_bits[h], dk, dv, S + it * ne, Q, r, c);
        write_block(pool + (long)slot * stride + offsets[h], head_bits[h], rb, dk, dv, Q, r, c);
        free(Q); free(r); free(c);
    }
    free(offsets);
    return bad ? -1 : clipped;
}

/* Dequantize the slots slot_ids[n] of a pool into S [n, H, dk, dv] (fp32). */
int oracle_pool_dump(int H, int dk, int dv, const int32_t *head_bits, int num_slots, const uint8_t *pool,
                     const int32_t *slot_ids, int n, float *S, int nthreads, const int32_t *row_bits)
{
    long *offsets = (long *)malloc((size_t)H * sizeof(long));
    long stride = oracle_head_offsets(H, head_bits, dk, dv, offsets, row_bits);
    int bad = 0;
    long items = (long)n * H;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(| : bad)
    for (long it = 0; it < items; it++) {
        int b = (int)(it / H), h = (int)(it % H);
        int slot = slot_ids[b];
        if (slot < 0 || slot >= num_slots) { bad |= 1; continue; }
        long ne = (long)dk * dv;
        if (head_bits[h] == 16) {
            double *Sp = (double *)malloc((size_t)ne * sizeof(double));
            read_pivot(pool + (long)slot * stride + offsets[h], ne, Sp);
            for (long e = 0; e < ne; e++) S[it * ne + e] = (float)Sp[e];
            free(Sp);
            continue;
        }
        int32_t *Q = (int32_t *)malloc((size_t)ne * sizeof(int32_t));
        float *r = (float *)malloc(4L * dk), *c = (float *)malloc(4L * dv);
        double *Sd = (double *)malloc((size_t)ne * sizeof(double));
        read_block(pool + (long)slot * stride + offsets[h], head_bits[h],
                   head_bits[h] ? NULL : row_bits + (long)h * dk, dk, dv, Q, r, c);
        oracle_dequantize(dk, dv, Q, r, c, Sd);
        for (long e = 0; e < ne; e++) S[it * ne + e] = (float)Sd[e];
        free(Q); free(r); free(c); free(Sd);
    }
    free(offsets);
    return bad ? -1 : 0;
}

/* One unquantized ("FP32-state") step for a batch of double states S [n, H, dk, dv]
 * (state index = request b, value head h; no pool, no slots).  When round_fp32 != 0
 * the state is rounded to fp32 after the step (an fp32-stored state, as in a
 * warm-up); otherwise it stays exact double (used for the error recursion). */
void oracle_fp_decode_step(int H, int Hk, int dk, int dv, int gate_mode, int n, double *S,
                           const float *q, const float *k, const float *v, const float *alpha,
                           const float *beta, float *y, int round_fp32, int nthreads)
{
    int group = H / Hk;
    long items = (long)n * H;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (long it = 0; it < items; it++) {
        int b = (int)(it / H), h = (int)(it % H);
        int g = h / group;
        long ne = (long)dk * dv;
        double *Sb = S + it * ne;
        float *al = (float *)malloc(4L * dk);
        double *yd = (double *)malloc(8L * dv);
        for (int i = 0; i < dk; i++)
            al[i] = gate_mode == 0 ? alpha[(long)b * H + h] : alpha[((long)b * H + h) * dk + i];
        oracle_delta_step(dk, dv, Sb, q + ((long)b * Hk + g) * dk, k + ((long)b * Hk + g) * dk,
                          v + ((long)b * H + h) * dv, al, beta[(long)b * H + h], yd);
        if (y)
            for (int j = 0; j < dv; j++) y[it * dv + j] = (float)yd[j];
        if (round_fp32)
            for (long e = 0; e < ne; e++) Sb[e] = (double)(float)Sb[e];
        free(al); free(yd);
    }
}
