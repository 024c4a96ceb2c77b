/*
 * oracle_driver.c -- runs every function of the CPU oracle (oracle/stepq_oracle.c) on seeded
 * random inputs, small shapes and edge cases, under AddressSanitizer, LeakSanitizer and
 * UndefinedBehaviorSanitizer.  Built and run by tests/test_sanitizers.py; exit status 0 means
 * no sanitizer report and every round trip held.  The numerical pins of the oracle live in
 * the Python tests; this driver looks for memory and undefined-behaviour faults.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

/* the oracle's entry points (definitions in oracle/stepq_oracle.c) */
int oracle_qmax(int bits);
long oracle_codes_bytes(int bits, int dk, int dv);
long oracle_block_bytes(int bits, int dk, int dv);
uint16_t oracle_fp16_from_double(double x);
double oracle_fp16_to_double(uint16_t h);
void oracle_pack_codes(int bits, int dk, int dv, const int32_t *Q, uint8_t *out);
void oracle_unpack_codes(int bits, int dk, int dv, const uint8_t *in, int32_t *Q);
void oracle_rows_order(int dk, const int32_t *rb, int32_t *order);
long oracle_rows_block_bytes(int dk, int dv, const int32_t *rb);
void oracle_rows_pack(int dk, int dv, const int32_t *rb, const int32_t *Q, uint8_t *out);
void oracle_rows_unpack(int dk, int dv, const int32_t *rb, const uint8_t *in, int32_t *Q);
int oracle_quantize(int bits, int dk, int dv, const float *S32, int32_t *Q, float *r, float *c);
int oracle_rows_quantize(int dk, int dv, const int32_t *rb, const float *S32, int32_t *Q, float *r, float *c);
void oracle_dequantize(int dk, int dv, const int32_t *Q, const float *r, const float *c, double *S);
void oracle_impact_normalize(int dk, const float *omega, float *w);
int oracle_quantize_impact(int bits, int dk, int dv, const float *S32, const float *w, int32_t *Q, float *r,
                           float *c);
long oracle_head_offsets(int H, const int32_t *head_bits, int dk, int dv, long *offsets, const int32_t *row_bits);
long oracle_decode_step(int H, int Hk, int dk, int dv, int gate_mode, const int32_t *head_bits, int num_slots,
                        uint8_t *pool, const int32_t *slot_ids, int n, const float *q, const float *k,
                        const float *v, const float *alpha, const float *beta, float *y, int nthreads,
                        const float *impact, const int32_t *row_bits);
long oracle_pool_load(int H, int dk, int dv, const int32_t *head_bits, int num_slots, uint8_t *pool,
                      const int32_t *slot_ids, int n, const float *S, int nthreads, const float *impact,
                      const int32_t *row_bits);
int oracle_pool_dump(int H, int dk, int dv, const int32_t *head_bits, int num_slots, const uint8_t *pool,
                     const int32_t *slot_ids, int n, float *S, int nthreads, const int32_t *row_bits);
void oracle_fp_decode_step(int H, int Hk, int dk, int dv, int gate_mode, int n, double *S, const float *q,
                           const float *k, const float *v, const float *alpha, const float *beta, float *y,
                           int round_fp32, int nthreads);

static int failures = 0;
#define CHECK(c)                                                                          \
    do {                                                                                  \
        if (!(c)) {                                                                       \
            ++failures;                                                                   \
            fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__, __LINE__, #c);         \
        }                                                                                 \
    } while (0)

static uint64_t rng_state = 0x9E3779B97F4A7C15ull;
static uint32_t rnd(void)
{
    rng_state ^= rng_state << 13;
    rng_state ^= rng_state >> 7;
    rng_state ^= rng_state << 17;
    return (uint32_t)(rng_state >> 11);
}
static double unif(void) { return (rnd() + 0.5) / 2097152.0 / 2048.0; }     /* (0, 1) */
static double gauss(void) { return sqrt(-2.0 * log(unif())) * cos(6.283185307179586 * unif()); }

static void test_codes(int dk, int dv)
{
    const int widths[3] = {4, 6, 8};
    int32_t *Q = malloc(sizeof(int32_t) * dk * dv), *Q2 = malloc(sizeof(int32_t) * dk * dv);
    for (int w = 0; w < 3; w++) {
        int b = widths[w], qm = oracle_qmax(b);
        uint8_t *buf = malloc((size_t)oracle_codes_bytes(b, dk, dv));
        for (int e = 0; e < dk * dv; e++) Q[e] = (int32_t)(rnd() % (2 * qm + 1)) - qm;
        oracle_pack_codes(b, dk, dv, Q, buf);
        oracle_unpack_codes(b, dk, dv, buf, Q2);
        CHECK(memcmp(Q, Q2, sizeof(int32_t) * dk * dv) == 0);
        free(buf);
    }
    /* per-key-row widths */
    int32_t *rb = malloc(sizeof(int32_t) * dk), *order = malloc(sizeof(int32_t) * dk);
    for (int i = 0; i < dk; i++) rb[i] = widths[rnd() % 3];
    for (int e = 0; e < dk * dv; e++) {
        int qm = oracle_qmax(rb[e / dv]);
        Q[e] = (int32_t)(rnd() % (2 * qm + 1)) - qm;
    }
    uint8_t *rbuf = calloc((size_t)oracle_rows_block_bytes(dk, dv, rb), 1);
    oracle_rows_pack(dk, dv, rb, Q, rbuf);
    oracle_rows_unpack(dk, dv, rb, rbuf, Q2);
    CHECK(memcmp(Q, Q2, sizeof(int32_t) * dk * dv) == 0);
    oracle_rows_order(dk, rb, order);
    free(rbuf); free(rb); free(order); free(Q); free(Q2);
}

static void test_fit(int dk, int dv)
{
    long ne = (long)dk * dv;
    float *S = malloc(sizeof(float) * ne), *r = malloc(4L * dk), *c = malloc(4L * dv), *w = malloc(4L * dk);
    float *om = malloc(4L * dk);
    int32_t *Q = malloc(sizeof(int32_t) * ne), *rb = malloc(sizeof(int32_t) * dk);
    double *D = malloc(sizeof(double) * ne);
    for (int trial = 0; trial < 4; trial++) {
        for (int i = 0; i < dk; i++) {
            double row = exp(gauss());
            for (int j = 0; j < dv; j++) S[i * dv + j] = (float)(row * gauss());
            om[i] = (float)exp(1.2 * gauss());
            rb[i] = 4 + 2 * (int)(rnd() % 3);
        }
        if (trial == 1) memset(S + dv, 0, sizeof(float) * dv);               /* a zero row */
        if (trial == 2) for (int i = 0; i < dk; i++) S[i * dv + 1] = 0.0f;   /* a zero column */
        if (trial == 3) for (int i = 0; i < dk; i++) S[i * dv + 2] = 1e-40f; /* subnormal column */
        for (int b = 4; b <= 8; b += 2) {
            CHECK(oracle_quantize(b, dk, dv, S, Q, r, c) == 0);
            oracle_dequantize(dk, dv, Q, r, c, D);
            oracle_impact_normalize(dk, om, w);
            (void)oracle_quantize_impact(b, dk, dv, S, w, Q, r, c);
        }
        CHECK(oracle_rows_quantize(dk, dv, rb, S, Q, r, c) == 0);
    }
    free(S); free(r); free(c); free(w); free(om); free(Q); free(rb); free(D);
}

static void test_fp16(void)
{
    const double special[8] = {0.0, -0.0, 65504.0, 65520.0, 1e-8, 5.960464477539063e-08, -2.9802322387695312e-08,
                               INFINITY};
    for (int k = 0; k < 8; k++) (void)oracle_fp16_from_double(special[k]);
    for (uint32_t h = 0; h < 65536; h++) {
        double x = oracle_fp16_to_double((uint16_t)h);
        if (x == x && (h & 0x7C00) != 0x7C00) CHECK(oracle_fp16_from_double(x) == (uint16_t)h || x == 0.0);
    }
}

/* a pool with every kind of head, GDN and KDA, through load, decode steps and dump */
static void test_pool(int gate_mode)
{
    const int dk = 128, dv = 128, H = 5, Hk = gate_mode ? 5 : 1, slots = 6, n = 4;
    int32_t bits[5] = {4, 6, 8, 16, 0};
    int32_t *row_bits = malloc(sizeof(int32_t) * H * dk);
    for (int e = 0; e < H * dk; e++) row_bits[e] = 4 + 2 * (int)(rnd() % 3);
    long offs[5];
    long stride = oracle_head_offsets(H, bits, dk, dv, offs, row_bits);
    uint8_t *pool = calloc((size_t)(stride * slots), 1);
    int32_t ids[4] = {5, 0, 3, 2};
    long ne = (long)dk * dv;
    float *S = malloc(sizeof(float) * n * H * ne), *S2 = malloc(sizeof(float) * n * H * ne);
    double *Sd = calloc((size_t)(n * H * ne), sizeof(double));
    float *q = malloc(4L * n * Hk * dk), *k = malloc(4L * n * Hk * dk), *v = malloc(4L * n * H * dv);
    float *al = malloc(4L * n * H * dk), *be = malloc(4L * n * H), *y = malloc(4L * n * H * dv);
    float *imp = malloc(4L * H * dk);
    for (int t = 0; t < 6; t++) {
        for (long e = 0; e < (long)n * Hk * dk; e++) { q[e] = (float)gauss() / 11.3f; k[e] = (float)gauss() / 11.3f; }
        for (long e = 0; e < (long)n * H * dv; e++) v[e] = (float)gauss();
        for (long e = 0; e < (long)n * H * dk; e++) al[e] = (float)(0.5 + 0.5 * unif());
        for (long e = 0; e < (long)n * H; e++) be[e] = (float)unif();
        oracle_fp_decode_step(H, Hk, dk, dv, gate_mode, n, Sd, q, k, v, al, be, y, 1, 1);
    }
    for (long e = 0; e < (long)n * H * ne; e++) S[e] = (float)Sd[e];
    for (long e = 0; e < (long)H * dk; e++) imp[e] = (float)(0.5 + unif());
    CHECK(oracle_pool_load(H, dk, dv, bits, slots, pool, ids, n, S, 1, NULL, row_bits) >= 0);
    CHECK(oracle_pool_dump(H, dk, dv, bits, slots, pool, ids, n, S2, 1, row_bits) == 0);
    for (int step = 0; step < 3; step++)
        CHECK(oracle_decode_step(H, Hk, dk, dv, gate_mode, bits, slots, pool, ids, n, q, k, v, al, be, y, 1,
                                 step == 1 ? imp : NULL, row_bits) >= 0);
    int32_t bad[2] = {1, 6};                              /* 6 is outside the pool: skipped, -1 */
    CHECK(oracle_decode_step(H, Hk, dk, dv, gate_mode, bits, slots, pool, bad, 2, q, k, v, al, be, y, 1, NULL,
                             row_bits) == -1);
    CHECK(oracle_pool_load(H, dk, dv, bits, slots, pool, ids, n, S, 1, imp, row_bits) >= 0);
    free(row_bits); free(pool); free(S); free(S2); free(Sd); free(q); free(k); free(v); free(al); free(be);
    free(y); free(imp);
}

int main(void)
{
    test_codes(128, 128);
    test_codes(16, 32);
    test_fit(128, 128);
    test_fit(16, 16);
    test_fp16();
    test_pool(0);
    test_pool(1);
    printf("oracle driver: %d failures\n", failures);
    return failures ? 1 : 0;
}
