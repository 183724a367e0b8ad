/*
 * moe_oracle.c -- plain CPU oracle of the routed MoE layer forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg load this library.  It shares no code, header,
 * table or helper with the CUDA path; both sides are handed the same seeded
 * input buffers and nothing else.
 *
 * What it computes (vLLM fused-MoE page, section 02 "what the fused MoE kernel
 * computes": a router picks the top-k of E experts for every token, each chosen
 * expert is a gate/up/down FFN with SwiGLU, and the top-k outputs are summed
 * with the gating weights; Weave review section 1.2 and the stepwise-vs-fused
 * comparison page section 2 give the same route -> dispatch -> expert FFN ->
 * combine data path):
 *
 *   l[t,e]  = sum_h x[t,h] * Wr[h,e]  (+ bias[e])           router logits
 *   S_t     = the k experts with the largest l[t,.], listed by descending
 *             logit, equal logits ordered by ascending expert index
 *   g[t,j]  = exp(l[t,S_j]) / sum_{i<k} exp(l[t,S_i])        softmax over the top-k
 *   out[t]  = sum_j g[t,j] * Wd_e ( silu(Wg_e x_t) * (Wu_e x_t) ),  e = S_j
 *   silu(a) = a / (1 + exp(-a))
 *
 * Readings taken where the pages are silent (each is listed in the design notes):
 *  - the router logit is an fp32 value with a fixed evaluation order: a chain of
 *    fused multiply-adds over h ascending starting from 0, the bias added last
 *    in fp32.  Routing is an integer decision made on that fp32 value, so both
 *    sides take it in the same precision.
 *  - ties in the top-k go to the lower expert index.
 *  - gates and the expert FFN are evaluated in fp64 from the bf16 inputs; no
 *    intermediate is rounded.
 *  - the permutation into expert groups is a stable counting sort of the flat
 *    assignment list (flat = t*k + j) by expert; group offsets carry no padding.
 *
 * FP8 block-scaled variant (GC-MoE page: block-scaled FP8/FP4 MMA with SwiGLU
 * and requantisation fused; vLLM fused-MoE page, section 03: fp8 weights with
 * [128,128] blocks): weights come as e4m3 codes with one fp32 scale per
 * 128x128 block; activations (x, and h after SwiGLU) are quantised per row per
 * 128-column group with s = amax/448 (fp32) and q = e4m3 round-to-nearest-even
 * of clamp(v/s, -448, 448) (fp32 division); amax = 0 gives s = 1, q = 0.  Each
 * GEMM is sum over 128-wide K blocks of sa[row,kb] * sb[nblk,kb] * (qa . qb)_kb,
 * evaluated in fp64 from the exact decoded codes.
 *
 * MX variant (GC-MoE page: FP8/FP4 block-scaled MMA on Blackwell; the element
 * and scale formats are those of the OCP Microscaling Formats spec v1.0): weights
 * as e2m1 codes and activations (x, and h after SwiGLU) as e4m3 codes, each with
 * one power-of-two e8m0 scale per 32 values along K; every GEMM is a sum over
 * 32-wide K blocks of 2^(Xa + Xb) * (codes . codes) in fp64 (oracle_combine_ffn_mx).
 *
 * Shared expert (GC-MoE page: "optional shared experts" fused into the expert
 * kernel, not defined there): one more SwiGLU FFN that every token passes through
 * with weight 1, added to the routed sum (oracle_shared_ffn; the caller adds).
 *
 * Deliberately slow and direct: no blocking, no fusion, no reordering.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- scalars */

static float bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static double bf16_to_f64(uint16_t b) { return (double)bf16_to_f32(b); }

static double silu(double a) { return a / (1.0 + exp(-a)); }

/* ------------------------------------------------------------ the router */

/* Router logits for one token: fp32 fused multiply-add chain over h ascending,
 * then + bias[e] in fp32.  Also returns the fp64 value of the same sum (for the
 * routing-margin diagnostics and the pins), when logit64 is not NULL. */
static void router_logits_token(int H, int E, const uint16_t *xt, const uint16_t *wr,
                                const float *bias, float *logit32, double *logit64)
{
    for (int e = 0; e < E; ++e) {
        float acc = 0.0f;
        double acc64 = 0.0;
        for (int h = 0; h < H; ++h) {
            float a = bf16_to_f32(xt[h]);
            float w = bf16_to_f32(wr[(size_t)h * E + e]);
            acc = fmaf(a, w, acc);
            acc64 += (double)a * (double)w;
        }
        if (bias) {
            acc = acc + bias[e];
            acc64 += (double)bias[e];
        }
        logit32[e] = acc;
        if (logit64) logit64[e] = acc64;
    }
}

/* Top-k by repeated arg-max: strictly larger wins, so among equal logits the
 * lower expert index is taken first. */
static void topk_token(int E, int k, const float *l, int32_t *idx, unsigned char *taken)
{
    memset(taken, 0, (size_t)E);
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (taken[e]) continue;
            if (best < 0 || l[e] > l[best]) best = e;
        }
        taken[best] = 1;
        idx[j] = best;
    }
}

/* Softmax over the k selected logits, in fp64. */
static void gates_token(int k, const float *l, const int32_t *idx, double *g)
{
    double m = (double)l[idx[0]];
    for (int j = 1; j < k; ++j)
        if ((double)l[idx[j]] > m) m = (double)l[idx[j]];
    double s = 0.0;
    for (int j = 0; j < k; ++j) s += exp((double)l[idx[j]] - m);
    for (int j = 0; j < k; ++j) g[j] = exp((double)l[idx[j]] - m) / s;
}

typedef struct {
    int T, H, E, k;
    const uint16_t *x, *wr;
    const float *bias;
    int32_t *idx;
    double *gate;
    float *logits32;
    double *logits64;
    int t0, t1;
} route_job;

static void *route_worker(void *p)
{
    route_job *j = (route_job *)p;
    float *l = (float *)malloc(sizeof(float) * (size_t)j->E);
    unsigned char *taken = (unsigned char *)malloc((size_t)j->E);
    for (int t = j->t0; t < j->t1; ++t) {
        double *l64 = j->logits64 ? j->logits64 + (size_t)t * j->E : NULL;
        router_logits_token(j->H, j->E, j->x + (size_t)t * j->H, j->wr, j->bias, l, l64);
        if (j->logits32) memcpy(j->logits32 + (size_t)t * j->E, l, sizeof(float) * (size_t)j->E);
        topk_token(j->E, j->k, l, j->idx + (size_t)t * j->k, taken);
        gates_token(j->k, l, j->idx + (size_t)t * j->k, j->gate + (size_t)t * j->k);
    }
    free(l);
    free(taken);
    return NULL;
}

/* Router + softmax top-k for all T tokens.
 *   x [T,H] bf16, wr [H,E] bf16, bias [E] fp32 or NULL
 *   -> idx [T,k] int32, gate [T,k] fp64, optional logits32 / logits64 [T,E]. */
int oracle_route(int T, int H, int E, int k, const uint16_t *x, const uint16_t *wr,
                 const float *bias, int32_t *idx, double *gate, float *logits32,
                 double *logits64, int nthreads)
{
    if (T < 0 || H <= 0 || E <= 0 || k < 1 || k > E) return 1;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > T) nthreads = T > 0 ? T : 1;
    pthread_t th[256];
    route_job jobs[256];
    if (nthreads > 256) nthreads = 256;
    for (int i = 0; i < nthreads; ++i) {
        route_job j = {T, H, E, k, x, wr, bias, idx, gate, logits32, logits64,
                       (int)((long)T * i / nthreads), (int)((long)T * (i + 1) / nthreads)};
        jobs[i] = j;
    }
    for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, route_worker, &jobs[i]);
    route_worker(&jobs[0]);
    for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
    return 0;
}

/* --------------------------------------------------------------- permute */

/* Stable counting sort of the flat assignment list by expert.
 *   idx [A] (A = T*k, flat = t*k + j)
 *   -> offsets [E+1], sorted_to_flat [A], flat_to_sorted [A]
 *   -> tile_list [3*n] of {expert, row_start, rows}: for e ascending, the
 *      row blocks of bm rows covering each group, and *num_tiles = n.
 * tile_list may be NULL (then only *num_tiles is produced). */
int oracle_permute(int A, int E, const int32_t *idx, int32_t *offsets, int32_t *sorted_to_flat,
                   int32_t *flat_to_sorted, int bm, int32_t *tile_list, int32_t *num_tiles)
{
    if (A < 0 || E <= 0 || bm <= 0) return 1;
    for (int f = 0; f < A; ++f)
        if (idx[f] < 0 || idx[f] >= E) return 2;
    int pos = 0;
    for (int e = 0; e < E; ++e) {
        offsets[e] = pos;
        for (int f = 0; f < A; ++f) {
            if (idx[f] == e) {
                sorted_to_flat[pos] = f;
                flat_to_sorted[f] = pos;
                ++pos;
            }
        }
    }
    offsets[E] = pos;
    int n = 0;
    for (int e = 0; e < E; ++e) {
        int c = offsets[e + 1] - offsets[e];
        for (int r = 0; r < c; r += bm) {
            if (tile_list) {
                tile_list[3 * n + 0] = e;
                tile_list[3 * n + 1] = offsets[e] + r;
                tile_list[3 * n + 2] = (c - r) < bm ? (c - r) : bm;
            }
            ++n;
        }
    }
    *num_tiles = n;
    return 0;
}

/* ----------------------------------------------------------- expert FFN */

/* One expert applied to one token, in fp64:
 *   y = Wd_e ( silu(Wg_e x) * (Wu_e x) )
 * wg, wu: [E,I,H] bf16; wd: [E,H,I] bf16; a: scratch [I]. */
static void expert_ffn(int H, int I, int e, const double *x, const uint16_t *wg,
                       const uint16_t *wu, const uint16_t *wd, double *a, double *y)
{
    const uint16_t *g = wg + (size_t)e * I * H;
    const uint16_t *u = wu + (size_t)e * I * H;
    const uint16_t *d = wd + (size_t)e * H * I;
    for (int i = 0; i < I; ++i) {
        double sg = 0.0, su = 0.0;
        for (int h = 0; h < H; ++h) {
            sg += bf16_to_f64(g[(size_t)i * H + h]) * x[h];
            su += bf16_to_f64(u[(size_t)i * H + h]) * x[h];
        }
        a[i] = silu(sg) * su;
    }
    for (int o = 0; o < H; ++o) {
        double s = 0.0;
        for (int i = 0; i < I; ++i) s += bf16_to_f64(d[(size_t)o * I + i]) * a[i];
        y[o] = s;
    }
}

typedef struct {
    int H, I, k;
    const uint16_t *x, *wg, *wu, *wd;
    const int32_t *idx;
    const double *gate;
    const int32_t *tokens;
    double *out;
    int n0, n1;
} ffn_job;

static void *ffn_worker(void *p)
{
    ffn_job *j = (ffn_job *)p;
    double *xt = (double *)malloc(sizeof(double) * (size_t)j->H);
    double *a = (double *)malloc(sizeof(double) * (size_t)j->I);
    double *y = (double *)malloc(sizeof(double) * (size_t)j->H);
    for (int n = j->n0; n < j->n1; ++n) {
        int t = j->tokens ? j->tokens[n] : n;
        for (int h = 0; h < j->H; ++h) xt[h] = bf16_to_f64(j->x[(size_t)t * j->H + h]);
        double *o = j->out + (size_t)n * j->H;
        for (int h = 0; h < j->H; ++h) o[h] = 0.0;
        for (int q = 0; q < j->k; ++q) {
            int e = j->idx[(size_t)t * j->k + q];
            double g = j->gate[(size_t)t * j->k + q];
            expert_ffn(j->H, j->I, e, xt, j->wg, j->wu, j->wd, a, y);
            for (int h = 0; h < j->H; ++h) o[h] += g * y[h];
        }
    }
    free(xt);
    free(a);
    free(y);
    return NULL;
}

/* Gate-weighted sum of the selected experts' FFN outputs, per token, in fp64.
 *   idx/gate: [T,k] routing (from oracle_route); tokens: the n token ids to
 *   evaluate (NULL = tokens 0..n-1)  ->  out [n,H] fp64. */
int oracle_combine_ffn(int H, int I, int k, const uint16_t *x, const int32_t *idx,
                       const double *gate, const uint16_t *wg, const uint16_t *wu,
                       const uint16_t *wd, int n, const int32_t *tokens, double *out,
                       int nthreads)
{
    if (H <= 0 || I <= 0 || k < 1 || n < 0) return 1;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > n) nthreads = n > 0 ? n : 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    ffn_job jobs[256];
    for (int i = 0; i < nthreads; ++i) {
        ffn_job j = {H, I, k, x, wg, wu, wd, idx, gate, tokens, out,
                     (int)((long)n * i / nthreads), (int)((long)n * (i + 1) / nthreads)};
        jobs[i] = j;
    }
    for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, ffn_worker, &jobs[i]);
    ffn_worker(&jobs[0]);
    for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
    return 0;
}

/* ---------------------------------------------------------- shared expert */

typedef struct {
    int H, I;
    const uint16_t *x, *wg, *wu, *wd;
    const int32_t *tokens;
    double *out;
    int n0, n1;
} shared_job;

static void *shared_worker(void *p)
{
    shared_job *j = (shared_job *)p;
    double *xt = (double *)malloc(sizeof(double) * (size_t)j->H);
    double *a = (double *)malloc(sizeof(double) * (size_t)j->I);
    for (int n = j->n0; n < j->n1; ++n) {
        int t = j->tokens ? j->tokens[n] : n;
        for (int h = 0; h < j->H; ++h) xt[h] = bf16_to_f64(j->x[(size_t)t * j->H + h]);
        expert_ffn(j->H, j->I, 0, xt, j->wg, j->wu, j->wd, a, j->out + (size_t)n * j->H);
    }
    free(xt);
    free(a);
    return NULL;
}

/* A shared expert: one gate/up/down SwiGLU FFN that every token passes through with
 * weight 1, its output added to the gate-weighted sum of the routed experts (the
 * GC-MoE page fuses "optional shared experts" into its expert kernel without
 * defining them; this is the plainest reading).  The caller adds the two:
 *   out[n] = oracle_combine_ffn(...)[n] + this[n].
 *   wg, wu: [I,H] bf16; wd: [H,I] bf16; tokens as in oracle_combine_ffn
 *   ->  out [n,H] fp64 (overwritten). */
int oracle_shared_ffn(int H, int I, const uint16_t *x, const uint16_t *wg, const uint16_t *wu,
                      const uint16_t *wd, int n, const int32_t *tokens, double *out, int nthreads)
{
    if (H <= 0 || I <= 0 || n < 0) return 1;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > n) nthreads = n > 0 ? n : 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    shared_job jobs[256];
    for (int i = 0; i < nthreads; ++i) {
        shared_job j = {H, I, x, wg, wu, wd, tokens, out,
                        (int)((long)n * i / nthreads), (int)((long)n * (i + 1) / nthreads)};
        jobs[i] = j;
    }
    for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, shared_worker, &jobs[i]);
    shared_worker(&jobs[0]);
    for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
    return 0;
}

/* -------------------------------------------------------------- FP8 e4m3 */

/* Value of an e4m3 (OCP "fn" variant) code: 1 sign bit, 4 exponent bits with
 * bias 7, 3 mantissa bits; exponent 0 is subnormal (m/8 * 2^-6); 0x7F/0xFF are
 * NaN (returned as NaN here); there is no infinity; the largest finite value
 * is 448. */
double oracle_e4m3_decode(uint8_t c)
{
    int sgn = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = (double)m / 8.0 * ldexp(1.0, -6);
    else
        v = (1.0 + (double)m / 8.0) * ldexp(1.0, e - 7);
    return sgn ? -v : v;
}

/* All 256 decoded codes, built once from oracle_e4m3_decode (a speed-up of the
 * GEMM loops only; the definition is the function above). */
static double g_e4m3[256];
static pthread_once_t g_e4m3_once = PTHREAD_ONCE_INIT;
static void build_e4m3_table(void)
{
    for (int c = 0; c < 256; ++c) g_e4m3[c] = oracle_e4m3_decode((uint8_t)c);
}
static double e4m3(uint8_t c) { return g_e4m3[c]; }

/* Round-to-nearest-even e4m3 code of a value already inside [-448, 448]:
 * the nearest finite code by brute force over all 127 magnitudes; on a tie the
 * code whose last mantissa bit is 0. */
uint8_t oracle_e4m3_encode(float v)
{
    double a = fabs((double)v);
    int best = 0;
    double bd = INFINITY;
    for (int c = 0; c < 127; ++c) {
        double d = fabs(oracle_e4m3_decode((uint8_t)c) - a);
        if (d < bd || (d == bd && (c & 1) == 0 && (best & 1) == 1)) {
            bd = d;
            best = c;
        }
    }
    if (best != 0 && v < 0) best |= 0x80;
    if (best == 0 && signbit(v)) best = 0x80;
    return (uint8_t)best;
}

/* Codes of n values already inside [-448, 448]. */
void oracle_e4m3_encode_array(int n, const float *v, uint8_t *q)
{
    for (int i = 0; i < n; ++i) q[i] = oracle_e4m3_encode(v[i]);
}

/* Quantise one group of n fp32 values: s = amax/448, q = e4m3(clamp(v/s)). */
static float quantize_group(const float *v, int n, uint8_t *q)
{
    float amax = 0.0f;
    for (int i = 0; i < n; ++i)
        if (fabsf(v[i]) > amax) amax = fabsf(v[i]);
    if (amax == 0.0f) {
        for (int i = 0; i < n; ++i) q[i] = 0;
        return 1.0f;
    }
    float s = amax / 448.0f;
    for (int i = 0; i < n; ++i) {
        float r = v[i] / s;
        if (r > 448.0f) r = 448.0f;
        if (r < -448.0f) r = -448.0f;
        q[i] = oracle_e4m3_encode(r);
    }
    return s;
}

/* Per-row, per-128-column-group quantisation of a bf16 matrix [R, K]
 * (K a multiple of 128): q [R, K] e4m3 codes, s [R, K/128] fp32 scales. */
int oracle_quantize_rows(int R, int K, const uint16_t *a, uint8_t *q, float *s)
{
    if (R < 0 || K <= 0 || K % 128) return 1;
    float buf[128];
    for (int r = 0; r < R; ++r)
        for (int g = 0; g < K / 128; ++g) {
            for (int i = 0; i < 128; ++i) buf[i] = bf16_to_f32(a[(size_t)r * K + g * 128 + i]);
            s[(size_t)r * (K / 128) + g] = quantize_group(buf, 128, q + (size_t)r * K + g * 128);
        }
    return 0;
}

/* One row of a block-scaled GEMM: out[n] = sum_kb sa[kb] * sb[n/128, kb] *
 * sum_{k in kb} qa[k] * qb[n, k], for n in [0, N); qb [N, K] codes, sb [N/128,
 * K/128] scales, qa [K] codes, sa [K/128] scales. */
static void fp8_row_gemm(int N, int K, const uint8_t *qa, const float *sa, const uint8_t *qb,
                         const float *sb, double *out)
{
    const int KB = K / 128;
    for (int n = 0; n < N; ++n) {
        double acc = 0.0;
        for (int kb = 0; kb < KB; ++kb) {
            double part = 0.0;
            for (int k = kb * 128; k < kb * 128 + 128; ++k)
                part += e4m3(qa[k]) * e4m3(qb[(size_t)n * K + k]);
            acc += (double)sa[kb] * (double)sb[(size_t)(n / 128) * KB + kb] * part;
        }
        out[n] = acc;
    }
}

typedef struct {
    int H, I, k;
    const uint16_t *x;
    const int32_t *idx;
    const double *gate;
    const uint8_t *wg, *wu, *wd;
    const float *sg, *su, *sd;
    const int32_t *tokens;
    double *out;
    int n0, n1;
} ffn8_job;

static void *ffn8_worker(void *p)
{
    ffn8_job *j = (ffn8_job *)p;
    const int H = j->H, I = j->I;
    uint8_t *qx = (uint8_t *)malloc((size_t)H);
    float *sx = (float *)malloc(sizeof(float) * (size_t)(H / 128));
    double *g = (double *)malloc(sizeof(double) * (size_t)I);
    double *u = (double *)malloc(sizeof(double) * (size_t)I);
    float *h = (float *)malloc(sizeof(float) * (size_t)I);
    uint8_t *qh = (uint8_t *)malloc((size_t)I);
    float *sh = (float *)malloc(sizeof(float) * (size_t)(I / 128));
    double *y = (double *)malloc(sizeof(double) * (size_t)H);
    for (int n = j->n0; n < j->n1; ++n) {
        int t = j->tokens ? j->tokens[n] : n;
        oracle_quantize_rows(1, H, j->x + (size_t)t * H, qx, sx);
        double *o = j->out + (size_t)n * H;
        for (int c = 0; c < H; ++c) o[c] = 0.0;
        for (int q = 0; q < j->k; ++q) {
            int e = j->idx[(size_t)t * j->k + q];
            double gt = j->gate[(size_t)t * j->k + q];
            fp8_row_gemm(I, H, qx, sx, j->wg + (size_t)e * I * H, j->sg + (size_t)e * (I / 128) * (H / 128), g);
            fp8_row_gemm(I, H, qx, sx, j->wu + (size_t)e * I * H, j->su + (size_t)e * (I / 128) * (H / 128), u);
            for (int i = 0; i < I; ++i) h[i] = (float)(silu(g[i]) * u[i]);
            for (int b = 0; b < I / 128; ++b) sh[b] = quantize_group(h + b * 128, 128, qh + b * 128);
            fp8_row_gemm(H, I, qh, sh, j->wd + (size_t)e * H * I, j->sd + (size_t)e * (H / 128) * (I / 128), y);
            for (int c = 0; c < H; ++c) o[c] += gt * y[c];
        }
    }
    free(qx); free(sx); free(g); free(u); free(h); free(qh); free(sh); free(y);
    return NULL;
}

/* FP8 variant of oracle_combine_ffn: x [T,H] bf16 is quantised per token per
 * 128 columns, each chosen expert's gate/up GEMMs are block-scaled sums, the
 * SwiGLU output h (rounded to fp32) is requantised per 128 columns, the down
 * GEMM is block-scaled, and the k results are summed with the gates in fp64.
 *   wg/wu [E,I,H] codes with sg/su [E,I/128,H/128]; wd [E,H,I] with sd [E,H/128,I/128]. */
int oracle_combine_ffn_fp8(int H, int I, int k, const uint16_t *x, const int32_t *idx,
                           const double *gate, const uint8_t *wg, const float *sg, const uint8_t *wu,
                           const float *su, const uint8_t *wd, const float *sd, int n,
                           const int32_t *tokens, double *out, int nthreads)
{
    if (H <= 0 || I <= 0 || H % 128 || I % 128 || k < 1 || n < 0) return 1;
    pthread_once(&g_e4m3_once, build_e4m3_table);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > n) nthreads = n > 0 ? n : 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    ffn8_job jobs[256];
    for (int i = 0; i < nthreads; ++i) {
        ffn8_job jb = {H, I, k, x, idx, gate, wg, wu, wd, sg, su, sd, tokens, out,
                       (int)((long)n * i / nthreads), (int)((long)n * (i + 1) / nthreads)};
        jobs[i] = jb;
    }
    for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, ffn8_worker, &jobs[i]);
    ffn8_worker(&jobs[0]);
    for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
    return 0;
}

/* ------------------------------------------------- MX (OCP microscaling) */

/* Value of an e2m1 (FP4) code, bits s eem: 1 sign bit, 2 exponent bits with bias
 * 1, 1 mantissa bit; exponent 0 is subnormal (m * 0.5).  The magnitudes are 0,
 * 0.5, 1, 1.5, 2, 3, 4, 6; there is no infinity or NaN. */
double oracle_e2m1_decode(uint8_t c)
{
    int sgn = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
    double v = e == 0 ? 0.5 * m : (1.0 + 0.5 * m) * ldexp(1.0, e - 1);
    return sgn ? -v : v;
}

/* Round-to-nearest-even code of a value inside the format's range: the nearest of
 * the nmag magnitudes (codes 0..nmag-1 in increasing order) by brute force; on a
 * tie the code whose last (mantissa) bit is 0.  sign_bit is the code's sign bit. */
static uint8_t encode_rne(double v, double (*decode)(uint8_t), int nmag, int sign_bit)
{
    double a = fabs(v);
    int best = 0;
    double bd = INFINITY;
    for (int c = 0; c < nmag; ++c) {
        double d = fabs(decode((uint8_t)c) - a);
        if (d < bd || (d == bd && !(c & 1) && (best & 1))) {  /* a tie goes to the even code */
            bd = d;
            best = c;
        }
    }
    if (best != 0 && v < 0) best |= 1 << sign_bit;
    return (uint8_t)best;
}

uint8_t oracle_e2m1_encode(float v) { return encode_rne((double)v, oracle_e2m1_decode, 8, 3); }

/* The two MX element formats used here: e4m3 (largest exponent emax = 8, largest
 * value 448) and e2m1 (emax = 2, largest value 6). */
enum { MX_E4M3 = 0, MX_E2M1 = 1 };
#define MX_BLOCK 32

/* One MX block of 32 fp32 values (OCP Microscaling Formats, v1.0, the conversion
 * of a block: the shared scale is 2^X with X = floor(log2(max |v|)) - emax of the
 * element format, stored as an e8m0 code X + 127; each element is v / 2^X rounded
 * to nearest-even in the element format, values past its largest magnitude
 * clamped to it).  Readings: X is clamped to [-127, 127]; an all-zero block gets
 * X = 0 and zero codes.  Returns the e8m0 code; q receives the element codes. */
static uint8_t mx_quantize_block(const float *v, int fmt, uint8_t *q)
{
    const int emax = fmt == MX_E4M3 ? 8 : 2;
    const double vmax = fmt == MX_E4M3 ? 448.0 : 6.0;
    double amax = 0.0;
    for (int i = 0; i < MX_BLOCK; ++i)
        if (fabs((double)v[i]) > amax) amax = fabs((double)v[i]);
    if (amax == 0.0) {
        for (int i = 0; i < MX_BLOCK; ++i) q[i] = 0;
        return 127;
    }
    int ex;
    frexp(amax, &ex);  /* amax = f * 2^ex, f in [0.5, 1): floor(log2(amax)) = ex - 1 */
    int X = ex - 1 - emax;
    if (X < -127) X = -127;
    if (X > 127) X = 127;
    for (int i = 0; i < MX_BLOCK; ++i) {
        double r = ldexp((double)v[i], -X);
        if (r > vmax) r = vmax;
        if (r < -vmax) r = -vmax;
        q[i] = fmt == MX_E4M3 ? encode_rne(r, oracle_e4m3_decode, 127, 7) : encode_rne(r, oracle_e2m1_decode, 8, 3);
    }
    return (uint8_t)(X + 127);
}

/* Per-row MX quantisation of an fp32 matrix [R, K] (K a multiple of 32):
 * q [R, K] element codes (one per byte), x [R, K/32] e8m0 scale codes. */
int oracle_mx_quantize_rows(int R, int K, const float *a, int fmt, uint8_t *q, uint8_t *x)
{
    if (R < 0 || K <= 0 || K % MX_BLOCK || (fmt != MX_E4M3 && fmt != MX_E2M1)) return 1;
    for (int r = 0; r < R; ++r)
        for (int b = 0; b < K / MX_BLOCK; ++b)
            x[(size_t)r * (K / MX_BLOCK) + b] =
                mx_quantize_block(a + (size_t)r * K + b * MX_BLOCK, fmt, q + (size_t)r * K + b * MX_BLOCK);
    return 0;
}

/* One row of an MX GEMM, activations e4m3 and weights e2m1:
 *   out[n] = sum_kb 2^(xa[kb] - 127) * 2^(xb[n,kb] - 127) * sum_{k in kb} a_k * b_{n,k}
 * over blocks kb of 32 along K; qb [N, K] e2m1 codes, xb [N, K/32]. */
static void mx_row_gemm(int N, int K, const uint8_t *qa, const uint8_t *xa, const uint8_t *qb,
                        const uint8_t *xb, double *out)
{
    const int KB = K / MX_BLOCK;
    for (int n = 0; n < N; ++n) {
        double acc = 0.0;
        for (int kb = 0; kb < KB; ++kb) {
            double part = 0.0;
            for (int k = kb * MX_BLOCK; k < kb * MX_BLOCK + MX_BLOCK; ++k)
                part += e4m3(qa[k]) * oracle_e2m1_decode(qb[(size_t)n * K + k]);
            acc += ldexp(1.0, (int)xa[kb] - 127) * ldexp(1.0, (int)xb[(size_t)n * KB + kb] - 127) * part;
        }
        out[n] = acc;
    }
}

typedef struct {
    int H, I, k;
    const uint16_t *x;
    const int32_t *idx;
    const double *gate;
    const uint8_t *wg, *wu, *wd, *xg, *xu, *xd;
    const int32_t *tokens;
    double *out;
    int n0, n1;
} ffnmx_job;

static void *ffnmx_worker(void *p)
{
    ffnmx_job *j = (ffnmx_job *)p;
    const int H = j->H, I = j->I;
    float *xf = (float *)malloc(sizeof(float) * (size_t)H);
    uint8_t *qx = (uint8_t *)malloc((size_t)H);
    uint8_t *sx = (uint8_t *)malloc((size_t)(H / MX_BLOCK));
    double *g = (double *)malloc(sizeof(double) * (size_t)I);
    double *u = (double *)malloc(sizeof(double) * (size_t)I);
    float *h = (float *)malloc(sizeof(float) * (size_t)I);
    uint8_t *qh = (uint8_t *)malloc((size_t)I);
    uint8_t *sh = (uint8_t *)malloc((size_t)(I / MX_BLOCK));
    double *y = (double *)malloc(sizeof(double) * (size_t)H);
    for (int n = j->n0; n < j->n1; ++n) {
        int t = j->tokens ? j->tokens[n] : n;
        for (int c = 0; c < H; ++c) xf[c] = bf16_to_f32(j->x[(size_t)t * H + c]);
        oracle_mx_quantize_rows(1, H, xf, MX_E4M3, qx, sx);
        double *o = j->out + (size_t)n * H;
        for (int c = 0; c < H; ++c) o[c] = 0.0;
        for (int q = 0; q < j->k; ++q) {
            int e = j->idx[(size_t)t * j->k + q];
            double gt = j->gate[(size_t)t * j->k + q];
            mx_row_gemm(I, H, qx, sx, j->wg + (size_t)e * I * H, j->xg + (size_t)e * I * (H / MX_BLOCK), g);
            mx_row_gemm(I, H, qx, sx, j->wu + (size_t)e * I * H, j->xu + (size_t)e * I * (H / MX_BLOCK), u);
            for (int i = 0; i < I; ++i) h[i] = (float)(silu(g[i]) * u[i]);
            oracle_mx_quantize_rows(1, I, h, MX_E4M3, qh, sh);
            mx_row_gemm(H, I, qh, sh, j->wd + (size_t)e * H * I, j->xd + (size_t)e * H * (I / MX_BLOCK), y);
            for (int c = 0; c < H; ++c) o[c] += gt * y[c];
        }
    }
    free(xf); free(qx); free(sx); free(g); free(u); free(h); free(qh); free(sh); free(y);
    return NULL;
}

/* MX variant of oracle_combine_ffn (FP4 weights, FP8 activations, each with one
 * power-of-two scale per 32 values along K): x [T,H] bf16 is quantised per token
 * to MX e4m3, each chosen expert's gate/up GEMMs are MX block sums against e2m1
 * weights, the SwiGLU output h (rounded to fp32) is requantised to MX e4m3, the
 * down GEMM is an MX block sum, and the k results are summed with the gates in fp64.
 *   wg/wu [E,I,H] e2m1 codes with xg/xu [E,I,H/32] e8m0 codes; wd [E,H,I] with
 *   xd [E,H,I/32]. */
int oracle_combine_ffn_mx(int H, int I, int k, const uint16_t *x, const int32_t *idx,
                          const double *gate, const uint8_t *wg, const uint8_t *xg, const uint8_t *wu,
                          const uint8_t *xu, const uint8_t *wd, const uint8_t *xd, int n,
                          const int32_t *tokens, double *out, int nthreads)
{
    if (H <= 0 || I <= 0 || H % MX_BLOCK || I % MX_BLOCK || k < 1 || n < 0) return 1;
    pthread_once(&g_e4m3_once, build_e4m3_table);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > n) nthreads = n > 0 ? n : 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    ffnmx_job jobs[256];
    for (int i = 0; i < nthreads; ++i) {
        ffnmx_job jb = {H, I, k, x, idx, gate, wg, wu, wd, xg, xu, xd, tokens, out,
                        (int)((long)n * i / nthreads), (int)((long)n * (i + 1) / nthreads)};
        jobs[i] = jb;
    }
    for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, ffnmx_worker, &jobs[i]);
    ffnmx_worker(&jobs[0]);
    for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
    return 0;
}
