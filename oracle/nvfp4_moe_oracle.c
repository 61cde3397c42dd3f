/*
 * FP64 CPU oracle for the routed NVFP4 mixture-of-experts FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY: loaded by the tests, the smoke check and the bench's
 * CPU-baseline leg; never by the layer itself. Plain loops, no blocking, no
 * fusion; every weight is decoded exactly and every sum is accumulated in FP64.
 *
 * Passages followed (pages' titles and sections):
 *   - Weight = E2M1 code x E4M3 scale of its group of 16 inputs x FP32 tensor
 *     scale: "TensorFold PR #906" first post (groups of 16 preserved, FP32 tensor
 *     scale unchanged); "Strata NVFP4" README, "How it differs from upstream
 *     Strata" (4.5-bit experts, calibrated scales, lossless repack). The E2M1 and
 *     E4M3 encodings themselves are the OCP Microscaling and OCP FP8 formats.
 *   - The per-expert FP32 scale multiplies each projection's output: same README,
 *     same section, first bullet.
 *   - Gate/up/down expert tensors with one global scale per projection: "#2727
 *     tools: add opt-in FP4-Local CSF checkpoint conversion", "Validation".
 *   - Softmax top-k renormalised routing, SwiGLU, routing-weighted combine: the
 *     pages name routed experts and a fused SwiGLU ("Strata NVFP4" README, the
 *     0.1.39-nvfp4.2 bullet) without writing the math; the oracle takes the
 *     textbook definitions, listed where each is used.
 */
#include "nvfp4_moe_oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* ---------------------------------------------------------------- decoders */

/* OCP MX E2M1: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0.
 * Exponent 0 is subnormal: value = mantissa * 2^(1-1) * 0.5. */
double orc_e2m1(uint32_t nib) {
    nib &= 0xFu;
    const int s = (nib >> 3) & 1, e = (nib >> 1) & 3, m = nib & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* OCP FP8 E4M3FN: sign bit 7, exponent bits 6..3 (bias 7), mantissa bits 2..0.
 * Exponent 0 is subnormal (m * 2^-9); S.1111.111 is NaN; no infinities. */
double orc_e4m3(uint32_t byte) {
    byte &= 0xFFu;
    const int s = (byte >> 7) & 1, e = (byte >> 3) & 0xF, m = byte & 7;
    if (e == 0xF && m == 7) return NAN;
    double mag = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* BF16 is the upper half of an IEEE binary32. */
double orc_bf16(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Nearest BF16 to an FP64 value, ties to even, by exhaustive neighbour choice:
 * take the two BF16 values that bracket v (found from the truncated FP32 bits)
 * and pick the nearer one, the one with an even last bit on a tie. */
uint16_t orc_bf16_rne(double v) {
    if (isnan(v)) return 0x7FC0;
    float f = (float)v; /* FP32 first only to find the bracket; decided in FP64 below */
    uint32_t u;
    memcpy(&u, &f, 4);
    uint16_t lo = (uint16_t)(u >> 16);
    /* candidates: lo and its neighbours one step away in magnitude */
    uint16_t best = lo;
    double bestd = fabs(orc_bf16(lo) - v);
    for (int d = -1; d <= 1; d += 2) {
        uint16_t c = (uint16_t)(lo + d);
        if (((c ^ lo) & 0x8000u) != 0) continue; /* crossed the sign bit */
        double cv = orc_bf16(c);
        if (isnan(cv)) continue;
        double cd = fabs(cv - v);
        if (cd < bestd || (cd == bestd && (c & 1u) == 0 && (best & 1u) == 1)) {
            best = c;
            bestd = cd;
        }
    }
    return best;
}

void orc_bf16_rne_array(int64_t n, const double *v, uint16_t *out) {
    for (int64_t i = 0; i < n; i++) out[i] = orc_bf16_rne(v[i]);
}

/* Tables built from the decoders above, once. */
static double g_e2m1[16], g_e4m3[256];
static pthread_once_t g_once = PTHREAD_ONCE_INIT;
static void build_tables(void) {
    for (int i = 0; i < 16; i++) g_e2m1[i] = orc_e2m1((uint32_t)i);
    for (int i = 0; i < 256; i++) g_e4m3[i] = orc_e4m3((uint32_t)i);
}
static void tables(void) { pthread_once(&g_once, build_tables); }

/* One weight: element (row, k) of a [rows][cols] matrix of one expert. */
static inline double weight(const uint8_t *codes, const uint8_t *scales, int cols, int row,
                            int k, double glob, int plant) {
    uint8_t byte = codes[(size_t)row * (cols / 2) + k / 2];
    int hi = (k & 1);
    if (plant == ORC_PLANT_NIBBLE_ORDER) hi = !hi;
    uint32_t nib = hi ? (byte >> 4) : (byte & 0xF);
    int grp = k / 16;
    if (plant == ORC_PLANT_GROUP_SHIFT) grp = (grp + 1) % (cols / 16);
    double s = g_e4m3[scales[(size_t)row * (cols / 16) + grp]];
    if (plant == ORC_PLANT_NO_GLOBAL) glob = 1.0;
    return g_e2m1[nib] * s * glob;
}

void orc_decode_matrix(int32_t rows, int32_t cols, const uint8_t *codes, const uint8_t *scales,
                       float glob, double *dst) {
    tables();
    for (int r = 0; r < rows; r++)
        for (int k = 0; k < cols; k++)
            dst[(size_t)r * cols + k] = weight(codes, scales, cols, r, k, (double)glob, 0);
}

/* ----------------------------------------------------------------- routing */

/* Key order for selection: larger logit first; NaN below every number; equal
 * logits -> lower expert id first. */
static int before(float a, int ia, float b, int ib) {
    int na = isnan(a), nb = isnan(b);
    if (na || nb) {
        if (na && nb) return ia < ib;
        return nb; /* a is a number, b is NaN */
    }
    if (a != b) return a > b;
    return ia < ib;
}

int orc_route(int32_t T, int32_t E, int32_t K, const float *logits, int32_t *ids, double *w) {
    int bad = 0;
    int *chosen = (int *)calloc((size_t)E, sizeof(int));
    for (int t = 0; t < T; t++) {
        const float *l = logits + (size_t)t * E;
        memset(chosen, 0, sizeof(int) * (size_t)E);
        /* selection: K passes, each taking the best unchosen expert */
        for (int j = 0; j < K; j++) {
            int best = -1;
            for (int e = 0; e < E; e++) {
                if (chosen[e]) continue;
                if (best < 0 || before(l[e], e, l[best], best)) best = e;
            }
            chosen[best] = 1;
            ids[(size_t)t * K + j] = best;
        }
        /* softmax over all E restricted to the K selected and renormalised:
         * w_j = exp(l_j) / sum_sel exp(l_i) = exp(l_j - l_max) / sum exp(l_i - l_max) */
        double lmax = (double)l[ids[(size_t)t * K]];
        int finite = 1;
        for (int j = 0; j < K; j++)
            if (!isfinite(l[ids[(size_t)t * K + j]])) finite = 0;
        if (!finite) bad++;
        double den = 0.0;
        for (int j = 0; j < K; j++) den += exp((double)l[ids[(size_t)t * K + j]] - lmax);
        for (int j = 0; j < K; j++)
            w[(size_t)t * K + j] = exp((double)l[ids[(size_t)t * K + j]] - lmax) / den;
    }
    free(chosen);
    return bad;
}

int orc_check_ids(int32_t T, int32_t E, int32_t K, const int32_t *ids) {
    int bad = 0;
    for (int t = 0; t < T; t++) {
        int ok = 1;
        for (int j = 0; j < K; j++) {
            int e = ids[(size_t)t * K + j];
            if (e < 0 || e >= E) ok = 0;
            for (int i = 0; i < j; i++)
                if (ids[(size_t)t * K + i] == e) ok = 0;
        }
        bad += !ok;
    }
    return bad;
}

void orc_sort(int32_t T, int32_t E, int32_t K, const int32_t *ids, int32_t *counts,
              int32_t *offsets, int32_t *perm) {
    for (int e = 0; e < E; e++) counts[e] = 0;
    for (int p = 0; p < T * K; p++) counts[ids[p]]++;
    offsets[0] = 0;
    for (int e = 0; e < E; e++) offsets[e + 1] = offsets[e] + counts[e];
    /* for each expert ascending, the pairs naming it in token order */
    int pos = 0;
    for (int e = 0; e < E; e++)
        for (int t = 0; t < T; t++)
            for (int j = 0; j < K; j++)
                if (ids[(size_t)t * K + j] == e) perm[pos++] = t * K + j;
}

/* --------------------------------------------------------------- quantiser */

/* RNE of a non-negative FP64 value <= 448 to an E4M3FN byte, by scanning the
 * 127 finite non-negative codes for the nearest value (ties -> even code). */
static uint8_t e4m3_nearest(double v) {
    if (v > 448.0) v = 448.0;
    int best = 0;
    double bd = fabs(g_e4m3[0] - v);
    for (int b = 1; b <= 0x7E; b++) {
        double d = fabs(g_e4m3[b] - v);
        if (d < bd || (d == bd && (b & 1) == 0)) {
            best = b;
            bd = d;
        }
    }
    return (uint8_t)best;
}

/* RNE of an FP64 ratio to an E2M1 nibble (nearest of the 8 magnitudes, ties ->
 * even mantissa bit, saturating at 6), sign in bit 3. */
static uint8_t e2m1_nearest(double r) {
    double a = fabs(r);
    int best = 0;
    double bd = fabs(g_e2m1[0] - a);
    for (int c = 1; c < 8; c++) {
        double d = fabs(g_e2m1[c] - a);
        if (d < bd || (d == bd && (c & 1) == 0)) {
            best = c;
            bd = d;
        }
    }
    return (uint8_t)(best | (r < 0 ? 8 : 0));
}

/* global = amax/(6*448) in FP64 stored as FP32; group scale = RNE_E4M3(group
 * amax / (6*global)); code = RNE_E2M1(w / (scale*global)); a zero scale or a
 * zero global gives zero codes. */
int orc_quantize(int32_t n_mat, int32_t rows, int32_t cols, const uint16_t *w_bf16,
                 uint8_t *codes, uint8_t *scales, float *glob) {
    if (cols % 16) return -1;
    tables();
    for (int n = 0; n < n_mat; n++) {
        const uint16_t *w = w_bf16 + (size_t)n * rows * cols;
        double amax = 0.0;
        for (size_t i = 0; i < (size_t)rows * cols; i++) {
            double a = fabs(orc_bf16(w[i]));
            if (a > amax) amax = a;
        }
        float g32 = (float)(amax / (6.0 * 448.0));
        glob[n] = g32;
        double g = (double)g32;
        for (int r = 0; r < rows; r++) {
            for (int gi = 0; gi < cols / 16; gi++) {
                double gam = 0.0;
                for (int k = 0; k < 16; k++) {
                    double a = fabs(orc_bf16(w[(size_t)r * cols + gi * 16 + k]));
                    if (a > gam) gam = a;
                }
                uint8_t sb = (g > 0.0) ? e4m3_nearest(gam / g / 6.0) : 0;
                scales[((size_t)n * rows + r) * (cols / 16) + gi] = sb;
                double step = g_e4m3[sb] * g;
                for (int k = 0; k < 16; k += 2) {
                    int kk = gi * 16 + k;
                    double r0 = step > 0 ? orc_bf16(w[(size_t)r * cols + kk]) / step : 0.0;
                    double r1 = step > 0 ? orc_bf16(w[(size_t)r * cols + kk + 1]) / step : 0.0;
                    codes[((size_t)n * rows + r) * (cols / 2) + kk / 2] =
                        (uint8_t)(e2m1_nearest(r0) | (e2m1_nearest(r1) << 4));
                }
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------- router projection */

/* Router logits from the layer's input: the projection that the pages keep on
 * FP32-exact inputs ("Strata NVFP4" README, "How it differs from upstream
 * Strata": the prompt path's BF16 projections -- router among them -- take
 * FP32-exact inputs):
 *   logits[t][e] = sum_k W_r[e][k] * x[t][k]
 * W_r is BF16, x is FP32 and is never rounded to BF16; every product and every
 * sum is FP64. */
void orc_router(int32_t T, int32_t E, int32_t H, const float *x, const uint16_t *w_r,
                double *logits) {
    for (int t = 0; t < T; t++)
        for (int e = 0; e < E; e++) {
            double s = 0.0;
            for (int k = 0; k < H; k++)
                s += orc_bf16(w_r[(size_t)e * H + k]) * (double)x[(size_t)t * H + k];
            logits[(size_t)t * E + e] = s;
        }
}

/* ------------------------------------------------------------------- layer */

static double act_value(int act_type, const void *row, int k) {
    if (act_type == 0) return orc_bf16(((const uint16_t *)row)[k]);
    return (double)((const int8_t *)row)[k];
}

/* SwiGLU of one (token, expert) pair:
 *   g = s_g * xs * sum_k G[i][k] x[k],  u = s_u * xs * sum_k U[i][k] x[k],
 *   h[i] = g / (1 + exp(-g)) * u
 * with xs = 1 for BF16 activations and the per-token scale for int8 ones. The
 * globals are applied after the sums (output-side scale). */
int orc_pair_h(const orc_dims *d, const orc_weights *w, int32_t act_type, const void *x_row,
               float x_scale, int32_t e, double *h, int32_t plant) {
    tables();
    const int H = d->H, I = d->I;
    const size_t gc = (size_t)e * I * (H / 2), gs = (size_t)e * I * (H / 16);
    const double xs = act_type == 0 ? 1.0 : (double)x_scale;
    for (int i = 0; i < I; i++) {
        double sg = 0.0, su = 0.0;
        for (int k = 0; k < H; k++) {
            double x = act_value(act_type, x_row, k);
            sg += weight(w->gate_codes + gc, w->gate_scales + gs, H, i, k, 1.0, plant) * x;
            su += weight(w->up_codes + gc, w->up_scales + gs, H, i, k, 1.0, plant) * x;
        }
        double gg = (plant == ORC_PLANT_NO_GLOBAL) ? 1.0 : (double)w->gate_global[e];
        double ug = (plant == ORC_PLANT_NO_GLOBAL) ? 1.0 : (double)w->up_global[e];
        double g = gg * xs * sg, u = ug * xs * su;
        if (plant == ORC_PLANT_SWAP_GATE_UP) {
            double t = g;
            g = u;
            u = t;
        }
        double silu = (plant == ORC_PLANT_SILU_SIGN) ? g / (1.0 + exp(g)) : g / (1.0 + exp(-g));
        h[i] = silu * u;
    }
    return 0;
}

typedef struct {
    const orc_dims *d;
    const orc_weights *w;
    int32_t T, act_type;
    const void *act;
    const float *act_scale;
    const int32_t *ids;
    const double *wts;
    int32_t n, tid, nthreads, plant;
    const int32_t *sample;
    double *out;
} job_t;

/* out_t = sum_j w_{t,j} * y_{t,e_j},  y = s_d * sum_i D[r][i] h[i]  (r = 0..H-1) */
static void *run_tokens(void *arg) {
    job_t *jb = (job_t *)arg;
    const orc_dims *d = jb->d;
    const int H = d->H, I = d->I, K = d->K;
    const size_t xrow = (size_t)H * (jb->act_type == 0 ? 2 : 1);
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
    for (int s = jb->tid; s < jb->n; s += jb->nthreads) {
        const int t = jb->sample ? jb->sample[s] : s;
        const void *xr = (const char *)jb->act + (size_t)t * xrow;
        const float xs = jb->act_type == 0 ? 1.0f : jb->act_scale[t];
        double *o = jb->out + (size_t)s * H;
        for (int r = 0; r < H; r++) o[r] = 0.0;
        for (int j = 0; j < K; j++) {
            const int e = jb->ids[(size_t)t * K + j];
            const double wj = (jb->plant == ORC_PLANT_EQUAL_WEIGHTS) ? 1.0 / K
                                                                     : jb->wts[(size_t)t * K + j];
            orc_pair_h(d, jb->w, jb->act_type, xr, xs, e, h, jb->plant);
            const size_t dc = (size_t)e * H * (I / 2), ds = (size_t)e * H * (I / 16);
            const double dg = (jb->plant == ORC_PLANT_NO_GLOBAL) ? 1.0 : (double)jb->w->down_global[e];
            for (int r = 0; r < H; r++) {
                double acc = 0.0;
                for (int i = 0; i < I; i++)
                    acc += weight(jb->w->down_codes + dc, jb->w->down_scales + ds, I, r, i, 1.0,
                                  jb->plant) * h[i];
                o[r] += wj * (dg * acc);
            }
        }
    }
    free(h);
    return NULL;
}

int orc_moe(const orc_dims *d, const orc_weights *w, int32_t T, int32_t act_type,
            const void *act, const float *act_scale, const int32_t *ids, const double *wts,
            int32_t n_sample, const int32_t *sample, double *out, int32_t nthreads,
            int32_t plant) {
    if (!d || !w || !act || !ids || !wts || !out || T < 0) return -1;
    if (d->H % 16 || d->I % 16 || d->K < 1 || d->K > d->E) return -1;
    if (act_type == 1 && !act_scale) return -1;
    tables();
    const int n = sample ? n_sample : T;
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads > n) nthreads = n > 0 ? n : 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    job_t *jobs = (job_t *)malloc(sizeof(job_t) * (size_t)nthreads);
    for (int i = 0; i < nthreads; i++) {
        jobs[i] = (job_t){d, w, T, act_type, act, act_scale, ids, wts, n, i, nthreads, plant,
                          sample, out};
        pthread_create(&th[i], NULL, run_tokens, &jobs[i]);
    }
    for (int i = 0; i < nthreads; i++) pthread_join(th[i], NULL);
    free(th);
    free(jobs);
    return 0;
}
